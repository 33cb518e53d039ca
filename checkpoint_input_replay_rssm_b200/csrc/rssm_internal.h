// rssm_internal.h -- host-side context shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/rssm.h"
#include "rssm_device.cuh"

namespace rssm {

struct Ctx {
    rssm_config cfg;
    rssm_workspace_layout lay;
    uint8_t *ws = nullptr;
    size_t ws_bytes = 0;
    cudaStream_t stream = nullptr;
    int pending = 0;            // K of an uncommitted verify (host mirror), 0 if none
    int len_lb = 0, len_ub = 0; // bounds of every sequence's committed buffer length (host mirror)
    int64_t launches = 0;       // kernels enqueued so far
    int num_sms = 148;          // SMs of the handle's device
    cudaEvent_t split_event = nullptr;  // recorded between prep and read kernels (measurement)
    std::string err;

    void *at(size_t off) const { return ws + off; }
    Counters counters() const {
        Counters c;
        c.seq_pos = (int64_t *)at(lay.seq_pos_off);
        c.ckpt_pos = (int64_t *)at(lay.ckpt_pos_off);
        c.pending = (int32_t *)at(lay.pending_off);
        c.flush_count = (int32_t *)at(lay.flush_count_off);
        c.arrive = (int32_t *)at(lay.arrive_off);
        c.err = (int32_t *)at(lay.error_off);
        return c;
    }
    // Replay: work list of the flush kernel, after the per-sequence hand-off
    // (int32 count, 3 pad words, then [batch] sequence indices).
    int *fold_count() const { return (int *)at(lay.seqinfo_off + (size_t)cfg.batch * 16); }
    int *fold_list() const { return fold_count() + 4; }
};

// Kernel launchers (one per layer kind).  op: Op; T tokens appended (0 for
// flush/export); in/y used by decode/verify, out by export.  mamba2_launch
// counts its launches and keeps the buffer-length bounds len_lb/len_ub.
cudaError_t mamba2_launch(Ctx &h, int op, int T, const rssm_inputs *in, float *y, float *out,
                          cudaStream_t st);
size_t mamba2_smem_bytes(const rssm_config &cf, int T);
cudaError_t gdn_launch(const Ctx &h, int op, int T, const rssm_inputs *in, float *y, float *out,
                       cudaStream_t st);
size_t gdn_smem_bytes(const rssm_config &cf, int T);

// The replay-read kernel (rssm_read.cu), shared by both kinds: queries Q[b][row][m][n]
// at the given element strides, q_group heads per query row.
cudaError_t launch_read(const Ctx &h, int op, int T, const void *Q, int q_bf16, int q_group, int64_t q_stride_b,
                        int64_t q_stride_row, int64_t q_stride_m, const void *xnew, const float *D,
                        float *y, cudaStream_t st);
int read_heads_per_cta(const rssm_config &cf);
size_t read_smem_bytes(const rssm_config &cf, int T);

// Kernels shared by both kinds (rssm_common.cu).
cudaError_t launch_commit(const Ctx &h, const int32_t *accept, cudaStream_t st);
cudaError_t launch_import(const Ctx &h, const float *S, cudaStream_t st);
cudaError_t launch_export_eager(const Ctx &h, float *out, cudaStream_t st);

}  // namespace rssm
