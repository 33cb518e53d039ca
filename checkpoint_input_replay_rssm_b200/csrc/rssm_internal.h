// rssm_internal.h -- host-side context shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/rssm.h"
#include "rssm_device.cuh"

namespace rssm {

// The prep kernel's per-call hand-off to the flush and read kernels: per
// sequence {entries replayed, ring slot of entry 0, folded, valid}, the flush
// kernel's work list, the replay decays and coefficients, and (Gated DeltaNet,
// KDA) the swept queries.
struct Handoff {
    int4 *seqinfo;    // [B]
    int *fold_count;  // one int32, zero between calls
    int *fold_list;   // [B]
    float *dec;       // [B][H][tq_max]
    float *coef;      // [B][H][tq_max][Emax], Emax = window + tq_max rounded up to 4
    float *query;     // Gated DeltaNet: [B][H][tq_max][dstate] swept queries
    int tq_max;
};

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
    cudaEvent_t split_event = nullptr;  // recorded between prep/flush and read kernels (measurement)
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
    // The hand-off in the handle's workspace.
    Handoff handoff() const {
        Handoff o{};
        if (!lay.seqinfo_bytes) return o;
        o.seqinfo = (int4 *)at(lay.seqinfo_off);
        o.fold_count = fold_count();
        o.fold_list = fold_list();
        o.dec = (float *)at(lay.dec_off);
        o.coef = (float *)at(lay.coef_off);
        o.query = lay.query_bytes ? (float *)at(lay.query_off) : nullptr;
        o.tq_max = (int)lay.tq_max;
        return o;
    }
};

// Kernel launchers (one per layer kind).  op: Op; T tokens appended (0 for
// flush/export); in/y used by decode/verify, out by export.  The launchers count
// their launches and keep the buffer-length bounds len_lb/len_ub.
// ho: where the replay decode/verify hand-off lives (nullptr: the workspace's).
cudaError_t mamba2_launch(Ctx &h, int op, int T, const rssm_inputs *in, float *y, float *out,
                          cudaStream_t st, const Handoff *ho = nullptr);
size_t mamba2_smem_bytes(const rssm_config &cf, int T);
cudaError_t gdn_launch(Ctx &h, int op, int T, const rssm_inputs *in, float *y, float *out,
                       cudaStream_t st, const Handoff *ho = nullptr);

// Bounds of every sequence's committed buffer length after a replay decode or
// verify of T tokens (a verify's commit keeps 0..T of them): a sequence that
// folded holds its kept tokens, the others add them to what they had.
inline void update_len_bounds(Ctx &h, int op, int T) {
    const int W = h.cfg.window, kept_min = op == OP_DECODE ? T : 0;
    if (h.len_lb + T > W) {          // every sequence folded
        h.len_lb = kept_min;
        h.len_ub = T;
    } else if (h.len_ub + T <= W) {  // none did
        h.len_lb += kept_min;
        h.len_ub += T;
    } else {                          // some may have
        h.len_lb = kept_min;
        h.len_ub = W;
    }
}
size_t gdn_smem_bytes(const rssm_config &cf, int T);

// The replay-read kernel (rssm_read.cu), shared by both kinds: queries Q[b][row][m][n]
// at the given element strides, q_group heads per query row.  `early`: no flush
// kernel ran in the call (every sequence is read); `pdl`: the kernel directly
// follows the prep kernel in the stream and is launched as its programmatic dependent.
cudaError_t launch_read(const Ctx &h, int op, int T, const void *Q, int q_bf16, int q_group, int64_t q_stride_b,
                        int64_t q_stride_row, int64_t q_stride_m, const void *xnew, const float *D,
                        float *y, const Handoff &ho, cudaStream_t st, bool early, bool pdl);
int read_heads_per_cta(const rssm_config &cf);
size_t read_smem_bytes(const rssm_config &cf, int T);

// Argument checks and error recording of the C ABI (rssm_api.cu).
rssm_status api_fail(Ctx *h, rssm_status st, const std::string &m);
rssm_status api_cuda_fail(Ctx *h, cudaError_t e, const char *what);
bool api_inputs_ok(const Ctx *h, const rssm_inputs *in);

// Kernels shared by both kinds (rssm_common.cu).
cudaError_t launch_commit(const Ctx &h, const int32_t *accept, cudaStream_t st);
cudaError_t launch_import(const Ctx &h, const float *S, cudaStream_t st);
cudaError_t launch_export_eager(const Ctx &h, float *out, cudaStream_t st);

}  // namespace rssm
