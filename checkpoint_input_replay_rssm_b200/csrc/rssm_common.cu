// rssm_common.cu -- kernels shared by both layer kinds: commit (replay and
// eager), state import (quantising the read copy), eager export.
#include "rssm_internal.h"

namespace rssm {

// Replay commit: the buffer pointer moves by the accepted draft count; the
// rejected drafts stay in their slots and are overwritten later, and the
// checkpoint is not touched (irisproject.cloud, "Un retour en arriere qui
// devient trivial": rollback is a pointer operation on the buffer).
__global__ void commit_replay_kernel(Counters c, const int32_t *accept, int B) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int a = accept[b];
    const int pend = c.pending[b];
    int take = a;
    if (a < 0 || a > pend) {
        report(c.err, DEV_BAD_ACCEPT, b, -1, a);
        take = 0;
    }
    c.seq_pos[b] += take;
    c.pending[b] = 0;
}

// Eager commit: copy the snapshot of the last accepted draft into the state
// (per-draft snapshots are what eager speculative decoding has to materialise;
// aikraft.ru, "Pochemu eto vazhno dlya industrii").  One CTA per (b, h).
__global__ void __launch_bounds__(kThreads)
commit_eager_kernel(Counters c, const int32_t *accept, int H, int tile_bytes, int P,
                    uint8_t *state, const uint8_t *snap, int64_t state_bytes, float *scale,
                    const float *snap_scale, int64_t scale_elems) {
    const int bh = blockIdx.x, b = bh / H;
    __shared__ int s_take;
    if (threadIdx.x == 0) {
        const int a = accept[b];
        const int pend = c.pending[b];
        int take = a;
        if (a < 0 || a > pend) {
            if (bh % H == 0) report(c.err, DEV_BAD_ACCEPT, b, -1, a);
            take = 0;
        }
        s_take = take;
        const int64_t sp = c.seq_pos[b];
        arrive_and_publish(c, b, H, sp + take, sp + take, 0, 0);
    }
    __syncthreads();
    const int take = s_take;
    if (take == 0) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(snap + (int64_t)(take - 1) * state_bytes +
                                                       (int64_t)bh * tile_bytes);
    uint4 *dst = reinterpret_cast<uint4 *>(state + (int64_t)bh * tile_bytes);
    for (int i = threadIdx.x; i < tile_bytes / 16; i += blockDim.x) dst[i] = src[i];
    if (scale) {
        for (int p = threadIdx.x; p < P; p += blockDim.x)
            scale[(int64_t)bh * P + p] = snap_scale[(int64_t)(take - 1) * scale_elems + (int64_t)bh * P + p];
    }
}

// Quantise fp32 rows [rows][N] into the storage dtype (one warp per row).
template <int SK>
__global__ void quant_rows_kernel(const float *src, void *dst, float *scale, int64_t rows, int N) {
    const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float *r = src + row * N;
    float am = 0.f;
    for (int n = lane; n < N; n += 32) am = fmaxf(am, fabsf(r[n]));
    am = group_max<32>(am);
    const float sc = fp8_scale(am);
    for (int n = lane; n < N; n += 32) {
        const float v = r[n];
        if (SK == SK_BF16) {
            reinterpret_cast<__nv_bfloat16 *>(dst)[row * N + n] = __float2bfloat16_rn(v);
        } else {
            reinterpret_cast<__nv_fp8_storage_t *>(dst)[row * N + n] =
                __nv_cvt_float_to_fp8(__fdiv_rn(v, sc), __NV_SATFINITE, __NV_E4M3);
        }
    }
    if (SK == SK_FP8 && lane == 0) scale[row] = sc;
}

// Dequantise stored rows to fp32 (eager export).
template <int SK>
__global__ void dequant_rows_kernel(const void *src, const float *scale, float *dst, int64_t rows,
                                    int N) {
    const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float sc = (SK == SK_FP8) ? scale[row] : 1.f;
    for (int n = lane; n < N; n += 32) {
        float v;
        if (SK == SK_F32) {
            v = reinterpret_cast<const float *>(src)[row * N + n];
        } else if (SK == SK_BF16) {
            v = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(src)[row * N + n]);
        } else {
            __half_raw hr = __nv_cvt_fp8_to_halfraw(
                reinterpret_cast<const __nv_fp8_storage_t *>(src)[row * N + n], __NV_E4M3);
            v = __half2float(*reinterpret_cast<__half *>(&hr)) * sc;
        }
        dst[row * N + n] = v;
    }
}

cudaError_t launch_commit(const Ctx &h, const int32_t *accept, cudaStream_t st) {
    const rssm_config &cf = h.cfg;
    if (cf.mode == RSSM_REPLAY) {
        commit_replay_kernel<<<(cf.batch + 255) / 256, 256, 0, st>>>(h.counters(), accept, cf.batch);
        return cudaGetLastError();
    }
    const int64_t elems = (int64_t)cf.batch * cf.nheads * cf.headdim * cf.dstate;
    const int eb = cf.state_dtype == RSSM_F32 ? 4 : (cf.state_dtype == RSSM_BF16 ? 2 : 1);
    uint8_t *state = (uint8_t *)h.at(cf.state_dtype == RSSM_F32 ? h.lay.ckpt_off : h.lay.rc_off);
    const uint8_t *snap = (const uint8_t *)h.at(h.lay.snap_off);
    float *scale = nullptr;
    const float *snap_scale = nullptr;
    const int64_t scale_elems = (int64_t)cf.batch * cf.nheads * cf.headdim;
    if (cf.state_dtype == RSSM_FP8E4M3) {
        scale = (float *)h.at(h.lay.rc_scale_off);
        snap_scale = (const float *)(snap + (int64_t)cf.max_draft * elems);
    }
    commit_eager_kernel<<<cf.batch * cf.nheads, kThreads, 0, st>>>(
        h.counters(), accept, cf.nheads, cf.headdim * cf.dstate * eb, cf.headdim, state, snap,
        elems * eb, scale, snap_scale, scale_elems);
    return cudaGetLastError();
}

cudaError_t launch_import(const Ctx &h, const float *S, cudaStream_t st) {
    const rssm_config &cf = h.cfg;
    const int64_t rows = (int64_t)cf.batch * cf.nheads * cf.headdim;
    const int64_t elems = rows * cf.dstate;
    cudaError_t e = cudaSuccess;
    if (h.lay.ckpt_bytes)
        e = cudaMemcpyAsync(h.at(h.lay.ckpt_off), S, elems * sizeof(float), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
    if (h.lay.rc_bytes) {
        const int grid = (int)((rows + kWarps - 1) / kWarps);
        if (cf.state_dtype == RSSM_BF16)
            quant_rows_kernel<SK_BF16><<<grid, kThreads, 0, st>>>(S, h.at(h.lay.rc_off), nullptr, rows, cf.dstate);
        else
            quant_rows_kernel<SK_FP8><<<grid, kThreads, 0, st>>>(
                S, h.at(h.lay.rc_off), (float *)h.at(h.lay.rc_scale_off), rows, cf.dstate);
        e = cudaGetLastError();
    }
    return e;
}

cudaError_t launch_export_eager(const Ctx &h, float *out, cudaStream_t st) {
    const rssm_config &cf = h.cfg;
    const int64_t rows = (int64_t)cf.batch * cf.nheads * cf.headdim;
    const int grid = (int)((rows + kWarps - 1) / kWarps);
    if (cf.state_dtype == RSSM_F32)
        dequant_rows_kernel<SK_F32><<<grid, kThreads, 0, st>>>(h.at(h.lay.ckpt_off), nullptr, out, rows, cf.dstate);
    else if (cf.state_dtype == RSSM_BF16)
        dequant_rows_kernel<SK_BF16><<<grid, kThreads, 0, st>>>(h.at(h.lay.rc_off), nullptr, out, rows, cf.dstate);
    else
        dequant_rows_kernel<SK_FP8><<<grid, kThreads, 0, st>>>(
            h.at(h.lay.rc_off), (const float *)h.at(h.lay.rc_scale_off), out, rows, cf.dstate);
    return cudaGetLastError();
}

}  // namespace rssm
