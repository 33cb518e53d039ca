// rssm_device.cuh -- device-side helpers shared by the Mamba-2 and Gated DeltaNet
// decode kernels (sm_100a).  No host code.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rssm {

constexpr int kThreads = 256;  // every kernel runs 8 warps per CTA
constexpr int kWarps = kThreads / 32;

enum Op : int { OP_DECODE = 0, OP_VERIFY = 1, OP_FLUSH = 2, OP_EXPORT = 3 };
enum StoreKind : int { SK_F32 = 0, SK_BF16 = 1, SK_FP8 = 2 };
enum DevErr : int { DEV_BAD_ACCEPT = 1, DEV_BAD_COUNTERS = 2 };

// Per-sequence bookkeeping, all in the workspace.
struct Counters {
    int64_t *seq_pos;
    int64_t *ckpt_pos;
    int32_t *pending;
    int32_t *flush_count;
    int32_t *arrive;  // per-sequence arrival count of the CTAs of one launch
    int32_t *err;     // {code, b, h, value}
};

// Elements of a state row held in one 16-byte chunk.
template <int SK> struct Chunk;
template <> struct Chunk<SK_F32> { static constexpr int EPC = 4; static constexpr int BYTES = 4; };
template <> struct Chunk<SK_BF16> { static constexpr int EPC = 8; static constexpr int BYTES = 2; };
template <> struct Chunk<SK_FP8> { static constexpr int EPC = 16; static constexpr int BYTES = 1; };

__device__ __forceinline__ void report(int32_t *err, int code, int b, int h, int value) {
    if (atomicCAS(err, 0, code) == 0) {
        err[1] = b;
        err[2] = h;
        err[3] = value;
    }
}

// Streaming 16-byte load that does not allocate in L1 (state tiles are read once).
__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

// Unpack one 16-byte chunk of a stored row to fp32.
template <int SK>
__device__ __forceinline__ void unpack(const uint4 &u, float *v);

template <>
__device__ __forceinline__ void unpack<SK_F32>(const uint4 &u, float *v) {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
}

template <>
__device__ __forceinline__ void unpack<SK_BF16>(const uint4 &u, float *v) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16_bits_to_float(w[i] & 0xFFFFu);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ float2 fp8x2_to_float2(uint32_t two_bytes) {
    __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two_bytes & 0xFFFFu), __NV_E4M3);
    __half2 h2 = *reinterpret_cast<__half2 *>(&hr);
    return __half22float2(h2);
}

template <>
__device__ __forceinline__ void unpack<SK_FP8>(const uint4 &u, float *v) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 lo = fp8x2_to_float2(w[i] & 0xFFFFu);
        float2 hi = fp8x2_to_float2(w[i] >> 16);
        v[4 * i + 0] = lo.x;
        v[4 * i + 1] = lo.y;
        v[4 * i + 2] = hi.x;
        v[4 * i + 3] = hi.y;
    }
}

// Four consecutive stored elements (an fp32-mapping quad) to fp32.
template <int SK>
__device__ __forceinline__ float4 load_quad(const void *base, int64_t elem);

template <>
__device__ __forceinline__ float4 load_quad<SK_F32>(const void *base, int64_t elem) {
    return __ldg(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + elem));
}
template <>
__device__ __forceinline__ float4 load_quad<SK_BF16>(const void *base, int64_t elem) {
    uint2 u = __ldg(reinterpret_cast<const uint2 *>(reinterpret_cast<const uint16_t *>(base) + elem));
    return make_float4(bf16_bits_to_float(u.x & 0xFFFFu), __uint_as_float(u.x & 0xFFFF0000u),
                       bf16_bits_to_float(u.y & 0xFFFFu), __uint_as_float(u.y & 0xFFFF0000u));
}
template <>
__device__ __forceinline__ float4 load_quad<SK_FP8>(const void *base, int64_t elem) {
    uint32_t u = __ldg(reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint8_t *>(base) + elem));
    float2 lo = fp8x2_to_float2(u & 0xFFFFu), hi = fp8x2_to_float2(u >> 16);
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// Quantise a quad and store it; returns the dequantised values the reads will see.
// For FP8 the caller supplies 1/scale and scale of the row.
template <int SK>
__device__ __forceinline__ float4 store_quad(void *base, int64_t elem, float4 s, float inv_scale,
                                             float scale);

template <>
__device__ __forceinline__ float4 store_quad<SK_F32>(void *base, int64_t elem, float4 s, float,
                                                     float) {
    *reinterpret_cast<float4 *>(reinterpret_cast<float *>(base) + elem) = s;
    return s;
}
template <>
__device__ __forceinline__ float4 store_quad<SK_BF16>(void *base, int64_t elem, float4 s, float,
                                                      float) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(s.z, s.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&lo);
    u.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(base) + elem) = u;
    return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
}
template <>
__device__ __forceinline__ float4 store_quad<SK_FP8>(void *base, int64_t elem, float4 s,
                                                     float inv_scale, float scale) {
    // code = e4m3(value / scale), round to nearest even, saturating at +-448
    __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(s.x, scale), __fdiv_rn(s.y, scale)), __NV_SATFINITE, __NV_E4M3);
    __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(s.z, scale), __fdiv_rn(s.w, scale)), __NV_SATFINITE, __NV_E4M3);
    (void)inv_scale;
    uint32_t u = (uint32_t)lo | ((uint32_t)hi << 16);
    *reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(base) + elem) = u;
    float2 a = fp8x2_to_float2(lo), b = fp8x2_to_float2(hi);
    return make_float4(a.x * scale, a.y * scale, b.x * scale, b.y * scale);
}

// Sum over aligned groups of G consecutive lanes (G a power of two <= 32); every
// lane of the warp must call it.
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
template <int G>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Sums of four row values over the Q lanes of a row group (Q >= 4, a power of
// two), exchanging halves first: 2 + 1 + log2(Q/4) shuffles instead of
// 4 log2(Q).  Lane q of the group returns the sum of row 2*(q >= Q/2) + ((q & Q/4) != 0).
// Every lane of the warp must call it.
template <int Q>
__device__ __forceinline__ float quad_rows_sum(float d0, float d1, float d2, float d3, int q) {
    const bool hi = (q & (Q / 2)) != 0, hi2 = (q & (Q / 4)) != 0;
    const float s0 = __shfl_xor_sync(0xffffffffu, hi ? d0 : d2, Q / 2);
    const float s1 = __shfl_xor_sync(0xffffffffu, hi ? d1 : d3, Q / 2);
    const float e0 = (hi ? d2 : d0) + s0, e1 = (hi ? d3 : d1) + s1;
    float f = (hi2 ? e1 : e0) + __shfl_xor_sync(0xffffffffu, hi2 ? e0 : e1, Q / 4);
#pragma unroll
    for (int o = Q / 8; o > 0; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
    return f;
}

__device__ __forceinline__ float ld_in(const void *p, int64_t i, int bf16) {
    return bf16 ? bf16_bits_to_float(reinterpret_cast<const uint16_t *>(p)[i])
                : reinterpret_cast<const float *>(p)[i];
}
__device__ __forceinline__ void copy_in(void *dst, int64_t di, const void *src, int64_t si,
                                        int bf16) {
    if (bf16)
        reinterpret_cast<uint16_t *>(dst)[di] = reinterpret_cast<const uint16_t *>(src)[si];
    else
        reinterpret_cast<float *>(dst)[di] = reinterpret_cast<const float *>(src)[si];
}

// FP8 row scale from the row's absolute maximum: amax / 448, or 1 for a zero row.
__device__ __forceinline__ float fp8_scale(float amax) {
    return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
}

// Read the counters of sequence b (thread 0 of a CTA), register this CTA's
// arrival, and let the last CTA of the sequence publish the new counters.
// Every CTA of the sequence reads before it arrives, so the last arriver's
// writes can no longer be seen by a reader of this launch.
struct SeqState {
    int64_t seq, ckpt;
    int ok;
};

__device__ __forceinline__ SeqState read_counters(const Counters &c, int b, int W) {
    SeqState s;
    s.seq = c.seq_pos[b];
    s.ckpt = c.ckpt_pos[b];
    const int64_t L = s.seq - s.ckpt;
    s.ok = (s.ckpt >= 0 && L >= 0 && L <= W) ? 1 : 0;
    return s;
}

// new_seq / new_ckpt < 0 leave the value unchanged; new_pending < 0 likewise.
__device__ __forceinline__ void arrive_and_publish(const Counters &c, int b, int ctas_per_seq,
                                                   int64_t new_seq, int64_t new_ckpt,
                                                   int new_pending, int flush_inc) {
    __threadfence();
    if (atomicAdd(&c.arrive[b], 1) == ctas_per_seq - 1) {
        c.arrive[b] = 0;
        if (new_seq >= 0) c.seq_pos[b] = new_seq;
        if (new_ckpt >= 0) c.ckpt_pos[b] = new_ckpt;
        if (new_pending >= 0) c.pending[b] = new_pending;
        if (flush_inc) c.flush_count[b] += flush_inc;
        __threadfence();
    }
}

}  // namespace rssm

namespace rssm {

// 16-byte global -> shared copy that bypasses registers (Ampere-style cp.async;
// completion is awaited with cp_async_wait_all + __syncthreads).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
// 4-byte global -> shared copy (cache-all variant; the 16-byte form is cache-global only).
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}
// Programmatic dependent launch.  A kernel that triggers lets the next kernel of
// its stream, when that one is launched with programmatic stream serialization,
// be scheduled once every CTA of this grid has triggered or exited; the next
// kernel's wait returns when this grid has completed and its writes are visible.
// Without such a launch both are no-ops.
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Close the copies issued so far into a group (an empty group is allowed), and
// wait until at most `Pending` of the most recent groups are still in flight.
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int Pending>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(Pending) : "memory");
}

// Element i of a raw input-dtype buffer (shared or global) as fp32.
__device__ __forceinline__ float raw_f(const void *p, int i, int bf16) {
    return bf16 ? bf16_bits_to_float(reinterpret_cast<const uint16_t *>(p)[i])
                : reinterpret_cast<const float *>(p)[i];
}

// Inclusive prefix sum over the warp of one value per lane.
__device__ __forceinline__ float warp_incl_scan(float v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

}  // namespace rssm
