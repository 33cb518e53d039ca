// rssm_prefill.cu -- chunked Mamba-2 prefill on the 5th-generation tensor cores:
// the outputs of a prompt and the fp32 state after it, the checkpoint a replay
// decode starts from (rssm_import_state).
//
// The prompt is cut into chunks of Q = 128 tokens.  With Lam_i the prefix sums
// of dt A_h over the chunk's tokens, s_j = dt_j (dt scales the input) or 1, and
// S the state at the chunk's start (headdim P x dstate N):
//   CB[i][j]  = C_i . B_j                                           (C B^T, group-shared)
//   M[i][j]   = e^{Lam_i - Lam_j} CB[i][j] s_j  for j <= i, else 0
//   y_i       = sum_j M[i][j] x_j + e^{Lam_i} (S C_i) + D x_i
//   S        <- e^{Lam_last} S + sum_j e^{Lam_last - Lam_j} s_j x_j B_j^T
// -- the checkpoint + buffered-inputs algebra of the replay read, with the chunk
// as the buffer (blog.thibaultmonteiro.fr, "Tenir le journal plutot que le
// solde").  The four products are dense contractions, so each is a tcgen05 MMA
// with bf16 operands and an fp32 accumulator in tensor memory:
//   MMA1  CB      = C [Q x N] . B [Q x N]^T                    (M = Q,  N = Q, K = N)
//   MMA3  Y_inter = C [Q x N] . S [P x N]^T                    (M = Q,  N = P, K = N)
//   MMA4  S^T    += B^T [N x Q] . (x w)^T [P x Q]^T             (M = N,  N = P, K = Q)
//   MMA2  Y_intra = M [Q x Q] . x^T [P x Q]^T                   (M = Q,  N = P, K = Q)
// x, B and C are bf16 and enter exactly; the fp32 operands (S, x w, M) enter as
// a (hi, lo) pair of bf16 matrices whose sum carries about 16 bits of mantissa,
// two MMAs each, so every product keeps near-fp32 accuracy.  The state stays
// in tensor memory, transposed (lane n, column p), across the chunks of a head.
//
// One CTA of 128 NG threads per (sequence, head): thread t owns tensor-memory
// lane t mod 128 (token i of the chunk, or state column n) and one of NG column
// groups of that row, so NG warps share each lane quarter (NG = 4 for headdim
// 64, 2 otherwise: a group's p columns stay a multiple of 16).  Per chunk:
// (A) the threads issue the chunk's global reads at once (C and B rows by
// cp.async into their swizzled rows, x into registers), then stage x and (x w),
// the state's (hi, lo) copy and, below headdim 64, B^T in shared memory -- at
// headdim 64 as MN-major tiles written 16 bytes at a time, otherwise transposed
// into K-major tiles -- and rescale the state by e^{Lam_last} in place; (B) one
// thread issues MMA1, MMA3 and MMA4; (C) the threads turn CB into M (hi, lo)
// (over B and B^T; at headdim 64 over B^T and (x w), while the next chunk's C
// and B rows land); (D) one thread issues MMA2; (E) the threads write y.  Waits
// on MMA completion are bounded (2 s) and report RSSM_DEV_PIPE_TIMEOUT.
#include <cuda_bf16.h>

#include "rssm_internal.h"
#include "rssm_umma.cuh"

namespace rssm {

namespace {

constexpr int kQ = 128;          // chunk length = MMA M
constexpr int kN = 128;          // dstate = MMA M of the state update
constexpr int kRows = 128;       // threads per column group: one tensor-memory lane (row) each
constexpr int kTileQN = kQ * kN * 2;  // one [128 x 128] bf16 tile
constexpr float kLog2e = 1.4426950408889634f;

struct PrefillArgs {
    int B, H, P, G, T, dt_scales;
    const __nv_bfloat16 *x;   // [B][T][H][P]
    const float *dt;          // [B][T][H]
    const __nv_bfloat16 *Bm;  // [B][T][G][N]
    const __nv_bfloat16 *Cm;  // [B][T][G][N]
    const float *A, *D;       // [H]
    const float *S0;          // [B][H][P][N] or nullptr (zero state)
    float *y;                 // [B][T][H][P]
    float *S_out;             // [B][H][P][N]
    int *err;                 // {code, b, h, value} or nullptr
};

// Shared memory (bytes from a 1024-aligned base).
struct PrefillLay {
    int C, Bk, Bt, Xt, XwHi, XwLo, SHi, SLo, lam, lam2, w, red, bar, tslot, bytes;
};
__host__ __device__ inline PrefillLay prefill_lay(int P) {
    PrefillLay L{};
    int o = 0;
    const int xp = P * kQ * 2;  // one [P x Q] bf16 tile
    const int sp = P * kN * 2;  // one [P x N] bf16 tile
    L.C = o;    o += kTileQN;   // C  [Q rows, K = N]
    L.Bk = o;   o += kTileQN;   // B  [Q rows, K = N]      (M hi afterwards)
    L.Bt = o;   o += kTileQN;   // B^T [N rows, K = Q]     (M lo afterwards)
    L.Xt = o;   o += xp;        // x^T [P rows, K = Q]
    L.XwHi = o; o += xp;        // (x w)^T hi
    L.XwLo = o; o += xp;        // (x w)^T lo
    L.SHi = o;  o += sp;        // S hi [P rows, K = N]
    L.SLo = o;  o += sp;        // S lo
    L.lam = o;  o += kQ * 4;    // Lam_i
    L.lam2 = o; o += kQ * 4;    // Lam_i log2(e)
    L.w = o;    o += kQ * 4;    // s_j (dt or 1)
    L.red = o;  o += 64;        // cross-warp scan carries
    L.bar = o;  o += 16;        // mbarrier
    L.tslot = o; o += 16;       // tensor-memory address
    L.bytes = o;
    return L;
}

__device__ __forceinline__ void report_err(int *err, int code, int b, int h, int v) {
    if (err && atomicCAS(err, 0, code) == 0) {
        err[1] = b;
        err[2] = h;
        err[3] = v;
    }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&t);
}

template <int P, int NG>
__global__ void __launch_bounds__(kRows * NG, 1) m2_prefill_kernel(const PrefillArgs a) {
    constexpr int PH = P / NG;  // p columns handled by each column group (a multiple of 16)
    static_assert(PH % 16 == 0, "a column group's p columns are loaded 16 at a time");
    // headdim 64: x, x w and the state copy are written as MN-major tiles (row = token
    // or state column, 128 bytes of p) and B is read MN-major by MMA4, so no operand
    // is transposed element by element; one MN block, so its stride is never used.
    constexpr bool kMN = (P == 64);
    constexpr uint32_t kMNBlock = 1024;
    extern __shared__ __align__(1024) uint8_t psm[];
    // the swizzled tiles need a 1024-byte aligned base
    uint8_t *sm = psm + ((1024 - (smem_u32(psm) & 1023)) & 1023);
    const PrefillLay Ly = prefill_lay(P);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = tid & (kQ - 1);  // tensor-memory lane: token i of the chunk, or state column n
    const int grp = tid >> 7;        // which column group this thread works on
    const int b = blockIdx.y, h = blockIdx.x;
    const int H = a.H, G = a.G, T = a.T;
    const int g = h / (H / G);
    uint8_t *sC = sm + Ly.C, *sBk = sm + Ly.Bk, *sBt = sm + Ly.Bt, *sXt = sm + Ly.Xt;
    uint8_t *sXwHi = sm + Ly.XwHi, *sXwLo = sm + Ly.XwLo, *sSHi = sm + Ly.SHi, *sSLo = sm + Ly.SLo;
    // M (hi, lo) for MMA2: over B and B^T; with headdim 64 (no B^T tile in use) over
    // B^T and the (x w) pair, so that C and B are free for the next chunk's rows.
    uint8_t *sMHi = kMN ? sBt : sBk, *sMLo = kMN ? sXwHi : sBt;
    float *slam = reinterpret_cast<float *>(sm + Ly.lam);
    float *slam2 = reinterpret_cast<float *>(sm + Ly.lam2);  // Lam log2(e): e^{Lam_i - Lam_j} = 2^{Lam2_i - Lam2_j}
    float *sw = reinterpret_cast<float *>(sm + Ly.w);
    float *sred = reinterpret_cast<float *>(sm + Ly.red);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + Ly.bar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + Ly.tslot);
    const uint32_t ncols = (128 + 2 * P) <= 256 ? 256u : 512u;
    // tensor-memory columns: CB (later Y_intra) at 0, Y_inter at 128, S^T at 128 + P
    const uint32_t cY1 = 0, cY2 = 128, cS = 128 + (uint32_t)P;

    if (warp == 0) tmem_alloc(tslot, ncols);
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init_fence();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // this warp's 32 lanes
    const float Ah = a.A[h], Dh = a.D[h];
    const int p_lo = grp * PH;  // this thread's p columns: [p_lo, p_lo + PH)
    const int64_t head = (int64_t)b * H + h;

    // The initial state, transposed into tensor memory: lane n holds S0[:, n].
    for (int j0 = 0; j0 < PH; j0 += 16) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = a.S0 ? a.S0[(head * P + p_lo + j0 + j) * kN + row] : 0.f;
        tmem_st16(lane_base + cS + p_lo + j0, v);
    }

    uint32_t phase = 0;
    bool failed = false;
    constexpr int CH = kN / 8 / NG;  // 16-byte row chunks per group
    // C and B rows of token `row` of chunk cc (this group's chunks), zeros past the prompt.
    auto stage_cb = [&](int cc) {
        const int tc0 = cc * kQ;
        const bool lv = row < min(kQ, T - tc0);
        const int64_t tk = (int64_t)b * T + tc0 + row;
        const uint8_t *Crow = reinterpret_cast<const uint8_t *>(a.Cm + (tk * G + g) * kN);
        const uint8_t *Brow = reinterpret_cast<const uint8_t *>(a.Bm + (tk * G + g) * kN);
#pragma unroll
        for (int k = 0; k < CH; ++k) {
            const int ch = grp * CH + k;
            if (lv) {
                cp_async16(sC + sw128_chunk(row, ch, kQ), Crow + 16 * ch);
                cp_async16(sBk + sw128_chunk(row, ch, kQ), Brow + 16 * ch);
            } else {
                *reinterpret_cast<uint4 *>(sC + sw128_chunk(row, ch, kQ)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sBk + sw128_chunk(row, ch, kQ)) = make_uint4(0, 0, 0, 0);
            }
        }
        cp_async_commit();
    };
    const int nchunks = (T + kQ - 1) / kQ;
    for (int c = 0; c < nchunks && !failed; ++c) {
        const int t0 = c * kQ, Lc = min(kQ, T - t0);
        const int i = row;  // token of the chunk owned by this thread
        const bool live = i < Lc;
        const int64_t tok = (int64_t)b * T + t0 + i;

        // (A) The chunk's global reads, all issued first: this group's 16-byte chunks
        //     of the C and B rows of token i by cp.async straight into their K-major
        //     rows (rows = tokens; with headdim 64 issued during the previous chunk),
        //     this group's part of x row i and dt_i into registers.
        if (!(kMN && c > 0)) stage_cb(c);
        uint4 xv[PH / 8];
        const uint4 *Xrow = reinterpret_cast<const uint4 *>(a.x + (tok * H + h) * P + p_lo);
#pragma unroll
        for (int k = 0; k < PH / 8; ++k) xv[k] = live ? Xrow[k] : make_uint4(0, 0, 0, 0);
        const float dti = live ? a.dt[tok * H + h] : 0.f;

        // Prefix sums of dt*A over the chunk (padding tokens add nothing); every
        // group scans, the first publishes.
        float v = dti * Ah;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        if (grp == 0 && lane == 31) sred[warp] = v;
        __syncthreads();
        float carry = 0.f;
        for (int w2 = 0; w2 < (warp & 3); ++w2) carry += sred[w2];
        const float lam = v + carry;
        if (grp == 0) {
            slam[i] = lam;
            slam2[i] = lam * kLog2e;
            sw[i] = live ? (a.dt_scales ? dti : 1.f) : 0.f;
        }
        __syncthreads();
        const float lam_last = slam[kQ - 1];

        // x and x w (w_i = e^{Lam_last - Lam_i} s_i, as (hi, lo)) for this group's p:
        // with headdim 64 as row i of MN-major tiles (one 16-byte chunk per 8 p),
        // otherwise as columns of the transposed K-major tiles.
        const float wi = live ? expf(lam_last - lam) * sw[i] : 0.f;
#pragma unroll
        for (int k = 0; k < PH / 8; ++k) {
            const __nv_bfloat16 *xe = reinterpret_cast<const __nv_bfloat16 *>(&xv[k]);
            if constexpr (kMN) {
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    __nv_bfloat16 h0, l0, h1, l1;
                    split_bf16(__bfloat162float(xe[2 * e2]) * wi, h0, l0);
                    split_bf16(__bfloat162float(xe[2 * e2 + 1]) * wi, h1, l1);
                    hw[e2] = pack2(__bfloat162float(h0), __bfloat162float(h1));
                    lw[e2] = pack2(__bfloat162float(l0), __bfloat162float(l1));
                }
                const uint32_t off = sw128_chunk(i, (p_lo >> 3) + k, kQ);
                *reinterpret_cast<uint4 *>(sXt + off) = xv[k];
                *reinterpret_cast<uint4 *>(sXwHi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(sXwLo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int p = p_lo + 8 * k + e;
                    *reinterpret_cast<__nv_bfloat16 *>(sXt + sw128_off(p, i, P)) = xe[e];
                    __nv_bfloat16 hi, lo;
                    split_bf16(__bfloat162float(xe[e]) * wi, hi, lo);
                    *reinterpret_cast<__nv_bfloat16 *>(sXwHi + sw128_off(p, i, P)) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(sXwLo + sw128_off(p, i, P)) = lo;
                }
            }
        }
        // The state at the chunk's start: (hi, lo) copy for MMA3 (S rows p, K = n;
        // with headdim 64 MN-major, row n holding this lane's p run), and
        // e^{Lam_last} S back into tensor memory for MMA4 to accumulate onto.
        const float dec = expf(lam_last);
        for (int j0 = 0; j0 < PH; j0 += 16) {
            float st[16];
            tmem_ld16(lane_base + cS + p_lo + j0, st);
            if constexpr (kMN) {
#pragma unroll
                for (int c8 = 0; c8 < 2; ++c8) {
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        __nv_bfloat16 h0, l0, h1, l1;
                        split_bf16(st[8 * c8 + 2 * e2], h0, l0);
                        split_bf16(st[8 * c8 + 2 * e2 + 1], h1, l1);
                        hw[e2] = pack2(__bfloat162float(h0), __bfloat162float(h1));
                        lw[e2] = pack2(__bfloat162float(l0), __bfloat162float(l1));
                    }
                    const uint32_t off = sw128_chunk(row, ((p_lo + j0) >> 3) + c8, kN);
                    *reinterpret_cast<uint4 *>(sSHi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4 *>(sSLo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) st[j] *= dec;
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    __nv_bfloat16 hi, lo;
                    split_bf16(st[j], hi, lo);
                    *reinterpret_cast<__nv_bfloat16 *>(sSHi + sw128_off(p_lo + j0 + j, row, P)) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(sSLo + sw128_off(p_lo + j0 + j, row, P)) = lo;
                    st[j] *= dec;
                }
            }
            tmem_st16(lane_base + cS + p_lo + j0, st);
        }
        cp_async_wait_all();
        // B^T columns from this thread's own B chunks once they have landed (with
        // headdim 64 MMA4 reads the B tile itself MN-major).
        if constexpr (!kMN) {
#pragma unroll
            for (int k = 0; k < CH; ++k) {
                const int ch = grp * CH + k;
                const uint4 bv = *reinterpret_cast<const uint4 *>(sBk + sw128_chunk(i, ch, kQ));
                const __nv_bfloat16 *be = reinterpret_cast<const __nv_bfloat16 *>(&bv);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    *reinterpret_cast<__nv_bfloat16 *>(sBt + sw128_off(8 * ch + e, i, kN)) = be[e];
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // (B) MMA1 (CB), MMA3 (Y_inter, hi and lo), MMA4 (state, hi and lo).
        if (tid == 0) {
            const uint32_t aC = smem_u32(sC), aB = smem_u32(sBk), aBt = smem_u32(sBt);
            for (int ks = 0; ks < kN / 16; ++ks)
                umma_bf16(tmem + cY1, sw128_desc(aC, kQ, ks), sw128_desc(aB, kQ, ks), idesc_bf16_f32(kQ, kQ), ks > 0);
            for (int hl = 0; hl < 2; ++hl) {
                const uint32_t aS = smem_u32(hl ? sSLo : sSHi);
                for (int ks = 0; ks < kN / 16; ++ks)
                    umma_bf16(tmem + cY2, sw128_desc(aC, kQ, ks),
                              kMN ? sw128_mn_desc(aS, kMNBlock, ks) : sw128_desc(aS, P, ks),
                              idesc_bf16_f32_mn(kQ, P, false, kMN), hl > 0 || ks > 0);
            }
            for (int hl = 0; hl < 2; ++hl) {
                const uint32_t aX = smem_u32(hl ? sXwLo : sXwHi);
                for (int ks = 0; ks < kQ / 16; ++ks)
                    umma_bf16(tmem + cS, kMN ? sw128_mn_desc(aB, kQ * 128, ks) : sw128_desc(aBt, kN, ks),
                              kMN ? sw128_mn_desc(aX, kMNBlock, ks) : sw128_desc(aX, P, ks),
                              idesc_bf16_f32_mn(kN, P, kMN, kMN), true);
            }
            umma_commit(bar);
        }
        __syncwarp();
        if (!mbar_wait(bar, phase & 1)) failed = true;
        ++phase;
        if (__syncthreads_or(failed)) {
            failed = true;
            break;
        }
        tc_fence_after();
        // The MMAs reading C and B have completed: with headdim 64 the next chunk's
        // rows go into them now and land while this chunk finishes.
        if constexpr (kMN) {
            if (c + 1 < nchunks) stage_cb(c + 1);
        }

        // (C) M = tril(e^{Lam_i - Lam_j}) (.) CB (.) s_j as (hi, lo): row i, this group's kQ / NG columns j.
        //     A warp holds rows 32 (w mod 4) .. + 31: a 32-column block wholly above their
        //     diagonal is zero and skips the exponentials (2^{Lam2_i - Lam2_j} elsewhere).
        const float lam2 = lam * kLog2e;
        const int warp_last_row = 32 * (warp & 3) + 31;
        for (int j0 = grp * (kQ / NG); j0 < (grp + 1) * (kQ / NG); j0 += 32) {
            if (j0 > warp_last_row) {  // warp-uniform
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const int chunk = (j0 >> 3) + ch;
                    *reinterpret_cast<uint4 *>(sMHi + sw128_chunk(i, chunk, kQ)) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(sMLo + sw128_chunk(i, chunk, kQ)) = make_uint4(0, 0, 0, 0);
                }
                continue;
            }
            float cb[32];
            tmem_ld32(lane_base + cY1 + j0, cb);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    float m2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int jj = 8 * ch + 2 * e2 + u, j = j0 + jj;
                        m2[u] = (j <= i) ? exp2f(lam2 - slam2[j]) * cb[jj] * sw[j] : 0.f;
                    }
                    __nv_bfloat16 h0, l0, h1, l1;
                    split_bf16(m2[0], h0, l0);
                    split_bf16(m2[1], h1, l1);
                    hw[e2] = pack2(__bfloat162float(h0), __bfloat162float(h1));
                    lw[e2] = pack2(__bfloat162float(l0), __bfloat162float(l1));
                }
                const int chunk = (j0 >> 3) + ch;
                *reinterpret_cast<uint4 *>(sMHi + sw128_chunk(i, chunk, kQ)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(sMLo + sw128_chunk(i, chunk, kQ)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // (D) MMA2: Y_intra = M x (hi and lo), over the CB columns.
        if (tid == 0) {
            const uint32_t aX = smem_u32(sXt);
            for (int hl = 0; hl < 2; ++hl) {
                const uint32_t aM = smem_u32(hl ? sMLo : sMHi);
                for (int ks = 0; ks < kQ / 16; ++ks)
                    umma_bf16(tmem + cY1, sw128_desc(aM, kQ, ks),
                              kMN ? sw128_mn_desc(aX, kMNBlock, ks) : sw128_desc(aX, P, ks),
                              idesc_bf16_f32_mn(kQ, P, false, kMN), hl > 0 || ks > 0);
            }
            umma_commit(bar);
        }
        __syncwarp();
        if (!mbar_wait(bar, phase & 1)) failed = true;
        ++phase;
        if (__syncthreads_or(failed)) {
            failed = true;
            break;
        }
        tc_fence_after();

        // (E) y_i = Y_intra + e^{Lam_i} Y_inter + D x_i over this group's p.
        const float di = expf(lam);
        for (int j0 = 0; j0 < PH; j0 += 16) {
            float y1[16], y2[16];
            tmem_ld16(lane_base + cY1 + p_lo + j0, y1);
            tmem_ld16(lane_base + cY2 + p_lo + j0, y2);
            if (live) {
                float4 *yr = reinterpret_cast<float4 *>(a.y + (tok * H + h) * P + p_lo + j0);
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4) {
                    float o[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = 4 * j4 + u;
                        const uint4 &xw = xv[(j0 + j) >> 3];
                        const __nv_bfloat16 *xe = reinterpret_cast<const __nv_bfloat16 *>(&xw);
                        o[u] = fmaf(di, y2[j], y1[j]) + Dh * __bfloat162float(xe[(j0 + j) & 7]);
                    }
                    yr[j4] = make_float4(o[0], o[1], o[2], o[3]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();  // shared memory and tensor-memory columns are reused by the next chunk
        tc_fence_after();
    }

    cp_async_wait_all();  // a chunk's rows still in flight after a failed wait
    if (failed) {
        if (tid == 0) report_err(a.err, DEV_PIPE_TIMEOUT, b, h, 0);
    } else {
        // The state after the prompt, S_out[b][h][p][n] from lane n.
        for (int j0 = 0; j0 < PH; j0 += 16) {
            float st[16];
            tmem_ld16(lane_base + cS + p_lo + j0, st);
#pragma unroll
            for (int j = 0; j < 16; ++j) a.S_out[(head * P + p_lo + j0 + j) * kN + row] = st[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace

size_t prefill_smem_bytes(int P) { return (size_t)prefill_lay(P).bytes + 1024; }

}  // namespace rssm

extern "C" RSSM_API rssm_status rssm_mamba2_prefill(const rssm_prefill_config *cfg, const float *A, const float *D,
                                                    const float *S0, const rssm_inputs *in, float *y, float *S_out,
                                                    int32_t *dev_error, void *stream) {
    using namespace rssm;
    if (!cfg || !A || !D || !in || !in->x || !in->dt || !in->Bm || !in->Cm || !y || !S_out)
        return RSSM_EINVAL;
    const rssm_prefill_config &c = *cfg;
    if (c.batch < 1 || c.nheads < 1 || c.ngroups < 1 || c.nheads % c.ngroups != 0 || c.T < 1) return RSSM_EINVAL;
    if (c.dstate != kN || c.headdim < 32 || c.headdim > 96 || c.headdim % 32 != 0) return RSSM_EINVAL;
    if (S0 && S0 == S_out) return RSSM_EINVAL;
    if (c.dt_scales_input != 0 && c.dt_scales_input != 1) return RSSM_EINVAL;
    auto al16 = [](const void *p) { return ((uintptr_t)p & 15) == 0; };
    if (!al16(in->x) || !al16(in->Bm) || !al16(in->Cm) || !al16(y)) return RSSM_EINVAL;
    PrefillArgs a{};
    a.B = c.batch; a.H = c.nheads; a.P = c.headdim; a.G = c.ngroups; a.T = c.T; a.dt_scales = c.dt_scales_input;
    a.x = (const __nv_bfloat16 *)in->x; a.dt = in->dt;
    a.Bm = (const __nv_bfloat16 *)in->Bm; a.Cm = (const __nv_bfloat16 *)in->Cm;
    a.A = A; a.D = D; a.S0 = S0; a.y = y; a.S_out = S_out; a.err = (int *)dev_error;
    const size_t smem = prefill_smem_bytes(c.headdim);
    const int ng = c.headdim == 64 ? 4 : 2;
    auto k = c.headdim == 32 ? m2_prefill_kernel<32, 2>
                             : (c.headdim == 64 ? m2_prefill_kernel<64, 4> : m2_prefill_kernel<96, 2>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return RSSM_ECUDA;
    k<<<dim3(c.nheads, c.batch), kRows * ng, smem, (cudaStream_t)stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? RSSM_OK : RSSM_ECUDA;
}
