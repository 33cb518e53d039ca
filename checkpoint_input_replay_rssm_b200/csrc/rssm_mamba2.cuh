// rssm_mamba2.cuh -- Mamba-2 decode kernels for sm_100a (templates; instantiated per dstate).
//
// Layer (per sequence b, head h, group g = h / (H/G)):
//   S_t = exp(dt_t A_h) S_{t-1} + (s_t x_t) B_t^T,   y_t = S_t C_t + D_h x_t
// Replay representation (ReplaySSM: the output comes from a checkpoint plus a
// buffer of recent inputs with no state write; the checkpoint is rewritten only
// when the buffer is full -- blog.thibaultmonteiro.fr, "Tenir le journal plutot
// que le solde").  With buffered entries 1..L (L counts the token being read)
// and prefix sums Lam_m = sum_{j<=m} dt_j A_h of the log decays:
//   y = e^{Lam_L} (S^ C) + sum_i e^{Lam_L - Lam_i} (B_i . C) s_i x_i + D x_L
//   fold: S_c <- e^{Lam_L} S_c + sum_i e^{Lam_L - Lam_i} s_i x_i B_i^T
// S^ is the read copy (bf16, per-row-scaled e4m3, or the fp32 checkpoint).
//
// One CTA per (b, h).  The replay kernel issues its read-copy loads (128-bit,
// L1 no-allocate) before anything else, reads the sequence counters, stages the
// buffered inputs in shared memory, and then either
//   * reads: dot products of every state row with C (and the K draft C's),
//     reduced with warp shuffles, or
//   * folds (the buffer is full): loads the fp32 checkpoint, applies the rank-L
//     update, stores fp32 + requantised copy, and reads the outputs from the
//     fresh copy -- so a flush never needs a second pass over the state.
// Then it writes y, appends the new tokens to the ring, and the last CTA of the
// sequence publishes the counters.
#pragma once
#include "rssm_device.cuh"
#include "rssm_internal.h"

namespace rssm {

struct M2Args {
    int B, H, P, G, W, R, T, op, in_bf16, dt_scales;
    Counters c;
    const float *A, *D;
    float *ckpt;        // fp32 [B][H][P][N]
    void *rc;           // read copy / low-precision state [B][H][P][N]
    float *rc_scale;    // [B][H][P] (FP8)
    void *xbuf;         // [B][H][R][P]
    float *dtbuf;       // [B][H][R]
    void *Bbuf;         // [B][G][R][N]
    void *snap;         // eager verify snapshots
    float *snap_scale;
    const void *x;      // [B][T][H][P]
    const float *dt;    // [B][T][H]
    const void *Bm;     // [B][T][G][N]
    const void *Cm;     // [B][T][G][N]
    const int32_t *accept;  // [B] (commit)
    float *y;           // [B][T][H][P]
    float *out;         // export target [B][H][P][N]
};

// Shared-memory carve-up for one CTA (floats unless noted).
struct M2Smem {
    float *sx, *sB, *sC, *sdot, *slam, *sdt, *su, *scoef, *sdec;
    int *si;
};

// Regions are padded to multiples of 4 floats so every one is 16-byte aligned.
__host__ __device__ constexpr int pad4(int n) { return (n + 3) & ~3; }

__host__ __device__ inline size_t m2_smem_floats(int P, int N, int W, int TQ) {
    const int E = W + TQ;
    return (size_t)pad4(E * P) + pad4(E * N) + pad4(TQ * N) + pad4(TQ * P) + 3 * (size_t)pad4(E) +
           pad4(TQ * E) + pad4(TQ) + 8;
}

__device__ __forceinline__ M2Smem m2_carve(float *sm, int P, int N, int W, int TQ) {
    const int E = W + TQ;
    M2Smem s;
    s.sx = sm;                           // [E][P]    x of entries (physical index)
    s.sB = s.sx + pad4(E * P);           // [E][N]    B of entries
    s.sC = s.sB + pad4(E * N);           // [TQ][N]   C of the query tokens
    s.sdot = s.sC + pad4(TQ * N);        // [TQ][P]   S^ C per row
    s.slam = s.sdot + pad4(TQ * P);      // [E]       prefix sums of log decay
    s.sdt = s.slam + pad4(E);            // [E]       dt of entries
    s.su = s.sdt + pad4(E);              // [E]       fold weights
    s.scoef = s.su + pad4(E);            // [TQ][E]   replay coefficients (logical entry index)
    s.sdec = s.scoef + pad4(TQ * E);     // [TQ]      decay applied to S^ C
    s.si = reinterpret_cast<int *>(s.sdec + pad4(TQ));
    return s;
}

// ---------------------------------------------------------------------------
// Replay kernel: decode (T = 1), verify (T = K), flush (T = 0), export (T = 0).
// ---------------------------------------------------------------------------
template <int N, int RK, int TQ>
__global__ void __launch_bounds__(kThreads) m2_replay_kernel(const M2Args a) {
    constexpr int EPC = Chunk<RK>::EPC;    // stored elements per 16-byte chunk
    constexpr int TPR = N / EPC;           // threads per row, read mapping
    constexpr int RPP = kThreads / TPR;    // rows per pass, read mapping
    constexpr int RB = 8;                  // rows per thread per batch
    constexpr int TPR4 = N / 4;            // threads per row, fp32 (quad) mapping
    constexpr int RPP4 = kThreads / TPR4;
    static_assert(TPR >= 1 && TPR <= 32 && (32 % TPR) == 0, "row must fit a warp");
    static_assert(TPR4 >= 1 && TPR4 <= 32, "row must fit a warp");

    extern __shared__ __align__(16) float smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.x;
    const int H = a.H, P = a.P, W = a.W, R = a.R, T = a.T, G = a.G;
    const int b = bh / H, h = bh - b * H;
    const int hpg = H / G, g = h / hpg;
    const int E = W + TQ;
    M2Smem s = m2_carve(smem, P, N, W, TQ);
    const int64_t tile0 = (int64_t)bh * P * N;
    const bool reads = (a.op == OP_DECODE || a.op == OP_VERIFY);

    // 1. Read-copy loads first: they do not depend on the counters, and on the
    //    steps that fold they are simply dropped.
    const int c = tid % TPR, r0 = tid / TPR;
    const uint8_t *rc_tile =
        (RK == SK_F32) ? reinterpret_cast<const uint8_t *>(a.ckpt + tile0)
                       : reinterpret_cast<const uint8_t *>(a.rc) + tile0 * Chunk<RK>::BYTES;
    uint4 rv[RB];
    float rscale[RB];
    if (reads) {
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k * RPP;
            if (r < P) rv[k] = ld_stream(rc_tile + ((size_t)r * TPR + c) * 16);
            if (RK == SK_FP8) rscale[k] = (r < P) ? __ldg(a.rc_scale + (int64_t)bh * P + r) : 0.f;
        }
    }

    // 2. Counters (thread 0), and the new tokens' inputs (independent of them).
    if (tid == 0) {
        SeqState ss = read_counters(a.c, b, W);
        const int L0 = (int)(ss.seq - ss.ckpt);
        int flush = 0;
        if (ss.ok) flush = (a.op == OP_FLUSH || a.op == OP_EXPORT) ? (L0 > 0) : (L0 + T > W);
        s.si[0] = ss.ok;
        s.si[1] = ss.ok ? L0 : 0;
        s.si[2] = flush;
        s.si[3] = (int)(ss.ckpt % R);
        s.si[4] = (int)(ss.seq % R);
        if (!ss.ok) {
            if (h == 0) report(a.c.err, DEV_BAD_COUNTERS, b, h, (int)(ss.seq - ss.ckpt));
        } else if (a.op != OP_EXPORT) {
            const int64_t new_seq = (a.op == OP_DECODE) ? ss.seq + 1 : -1;
            const int64_t new_ckpt = flush ? ss.seq : -1;
            const int new_pending = (a.op == OP_VERIFY) ? T : -1;
            arrive_and_publish(a.c, b, H, new_seq, new_ckpt, new_pending, flush);
        }
    }
    for (int i = tid; i < T * P; i += kThreads) {
        const int m = i / P, p = i - m * P;
        s.sx[(W + m) * P + p] = ld_in(a.x, ((int64_t)(b * T + m) * H + h) * P + p, a.in_bf16);
    }
    for (int i = tid; i < T * N; i += kThreads) {
        const int m = i / N, n = i - m * N;
        const int64_t src = ((int64_t)(b * T + m) * G + g) * N + n;
        s.sB[(W + m) * N + n] = ld_in(a.Bm, src, a.in_bf16);
        s.sC[m * N + n] = ld_in(a.Cm, src, a.in_bf16);
    }
    if (tid < T) s.sdt[W + tid] = a.dt[(int64_t)(b * T + tid) * H + h];
    __syncthreads();
    if (!s.si[0]) return;  // counters corrupted: error reported, sequence skipped
    const int L0 = s.si[1], flush = s.si[2], ckmod = s.si[3], spmod = s.si[4];
    const int base = W - L0;  // buffered entries sit right-aligned before the new tokens
    const int nE = L0 + T;

    // 3. Buffered entries (logical 0..L0-1 -> physical base..W-1).
    for (int i = tid; i < L0 * P; i += kThreads) {
        const int e = i / P, p = i - e * P;
        const int slot = (ckmod + e) % R;
        s.sx[(base + e) * P + p] = ld_in(a.xbuf, ((int64_t)bh * R + slot) * P + p, a.in_bf16);
    }
    for (int i = tid; i < L0 * N; i += kThreads) {
        const int e = i / N, n = i - e * N;
        const int slot = (ckmod + e) % R;
        s.sB[(base + e) * N + n] = ld_in(a.Bbuf, ((int64_t)(b * G + g) * R + slot) * N + n, a.in_bf16);
    }
    for (int e = tid; e < L0; e += kThreads) s.sdt[base + e] = a.dtbuf[(int64_t)bh * R + (ckmod + e) % R];
    __syncthreads();

    // 4. Prefix sums of the log decays, fold weights, replay coefficients.
    const float Ah = a.A[h];
    if (tid == 0) {
        float acc = 0.f;
        for (int e = 0; e < nE; ++e) {
            acc += s.sdt[base + e] * Ah;
            s.slam[base + e] = acc;
        }
    }
    __syncthreads();
    const int e0 = flush ? L0 : 0;  // first entry the outputs replay
    const float lam_fold = (L0 > 0) ? s.slam[base + L0 - 1] : 0.f;
    const float lam_base = flush ? lam_fold : 0.f;
    if (flush) {
        for (int e = tid; e < L0; e += kThreads)
            s.su[e] = expf(lam_fold - s.slam[base + e]) * (a.dt_scales ? s.sdt[base + e] : 1.f);
    }
    if (reads) {
        const int npairs = T * nE;
        for (int pr = warp; pr < npairs; pr += kWarps) {
            const int m = pr / nE, e = pr - m * nE;
            if (e < e0 || e > L0 + m) continue;  // warp-uniform
            float d = 0.f;
            for (int n = lane; n < N; n += 32) d += s.sB[(base + e) * N + n] * s.sC[m * N + n];
            d = group_sum<32>(d);
            if (lane == 0)
                s.scoef[m * E + e] = expf(s.slam[base + L0 + m] - s.slam[base + e]) * d *
                                     (a.dt_scales ? s.sdt[base + e] : 1.f);
        }
        if (tid < T) s.sdec[tid] = expf(s.slam[base + L0 + tid] - lam_base);
    }
    __syncthreads();

    if (flush) {
        // 5a. Fold: fp32 checkpoint rows in quads, TPR4 lanes per row.
        const int c4 = tid % TPR4, q0 = tid / TPR4;
        const float dec_all = expf(lam_fold);
        float4 Cq[TQ];
#pragma unroll
        for (int m = 0; m < TQ; ++m)
            Cq[m] = (reads && m < T) ? reinterpret_cast<const float4 *>(s.sC + m * N)[c4]
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int rb = 0; rb < P; rb += RB * RPP4) {
            float4 st[RB];
#pragma unroll
            for (int k = 0; k < RB; ++k) {
                const int r = rb + q0 + k * RPP4;
                st[k] = (r < P) ? load_quad<SK_F32>(a.ckpt, tile0 + (int64_t)r * N + 4 * c4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < RB; ++k) {
                const int r = rb + q0 + k * RPP4;
                const bool valid = r < P;
                float4 v = st[k];
                v.x *= dec_all; v.y *= dec_all; v.z *= dec_all; v.w *= dec_all;
                if (valid) {
                    for (int e = 0; e < L0; ++e) {
                        const float w = s.su[e] * s.sx[(base + e) * P + r];
                        const float4 Bq = reinterpret_cast<const float4 *>(s.sB + (base + e) * N)[c4];
                        v.x = fmaf(w, Bq.x, v.x); v.y = fmaf(w, Bq.y, v.y);
                        v.z = fmaf(w, Bq.z, v.z); v.w = fmaf(w, Bq.w, v.w);
                    }
                }
                const int64_t el = tile0 + (int64_t)(valid ? r : 0) * N + 4 * c4;
                if (a.op == OP_EXPORT) {
                    if (valid) *reinterpret_cast<float4 *>(a.out + el) = v;
                    continue;
                }
                if (valid) *reinterpret_cast<float4 *>(a.ckpt + el) = v;
                float4 rd = v;  // what the outputs read: the fresh read copy
                if (RK == SK_BF16) {
                    if (valid) rd = store_quad<SK_BF16>(a.rc, el, v, 0.f, 0.f);
                } else if (RK == SK_FP8) {
                    float am = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
                    am = group_max<TPR4>(am);
                    const float sc = fp8_scale(am);
                    if (valid) {
                        rd = store_quad<SK_FP8>(a.rc, el, v, 0.f, sc);
                        if (c4 == 0) a.rc_scale[(int64_t)bh * P + r] = sc;
                    }
                }
                if (reads) {
#pragma unroll
                    for (int m = 0; m < TQ; ++m) {
                        float d = rd.x * Cq[m].x + rd.y * Cq[m].y + rd.z * Cq[m].z + rd.w * Cq[m].w;
                        d = group_sum<TPR4>(d);
                        if (c4 == 0 && valid && m < T) s.sdot[m * P + r] = d;
                    }
                }
            }
        }
    } else if (reads) {
        // 5b. Read: dot products of the read-copy rows with the query C's.
        float Cr[TQ][EPC];
#pragma unroll
        for (int m = 0; m < TQ; ++m)
#pragma unroll
            for (int j = 0; j < EPC; ++j) Cr[m][j] = (m < T) ? s.sC[m * N + c * EPC + j] : 0.f;
        for (int rb = 0; rb < P; rb += RB * RPP) {
            if (rb > 0) {
#pragma unroll
                for (int k = 0; k < RB; ++k) {
                    const int r = rb + r0 + k * RPP;
                    if (r < P) rv[k] = ld_stream(rc_tile + ((size_t)r * TPR + c) * 16);
                    if (RK == SK_FP8) rscale[k] = (r < P) ? __ldg(a.rc_scale + (int64_t)bh * P + r) : 0.f;
                }
            }
#pragma unroll
            for (int k = 0; k < RB; ++k) {
                const int r = rb + r0 + k * RPP;
                float v[EPC];
                if (r < P) unpack<RK>(rv[k], v);
                else {
#pragma unroll
                    for (int j = 0; j < EPC; ++j) v[j] = 0.f;
                }
#pragma unroll
                for (int m = 0; m < TQ; ++m) {
                    float d = 0.f;
#pragma unroll
                    for (int j = 0; j < EPC; ++j) d = fmaf(v[j], Cr[m][j], d);
                    d = group_sum<TPR>(d);
                    if (RK == SK_FP8) d *= rscale[k];
                    if (c == 0 && r < P && m < T) s.sdot[m * P + r] = d;
                }
            }
        }
    }
    if (!reads) return;
    __syncthreads();

    // 6. Outputs y[b, m, h, :].
    const float Dh = a.D[h];
    for (int i = tid; i < T * P; i += kThreads) {
        const int m = i / P, p = i - m * P;
        float yv = s.sdec[m] * s.sdot[m * P + p];
        for (int e = e0; e <= L0 + m; ++e) yv = fmaf(s.scoef[m * E + e], s.sx[(base + e) * P + p], yv);
        yv = fmaf(Dh, s.sx[(W + m) * P + p], yv);
        a.y[((int64_t)(b * T + m) * H + h) * P + p] = yv;
    }

    // 7. Append the new tokens to the ring (slots seq_pos + m mod R).
    for (int i = tid; i < T * P; i += kThreads) {
        const int m = i / P, p = i - m * P;
        const int slot = (spmod + m) % R;
        copy_in(a.xbuf, ((int64_t)bh * R + slot) * P + p, a.x, ((int64_t)(b * T + m) * H + h) * P + p,
                a.in_bf16);
    }
    if (tid < T) a.dtbuf[(int64_t)bh * R + (spmod + tid) % R] = s.sdt[W + tid];
    if (h % hpg == 0) {  // one head per group writes the group's B
        for (int i = tid; i < T * N; i += kThreads) {
            const int m = i / N, n = i - m * N;
            const int slot = (spmod + m) % R;
            copy_in(a.Bbuf, ((int64_t)(b * G + g) * R + slot) * N + n, a.Bm,
                    ((int64_t)(b * T + m) * G + g) * N + n, a.in_bf16);
        }
    }
}

// ---------------------------------------------------------------------------
// Eager read-modify-write baseline: decode (T = 1, state rewritten) and verify
// (T = K drafts applied in registers, K snapshots written, state untouched).
// The per-token state rewrite is the baseline the ReplaySSM reports start from
// (blog.thibaultmonteiro.fr, "La fiche qu'on reecrit a chaque token").
// ---------------------------------------------------------------------------
template <int N, int SK, int TQ>
__global__ void __launch_bounds__(kThreads) m2_eager_kernel(const M2Args a) {
    constexpr int TPR4 = N / 4;
    constexpr int RPP4 = kThreads / TPR4;
    constexpr int RB = 8;
    extern __shared__ __align__(16) float smem[];
    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int H = a.H, P = a.P, T = a.T, G = a.G;
    const int b = bh / H, h = bh - b * H;
    const int g = h / (H / G);
    float *sx = smem;                   // [TQ][P]
    float *sB = sx + pad4(TQ * P);      // [TQ][N]
    float *sC = sB + pad4(TQ * N);      // [TQ][N]
    float *sdot = sC + pad4(TQ * N);    // [TQ][P]
    float *sa = sdot + pad4(TQ * P);    // [TQ] decay
    float *ss = sa + pad4(TQ);          // [TQ] input scale
    const int64_t tile0 = (int64_t)bh * P * N;
    void *state = (SK == SK_F32) ? (void *)a.ckpt : a.rc;
    const int64_t state_elems = (int64_t)a.B * H * P * N;

    if (tid == 0) {
        SeqState st = read_counters(a.c, b, a.W);
        if (a.op == OP_DECODE)
            arrive_and_publish(a.c, b, H, st.seq + 1, st.seq + 1, -1, 0);
        else
            arrive_and_publish(a.c, b, H, -1, -1, T, 0);
    }
    for (int i = tid; i < T * P; i += kThreads) {
        const int m = i / P, p = i - m * P;
        sx[m * P + p] = ld_in(a.x, ((int64_t)(b * T + m) * H + h) * P + p, a.in_bf16);
    }
    for (int i = tid; i < T * N; i += kThreads) {
        const int m = i / N, n = i - m * N;
        const int64_t src = ((int64_t)(b * T + m) * G + g) * N + n;
        sB[m * N + n] = ld_in(a.Bm, src, a.in_bf16);
        sC[m * N + n] = ld_in(a.Cm, src, a.in_bf16);
    }
    if (tid < T) {
        const float dtv = a.dt[(int64_t)(b * T + tid) * H + h];
        sa[tid] = expf(dtv * a.A[h]);
        ss[tid] = a.dt_scales ? dtv : 1.f;
    }
    __syncthreads();

    const int c4 = tid % TPR4, q0 = tid / TPR4;
    for (int rb = 0; rb < P; rb += RB * RPP4) {
        float4 st[RB];
        float scl[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = rb + q0 + k * RPP4;
            st[k] = (r < P) ? load_quad<SK>(state, tile0 + (int64_t)r * N + 4 * c4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            scl[k] = (SK == SK_FP8 && r < P) ? __ldg(a.rc_scale + (int64_t)bh * P + r) : 1.f;
        }
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = rb + q0 + k * RPP4;
            const bool valid = r < P;
            const int64_t el = tile0 + (int64_t)(valid ? r : 0) * N + 4 * c4;
            float4 v = st[k];
            if (SK == SK_FP8) { v.x *= scl[k]; v.y *= scl[k]; v.z *= scl[k]; v.w *= scl[k]; }
            for (int m = 0; m < T; ++m) {
                const float w = ss[m] * (valid ? sx[m * P + r] : 0.f);
                const float4 Bq = reinterpret_cast<const float4 *>(sB + m * N)[c4];
                const float am = sa[m];
                v.x = fmaf(am, v.x, w * Bq.x); v.y = fmaf(am, v.y, w * Bq.y);
                v.z = fmaf(am, v.z, w * Bq.z); v.w = fmaf(am, v.w, w * Bq.w);
                const float4 Cq = reinterpret_cast<const float4 *>(sC + m * N)[c4];
                float d = v.x * Cq.x + v.y * Cq.y + v.z * Cq.z + v.w * Cq.w;
                d = group_sum<TPR4>(d);
                if (c4 == 0 && valid) sdot[m * P + r] = d;  // output from the fp32 value
                if (a.op == OP_VERIFY) {  // snapshot after draft m, in the state's storage type
                    void *snap = (SK == SK_F32)
                        ? (void *)(reinterpret_cast<float *>(a.snap) + m * state_elems)
                        : (void *)(reinterpret_cast<uint8_t *>(a.snap) + m * state_elems * Chunk<SK>::BYTES);
                    float sc = 1.f;
                    if (SK == SK_FP8) {
                        float amx = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
                        sc = fp8_scale(group_max<TPR4>(amx));
                        if (valid && c4 == 0) a.snap_scale[(int64_t)m * a.B * H * P + (int64_t)bh * P + r] = sc;
                    }
                    if (valid) store_quad<SK>(snap, el, v, 0.f, sc);
                }
            }
            if (a.op == OP_DECODE) {
                float sc = 1.f;
                if (SK == SK_FP8) {
                    float amx = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
                    sc = fp8_scale(group_max<TPR4>(amx));
                    if (valid && c4 == 0) a.rc_scale[(int64_t)bh * P + r] = sc;
                }
                if (valid) store_quad<SK>(state, el, v, 0.f, sc);
            }
        }
    }
    __syncthreads();
    const float Dh = a.D[h];
    for (int i = tid; i < T * P; i += kThreads) {
        const int m = i / P, p = i - m * P;
        a.y[((int64_t)(b * T + m) * H + h) * P + p] = sdot[m * P + p] + Dh * sx[m * P + p];
    }
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
template <int N, int RK, int TQ>
inline cudaError_t launch_replay_t(const M2Args &a, size_t smem, cudaStream_t st) {
    auto k = m2_replay_kernel<N, RK, TQ>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<a.B * a.H, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}
template <int N, int SK, int TQ>
inline cudaError_t launch_eager_t(const M2Args &a, size_t smem, cudaStream_t st) {
    auto k = m2_eager_kernel<N, SK, TQ>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<a.B * a.H, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int N, int TQ>
inline cudaError_t dispatch_rk(bool eager, int rk, const M2Args &a, size_t smem, cudaStream_t st) {
    switch (rk) {
        case SK_F32: return eager ? launch_eager_t<N, SK_F32, TQ>(a, smem, st) : launch_replay_t<N, SK_F32, TQ>(a, smem, st);
        case SK_BF16: return eager ? launch_eager_t<N, SK_BF16, TQ>(a, smem, st) : launch_replay_t<N, SK_BF16, TQ>(a, smem, st);
        default: return eager ? launch_eager_t<N, SK_FP8, TQ>(a, smem, st) : launch_replay_t<N, SK_FP8, TQ>(a, smem, st);
    }
}
template <int N>
inline cudaError_t dispatch_tq(bool eager, int rk, int TQ, const M2Args &a, size_t smem, cudaStream_t st) {
    if (TQ == 1) return dispatch_rk<N, 1>(eager, rk, a, smem, st);
    if (TQ == 4) return dispatch_rk<N, 4>(eager, rk, a, smem, st);
    return dispatch_rk<N, 8>(eager, rk, a, smem, st);
}

// Per-dstate entry point; each instantiation lives in its own translation unit.
template <int N>
cudaError_t m2_dispatch_n(bool eager, int rk, int TQ, const M2Args &a, size_t smem, cudaStream_t st) {
    return dispatch_tq<N>(eager, rk, TQ, a, smem, st);
}

}  // namespace rssm
