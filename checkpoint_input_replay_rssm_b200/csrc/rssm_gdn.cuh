// rssm_gdn.cuh -- Gated DeltaNet decode kernels for sm_100a (templates; instantiated per dstate).
//
// Layer (per sequence b, head h; S is d_v x d_k, rows contiguous along d_k):
//   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t
// GDN's update is the Mamba-2 form plus a delta-rule correction
// (blog.thibaultmonteiro.fr, "La fiche qu'on reecrit a chaque token"), so the
// same checkpoint + input-buffer replay applies.  With M_j = alpha_j (I - beta_j k_j k_j^T)
// and buffered entries 1..L (L counts the query token):
//   o = S_c M_1 ... M_L q + sum_i beta_i v_i (k_i . M_{i+1} ... M_L q)
// Sweep r <- q; for j = L..1: c_j = beta_j (k_j . r), r <- alpha_j (r - c_j k_j);
// then o = S^ r + sum_j c_j v_j.  The kernel never forms r during the sweep: it
// tracks t_e = k_e . r for every earlier entry e, which obeys
//   t_e <- alpha_j (t_e - c_j (k_e . k_j)),
// so with the Gram matrix k_e . k_j computed up front (all warps, in parallel)
// the serial chain is one shuffle per entry, and
//   r = (prod_{l} alpha_l) q - sum_i (prod_{l<=i} alpha_l) c_i k_i
// is assembled afterwards in parallel.  The fold applies the per-token updates
// in order to each fp32 checkpoint row in registers:
//   s <- alpha s + (beta v[row] - alpha beta (s . k)) k.
#pragma once
#include "rssm_device.cuh"
#include "rssm_pair.cuh"
#include "rssm_internal.h"

namespace rssm {

struct GArgs {
    int B, H, P, W, R, Rs, T, op, in_bf16;  // Rs: row length of the scalar rings
    Counters c;
    float *ckpt;
    void *rc;
    float *rc_scale;
    void *kbuf, *vbuf;   // [B][H][R][N], [B][H][R][P] input dtype
    float *abuf, *bbuf;  // GDN [B][H][Rs] each; KDA alpha [B][H][R][N]
    void *snap;
    float *snap_scale;
    const void *q, *k, *v;      // [B][T][H][N|P]
    const float *alpha, *beta;  // [B][T][H]; KDA alpha [B][T][H][N]
    float *y;                   // [B][T][H][P]
    float *out;                 // export target
    // replay decode/verify: hand-off of the prep kernel to the read kernel
    int4 *seqinfo;              // [B] {L0 replayed, ring slot of entry 0, folded, valid}
    float *dec;                 // [B][H][TQmax] (1: the decays are inside the swept query)
    float *coef;                // [B][H][TQmax][Emax] sweep coefficients c_e
    float *query;               // [B][H][TQmax][N] swept queries r
    int TQmax, Emax;
    int fold_launched;          // the fold-only launch of gdn_replay_kernel follows in this call
    int fold_only;              // gdn_replay_kernel: only fold (and serve) sequences whose buffer is full
    int prep_heads;             // gdn_prep_kernel: heads (warps at work) per CTA, <= 8
    int kda;                    // Kimi Delta Attention: alpha is a gate per key channel
};

__host__ __device__ constexpr int gpad4(int n) { return (n + 3) & ~3; }

// KDA keeps a gate row [E][N] where GDN keeps one gate per entry.  After the
// working arrays, the raw rings (k, v in the input dtype, gates and beta fp32) as
// staged from global memory, ring slot order, R <= W + 8 slots.
__host__ __device__ inline size_t gdn_raw_floats(int P, int N, int W, int ib, int kda) {
    const int Rm = W + 8;
    return (size_t)gpad4(Rm * N * ib / 4) + gpad4(Rm * P * ib / 4) + gpad4(kda ? Rm * N : Rm) + gpad4(Rm);
}
__host__ __device__ inline size_t gdn_smem_floats(int P, int N, int W, int TQ, int kda, int ib) {
    const int E = W + TQ;
    return (size_t)gpad4(E * N) + gpad4(E * P) + gpad4(kda ? E * N : E) + 2 * (size_t)gpad4(E) + gpad4(TQ * N) +
           gpad4(E * E) + 2 * (size_t)gpad4(TQ * E) + gpad4(TQ * N) + gpad4(TQ * P) + gpad4(TQ) + 8 +
           gdn_raw_floats(P, N, W, ib, kda);
}

struct GSmem {
    float *sk, *sv, *sal, *sbe, *spr, *sq, *sG, *shq, *sc, *sr, *sdot, *srq;
    int *si;
    uint8_t *rk, *rv;  // raw k, v rings [R][N], [R][P] (input dtype)
    float *ra, *rb;    // raw gate ring ([Rs], KDA [R][N]) and beta ring [Rs]
};

__device__ __forceinline__ GSmem gdn_carve(float *sm, int P, int N, int W, int TQ, int kda, int ib) {
    const int E = W + TQ;
    GSmem s;
    s.sk = sm;                            // [E][N]  k of entries (physical)
    s.sv = s.sk + gpad4(E * N);           // [E][P]  v of entries (physical)
    s.sal = s.sv + gpad4(E * P);          // [E]     alpha (physical); KDA [E][N]
    s.sbe = s.sal + gpad4(kda ? E * N : E);  // [E]  beta (physical)
    s.spr = s.sbe + gpad4(E);             // [E]     prefix products of alpha from e0 (logical)
    s.sq = s.spr + gpad4(E);              // [TQ][N] queries
    s.sG = s.sq + gpad4(TQ * N);          // [E][E]  Gram k_e . k_j (logical)
    s.shq = s.sG + gpad4(E * E);          // [TQ][E] k_e . q_m (logical)
    s.sc = s.shq + gpad4(TQ * E);         // [TQ][E] sweep coefficients c (logical)
    s.sr = s.sc + gpad4(TQ * E);          // [TQ][N] swept query r
    s.sdot = s.sr + gpad4(TQ * N);        // [TQ][P] S^ r per row
    s.srq = s.sdot + gpad4(TQ * P);       // [TQ]    unused pad
    s.si = reinterpret_cast<int *>(s.srq + gpad4(TQ));
    float *raw = s.srq + gpad4(TQ) + 8;
    const int Rm = W + 8;
    s.rk = reinterpret_cast<uint8_t *>(raw);
    s.rv = s.rk + 4 * gpad4(Rm * N * ib / 4);
    s.ra = reinterpret_cast<float *>(s.rv + 4 * gpad4(Rm * P * ib / 4));
    s.rb = s.ra + gpad4(kda ? Rm * N : Rm);
    return s;
}

// 16 bytes of raw inputs (8 bf16 or 4 fp32) to fp32 in shared memory.
__device__ __forceinline__ void raw16_to_f32(const uint8_t *src, float *dst, int bf16) {
    const uint4 u = *reinterpret_cast<const uint4 *>(src);
    if (bf16) {
        reinterpret_cast<float4 *>(dst)[0] = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                                                         __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
        reinterpret_cast<float4 *>(dst)[1] = make_float4(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xffff0000u),
                                                         __uint_as_float(u.w << 16), __uint_as_float(u.w & 0xffff0000u));
    } else {
        *reinterpret_cast<float4 *>(dst) = make_float4(__uint_as_float(u.x), __uint_as_float(u.y),
                                                       __uint_as_float(u.z), __uint_as_float(u.w));
    }
}

// Fold-mapping: TPRF lanes per state row, NPT contiguous elements per lane
// (16 lanes x 8 at d_k = 128: half the state registers of 8 x 16, so three CTAs
// share an SM and hide the per-token reduction chain).
template <int N> struct FoldMap {
    static constexpr int TPRF = (N >= 64) ? 16 : (N >= 32 ? 8 : N / 4);
    static constexpr int NPT = N / TPRF;
    static constexpr int RPPF = kThreads / TPRF;
};

// Stage the new tokens' inputs at physical entries W..W+T-1 and queries.
__device__ __forceinline__ void gdn_stage_new(const GArgs &a, const GSmem &s, int b, int h, int N,
                                              int tid) {
    const int H = a.H, P = a.P, T = a.T, W = a.W;
    for (int i = tid; i < T * N; i += kThreads) {
        const int m = i / N, n = i - m * N;
        const int64_t src = ((int64_t)(b * T + m) * H + h) * N + n;
        s.sk[(W + m) * N + n] = ld_in(a.k, src, a.in_bf16);
        s.sq[m * N + n] = ld_in(a.q, src, a.in_bf16);
    }
    for (int i = tid; i < T * P; i += kThreads) {
        const int m = i / P, p = i - m * P;
        s.sv[(W + m) * P + p] = ld_in(a.v, ((int64_t)(b * T + m) * H + h) * P + p, a.in_bf16);
    }
    if (a.kda) {
        for (int i = tid; i < T * N; i += kThreads) {
            const int m = i / N, n = i - m * N;
            s.sal[(W + m) * N + n] = a.alpha[((int64_t)(b * T + m) * H + h) * N + n];
        }
    } else if (tid < T) {
        s.sal[W + tid] = a.alpha[(int64_t)(b * T + tid) * H + h];
    }
    if (tid < T) s.sbe[W + tid] = a.beta[(int64_t)(b * T + tid) * H + h];
}

// Apply entries [0, L0) (physical base..) to the NR = 4 rows a thread holds as
// NPT-element lane segments (TPRF lanes per row).  Rows are independent; every
// lane of the warp must call this.
// GDN:  s <- alpha s + (beta v[row] - alpha beta (s . k)) k
// KDA:  u = alpha (.) s;  s <- u + beta (v[row] - u . k) k
// The row segments are held as packed pairs for the length of the call, so the
// per-entry dot and update take one .f32x2 instruction per two elements.  The
// four rows' dots are reduced together (quad_rows_sum: 5 shuffles instead of
// 4 log2(TPRF)); each lane then holds one row's sum, reads that row's v and
// forms its coefficient, and the four coefficients are broadcast back from the
// lanes that hold them.
template <int N, int NR>
__device__ __forceinline__ void gdn_fold_rows(float (&st)[NR][FoldMap<N>::NPT], const int (&rows)[NR],
                                              int P, const GSmem &s, int base, int L0, int cseg, int kda) {
    constexpr int NPT = FoldMap<N>::NPT, TPRF = FoldMap<N>::TPRF, NP2 = NPT / 2;
    static_assert(NR == 4 && TPRF >= 4, "four rows per thread, reduced over at least four lanes");
    const int lane = threadIdx.x & 31;
    const int qrow = 2 * ((cseg & (TPRF / 2)) != 0) + ((cseg & (TPRF / 4)) != 0);  // the row this lane's sum belongs to
    const int myrow = qrow == 0 ? rows[0] : (qrow == 1 ? rows[1] : (qrow == 2 ? rows[2] : rows[3]));
    const bool myvalid = myrow < P;
    const int gbase = lane & ~(TPRF - 1);  // first lane of this row group
    unsigned long long s2[NR][NP2];
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int j = 0; j < NP2; ++j) s2[r][j] = f2_pack(st[r][2 * j], st[r][2 * j + 1]);
    for (int e = 0; e < L0; ++e) {
        const float be = s.sbe[base + e];
        unsigned long long k2[NP2];
#pragma unroll
        for (int j = 0; j < NPT; j += 4) {
            const float4 k4 = *reinterpret_cast<const float4 *>(s.sk + (base + e) * N + cseg * NPT + j);
            k2[j / 2] = f2_pack(k4.x, k4.y);
            k2[j / 2 + 1] = f2_pack(k4.z, k4.w);
        }
        float dp[NR];
        if (kda) {  // warp-uniform
            unsigned long long g2[NP2];
#pragma unroll
            for (int j = 0; j < NPT; j += 4) {
                const float4 g4 = *reinterpret_cast<const float4 *>(s.sal + (base + e) * N + cseg * NPT + j);
                g2[j / 2] = f2_pack(g4.x, g4.y);
                g2[j / 2 + 1] = f2_pack(g4.z, g4.w);
            }
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                unsigned long long d2 = 0ull;
#pragma unroll
                for (int j = 0; j < NP2; ++j) {
                    s2[r][j] = f2_mul(s2[r][j], g2[j]);
                    d2 = f2_fma(s2[r][j], k2[j], d2);
                }
                float dl, dh;
                f2_unpack(d2, dl, dh);
                dp[r] = dl + dh;
            }
        } else {
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                unsigned long long d2 = 0ull;
#pragma unroll
                for (int j = 0; j < NP2; ++j) d2 = f2_fma(s2[r][j], k2[j], d2);
                float dl, dh;
                f2_unpack(d2, dl, dh);
                dp[r] = dl + dh;
            }
        }
        const float d = quad_rows_sum<TPRF>(dp[0], dp[1], dp[2], dp[3], cseg);
        const float vr = myvalid ? s.sv[(base + e) * P + myrow] : 0.f;
        const float al = kda ? 1.f : s.sal[base + e];
        const float coef = kda ? be * (vr - d) : be * vr - al * be * d;
        float cr[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) cr[r] = __shfl_sync(0xffffffffu, coef, gbase + r * (TPRF / 4));
        if (kda) {
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                const unsigned long long c2 = f2_pack(cr[r], cr[r]);
#pragma unroll
                for (int j = 0; j < NP2; ++j) s2[r][j] = f2_fma(c2, k2[j], s2[r][j]);
            }
        } else {
            const unsigned long long a2 = f2_pack(al, al);
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                const unsigned long long c2 = f2_pack(cr[r], cr[r]);
#pragma unroll
                for (int j = 0; j < NP2; ++j) s2[r][j] = f2_fma(a2, s2[r][j], f2_mul(c2, k2[j]));
            }
        }
    }
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int j = 0; j < NP2; ++j) f2_unpack(s2[r][j], st[r][2 * j], st[r][2 * j + 1]);
}

// ---------------------------------------------------------------------------
// Replay kernel: decode (T = 1), verify (T = K), flush (T = 0), export (T = 0).
// ---------------------------------------------------------------------------
template <int N, int RK, int TQ>
__global__ void __launch_bounds__(kThreads, TQ == 1 ? 3 : 1) gdn_replay_kernel(const GArgs a) {
    constexpr int EPC = Chunk<RK>::EPC;
    constexpr int TPR = N / EPC;
    constexpr int RPP = kThreads / TPR;
    constexpr int RB = 8;
    using FM = FoldMap<N>;
    constexpr int NPT = FM::NPT, TPRF = FM::TPRF, RPPF = FM::RPPF, RBF = 4;
    static_assert(TPR >= 1 && TPR <= 32 && (32 % TPR) == 0, "row must fit a warp");

    extern __shared__ __align__(16) float smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.x;
    const int H = a.H, P = a.P, W = a.W, R = a.R, T = a.T;
    const int b = bh / H, h = bh - b * H;
    const int E = W + TQ;
    const int ib = a.in_bf16 ? 2 : 4;
    GSmem s = gdn_carve(smem, P, N, W, TQ, a.kda, ib);
    const int64_t tile0 = (int64_t)bh * P * N;
    const bool reads = (a.op == OP_DECODE || a.op == OP_VERIFY);

    // 1. Read-copy loads first (dropped on folding steps; none in fold-only mode,
    //    which serves only sequences that fold).
    const int c = tid % TPR, r0 = tid / TPR;
    const uint8_t *rc_tile =
        (RK == SK_F32) ? reinterpret_cast<const uint8_t *>(a.ckpt + tile0)
                       : reinterpret_cast<const uint8_t *>(a.rc) + tile0 * Chunk<RK>::BYTES;
    uint4 rv[RB];
    float rscale[RB];
    if (reads && !a.fold_only) {
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k * RPP;
            if (r < P) rv[k] = ld_stream(rc_tile + ((size_t)r * TPR + c) * 16);
            if (RK == SK_FP8) rscale[k] = (r < P) ? __ldg(a.rc_scale + (int64_t)bh * P + r) : 0.f;
        }
    }

    // 2. The whole rings (raw, slot order: none of it depends on the counters),
    //    the counters and the new tokens, in one round trip.
    {
        const uint8_t *ks = reinterpret_cast<const uint8_t *>(a.kbuf) + (int64_t)bh * R * N * ib;
        for (int i = tid; i < R * N * ib / 16; i += kThreads) cp_async16(s.rk + 16 * i, ks + 16 * i);
        const uint8_t *vs = reinterpret_cast<const uint8_t *>(a.vbuf) + (int64_t)bh * R * P * ib;
        for (int i = tid; i < R * P * ib / 16; i += kThreads) cp_async16(s.rv + 16 * i, vs + 16 * i);
        if (a.kda) {
            const float *as = a.abuf + (int64_t)bh * R * N;
            for (int i = tid; i < R * N / 4; i += kThreads) cp_async16(s.ra + 4 * i, as + 4 * i);
        } else {
            for (int i = tid; i < a.Rs / 4; i += kThreads) cp_async16(s.ra + 4 * i, a.abuf + (int64_t)bh * a.Rs + 4 * i);
        }
        for (int i = tid; i < a.Rs / 4; i += kThreads) cp_async16(s.rb + 4 * i, a.bbuf + (int64_t)bh * a.Rs + 4 * i);
    }
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
            if (h == 0 && !a.fold_only) report(a.c.err, DEV_BAD_COUNTERS, b, h, (int)(ss.seq - ss.ckpt));
        } else if (a.op != OP_EXPORT && !a.fold_only) {
            const int64_t new_seq = (a.op == OP_DECODE) ? ss.seq + 1 : -1;
            const int64_t new_ckpt = flush ? ss.seq : -1;
            const int new_pending = (a.op == OP_VERIFY) ? T : -1;
            arrive_and_publish(a.c, b, H, new_seq, new_ckpt, new_pending, flush);
        }
    }
    gdn_stage_new(a, s, b, h, N, tid);
    cp_async_wait_all();
    __syncthreads();
    if (!s.si[0]) return;
    const int L0 = s.si[1], flush = s.si[2], ckmod = s.si[3], spmod = s.si[4];
    if (a.fold_only && !flush) return;  // served by the prep and read kernels
    const int base = W - L0;
    const int nE = L0 + T;
    const int e0 = flush ? L0 : 0;

    // 3. Buffered entries, from the staged rings (slot (ckmod + e) mod R) to fp32
    //    rows at their physical entries base + e.
    {
        const int kc = N * ib / 16, vc = P * ib / 16;  // 16-byte chunks per row
        auto slot_of = [&](int e) { const int sl = ckmod + e; return sl >= R ? sl - R : sl; };
        for (int i = tid; i < L0 * kc; i += kThreads) {
            const int e = i / kc, c2 = i - e * kc;
            raw16_to_f32(s.rk + (slot_of(e) * kc + c2) * 16, s.sk + (base + e) * N + c2 * (16 / ib), a.in_bf16);
        }
        for (int i = tid; i < L0 * vc; i += kThreads) {
            const int e = i / vc, c2 = i - e * vc;
            raw16_to_f32(s.rv + (slot_of(e) * vc + c2) * 16, s.sv + (base + e) * P + c2 * (16 / ib), a.in_bf16);
        }
        if (a.kda) {
            for (int i = tid; i < L0 * (N / 4); i += kThreads) {
                const int e = i / (N / 4), c4 = i - e * (N / 4);
                *reinterpret_cast<float4 *>(s.sal + (base + e) * N + 4 * c4) =
                    *reinterpret_cast<const float4 *>(s.ra + slot_of(e) * N + 4 * c4);
            }
        }
        for (int e = tid; e < L0; e += kThreads) {
            if (!a.kda) s.sal[base + e] = s.ra[slot_of(e)];
            s.sbe[base + e] = s.rb[slot_of(e)];
        }
    }
    __syncthreads();

    if (reads && a.kda) {
        // 4-6 (KDA). One warp per query: the backward sweep applied to the query
        // itself, r <- alpha_i (.) (r - c_i k_i), c_i = beta_i (k_i . r).
        if (warp < T) {
            const int m = warp, em = L0 + m;
            float *r = s.sr + m * N;
            for (int x = lane; x < N; x += 32) r[x] = s.sq[m * N + x];
            __syncwarp();
            for (int i = em; i >= e0; --i) {
                const float *ki = s.sk + (base + i) * N, *gi = s.sal + (base + i) * N;
                float d = 0.f;
                for (int x = lane; x < N; x += 32) d = fmaf(ki[x], r[x], d);
                d = group_sum<32>(d);
                const float ci = s.sbe[base + i] * d;
                if (lane == 0) s.sc[m * E + i] = ci;
                for (int x = lane; x < N; x += 32) r[x] = gi[x] * fmaf(-ci, ki[x], r[x]);
                __syncwarp();
            }
        }
        __syncthreads();
    } else if (reads) {
        // 4. Gram matrix of the replayed keys and their products with the queries.
        const int n = nE - e0;                       // replayed entries
        const int ngram = n * (n - 1) / 2;
        const int nq = T * n;
        for (int pr = warp; pr < ngram + nq; pr += kWarps) {
            int ea, eb;
            const float *va, *vb;
            if (pr < ngram) {  // unrank pr -> (i < j) over [0, n)
                int j = (int)((1.f + sqrtf(1.f + 8.f * (float)pr)) * 0.5f);
                while (j * (j - 1) / 2 > pr) --j;
                while ((j + 1) * j / 2 <= pr) ++j;
                const int i = pr - j * (j - 1) / 2;
                ea = e0 + i; eb = e0 + j;
                va = s.sk + (base + ea) * N;
                vb = s.sk + (base + eb) * N;
            } else {
                const int m = (pr - ngram) / n;
                ea = e0 + (pr - ngram) - m * n;
                eb = -1 - m;
                va = s.sk + (base + ea) * N;
                vb = s.sq + m * N;
            }
            float d = 0.f;
            for (int x = lane; x < N; x += 32) d = fmaf(va[x], vb[x], d);
            d = group_sum<32>(d);
            if (lane == 0) {
                if (eb >= 0) s.sG[ea * E + eb] = d;
                else s.shq[(-1 - eb) * E + ea] = d;
            }
        }
        if (tid == 0) {  // prefix products of alpha from e0
            float acc = 1.f;
            for (int e = e0; e < nE; ++e) { acc *= s.sal[base + e]; s.spr[e] = acc; }
        }
        __syncthreads();
        // 5. One warp per query: the backward sweep as a lane-parallel chain.
        constexpr int CH = (64 + TQ + 31) / 32;  // entries per lane (W <= 64)
        if (warp < T) {
            const int m = warp, em = L0 + m;
            float t[CH];
#pragma unroll
            for (int j = 0; j < CH; ++j) {
                const int e = e0 + lane + 32 * j;
                t[j] = (e <= em) ? s.shq[m * E + e] : 0.f;
            }
            for (int i = em; i >= e0; --i) {
                const int li = i - e0, src = li & 31, ji = li >> 5;
                float ti = 0.f;
#pragma unroll
                for (int j = 0; j < CH; ++j) if (j == ji) ti = t[j];
                const float ci = s.sbe[base + i] * __shfl_sync(0xffffffffu, ti, src);
                const float al = s.sal[base + i];
                if (lane == 0) s.sc[m * E + i] = ci;
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    const int e = e0 + lane + 32 * j;
                    if (e < i) t[j] = al * (t[j] - ci * s.sG[e * E + i]);
                }
            }
        }
        __syncthreads();
        // 6. r_m = P_{em} q_m - sum_i P_i c_{m,i} k_i  (P_i: prefix products of alpha).
        for (int idx = tid; idx < T * N; idx += kThreads) {
            const int m = idx / N, x = idx - m * N, em = L0 + m;
            float r = s.spr[em] * s.sq[m * N + x];
            for (int i = e0; i <= em; ++i) r = fmaf(-s.spr[i] * s.sc[m * E + i], s.sk[(base + i) * N + x], r);
            s.sr[m * N + x] = r;
        }
        __syncthreads();
    }

    if (flush) {
        // 7a. Fold the committed entries into the fp32 checkpoint rows.
        const int cseg = tid % TPRF, q0 = tid / TPRF;
        for (int rb = 0; rb < P; rb += RBF * RPPF) {
            float st[RBF][NPT];
            int rows[RBF];
#pragma unroll
            for (int k = 0; k < RBF; ++k) {
                rows[k] = rb + q0 + k * RPPF;
#pragma unroll
                for (int j = 0; j < NPT; j += 4) {
                    float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (rows[k] < P) v4 = load_quad<SK_F32>(a.ckpt, tile0 + (int64_t)rows[k] * N + cseg * NPT + j);
                    st[k][j] = v4.x; st[k][j + 1] = v4.y; st[k][j + 2] = v4.z; st[k][j + 3] = v4.w;
                }
            }
            gdn_fold_rows<N, RBF>(st, rows, P, s, base, L0, cseg, a.kda);
#pragma unroll
            for (int k = 0; k < RBF; ++k) {
                const bool valid = rows[k] < P;
                const int64_t el = tile0 + (int64_t)(valid ? rows[k] : 0) * N + cseg * NPT;
                if (a.op == OP_EXPORT) {
                    if (valid)
#pragma unroll
                        for (int j = 0; j < NPT; j += 4)
                            *reinterpret_cast<float4 *>(a.out + el + j) =
                                make_float4(st[k][j], st[k][j + 1], st[k][j + 2], st[k][j + 3]);
                    continue;
                }
                float sc = 1.f;
                if (RK == SK_FP8) {
                    float am = 0.f;
#pragma unroll
                    for (int j = 0; j < NPT; ++j) am = fmaxf(am, fabsf(st[k][j]));
                    sc = fp8_scale(group_max<TPRF>(am));
                    if (valid && cseg == 0) a.rc_scale[(int64_t)bh * P + rows[k]] = sc;
                }
                float dots[TQ];
#pragma unroll
                for (int m = 0; m < TQ; ++m) dots[m] = 0.f;
#pragma unroll
                for (int j = 0; j < NPT; j += 4) {
                    float4 v4 = make_float4(st[k][j], st[k][j + 1], st[k][j + 2], st[k][j + 3]);
                    float4 rd = v4;
                    if (valid) {
                        store_quad<SK_F32>(a.ckpt, el + j, v4, 0.f, 0.f);
                        if (RK == SK_BF16) rd = store_quad<SK_BF16>(a.rc, el + j, v4, 0.f, 0.f);
                        if (RK == SK_FP8) rd = store_quad<SK_FP8>(a.rc, el + j, v4, 0.f, sc);
                    }
                    if (reads) {
#pragma unroll
                        for (int m = 0; m < TQ; ++m) {
                            const float4 r4 = *reinterpret_cast<const float4 *>(s.sr + m * N + cseg * NPT + j);
                            dots[m] += rd.x * r4.x + rd.y * r4.y + rd.z * r4.z + rd.w * r4.w;
                        }
                    }
                }
                if (reads) {
#pragma unroll
                    for (int m = 0; m < TQ; ++m) {
                        const float d = group_sum<TPRF>(dots[m]);
                        if (valid && cseg == 0 && m < T) s.sdot[m * P + rows[k]] = d;
                    }
                }
            }
        }
    } else if (reads) {
        // 7b. Read: dot products of the read-copy rows with the swept queries.
        float Rr[TQ][EPC];
#pragma unroll
        for (int m = 0; m < TQ; ++m)
#pragma unroll
            for (int j = 0; j < EPC; ++j) Rr[m][j] = (m < T) ? s.sr[m * N + c * EPC + j] : 0.f;
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
                    for (int j = 0; j < EPC; ++j) d = fmaf(v[j], Rr[m][j], d);
                    d = group_sum<TPR>(d);
                    if (RK == SK_FP8) d *= rscale[k];
                    if (c == 0 && r < P && m < T) s.sdot[m * P + r] = d;
                }
            }
        }
    }
    if (!reads) return;
    __syncthreads();

    // 8. Outputs o_m = S^ r_m + sum_i c_{m,i} v_i.
    for (int i = tid; i < T * P; i += kThreads) {
        const int m = i / P, p = i - m * P;
        float o = s.sdot[m * P + p];
        for (int e = e0; e <= L0 + m; ++e) o = fmaf(s.sc[m * E + e], s.sv[(base + e) * P + p], o);
        a.y[((int64_t)(b * T + m) * H + h) * P + p] = o;
    }

    // 9. Append the new tokens to the ring (fold-only mode: the prep kernel did).
    if (a.fold_only) return;
    for (int i = tid; i < T * N; i += kThreads) {
        const int m = i / N, n = i - m * N;
        copy_in(a.kbuf, ((int64_t)bh * R + (spmod + m) % R) * N + n, a.k,
                ((int64_t)(b * T + m) * H + h) * N + n, a.in_bf16);
    }
    for (int i = tid; i < T * P; i += kThreads) {
        const int m = i / P, p = i - m * P;
        copy_in(a.vbuf, ((int64_t)bh * R + (spmod + m) % R) * P + p, a.v,
                ((int64_t)(b * T + m) * H + h) * P + p, a.in_bf16);
    }
    if (tid < T) {
        const int64_t slot = (int64_t)bh * a.Rs + (spmod + tid) % R;
        if (!a.kda) a.abuf[slot] = s.sal[W + tid];
        a.bbuf[slot] = s.sbe[W + tid];
    }
    if (a.kda)
        for (int i = tid; i < T * N; i += kThreads) {
            const int m = i / N, n = i - m * N;
            a.abuf[((int64_t)bh * R + (spmod + m) % R) * N + n] = s.sal[(W + m) * N + n];
        }
}

// ---------------------------------------------------------------------------
// Prep kernel of a replay decode/verify: one CTA per (sequence, up to 8 heads),
// one warp per head.  Thread 0 reads the sequence's counters; each warp stages its
// head's buffered keys and gates and the call's k, q, then runs the backward
// sweep for every query m (entries L0+m .. 0):
//     c_e = beta_e (k_e . r),   r <- alpha_e (r - c_e k_e),   starting from r = q_m,
// leaving the swept query r_m and the coefficients c for the read kernel,
// which computes o_m = S^ r_m + sum_e c_e v_e (decay 1: it is inside r).
// Sequences whose buffer must be folded first (len + T > W) are left to the
// fold-only launch of gdn_replay_kernel.  Every sequence's tokens are appended
// to the ring (slots seq_pos + m mod R, never an entry read in this call).
// ---------------------------------------------------------------------------
// Per warp: raw k rows [E][N] and q rows [TQ][N], then the gates (GDN [Ea], KDA
// [E][N] fp32) and beta [Ea].
__host__ __device__ inline int gdn_prep_warp_bytes(int N, int W, int TQ, int ib, int kda) {
    const int E = W + TQ, Ea = (E + 3) & ~3;
    return ((E + TQ) * N * ib + (kda ? E * N : Ea) * 4 + Ea * 4 + 15) & ~15;
}

template <int N, int TQ, bool BF>
__global__ void __launch_bounds__(kThreads) gdn_prep_kernel(const GArgs a) {
    constexpr int IB = BF ? 2 : 4;
    constexpr int NL = N >= 32 ? N / 32 : 1;  // key elements per lane (lanes >= N idle when N < 32)
    extern __shared__ __align__(16) uint8_t gsm[];
    __shared__ int si[6];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, P = a.P, W = a.W, R = a.R, T = a.T;
    const int E = W + TQ, Ea = (E + 3) & ~3;
    const int b = blockIdx.y, h = blockIdx.x * a.prep_heads + warp;
    pdl_trigger();  // the read kernel may be scheduled as this grid's last CTAs run
    if (tid == 0) {
        const SeqState ss = read_counters(a.c, b, W);
        const int L0 = (int)(ss.seq - ss.ckpt);
        const int fold = ss.ok && (L0 + T > W);
        bool valid = ss.ok;
        if (blockIdx.x == 0) {
            if (!ss.ok) report(a.c.err, DEV_BAD_COUNTERS, b, 0, L0);
            if (fold && !a.fold_launched) {  // the host's bound on buffer lengths was wrong
                report(a.c.err, DEV_BAD_COUNTERS, b, 0, L0);
                valid = false;
            }
            a.seqinfo[b] = valid ? make_int4(fold ? 0 : L0, (int)(ss.ckpt % R), fold, 1) : make_int4(0, 0, 1, 0);
        }
        si[0] = ss.ok;
        si[1] = ss.ok ? L0 : 0;
        si[2] = fold;
        si[3] = (int)(ss.ckpt % R);
        si[4] = (int)(ss.seq % R);
    }
    __syncthreads();
    if (!si[0] || warp >= a.prep_heads || h >= H) return;
    const int L0 = si[1], fold = si[2], ckmod = si[3], spmod = si[4];
    const int64_t bh = (int64_t)b * H + h;
    const int krow = N * IB, kch = krow / 16;
    const int kda = a.kda;
    uint8_t *wk = gsm + warp * gdn_prep_warp_bytes(N, W, TQ, IB, kda);  // k rows [E][N] raw
    uint8_t *wq = wk + E * krow;                                   // q rows [TQ][N] raw
    float *wal = reinterpret_cast<float *>(wq + TQ * krow);        // alpha [E]; KDA [E][N]
    float *wbe = wal + (kda ? E * N : Ea);                         // beta  [E]
    auto run = [&](uint8_t *dst, const uint8_t *src, int n) {
        for (int j = lane; j < n; j += 32) cp_async16(dst + 16 * j, src + 16 * j);
    };
    const uint8_t *kin = reinterpret_cast<const uint8_t *>(a.k), *qin = reinterpret_cast<const uint8_t *>(a.q);
    for (int m = 0; m < T; ++m) {
        const int64_t row = ((int64_t)b * T + m) * H + h;
        run(wk + (L0 + m) * krow, kin + row * krow, kch);
        run(wq + m * krow, qin + row * krow, kch);
    }
    const int gch = N * 4 / 16;  // 16-byte chunks of a KDA gate row
    if (!fold) {
        const int n1 = min(L0, R - ckmod);
        const uint8_t *kr = reinterpret_cast<const uint8_t *>(a.kbuf) + bh * R * krow;
        run(wk, kr + ckmod * krow, n1 * kch);
        run(wk + n1 * krow, kr, (L0 - n1) * kch);
        if (kda) {
            const uint8_t *gr = reinterpret_cast<const uint8_t *>(a.abuf) + bh * R * N * 4;
            run(reinterpret_cast<uint8_t *>(wal), gr + ckmod * N * 4, n1 * gch);
            run(reinterpret_cast<uint8_t *>(wal + n1 * N), gr, (L0 - n1) * gch);
        }
        for (int e = lane; e < L0; e += 32) {
            const int s2 = ckmod + e >= R ? ckmod + e - R : ckmod + e;
            if (!kda) wal[e] = a.abuf[bh * a.Rs + s2];
            wbe[e] = a.bbuf[bh * a.Rs + s2];
        }
    }
    if (kda)
        for (int m = 0; m < T; ++m)
            run(reinterpret_cast<uint8_t *>(wal + (L0 + m) * N),
                reinterpret_cast<const uint8_t *>(a.alpha + (((int64_t)b * T + m) * H + h) * N), gch);
    if (lane < T) {
        if (!kda) wal[L0 + lane] = a.alpha[((int64_t)b * T + lane) * H + h];
        wbe[L0 + lane] = a.beta[((int64_t)b * T + lane) * H + h];
    }
    cp_async_wait_all();
    __syncwarp();
    auto lde = [&](const uint8_t *row, float (&v)[NL]) {  // this lane's NL elements of a raw row
        if (NL * lane >= N) {
#pragma unroll
            for (int i = 0; i < NL; ++i) v[i] = 0.f;
            return;
        }
#pragma unroll
        for (int i = 0; i < NL; ++i) {
            const uint8_t *q = row + (NL * lane + i) * IB;
            v[i] = BF ? bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(q)) : *reinterpret_cast<const float *>(q);
        }
    };
    if (!fold) {
        for (int m = 0; m < T; ++m) {
            float r[NL];
            lde(wq + m * krow, r);
            float *crow = a.coef + (bh * a.TQmax + m) * a.Emax;
            for (int e = L0 + m; e >= 0; --e) {
                float kv[NL];
                lde(wk + e * krow, kv);
                float d = 0.f;
#pragma unroll
                for (int i = 0; i < NL; ++i) d = fmaf(kv[i], r[i], d);
                d = group_sum<32>(d);
                const float ce = wbe[e] * d;
                if (kda) {  // gate per key channel; lanes past N hold zeros
#pragma unroll
                    for (int i = 0; i < NL; ++i) {
                        const float g = NL * lane < N ? wal[e * N + NL * lane + i] : 0.f;
                        r[i] = g * fmaf(-ce, kv[i], r[i]);
                    }
                } else {
                    const float al = wal[e];
#pragma unroll
                    for (int i = 0; i < NL; ++i) r[i] = al * fmaf(-ce, kv[i], r[i]);
                }
                if (lane == 0) crow[e] = ce;
            }
            if (NL * lane < N) {
                float *qo = a.query + (bh * a.TQmax + m) * N + NL * lane;
#pragma unroll
                for (int i = 0; i < NL; ++i) qo[i] = r[i];
            }
            if (lane == 0) a.dec[bh * a.TQmax + m] = 1.f;
        }
    }
    // Append the call's tokens: k from the staged rows, v straight from the
    // inputs, the gates.
    const int vch = P * IB / 16;
    for (int m = 0; m < T; ++m) {
        const int sl = spmod + m >= R ? spmod + m - R : spmod + m;
        uint8_t *kd = reinterpret_cast<uint8_t *>(a.kbuf) + (bh * R + sl) * krow;
        for (int j = lane; j < kch; j += 32)
            *reinterpret_cast<uint4 *>(kd + 16 * j) = *reinterpret_cast<const uint4 *>(wk + (L0 + m) * krow + 16 * j);
        uint8_t *vd = reinterpret_cast<uint8_t *>(a.vbuf) + (bh * R + sl) * P * IB;
        const uint8_t *vs = reinterpret_cast<const uint8_t *>(a.v) + (((int64_t)b * T + m) * H + h) * P * IB;
        for (int j = lane; j < vch; j += 32)
            *reinterpret_cast<uint4 *>(vd + 16 * j) = *reinterpret_cast<const uint4 *>(vs + 16 * j);
        if (kda) {
            float *gd = a.abuf + (bh * R + sl) * N;
            for (int j = lane; j < N / 4; j += 32)
                *reinterpret_cast<float4 *>(gd + 4 * j) = *reinterpret_cast<const float4 *>(wal + (L0 + m) * N + 4 * j);
        }
        if (lane == 0) {
            if (!kda) a.abuf[bh * a.Rs + sl] = wal[L0 + m];
            a.bbuf[bh * a.Rs + sl] = wbe[L0 + m];
        }
    }
}

// ---------------------------------------------------------------------------
// Eager baseline: decode (state rewritten every token) and verify (K snapshots).
// ---------------------------------------------------------------------------
template <int N, int SK, int TQ>
__global__ void __launch_bounds__(kThreads) gdn_eager_kernel(const GArgs a) {
    using FM = FoldMap<N>;
    constexpr int NPT = FM::NPT, TPRF = FM::TPRF, RPPF = FM::RPPF, RBF = 4;
    extern __shared__ __align__(16) float smem[];
    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int H = a.H, P = a.P, T = a.T, W = a.W;
    const int b = bh / H, h = bh - b * H;
    GSmem s = gdn_carve(smem, P, N, W, TQ, a.kda, a.in_bf16 ? 2 : 4);
    const int64_t tile0 = (int64_t)bh * P * N;
    void *state = (SK == SK_F32) ? (void *)a.ckpt : a.rc;
    const int64_t state_elems = (int64_t)a.B * H * P * N;

    // No other CTA of an eager launch reads the counters, so the sequence's first
    // head's CTA rewrites them alone (no arrival count, no fence).
    if (tid == 0 && h == 0) {
        if (a.op == OP_DECODE) {
            const int64_t s1 = a.c.seq_pos[b] + 1;
            a.c.seq_pos[b] = s1;
            a.c.ckpt_pos[b] = s1;
        } else {
            a.c.pending[b] = T;
        }
    }
    gdn_stage_new(a, s, b, h, N, tid);
    __syncthreads();

    const int cseg = tid % TPRF, q0 = tid / TPRF;
    for (int rb = 0; rb < P; rb += RBF * RPPF) {
        float st[RBF][NPT];
        int rows[RBF];
#pragma unroll
        for (int k = 0; k < RBF; ++k) {
            rows[k] = rb + q0 + k * RPPF;
            const float scl = (SK == SK_FP8 && rows[k] < P) ? __ldg(a.rc_scale + (int64_t)bh * P + rows[k]) : 1.f;
#pragma unroll
            for (int j = 0; j < NPT; j += 4) {
                float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (rows[k] < P) v4 = load_quad<SK>(state, tile0 + (int64_t)rows[k] * N + cseg * NPT + j);
                st[k][j] = v4.x * scl; st[k][j + 1] = v4.y * scl; st[k][j + 2] = v4.z * scl; st[k][j + 3] = v4.w * scl;
            }
        }
        for (int m = 0; m < T; ++m) {
            // one token: entry m sits at physical W + m
            gdn_fold_rows<N, RBF>(st, rows, P, s, W + m, 1, cseg, a.kda);
#pragma unroll
            for (int k = 0; k < RBF; ++k) {
                const bool valid = rows[k] < P;
                float d = 0.f;
#pragma unroll
                for (int j = 0; j < NPT; ++j) d = fmaf(st[k][j], s.sq[m * N + cseg * NPT + j], d);
                d = group_sum<TPRF>(d);
                if (valid && cseg == 0) s.sdot[m * P + rows[k]] = d;
                const bool last = (m == T - 1);
                if (a.op == OP_VERIFY || (a.op == OP_DECODE && last)) {
                    void *dst = state;
                    float *dscale = a.rc_scale;
                    if (a.op == OP_VERIFY) {
                        dst = (SK == SK_F32) ? (void *)(reinterpret_cast<float *>(a.snap) + m * state_elems)
                                             : (void *)(reinterpret_cast<uint8_t *>(a.snap) + m * state_elems * Chunk<SK>::BYTES);
                        dscale = a.snap_scale ? a.snap_scale + (int64_t)m * a.B * H * P : nullptr;
                    }
                    float sc = 1.f;
                    if (SK == SK_FP8) {
                        float am = 0.f;
#pragma unroll
                        for (int j = 0; j < NPT; ++j) am = fmaxf(am, fabsf(st[k][j]));
                        sc = fp8_scale(group_max<TPRF>(am));
                        if (valid && cseg == 0) dscale[(int64_t)bh * P + rows[k]] = sc;
                    }
                    if (valid) {
                        const int64_t el = tile0 + (int64_t)rows[k] * N + cseg * NPT;
#pragma unroll
                        for (int j = 0; j < NPT; j += 4)
                            store_quad<SK>(dst, el + j, make_float4(st[k][j], st[k][j + 1], st[k][j + 2], st[k][j + 3]), 0.f, sc);
                    }
                }
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < T * P; i += kThreads) {
        const int m = i / P, p = i - m * P;
        a.y[((int64_t)(b * T + m) * H + h) * P + p] = s.sdot[m * P + p];
    }
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
template <int N, int RK, int TQ>
inline cudaError_t glaunch_replay(const GArgs &a, size_t smem, cudaStream_t st) {
    auto k = gdn_replay_kernel<N, RK, TQ>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<a.B * a.H, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}
template <int N, int SK, int TQ>
inline cudaError_t glaunch_eager(const GArgs &a, size_t smem, cudaStream_t st) {
    auto k = gdn_eager_kernel<N, SK, TQ>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<a.B * a.H, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}
template <int N, int TQ>
inline cudaError_t gdispatch_rk(bool eager, int rk, const GArgs &a, size_t smem, cudaStream_t st) {
    switch (rk) {
        case SK_F32: return eager ? glaunch_eager<N, SK_F32, TQ>(a, smem, st) : glaunch_replay<N, SK_F32, TQ>(a, smem, st);
        case SK_BF16: return eager ? glaunch_eager<N, SK_BF16, TQ>(a, smem, st) : glaunch_replay<N, SK_BF16, TQ>(a, smem, st);
        default: return eager ? glaunch_eager<N, SK_FP8, TQ>(a, smem, st) : glaunch_replay<N, SK_FP8, TQ>(a, smem, st);
    }
}
template <int N>
inline cudaError_t gdispatch_tq(bool eager, int rk, int TQ, const GArgs &a, size_t smem, cudaStream_t st) {
    if (TQ == 1) return gdispatch_rk<N, 1>(eager, rk, a, smem, st);
    if (TQ == 4) return gdispatch_rk<N, 4>(eager, rk, a, smem, st);
    return gdispatch_rk<N, 8>(eager, rk, a, smem, st);
}

// Per-dstate entry point; each instantiation lives in its own translation unit.
template <int N>
cudaError_t g_dispatch_n(bool eager, int rk, int TQ, const GArgs &a, size_t smem, cudaStream_t st) {
    return gdispatch_tq<N>(eager, rk, TQ, a, smem, st);
}

template <int N, int TQ>
inline cudaError_t launch_gprep_t(const GArgs &a, cudaStream_t st) {
    auto k = a.in_bf16 ? gdn_prep_kernel<N, TQ, true> : gdn_prep_kernel<N, TQ, false>;
    const int smem = a.prep_heads * gdn_prep_warp_bytes(N, a.W, TQ, a.in_bf16 ? 2 : 4, a.kda);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k<<<dim3((a.H + a.prep_heads - 1) / a.prep_heads, a.B), kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int N>
cudaError_t g_prep_dispatch_n(int TQ, const GArgs &a, cudaStream_t st) {
    if (TQ == 1) return launch_gprep_t<N, 1>(a, st);
    if (TQ == 4) return launch_gprep_t<N, 4>(a, st);
    return launch_gprep_t<N, 8>(a, st);
}

}  // namespace rssm
