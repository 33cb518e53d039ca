// rssm_read.cuh -- the replay-read kernel (sm_100a), shared by Mamba-2 and Gated DeltaNet.
//
// ReplaySSM computes a token's output from the checkpoint and the buffered inputs
// without writing state ("Tenir le journal plutot que le solde",
// blog.thibaultmonteiro.fr).  After the prep kernel has turned the buffer into a
// per-head coefficient table, the output of query m of head h is
//   y[b,m,h,p] = dec[b,h,m] * (S^[b,h,p,:] . Q[b,h,m,:])
//                + sum_{e <= L0+m} coef[b,h,m,e] * X_e[p]  + D_h X_{L0+m}[p]
// with S^ the read copy, X_e the buffered entries (Mamba-2 x, GDN v; e < L0 from
// the ring, the call's own tokens after), Q the query (Mamba-2 C of the head's
// group straight from the inputs; GDN the swept query r from the prep kernel).
// Sequences whose buffer was folded in this call were fully served by the prep
// kernel and are skipped.
//
// One CTA per (sequence, HC heads).  Every thread issues its read-copy chunks
// (128-bit, L1 no-allocate) first -- they depend on nothing -- then the CTA
// stages the small operands, dots the rows with the query (LPR lanes per row,
// chunks interleaved so each warp load covers whole 64-byte row segments), and
// applies the replay term.  Only ordinary loads and cp.async are used.  When no
// flush kernel ran in the call, the kernel is launched as a programmatic
// dependent of the prep kernel: its first round of copy loads overlaps the prep
// kernel's last CTAs, and it waits for the prep kernel's hand-off before
// reading anything the prep kernel wrote (or rewriting the counters it read).
// After a flush kernel, the CTA first learns whether its sequence was folded
// (a folded sequence needs no read copy).
#pragma once

#include "rssm_device.cuh"

namespace rssm {

// Shared memory of the read kernel (bytes, 16-byte aligned regions).
struct ReadLay {
    int q, x, coef, dec, dot, scale, info, bytes;
};
inline ReadLay read_lay(int HC, int P, int N, int W, int TQ, int ib, int Ep) {
    auto al = [](int v) { return (v + 15) & ~15; };
    const int E = W + TQ;
    ReadLay L{};
    int o = 0;
    L.q = o;    o += al(HC * TQ * N * 4);     // queries as fp32   [HC or 1][TQ][N]
    L.x = o;    o += al(HC * E * P * ib);     // entries           [HC][E][P] raw
    L.coef = o; o += al(HC * TQ * Ep * 4);    // coefficients      [HC][TQ][Ep]
    L.dec = o;  o += al(HC * TQ * 4);         // decays            [HC][TQ]
    L.dot = o;  o += al(HC * P * TQ * 4);     // S^ . Q per row    [HC*P][TQ]
    L.scale = o; o += al(HC * P * 4);         // fp8 row scales    [HC*P]
    L.info = o; o += 16;
    L.bytes = o;
    return L;
}

struct ReadArgs {
    int B, H, P, R, W, T, HC, in_bf16;
    int q_group;            // heads per query row (Mamba-2: H / G; GDN: 1)
    int q_bf16;             // query dtype: 1 = input bf16, 0 = fp32
    int64_t q_stride_m;     // elements between queries m and m+1 of one (b, query row)
    int64_t q_stride_b;     // elements between sequences
    int64_t q_stride_row;   // elements between query rows
    const void *Q;          // query vectors
    const void *rc;         // read copy (or the fp32 checkpoint): [B][H][P][N]
    const float *rc_scale;  // fp8 row scales [B][H][P]
    const void *xring;      // buffered entries [B][H][R][P] (input dtype)
    const void *xnew;       // the call's own entries [B][T][H][P] (input dtype)
    const float *D;         // per-head skip (nullptr: none)
    const int4 *seqinfo;    // per sequence {L0 replayed from the ring, ring slot of entry 0, folded, valid}
    Counters c;             // published by the first CTA of each sequence
    int *fold_count;        // flush kernel work-list length, reset here for the next call
    int op;                 // OP_DECODE | OP_VERIFY
    const float *dec;       // [B][H][TQmax]
    const float *coef;      // [B][H][TQmax][Emax]
    int TQmax, Emax;        // Emax: padded row length of the coefficient table
    ReadLay lay;            // shared memory, computed on the host
    float *y;               // [B][T][H][P]
    int early;              // no flush kernel ran in this call: every sequence is read, so the
                            // first read-copy round is issued before anything else
    int pdl;                // launched as a programmatic dependent of the prep kernel
    int q_ready;            // the queries are the caller's input, not the prep kernel's output
};

template <int N, int RK, int TQ, bool BF>
__global__ void __launch_bounds__(kThreads, TQ == 1 ? 4 : 2) replay_read_kernel(const ReadArgs a) {
    constexpr int EPC = Chunk<RK>::EPC;   // stored elements per 16-byte chunk
    constexpr int TPR = N / EPC;          // chunks per state row
    constexpr int RCB = Chunk<RK>::BYTES;
    constexpr int LPR = TPR < 4 ? TPR : 4;  // lanes per row
    constexpr int CPL = TPR / LPR;          // chunks per lane per row
    constexpr int RPP = kThreads / LPR;     // rows per pass
    constexpr int MAXC = 8;                 // chunks in flight per thread
    constexpr int PPR = MAXC / CPL > 0 ? MAXC / CPL : 1;  // passes per round
    constexpr int IB = BF ? 2 : 4;
    static_assert(CPL <= MAXC, "a lane's chunks of one row must fit a round");

    extern __shared__ __align__(128) uint8_t smraw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, P = a.P, R = a.R, W = a.W, T = a.T, HC = a.HC;
    const int b = blockIdx.y;
    const int h0 = blockIdx.x * HC;
    const int E = W + TQ, Ep = a.Emax;
    const ReadLay &Ly = a.lay;
    float *sq = reinterpret_cast<float *>(smraw + Ly.q);
    uint8_t *sx = smraw + Ly.x;
    float *scoef = reinterpret_cast<float *>(smraw + Ly.coef);
    float *sdec = reinterpret_cast<float *>(smraw + Ly.dec);
    float *sdot = reinterpret_cast<float *>(smraw + Ly.dot);
    float *ssc = reinterpret_cast<float *>(smraw + Ly.scale);
    int *sinfo = reinterpret_cast<int *>(smraw + Ly.info);
    const int64_t row0 = (int64_t)b * H + h0;
    const int nrows = HC * P;
    const uint8_t *tile = reinterpret_cast<const uint8_t *>(a.rc) + row0 * P * N * RCB;
    const int q = tid % LPR, rrow = tid / LPR;
    const int xrow = P * IB, xch = xrow / 16;

    // 1. First round of read-copy chunks.
    uint4 rv[MAXC];
    auto issue_pass = [&](int pass, int off) {  // the pass's chunks into rv[off ..]
        const int r = pass * RPP + rrow;
#pragma unroll
        for (int k = 0; k < CPL; ++k)
            if (r < nrows) rv[off + k] = ld_stream(tile + ((size_t)r * TPR + q + LPR * k) * 16);
    };
    bool skip_copy = false;  // folded in this call: served by the flush kernel
    if (!a.early) {          // a flush kernel ran in this call
        if (tid == 0) sinfo[2] = a.seqinfo[b].z;
        __syncthreads();
        skip_copy = sinfo[2] != 0;
    }
    if (!skip_copy) {
#pragma unroll
        for (int j = 0; j < PPR; ++j) issue_pass(j, j * CPL);
    }
    // The read copy, its fp8 row scales and (for Mamba-2) the queries are not
    // written by the prep kernel.  When no flush kernel runs in this call and the
    // queries are the caller's input, every round of the stream is dotted before
    // the prep kernel's hand-off is awaited; otherwise it is awaited here.
    const bool stream_first = a.early && a.q_ready;
    if (!stream_first) pdl_wait();  // the prep kernel's hand-off is complete and visible

    // Queries: one row for the CTA when its heads share a query row (Mamba-2
    // groups), else one per head; fp8 row scales.
    const bool shared_q = (h0 / a.q_group) == ((h0 + HC - 1) / a.q_group);
    const int nq = shared_q ? 1 : HC;
    auto stage_queries = [&]() {
        for (int i = tid; i < nq * T * N; i += kThreads) {
            const int hq = i / (T * N), r2 = i - hq * T * N;
            const int m = r2 / N, n = r2 - m * N;
            const int64_t qi = (int64_t)b * a.q_stride_b + (int64_t)((h0 + hq) / a.q_group) * a.q_stride_row +
                               (int64_t)m * a.q_stride_m + n;
            sq[(hq * TQ + m) * N + n] = a.q_bf16 ? bf16_bits_to_float(reinterpret_cast<const uint16_t *>(a.Q)[qi])
                                                 : reinterpret_cast<const float *>(a.Q)[qi];
        }
        if (RK == SK_FP8)
            for (int i = tid; i < nrows / 4; i += kThreads) cp_async16(ssc + 4 * i, a.rc_scale + row0 * P + 4 * i);
    };
    // The prep kernel's hand-off: per-sequence info (and the counters it read,
    // rewritten by the sequence's first CTA), the call's entries, decays and the
    // coefficient rows of the CTA's heads (contiguous).
    auto stage_handoff = [&]() {
        if (tid == 0) {
            const int4 si = a.seqinfo[b];
            sinfo[0] = si.x; sinfo[1] = si.y; sinfo[2] = si.z;
            // Every prep CTA has read the counters (the prep kernel has completed),
            // so the first CTA of the sequence rewrites them.
            if (blockIdx.x == 0 && b == 0) *a.fold_count = 0;  // the flush kernel has run
            if (blockIdx.x == 0 && si.w) {
                const int64_t sp = a.c.seq_pos[b];
                if (si.z) {
                    a.c.ckpt_pos[b] = sp;
                    a.c.flush_count[b] += 1;
                }
                if (a.op == OP_DECODE) a.c.seq_pos[b] = sp + 1;
                else a.c.pending[b] = T;
            }
        }
        for (int row = warp; row < T * HC; row += kWarps) {  // x of token m, head hh
            const int m = row / HC, hh = row - m * HC;
            const uint8_t *src = reinterpret_cast<const uint8_t *>(a.xnew) + (((int64_t)(b * T + m) * H + h0 + hh) * P) * IB;
            for (int k = lane; k < xch; k += 32) cp_async16(sx + (hh * E + W + m) * xrow + k * 16, src + k * 16);
        }
        {  // rows m < T of each head's [TQmax][Ep] table, to [HC][TQ][Ep]
            const int per = T * Ep / 4;  // 16-byte chunks per head
            for (int i = tid; i < HC * per; i += kThreads) {
                const int hh = i / per, j = i - hh * per;
                cp_async16(scoef + hh * TQ * Ep + 4 * j, a.coef + (row0 + hh) * a.TQmax * Ep + 4 * j);
            }
        }
        for (int i = tid; i < HC * T; i += kThreads) {
            const int hh = i / T, m = i - hh * T;
            sdec[hh * TQ + m] = a.dec[(row0 + hh) * a.TQmax + m];
        }
    };
    // The rows dotted with their query, round after round of the copy.  A round
    // is two halves; a half's next chunks go out as soon as it has been dotted,
    // so the other half's loads are in flight while it is.
    auto dot_pass = [&](int pass, int off) {
        const int r = pass * RPP + rrow;
        const bool valid = r < nrows;
        float acc[TQ];
#pragma unroll
        for (int m = 0; m < TQ; ++m) acc[m] = 0.f;
        const float *qv = sq + (shared_q ? 0 : (valid ? r / P : 0)) * TQ * N;
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            float v[EPC];
            if (valid) unpack<RK>(rv[off + k], v);
            else {
#pragma unroll
                for (int e = 0; e < EPC; ++e) v[e] = 0.f;
            }
            const int c0 = (q + LPR * k) * EPC;
#pragma unroll
            for (int m = 0; m < TQ; ++m) {
                const float4 *q4 = reinterpret_cast<const float4 *>(qv + m * N + c0);
#pragma unroll
                for (int e4 = 0; e4 < EPC / 4; ++e4) {
                    const float4 w = q4[e4];
                    acc[m] = fmaf(v[4 * e4], w.x, acc[m]);
                    acc[m] = fmaf(v[4 * e4 + 1], w.y, acc[m]);
                    acc[m] = fmaf(v[4 * e4 + 2], w.z, acc[m]);
                    acc[m] = fmaf(v[4 * e4 + 3], w.w, acc[m]);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < TQ; ++m) {
            const float d = group_sum<LPR>(acc[m]);
            if (q == 0 && valid && m < T)
                sdot[r * TQ + m] = (RK == SK_FP8) ? d * ssc[r] : d;
        }
    };
    auto stream = [&]() {
        constexpr int HP = PPR / 2;  // passes in a round's first half (0: one pass per round)
        const int npass = (nrows + RPP - 1) / RPP;
        for (int p0 = 0; p0 < npass; p0 += PPR) {
            const bool more = p0 + PPR < npass;
#pragma unroll
            for (int j = 0; j < HP; ++j) dot_pass(p0 + j, j * CPL);
            if (more) {
#pragma unroll
                for (int j = 0; j < HP; ++j) issue_pass(p0 + PPR + j, j * CPL);
            }
#pragma unroll
            for (int j = HP; j < PPR; ++j) dot_pass(p0 + j, j * CPL);
            if (more) {
#pragma unroll
                for (int j = HP; j < PPR; ++j) issue_pass(p0 + PPR + j, j * CPL);
            }
        }
    };

    if (stream_first) {
        stage_queries();
        cp_async_wait_all();  // fp8 row scales
        __syncthreads();
        stream();
        pdl_wait();  // the prep kernel's hand-off is complete and visible
        stage_handoff();
        __syncthreads();
    } else {
        stage_handoff();
        stage_queries();
        __syncthreads();
    }
    const int L0 = sinfo[0], ckmod = sinfo[1], folded = sinfo[2];
    if (folded) {  // served by the flush kernel
        cp_async_wait_all();
        return;
    }
    const int base = W - L0;
    const int n1 = min(L0, R - ckmod);  // buffered entries before the ring wraps
    for (int row = warp; row < 2 * HC; row += kWarps) {  // two contiguous runs of slots per head
        const int hh = row >> 1, second = row & 1;
        const int cnt = second ? L0 - n1 : n1;
        const uint8_t *src = reinterpret_cast<const uint8_t *>(a.xring) +
                             (((row0 + hh) * R + (second ? 0 : ckmod)) * P) * IB;
        uint8_t *dst = sx + (hh * E + base + (second ? n1 : 0)) * xrow;
        for (int k = lane; k < cnt * xch; k += 32) cp_async16(dst + k * 16, src + k * 16);
    }
    if (!stream_first) {
        if (RK == SK_FP8) {  // the row scales must have landed before the first dot is scaled
            cp_async_wait_all();
            __syncthreads();
        }
        stream();
    }
    cp_async_wait_all();
    __syncthreads();

    // 4. y = dec * (S^ . Q) + replay term (+ D x).
    for (int i = tid; i < T * nrows; i += kThreads) {
        const int m = i / nrows, r2 = i - m * nrows;
        const int hh = r2 / P, p = r2 - hh * P;
        float yv = sdec[hh * TQ + m] * sdot[r2 * TQ + m];
        const float *cf = scoef + (hh * TQ + m) * Ep;
        const uint8_t *xs = sx + (hh * E + base) * xrow + p * IB;
        for (int e = 0; e <= L0 + m; ++e) {
            const float xv = BF ? bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(xs + e * xrow))
                                : *reinterpret_cast<const float *>(xs + e * xrow);
            yv = fmaf(cf[e], xv, yv);
        }
        if (a.D) {
            const uint8_t *xn = sx + (hh * E + W + m) * xrow + p * IB;
            const float xv = BF ? bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(xn))
                                : *reinterpret_cast<const float *>(xn);
            yv = fmaf(a.D[h0 + hh], xv, yv);
        }
        a.y[((int64_t)(b * T + m) * H + h0 + hh) * P + p] = yv;
    }
}

// Host-side launch of one instantiation, and the per-dstate entry point (each
// dstate is compiled in its own translation unit, rssm_read_n*.cu).
template <int N, int RK, int TQ>
inline cudaError_t launch_read_t(const ReadArgs &r, size_t smem, cudaStream_t st) {
    auto k = r.in_bf16 ? replay_read_kernel<N, RK, TQ, true> : replay_read_kernel<N, RK, TQ, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(r.H / r.HC, r.B);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = r.pdl ? 1 : 0;  // a programmatic dependent of the prep kernel
    return cudaLaunchKernelEx(&cfg, k, r);
}

template <int N>
cudaError_t read_dispatch_n(int rk, int TQ, const ReadArgs &r, size_t smem, cudaStream_t st) {
    if (TQ == 1) {
        if (rk == SK_F32) return launch_read_t<N, SK_F32, 1>(r, smem, st);
        if (rk == SK_BF16) return launch_read_t<N, SK_BF16, 1>(r, smem, st);
        return launch_read_t<N, SK_FP8, 1>(r, smem, st);
    }
    if (TQ == 4) {
        if (rk == SK_F32) return launch_read_t<N, SK_F32, 4>(r, smem, st);
        if (rk == SK_BF16) return launch_read_t<N, SK_BF16, 4>(r, smem, st);
        return launch_read_t<N, SK_FP8, 4>(r, smem, st);
    }
    if (rk == SK_F32) return launch_read_t<N, SK_F32, 8>(r, smem, st);
    if (rk == SK_BF16) return launch_read_t<N, SK_BF16, 8>(r, smem, st);
    return launch_read_t<N, SK_FP8, 8>(r, smem, st);
}

}  // namespace rssm
