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
#include "rssm_pipe.cuh"

namespace rssm {

struct M2Args {
    int B, H, P, G, W, R, Rs, T, op, in_bf16, dt_scales;  // Rs: dt ring row length
    int HC;             // heads per replay item (divides H / G)
    int NS;             // pipeline stages of the replay kernel
    int grid;           // persistent CTAs of the replay kernel
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

__host__ __device__ constexpr int a16(int v) { return (v + 15) & ~15; }
__host__ __device__ constexpr int pad4(int n) { return (n + 3) & ~3; }

// One pipeline stage of the persistent replay kernel (bytes, 16-byte aligned
// regions).  A stage carries one unit of work: the state tile of an item (the
// read copy of HC heads, or one part of their fp32 checkpoint when the item
// folds) plus everything the item needs from the ring and from this call's
// tokens.  Entry slots: E = W + TQ; committed entries sit right-aligned before
// slot W and this call's tokens at W..W+T-1.
struct M2Stage {
    int tile, scale, x, B, C, dt, dtn, info, bytes;
};
// Upper bound of a dt ring row in bytes: the ring has R = W + max(max_draft, 1) <= W + 8
// slots, rows padded to 4 floats.
__host__ __device__ constexpr int dt_row_max_bytes(int W) { return ((W + 8 + 3) & ~3) * 4; }
constexpr int kTileCap = 32 * 1024;  // bytes of state rows per pipeline unit

__host__ __device__ inline M2Stage m2_stage(int HC, int P, int N, int W, int TQ, int ib, int rcb) {
    const int E = W + TQ;
    M2Stage S{};
    int o = 0;
    S.tile = o;  o += kTileCap;                                  // state rows of the unit
    S.scale = o; o += (rcb == 1) ? a16(kTileCap / N * 4) : 0;    // fp8 row scales
    S.x = o;     o += a16(HC * E * P * ib);            // x of entries   [HC][E][P]
    S.B = o;     o += a16(E * N * ib);                 // B of entries   [E][N]
    S.C = o;     o += a16(TQ * N * ib);                // C of queries   [TQ][N]
    S.dt = o;    o += a16(HC * dt_row_max_bytes(W));   // dt ring rows   [HC][Rs]
    S.dtn = o;   o += a16(TQ * HC * 4);                // dt of this call's tokens [TQ][HC]
    S.info = o;  o += 64;                              // unit descriptor
    S.bytes = o;
    return S;
}

// Consumer-side scratch, shared by all units (bytes).
struct M2Scratch {
    int sd, slam, scoef, sdec, su, sfdec, sdot, sCf, pdt, bytes;
};
__host__ __device__ inline M2Scratch m2_scratch(int HC, int P, int N, int W, int TQ) {
    const int E = W + TQ;
    M2Scratch S{};
    int o = 0;
    S.sd = o;    o += a16(TQ * E * 4);       // B_e . C_m             [TQ][E]
    S.slam = o;  o += a16(HC * E * 4);       // prefix sums of dt*A   [HC][E]
    S.scoef = o; o += a16(HC * TQ * E * 4);  // replay coefficients   [HC][TQ][E]
    S.sdec = o;  o += a16(HC * TQ * 4);      // decay of S^ C         [HC][TQ]
    S.su = o;    o += a16(HC * E * 4);       // fold weights          [HC][E]
    S.sfdec = o; o += a16(HC * 4);           // decay of the folded checkpoint [HC]
    S.sdot = o;  o += a16(HC * P * TQ * 4);  // S^ C per state row    [HC*P][TQ]
    S.sCf = o;   o += a16(TQ * N * 4);       // C as fp32             [TQ][N]
    S.pdt = o;   o += a16(32 * HC * TQ * 4); // producer: dt of its 32 prefetched items
    S.bytes = o;
    return S;
}

__host__ __device__ inline int m2_smem_total(int NS, int HC, int P, int N, int W, int TQ, int ib, int rcb) {
    return 16 * NS + NS * m2_stage(HC, P, N, W, TQ, ib, rcb).bytes + m2_scratch(HC, P, N, W, TQ).bytes;
}

enum { INFO_ITEM = 0, INFO_PART, INFO_NPARTS, INFO_L0, INFO_FLUSH, INFO_CKMOD, INFO_SPMOD };

// ---------------------------------------------------------------------------
// Replay kernel: decode (T = 1), verify (T = K), flush (T = 0), export (T = 0).
//
// Persistent: one CTA per SM walks the items (sequence b, group g, chunk of HC
// heads of the group; the HC state tiles are contiguous) with stride gridDim.
// Warp 8 is the producer: for each item it reads the sequence counters, decides
// whether the item folds, and fills the next free stage of an NS-deep ring in
// shared memory with bulk copies (the read-copy tile, or the fp32 checkpoint in
// parts when folding, plus the buffered entries and this call's tokens), so up
// to NS tiles are in flight while the eight consumer warps work.  Consumers,
// per unit: B_e . C_m and per-head prefix sums of the log decays (first part of
// an item), then either the read-copy rows dotted with C or the fold of the
// checkpoint rows (stored with the requantised copy), then outputs and ring
// appends (last part), and release the stage.  Every barrier wait is bounded.
// ---------------------------------------------------------------------------
template <int N, int RK, int TQ>
__global__ void __maxnreg__(112) m2_replay_kernel(const M2Args a) {
    constexpr int EPC = Chunk<RK>::EPC;    // stored elements per 16-byte chunk
    constexpr int TPR = N / EPC;           // lanes per state row, read mapping
    constexpr int RCB = Chunk<RK>::BYTES;  // bytes per stored element
    constexpr int TPR4 = N / 4;            // lanes per row, fp32 quad mapping (fold)
    constexpr int RPP4 = kThreads / TPR4;
    static_assert(TPR >= 1 && TPR <= 32 && (32 % TPR) == 0, "row must fit a warp");

    extern __shared__ __align__(128) uint8_t smraw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, P = a.P, W = a.W, R = a.R, T = a.T, G = a.G, HC = a.HC, NS = a.NS;
    const int hpg = H / G, cpg = hpg / HC;
    const int E = W + TQ;
    const int bf = a.in_bf16, ib = bf ? 2 : 4;
    const int nrows = HC * P;
    const bool reads = (a.op == OP_DECODE || a.op == OP_VERIFY);
    const int rpp_read = kTileCap / (N * RCB);  // read-copy rows per unit
    const int rpp_fold = kTileCap / (N * 4);    // fp32 checkpoint rows per unit
    const int read_parts = (nrows + rpp_read - 1) / rpp_read;
    const int fold_parts = (nrows + rpp_fold - 1) / rpp_fold;
    const int xrow = P * ib, brow = N * ib;
    const M2Stage SG = m2_stage(HC, P, N, W, TQ, ib, RCB);
    const M2Scratch SC = m2_scratch(HC, P, N, W, TQ);
    uint64_t *full = reinterpret_cast<uint64_t *>(smraw);
    uint64_t *empty = full + NS;
    uint8_t *stages = smraw + 16 * NS;
    uint8_t *scr = stages + NS * SG.bytes;
    const int nitems = a.B * (H / HC);

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 32);       // the producer warp's lanes (+ bulk-copy bytes)
            mbar_init(&empty[i], kWarps);  // one arrival per consumer warp
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == kWarps) {
        // ================================ producer ================================
        // Items are taken 32 at a time: lane j loads the counters and the token dt's
        // of the j-th item of the batch (one memory round trip per 32 items); then
        // the items' units are queued in order.
        float *pdt = reinterpret_cast<float *>(scr + SC.pdt);
        const int HT = HC * T;
        const int nper = H / HC;  // items per sequence
        int s = 0;
        uint32_t used = 0, ephase = 0;
        bool dead = false;
        auto acquire = [&](int st) -> bool {  // warp-uniform
            if (used & (1u << st)) {
                int got = 0;
                if (lane == 0) got = mbar_wait(&empty[st], (ephase >> st) & 1u) ? 1 : 0;
                got = __shfl_sync(0xffffffffu, got, 0);
                __syncwarp();
                if (!got) return false;
                ephase ^= 1u << st;
            }
            used |= 1u << st;
            return true;
        };
        for (int bstart = blockIdx.x; bstart < nitems && !dead; bstart += 32 * gridDim.x) {
            const int mine = bstart + lane * gridDim.x;
            int ok = 0, L0 = 0, flush = 0, ckmod = 0, spmod = 0;
            if (mine < nitems) {
                const int b = mine / nper, rem = mine - b * nper;
                const int g = rem / cpg, hc = rem - g * cpg, h0 = g * hpg + hc * HC;
                for (int i = 0; i < HT; ++i) {
                    const int m = i / HC, hh = i - m * HC;
                    pdt[lane * HT + i] = a.dt[(int64_t)(b * T + m) * H + h0 + hh];
                }
                SeqState ss = read_counters(a.c, b, W);
                ok = ss.ok;
                L0 = (int)(ss.seq - ss.ckpt);
                if (ok) flush = (a.op == OP_FLUSH || a.op == OP_EXPORT) ? (L0 > 0) : (L0 + T > W);
                ckmod = (int)(ss.ckpt % R);
                spmod = (int)(ss.seq % R);
                if (!ok && g == 0 && hc == 0) report(a.c.err, DEV_BAD_COUNTERS, b, h0, L0);
            }
            __syncwarp();
            for (int j = 0; j < 32 && !dead; ++j) {
                const int item = bstart + j * gridDim.x;
                if (item >= nitems) break;
                const int iok = __shfl_sync(0xffffffffu, ok, j);
                const int iL0 = __shfl_sync(0xffffffffu, L0, j);
                const int ifl = __shfl_sync(0xffffffffu, flush, j);
                const int ick = __shfl_sync(0xffffffffu, ckmod, j);
                const int isp = __shfl_sync(0xffffffffu, spmod, j);
                const int b = item / nper, rem = item - b * nper;
                const int g = rem / cpg, hc = rem - g * cpg, h0 = g * hpg + hc * HC;
                const int64_t row0 = (int64_t)b * H + h0;
                const int64_t tile0 = row0 * P * N;
                const int nparts = !iok ? 0 : (ifl ? fold_parts : (reads ? read_parts : 0));
                const int base = W - iL0;
                const int n1 = min(iL0, R - ick);  // entries before the ring wraps
                for (int part = 0; part < nparts; ++part) {
                    if (!acquire(s)) {
                        if (lane == 0) report(a.c.err, DEV_PIPE_TIMEOUT, b, h0, 1);
                        dead = true;
                        break;
                    }
                    uint8_t *st = stages + s * SG.bytes;
                    int *info = reinterpret_cast<int *>(st + SG.info);
                    float *dtn = reinterpret_cast<float *>(st + SG.dtn);
                    if (lane == 0) {
                        info[INFO_ITEM] = item; info[INFO_PART] = part; info[INFO_NPARTS] = nparts;
                        info[INFO_L0] = iL0; info[INFO_FLUSH] = ifl; info[INFO_CKMOD] = ick;
                        info[INFO_SPMOD] = isp;
                    }
                    for (int i = lane; i < HT; i += 32) dtn[i] = pdt[j * HT + i];
                    // The unit's bulk copies: the same list is walked twice, once to
                    // total the bytes, once to issue (copy k by lane k mod 32).
                    uint32_t tx = 0;
                    int ci = 0;
                    auto copy = [&](bool issue, void *dst, const void *src, uint32_t bytes) {
                        if (bytes == 0) return;
                        if (!issue) tx += bytes;
                        else if ((ci & 31) == lane) bulk_g2s(dst, src, bytes, &full[s]);
                        ++ci;
                    };
                    auto walk = [&](bool issue) {
                        ci = 0;
                        if (ifl) {
                            const int r0 = part * rpp_fold, r1 = min(nrows, r0 + rpp_fold);
                            copy(issue, st + SG.tile, a.ckpt + tile0 + (int64_t)r0 * N, (uint32_t)((r1 - r0) * N * 4));
                        } else {
                            const int r0 = part * rpp_read, r1 = min(nrows, r0 + rpp_read);
                            const uint8_t *rc = (RK == SK_F32) ? reinterpret_cast<const uint8_t *>(a.ckpt + tile0)
                                                               : reinterpret_cast<const uint8_t *>(a.rc) + tile0 * RCB;
                            copy(issue, st + SG.tile, rc + (int64_t)r0 * N * RCB, (uint32_t)((r1 - r0) * N * RCB));
                            if (RK == SK_FP8)
                                copy(issue, st + SG.scale, a.rc_scale + row0 * P + r0, (uint32_t)((r1 - r0) * 4));
                        }
                        copy(issue, st + SG.dt, a.dtbuf + row0 * a.Rs, (uint32_t)(HC * a.Rs * 4));
                        const uint8_t *Bb = reinterpret_cast<const uint8_t *>(a.Bbuf) + ((int64_t)(b * G + g) * R) * brow;
                        copy(issue, st + SG.B + base * brow, Bb + (int64_t)ick * brow, (uint32_t)(n1 * brow));
                        copy(issue, st + SG.B + (base + n1) * brow, Bb, (uint32_t)((iL0 - n1) * brow));
                        for (int hh = 0; hh < HC; ++hh) {
                            const uint8_t *xb = reinterpret_cast<const uint8_t *>(a.xbuf) + ((row0 + hh) * R) * xrow;
                            uint8_t *xd = st + SG.x + (hh * E + base) * xrow;
                            copy(issue, xd, xb + (int64_t)ick * xrow, (uint32_t)(n1 * xrow));
                            copy(issue, xd + n1 * xrow, xb, (uint32_t)((iL0 - n1) * xrow));
                        }
                        for (int m = 0; m < T; ++m) {
                            const int64_t gsrc = (((int64_t)(b * T + m) * G + g) * N) * ib;
                            copy(issue, st + SG.C + m * brow, reinterpret_cast<const uint8_t *>(a.Cm) + gsrc, (uint32_t)brow);
                            copy(issue, st + SG.B + (W + m) * brow, reinterpret_cast<const uint8_t *>(a.Bm) + gsrc, (uint32_t)brow);
                            const uint8_t *xs = reinterpret_cast<const uint8_t *>(a.x) + (((int64_t)(b * T + m) * H + h0) * P) * ib;
                            for (int hh = 0; hh < HC; ++hh)
                                copy(issue, st + SG.x + (hh * E + W + m) * xrow, xs + hh * xrow, (uint32_t)xrow);
                        }
                    };
                    walk(false);
                    if (lane == 0) mbar_arrive_expect_tx(&full[s], tx);
                    else mbar_arrive(&full[s]);
                    __syncwarp();
                    walk(true);
                    s = (s + 1 == NS) ? 0 : s + 1;
                }
            }
        }
        if (!dead && acquire(s)) {  // end-of-work unit
            if (lane == 0) reinterpret_cast<int *>(stages + s * SG.bytes + SG.info)[INFO_ITEM] = -1;
            mbar_arrive(&full[s]);
        } else if (lane == 0 && !dead) {
            report(a.c.err, DEV_PIPE_TIMEOUT, -1, -1, 2);
        }
        // Counters: every CTA has read all of its items' counters by now; the last
        // CTA to get here publishes the new counters of every sequence.
        if (a.op != OP_EXPORT) {
            int last = 0;
            if (lane == 0) {
                __threadfence();
                last = (atomicAdd(&a.c.err[4], 1) == (int)gridDim.x - 1) ? 1 : 0;
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                __threadfence();
                for (int b = lane; b < a.B; b += 32) {
                    SeqState ss = read_counters(a.c, b, W);
                    if (!ss.ok) continue;
                    const int L0 = (int)(ss.seq - ss.ckpt);
                    const int flush = (a.op == OP_FLUSH) ? (L0 > 0) : (L0 + T > W);
                    if (flush) {
                        a.c.ckpt_pos[b] = ss.seq;
                        a.c.flush_count[b] += 1;
                    }
                    if (a.op == OP_DECODE) a.c.seq_pos[b] = ss.seq + 1;
                    if (a.op == OP_VERIFY) a.c.pending[b] = T;
                }
                __syncwarp();
                if (lane == 0) a.c.err[4] = 0;
                __threadfence();
            }
        }
        return;
    }

    // ================================ consumers ================================
    float *sd = reinterpret_cast<float *>(scr + SC.sd);
    float *slam = reinterpret_cast<float *>(scr + SC.slam);
    float *scoef = reinterpret_cast<float *>(scr + SC.scoef);
    float *sdec = reinterpret_cast<float *>(scr + SC.sdec);
    float *su = reinterpret_cast<float *>(scr + SC.su);
    float *sfdec = reinterpret_cast<float *>(scr + SC.sfdec);
    float *sdot = reinterpret_cast<float *>(scr + SC.sdot);
    float *sCf = reinterpret_cast<float *>(scr + SC.sCf);
    // read mapping: LPR lanes per state row, CPL chunks per lane, rotated so the
    // rows of a warp spread over all shared-memory banks
    constexpr int LPR = TPR < 4 ? TPR : 4;
    constexpr int CPL = TPR / LPR;
    constexpr int RPPR = kThreads / LPR;
    constexpr bool kCregs = TQ * CPL * EPC <= 32;
    const int q = tid % LPR, rrow = tid / LPR, rot = rrow % CPL;
    // fold mapping: TPR4 lanes per row (quads), FR rows per thread per unit
    constexpr int FR = 8;  // = (kTileCap / (N * 4)) / RPP4 for every N
    static_assert(FR * RPP4 * N * 4 == kTileCap, "fold unit is FR rows per thread");
    const int c4 = tid % TPR4, q0 = tid / TPR4;
    int s = 0;
    uint32_t fphase = 0;
    for (;;) {
        const bool got = mbar_wait(&full[s], (fphase >> s) & 1u);
        if (consumer_sync_any(!got)) {
            if (tid == 0) report(a.c.err, DEV_PIPE_TIMEOUT, -1, -1, 3);
            break;
        }
        fphase ^= 1u << s;
        const uint8_t *st = stages + s * SG.bytes;
        const int *info = reinterpret_cast<const int *>(st + SG.info);
        const int item = info[INFO_ITEM];
        if (item < 0) break;
        const int part = info[INFO_PART], nparts = info[INFO_NPARTS];
        const int L0 = info[INFO_L0], flush = info[INFO_FLUSH], spmod = info[INFO_SPMOD];
        const int ckmod = info[INFO_CKMOD];
        const int b = item / (H / HC);
        const int rem = item - b * (H / HC);
        const int g = rem / cpg, hc = rem - g * cpg;
        const int h0 = g * hpg + hc * HC;
        const int64_t row0 = (int64_t)b * H + h0;
        const int64_t tile0 = row0 * P * N;
        const int base = W - L0, nE = L0 + T;
        const int e0 = flush ? L0 : 0;  // first entry the outputs replay
        const uint8_t *sx = st + SG.x;
        const uint8_t *sB = st + SG.B;
        const uint8_t *sC = st + SG.C;
        const float *dring = reinterpret_cast<const float *>(st + SG.dt);
        const float *dtn = reinterpret_cast<const float *>(st + SG.dtn);
        // dt of logical entry e (committed entries from the ring, then this call's tokens)
        auto dt_of = [&](int hh, int e) -> float {
            return e < L0 ? dring[hh * a.Rs + (ckmod + e) % R] : dtn[(e - L0) * HC + hh];
        };

        if (part == 0) {
            // B_e . C_m once per item; C to fp32; prefix sums of dt*A per head.
            if (reads) {
                for (int pr = warp; pr < T * nE; pr += kWarps) {
                    const int m = pr / nE, e = pr - m * nE;
                    if (e < e0 || e > L0 + m) continue;  // warp-uniform
                    float d = 0.f;
                    for (int n = lane; n < N; n += 32)
                        d = fmaf(raw_f(sB + (base + e) * brow, n, bf), raw_f(sC + m * brow, n, bf), d);
                    d = group_sum<32>(d);
                    if (lane == 0) sd[m * E + e] = d;
                }
                for (int i = tid; i < T * N; i += kThreads) sCf[i] = raw_f(sC, i, bf);
            }
            for (int hh = warp; hh < HC; hh += kWarps) {
                const float Ah = a.A[h0 + hh];
                float carry = 0.f;
                for (int k0 = 0; k0 < nE; k0 += 32) {
                    const int e = k0 + lane;
                    float v = (e < nE) ? dt_of(hh, e) * Ah : 0.f;
                    v = warp_incl_scan(v) + carry;
                    if (e < nE) slam[hh * E + base + e] = v;
                    carry = __shfl_sync(0xffffffffu, v, 31);
                }
            }
            consumer_sync();
            for (int i = tid; i < HC * nE; i += kThreads) {
                const int hh = i / nE, e = i - hh * nE;
                const float *lam = slam + hh * E + base;
                const float se = a.dt_scales ? dt_of(hh, e) : 1.f;
                if (reads) {
#pragma unroll
                    for (int m = 0; m < TQ; ++m)
                        if (m < T && e >= e0 && e <= L0 + m)
                            scoef[(hh * TQ + m) * E + e] = expf(lam[L0 + m] - lam[e]) * sd[m * E + e] * se;
                }
                if (flush && e < L0) su[hh * E + e] = expf(lam[L0 - 1] - lam[e]) * se;
            }
            for (int i = tid; i < HC; i += kThreads) {
                const float *lam = slam + i * E + base;
                sfdec[i] = flush ? expf(lam[L0 - 1]) : 1.f;
#pragma unroll
                for (int m = 0; m < TQ; ++m)
                    if (reads && m < T) sdec[i * TQ + m] = expf(lam[L0 + m] - (flush ? lam[L0 - 1] : 0.f));
            }
            consumer_sync();
        }

        if (flush) {
            // Fold this part's fp32 checkpoint rows (staged), FR rows per thread held
            // in registers, buffered B applied 8 entries at a time; store the
            // checkpoint and the requantised copy, dot the fresh copy with C.
            const int r0 = part * rpp_fold, nr = min(nrows, r0 + rpp_fold) - r0;
            const float *tf = reinterpret_cast<const float *>(st + SG.tile);
            float4 Cq[TQ];
#pragma unroll
            for (int m = 0; m < TQ; ++m)
                Cq[m] = (reads && m < T) ? *reinterpret_cast<const float4 *>(sCf + m * N + 4 * c4)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
            constexpr int FH = 4;  // rows in registers at a time
#pragma unroll 1
            for (int kh = 0; kh < FR; kh += FH) {
                float4 v[FH];
#pragma unroll
                for (int k = 0; k < FH; ++k) {
                    const int rl = q0 + (kh + k) * RPP4;
                    v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (rl < nr) {
                        v[k] = *reinterpret_cast<const float4 *>(tf + rl * N + 4 * c4);
                        const float dc = sfdec[(r0 + rl) / P];
                        v[k].x *= dc; v[k].y *= dc; v[k].z *= dc; v[k].w *= dc;
                    }
                }
#pragma unroll 1
                for (int eb = 0; eb < L0; eb += 8) {
                    float4 Bq[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint8_t *Br = sB + (base + eb + j) * brow;
                        Bq[j] = (eb + j < L0) ? make_float4(raw_f(Br, 4 * c4, bf), raw_f(Br, 4 * c4 + 1, bf),
                                                            raw_f(Br, 4 * c4 + 2, bf), raw_f(Br, 4 * c4 + 3, bf))
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int k = 0; k < FH; ++k) {
                        const int rl = q0 + (kh + k) * RPP4;
                        if (rl >= nr) continue;
                        const int gr = r0 + rl, hh = gr / P, p = gr - hh * P;
                        const uint8_t *xr = sx + (hh * E + base + eb) * xrow;
                        const float *uw = su + hh * E + eb;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            if (eb + j < L0) {
                                const float w = uw[j] * raw_f(xr + j * xrow, p, bf);
                                v[k].x = fmaf(w, Bq[j].x, v[k].x); v[k].y = fmaf(w, Bq[j].y, v[k].y);
                                v[k].z = fmaf(w, Bq[j].z, v[k].z); v[k].w = fmaf(w, Bq[j].w, v[k].w);
                            }
                        }
                    }
                }
#pragma unroll
                for (int k = 0; k < FH; ++k) {
                    const int rl = q0 + (kh + k) * RPP4;
                    const bool valid = rl < nr;
                    const int gr = r0 + rl;
                    const int64_t el = tile0 + (int64_t)(valid ? gr : 0) * N + 4 * c4;
                    if (a.op == OP_EXPORT) {
                        if (valid) *reinterpret_cast<float4 *>(a.out + el) = v[k];
                        continue;
                    }
                    if (valid) *reinterpret_cast<float4 *>(a.ckpt + el) = v[k];
                    float4 rd = v[k];
                    if (RK == SK_BF16) {
                        if (valid) rd = store_quad<SK_BF16>(a.rc, el, v[k], 0.f, 0.f);
                    } else if (RK == SK_FP8) {
                        float am = fmaxf(fmaxf(fabsf(v[k].x), fabsf(v[k].y)), fmaxf(fabsf(v[k].z), fabsf(v[k].w)));
                        am = group_max<TPR4>(am);
                        const float sc = fp8_scale(am);
                        if (valid) {
                            rd = store_quad<SK_FP8>(a.rc, el, v[k], 0.f, sc);
                            if (c4 == 0) a.rc_scale[row0 * P + gr] = sc;
                        }
                    }
                    if (reads) {
#pragma unroll
                        for (int m = 0; m < TQ; ++m) {
                            float d = rd.x * Cq[m].x + rd.y * Cq[m].y + rd.z * Cq[m].z + rd.w * Cq[m].w;
                            d = group_sum<TPR4>(d);
                            if (c4 == 0 && valid && m < T) sdot[gr * TQ + m] = d;
                        }
                    }
                }
            }
        } else if (reads) {
            // Read: LPR lanes per staged read-copy row, C fragments in registers.
            float Cf[kCregs ? TQ : 1][kCregs ? CPL * EPC : 1];
            if (kCregs) {
#pragma unroll
                for (int m = 0; m < (kCregs ? TQ : 1); ++m)
#pragma unroll
                    for (int k = 0; k < (kCregs ? CPL : 1); ++k)
#pragma unroll
                        for (int e = 0; e < (kCregs ? EPC : 1); ++e)
                            Cf[m][k * EPC + e] =
                                (m < T) ? sCf[m * N + (q + LPR * ((k + rot) % CPL)) * EPC + e] : 0.f;
            }
            const uint4 *tile = reinterpret_cast<const uint4 *>(st + SG.tile);
            const float *ssc = reinterpret_cast<const float *>(st + SG.scale);
            const int r0 = part * rpp_read, nr = min(nrows, r0 + rpp_read) - r0;
            for (int rb = 0; rb < nr; rb += RPPR) {  // same trip count for every lane
                const int rl = rb + rrow;
                const bool valid = rl < nr;
                float acc[TQ];
#pragma unroll
                for (int m = 0; m < TQ; ++m) acc[m] = 0.f;
#pragma unroll
                for (int k = 0; k < CPL; ++k) {
                    const int ch = q + LPR * ((k + rot) % CPL);
                    float vv[EPC];
                    if (valid) unpack<RK>(tile[rl * TPR + ch], vv);
                    else {
#pragma unroll
                        for (int e = 0; e < EPC; ++e) vv[e] = 0.f;
                    }
#pragma unroll
                    for (int m = 0; m < TQ; ++m)
#pragma unroll
                        for (int e = 0; e < EPC; ++e)
                            acc[m] = fmaf(vv[e], kCregs ? Cf[kCregs ? m : 0][kCregs ? k * EPC + e : 0]
                                                        : sCf[m * N + ch * EPC + e], acc[m]);
                }
#pragma unroll
                for (int m = 0; m < TQ; ++m) {
                    const float d = group_sum<LPR>(acc[m]);
                    if (q == 0 && valid && m < T)
                        sdot[(r0 + rl) * TQ + m] = (RK == SK_FP8) ? d * ssc[rl] : d;
                }
            }
        }

        if (reads && part == nparts - 1) {
            consumer_sync();
            // Outputs y[b, m, h0 + hh, :] and ring appends (slots seq_pos + m mod R).
            for (int i = tid; i < T * HC * P; i += kThreads) {
                const int m = i / (HC * P), r2 = i - m * HC * P;
                const int hh = r2 / P, p = r2 - hh * P;
                float yv = sdec[hh * TQ + m] * sdot[(hh * P + p) * TQ + m];
                const float *cf = scoef + (hh * TQ + m) * E;
                const uint8_t *xs = sx + (hh * E + base) * xrow;
                for (int e = e0; e <= L0 + m; ++e) yv = fmaf(cf[e], raw_f(xs + e * xrow, p, bf), yv);
                yv = fmaf(a.D[h0 + hh], raw_f(sx + (hh * E + W + m) * xrow, p, bf), yv);
                a.y[((int64_t)(b * T + m) * H + h0 + hh) * P + p] = yv;
            }
            const int xch = xrow / 16, bch = brow / 16;
            for (int i = tid; i < T * HC * xch; i += kThreads) {
                const int m = i / (HC * xch), r2 = i - m * HC * xch;
                const int hh = r2 / xch, k = r2 - hh * xch;
                const int slot = (spmod + m) % R;
                *reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(a.xbuf) + (((row0 + hh) * R + slot) * P) * ib + k * 16) =
                    *reinterpret_cast<const uint4 *>(sx + (hh * E + W + m) * xrow + k * 16);
            }
            if (tid < T * HC) {
                const int m = tid / HC, hh = tid - m * HC;
                a.dtbuf[(row0 + hh) * a.Rs + (spmod + m) % R] = dtn[m * HC + hh];
            }
            if (hc == 0) {  // the group's first item writes the group's B
                for (int i = tid; i < T * bch; i += kThreads) {
                    const int m = i / bch, k = i - m * bch;
                    const int slot = (spmod + m) % R;
                    *reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(a.Bbuf) + (((int64_t)(b * G + g) * R + slot) * N) * ib + k * 16) =
                        *reinterpret_cast<const uint4 *>(sB + (W + m) * brow + k * 16);
                }
            }
        }
        consumer_sync();  // every consumer is done with the stage
        if (lane == 0) mbar_arrive(&empty[s]);
        s = (s + 1 == NS) ? 0 : s + 1;
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
    k<<<a.grid, kThreads + 32, smem, st>>>(a);
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
