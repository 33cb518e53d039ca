// rssm_mamba2.cuh -- Mamba-2 decode kernels for sm_100a (templates; instantiated per dstate).
//
// Layer (per sequence b, head h, group g = h / (H/G)):
//   S_t = exp(dt_t A_h) S_{t-1} + (s_t x_t) B_t^T,   y_t = S_t C_t + D_h x_t
// Replay representation (ReplaySSM: the output comes from a checkpoint plus a
// buffer of recent inputs with no state write; the checkpoint is rewritten only
// when the buffer is full -- blog.thibaultmonteiro.fr, "Tenir le journal plutot
// que le solde").  With buffered entries e = 0..L-1 (the last being the token
// read) and prefix sums Lam_e = sum_{j<=e} dt_j A_h of the log decays:
//   y = e^{Lam_{L-1}} (S^ C) + sum_e e^{Lam_{L-1} - Lam_e} (B_e . C) s_e x_e + D x_{L-1}
//   fold: S_c <- e^{Lam_{L-1}} S_c + sum_e e^{Lam_{L-1} - Lam_e} s_e x_e B_e^T
// S^ is the read copy (bf16, per-row-scaled e4m3, or the fp32 checkpoint).
//
// A replay decode/verify runs this file's prep/flush kernel, which turns the
// buffer into per-head replay coefficients (and folds when the buffer is full),
// then the shared replay-read kernel (rssm_read.cuh).  The eager baseline below
// rewrites the whole state every token.
#pragma once
#include "rssm_device.cuh"
#include "rssm_pair.cuh"
#include "rssm_internal.h"
#include "rssm_pipe.cuh"
#include "rssm_read.cuh"

namespace rssm {

__host__ __device__ constexpr int a16(int v) { return (v + 15) & ~15; }
__host__ __device__ constexpr int pad4(int n) { return (n + 3) & ~3; }

// Upper bound of a dt ring row in bytes: the ring has R = W + max(max_draft, 1) <= W + 8
// slots, rows padded to 4 floats.
__host__ __device__ constexpr int dt_row_max_bytes(int W) { return ((W + 8 + 3) & ~3) * 4; }

constexpr int kFoldChunk = 16 * 1024;  // bytes of fp32 checkpoint rows per fold stage

// Shared memory of the prep kernel (bytes, 16-byte aligned regions), computed on
// the host.  The group's B ring is staged whole (R <= W + 8 rows).
struct M2PrepLay {
    int sC, sBr, sBn, sx, dring, dtn, sA, sd, slam, si, bytes;
};
inline M2PrepLay m2_prep_lay(int HC, int P, int N, int W, int TQ, int ib) {
    const int E = W + TQ;
    M2PrepLay L{};
    int o = 0;
    L.sC = o;    o += a16(TQ * N * ib);          // raw C of the queries     [TQ][N]
    L.sBr = o;   o += a16((W + 8) * N * ib);     // raw B ring of the group  [R][N]
    L.sBn = o;   o += a16(TQ * N * ib);          // raw B of the call's tokens [TQ][N]
    L.sx = o;    o += a16(TQ * HC * P * ib);     // raw x of the call's tokens [TQ][HC][P]
    L.dring = o; o += a16(HC * dt_row_max_bytes(W));  // dt ring rows        [HC][Rs]
    L.dtn = o;   o += a16(TQ * HC * 4);          // dt of the call's tokens  [TQ][HC]
    L.sA = o;    o += a16(HC * 4);               // A of the heads           [HC]
    L.sd = o;    o += a16(TQ * E * 4);           // B_e . C_m                [TQ][E]
    L.slam = o;  o += a16(HC * E * 4);           // prefix sums of dt*A      [HC][E]
    L.si = o;    o += 32;
    L.bytes = o;
    return L;
}

struct M2Args {
    int B, H, P, G, W, R, Rs, T, op, in_bf16, dt_scales;  // Rs: dt ring row length
    int HC, cpg;        // heads per CTA (divides H / G); CTAs per group
    M2PrepLay lay;      // prep kernel shared memory
    int4 *seqinfo;      // per sequence, for the read kernel: {L0, ring slot of entry 0, folded, valid}
    int *fold_count;    // sequences the flush kernel folds in this call (reset by the read kernel)
    int *fold_list;     // [B] their indices
    int fold_launched;  // the host launches the flush kernel in this call
    float *dec;         // [B][H][TQmax] decay of S^ C
    float *coef;        // [B][H][TQmax][Emax] replay coefficients
    int TQmax, Emax;    // Emax: padded row length of the coefficient table
    Counters c;
    const float *A, *D;
    float *ckpt;        // fp32 [B][H][P][N]
    void *rc;           // read copy / low-precision state [B][H][P][N]
    float *rc_scale;    // [B][H][P] (FP8)
    void *xbuf;         // [B][H][R][P]
    float *dtbuf;       // [B][H][Rs]
    void *Bbuf;         // [B][G][R][N]
    void *snap;         // eager verify snapshots
    float *snap_scale;
    const void *x;      // [B][T][H][P]
    const float *dt;    // [B][T][H]
    const void *Bm;     // [B][T][G][N]
    const void *Cm;     // [B][T][G][N]
    float *y;           // [B][T][H][P]
    float *out;         // export target [B][H][P][N]
};

// ---------------------------------------------------------------------------
// Prep kernel: decode (T = 1) and verify (T = K).
//
// One CTA per (group chunk of HC heads, sequence b).  In one round trip it reads
// the sequence's counters and stages the group's whole B ring, the heads' dt
// ring rows and the call's tokens.  A sequence whose buffer must be folded first
// (len + T > W) is left to the flush kernel (m2_fold_kernel).  Otherwise it
// computes B_e . C_m once for the group and, per head (one warp each), the
// prefix sums Lam of dt*A and the replay coefficients for the read kernel:
//     coef[m][e] = e^{Lam_{L0+m} - Lam_e} (B_e . C_m) s_e,   dec[m] = e^{Lam_{L0+m}}.
// Every sequence's tokens are appended to the ring (slots seq_pos + m mod R);
// the slots of the entries a fold reads are never among them (R >= W + T).
// ---------------------------------------------------------------------------
template <int N, int TQ, bool BF>
__global__ void __launch_bounds__(kThreads, 6) m2_prep_kernel(const M2Args a) {
    constexpr int IB = BF ? 2 : 4;
    extern __shared__ __align__(128) uint8_t smraw[];
    const M2PrepLay &Ly = a.lay;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, P = a.P, W = a.W, R = a.R, T = a.T, G = a.G, HC = a.HC;
    const int hpg = H / G;
    const int b = blockIdx.y;
    const int g = blockIdx.x / a.cpg, hc = blockIdx.x - g * a.cpg;
    const int h0 = g * hpg + hc * HC;
    const int E = W + TQ;
    uint8_t *sC = smraw + Ly.sC, *sBr = smraw + Ly.sBr, *sBn = smraw + Ly.sBn, *sx = smraw + Ly.sx;
    float *dring = reinterpret_cast<float *>(smraw + Ly.dring);
    float *dtn = reinterpret_cast<float *>(smraw + Ly.dtn);
    float *sA = reinterpret_cast<float *>(smraw + Ly.sA);
    float *sd = reinterpret_cast<float *>(smraw + Ly.sd);
    float *slam = reinterpret_cast<float *>(smraw + Ly.slam);
    int *si = reinterpret_cast<int *>(smraw + Ly.si);
    const int64_t row0 = (int64_t)b * H + h0;
    const int xrow = P * IB, brow = N * IB, xch = xrow / 16, bch = brow / 16;
    const int Rs = a.Rs;
    auto ldx = [](const uint8_t *p) -> float {
        return BF ? bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(p)) : *reinterpret_cast<const float *>(p);
    };

    pdl_trigger();  // the read kernel may be scheduled as this grid's last CTAs run

    // 1. Counters (thread 0) and everything that does not depend on them, at once.
    if (tid == 0) {
        const SeqState ss = read_counters(a.c, b, W);
        const int L0 = (int)(ss.seq - ss.ckpt);
        const int fold = ss.ok && (L0 + T > W);
        si[0] = ss.ok;
        si[1] = ss.ok ? L0 : 0;
        si[2] = fold;
        si[3] = (int)(ss.ckpt % R);
        si[4] = (int)(ss.seq % R);
        // seqinfo: {ring entries the read kernel replays, ring slot of entry 0,
        // folded by the flush kernel, counters valid}; the read kernel also
        // publishes the sequence's new counters from it
        if (blockIdx.x == 0) {
            bool valid = ss.ok;
            if (!ss.ok) report(a.c.err, DEV_BAD_COUNTERS, b, h0, L0);
            if (fold) {  // list the sequence for the flush kernel
                if (a.fold_launched) {
                    const int j = atomicAdd(a.fold_count, 1);
                    if (j < a.B) a.fold_list[j] = b;
                } else {  // the host's bound on buffer lengths was wrong: counters changed outside the API
                    report(a.c.err, DEV_BAD_COUNTERS, b, h0, L0);
                    valid = false;
                }
            }
            a.seqinfo[b] = valid ? make_int4(fold ? 0 : L0, (int)(ss.ckpt % R), fold, 1) : make_int4(0, 0, 1, 0);
        }
    }
    {
        const uint8_t *src = reinterpret_cast<const uint8_t *>(a.Bbuf) + ((int64_t)(b * G + g) * R) * brow;
        for (int i = tid; i < R * bch; i += kThreads) cp_async16(sBr + i * 16, src + i * 16);
    }
    for (int i = tid; i < HC * Rs / 4; i += kThreads) cp_async16(dring + 4 * i, a.dtbuf + row0 * Rs + 4 * i);
    for (int row = warp; row < T; row += kWarps) {
        const int64_t src = (((int64_t)(b * T + row) * G + g) * N) * IB;
        for (int k = lane; k < bch; k += 32) {
            cp_async16(sC + row * brow + k * 16, reinterpret_cast<const uint8_t *>(a.Cm) + src + k * 16);
            cp_async16(sBn + row * brow + k * 16, reinterpret_cast<const uint8_t *>(a.Bm) + src + k * 16);
        }
    }
    for (int row = warp; row < T * HC; row += kWarps) {
        const int m = row / HC, hh = row - m * HC;
        const uint8_t *src = reinterpret_cast<const uint8_t *>(a.x) + (((int64_t)(b * T + m) * H + h0 + hh) * P) * IB;
        for (int k = lane; k < xch; k += 32) cp_async16(sx + (m * HC + hh) * xrow + k * 16, src + k * 16);
    }
    for (int i = tid; i < T * HC; i += kThreads) {
        const int m = i / HC, hh = i - m * HC;
        dtn[m * HC + hh] = a.dt[(int64_t)(b * T + m) * H + h0 + hh];
    }
    for (int i = tid; i < HC; i += kThreads) sA[i] = a.A[h0 + i];
    cp_async_wait_all();
    __syncthreads();
    if (!si[0]) return;  // counters corrupted: reported, sequence skipped
    const int L0 = si[1], fold = si[2], ckmod = si[3], spmod = si[4];
    const int nE = L0 + T;
    auto slot_of = [&](int e) { const int s = ckmod + e; return s >= R ? s - R : s; };

    if (!fold) {
        // 2. B_e . C_m once for the group: a row is bch 16-byte chunks, one lane
        //    each, so a warp takes 32 / bch dots at a time.
        {
            const int dpw = 32 / bch, dl = lane / bch, c = lane - dl * bch;
            const int ndots = T * nE;
            for (int pr0 = warp * dpw; pr0 < ndots; pr0 += kWarps * dpw) {  // warp-uniform
                const int pr = pr0 + dl;
                const int m = pr / nE, e = pr - m * nE;
                float d = 0.f;
                if (pr < ndots && e <= L0 + m) {
                    const uint8_t *Bp = e < L0 ? sBr + slot_of(e) * brow : sBn + (e - L0) * brow;
                    const uint4 bu = *reinterpret_cast<const uint4 *>(Bp + c * 16);
                    const uint4 cu = *reinterpret_cast<const uint4 *>(sC + m * brow + c * 16);
                    if (BF) {
                        const uint32_t bw[4] = {bu.x, bu.y, bu.z, bu.w}, cw[4] = {cu.x, cu.y, cu.z, cu.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            d = fmaf(bf16_bits_to_float(bw[k] & 0xFFFFu), bf16_bits_to_float(cw[k] & 0xFFFFu), d);
                            d = fmaf(__uint_as_float(bw[k] & 0xFFFF0000u), __uint_as_float(cw[k] & 0xFFFF0000u), d);
                        }
                    } else {
                        d = __uint_as_float(bu.x) * __uint_as_float(cu.x) + __uint_as_float(bu.y) * __uint_as_float(cu.y) +
                            __uint_as_float(bu.z) * __uint_as_float(cu.z) + __uint_as_float(bu.w) * __uint_as_float(cu.w);
                    }
                }
                for (int o = bch / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                if (c == 0 && pr < ndots && e <= L0 + m) sd[m * E + e] = d;
            }
        }
        __syncthreads();
        // 3. Per head (one warp): prefix sums of dt*A, coefficients, decays.
        for (int hh = warp; hh < HC; hh += kWarps) {
            const float Ah = sA[hh];
            float *lam = slam + hh * E;
            float carry = 0.f;
            for (int k0 = 0; k0 < nE; k0 += 32) {
                const int e = k0 + lane;
                float v = 0.f;
                if (e < nE) v = (e < L0 ? dring[hh * Rs + slot_of(e)] : dtn[(e - L0) * HC + hh]) * Ah;
                v = warp_incl_scan(v) + carry;
                if (e < nE) lam[e] = v;
                carry = __shfl_sync(0xffffffffu, v, 31);
            }
            __syncwarp();
            float *crow = a.coef + (row0 + hh) * a.TQmax * a.Emax;
            for (int e = lane; e < nE; e += 32) {
                const float se = a.dt_scales ? (e < L0 ? dring[hh * Rs + slot_of(e)] : dtn[(e - L0) * HC + hh]) : 1.f;
#pragma unroll
                for (int m = 0; m < TQ; ++m)
                    if (m < T && e <= L0 + m) crow[m * a.Emax + e] = expf(lam[L0 + m] - lam[e]) * sd[m * E + e] * se;
            }
            if (lane < T) a.dec[(row0 + hh) * a.TQmax + lane] = expf(lam[L0 + lane]);
        }
    }

    // 4. Append the call's tokens to the ring.
    for (int row = warp; row < T * HC; row += kWarps) {
        const int m = row / HC, hh = row - m * HC;
        const int slot = spmod + m >= R ? spmod + m - R : spmod + m;
        uint8_t *dst = reinterpret_cast<uint8_t *>(a.xbuf) + (((row0 + hh) * R + slot) * P) * IB;
        const uint8_t *src = sx + (m * HC + hh) * xrow;
        for (int k = lane; k < xch; k += 32)
            *reinterpret_cast<uint4 *>(dst + k * 16) = *reinterpret_cast<const uint4 *>(src + k * 16);
    }
    for (int i = tid; i < T * HC; i += kThreads) {
        const int m = i / HC, hh = i - m * HC;
        const int slot = spmod + m >= R ? spmod + m - R : spmod + m;
        a.dtbuf[(row0 + hh) * Rs + slot] = dtn[m * HC + hh];
    }
    if (hc == 0) {  // the group's first chunk writes the group's B
        for (int row = warp; row < T; row += kWarps) {
            const int slot = spmod + row >= R ? spmod + row - R : spmod + row;
            uint8_t *dst = reinterpret_cast<uint8_t *>(a.Bbuf) + (((int64_t)(b * G + g) * R + slot) * N) * IB;
            for (int k = lane; k < bch; k += 32)
                *reinterpret_cast<uint4 *>(dst + k * 16) = *reinterpret_cast<const uint4 *>(sBn + row * brow + k * 16);
        }
    }
}

// ---------------------------------------------------------------------------
// Flush kernel: fold the committed buffer into the fp32 checkpoint and
// requantise the read copy ("the checkpoint is rewritten only when the buffer
// is full", blog.thibaultmonteiro.fr, "Tenir le journal plutot que le solde").
// Runs for decode/verify calls that find a full buffer (len + T > W; it then
// also serves that sequence's outputs), and for flush (len > 0) and export
// (writing the folded state out instead).
//
//     S_c <- e^{Lam_{L0-1}} S_c + sum_{e < L0} U_e B_e^T,   U_e[p] = e^{Lam_{L0-1} - Lam_e} s_e x_e[p]
//
// is a rank-L0 update: U and B (fp32, in shared memory) give each thread a 4x4
// register block (4 consecutive rows x 4 columns) updated with two 128-bit
// shared loads and 16 FMAs per entry.  The checkpoint rows arrive in 16 KiB
// bulk-copy stages, two in flight per CTA (three CTAs per SM); all waits are bounded.
//
// The kernel is persistent and each CTA walks a list of work items (sequence,
// HC heads of one group).  What an item's prefix sums, fold weights and
// coefficients read (the whole B, x and dt rings, A, the call's C, B and dt) and
// its counters are fetched while the previous item's rows are folded, since
// none of it depends on the counters; that phase then takes one barrier.  In a
// decode/verify every listed sequence folds, so the checkpoint stages of a CTA's
// items form one stream: the next item's first stages are issued while the
// current item's last stages are folded, and a new item starts with its rows
// already landing.
// ---------------------------------------------------------------------------
struct M2FoldLay {
    int stage, bar, sC, sBr, sBn, sxr, sxn, dring, dtn, sA, sD, U, Bf, scoef, sdec, sfdec, sCf, sdot, si, bytes;
};
constexpr int kFoldStages = 2;
// R: ring slots (W + max(max_draft, 1)).
inline M2FoldLay m2_fold_lay(int HC, int P, int N, int W, int R, int TQ, int ib) {
    M2FoldLay L{};
    int o = 0;
    L.stage = o; o += kFoldStages * kFoldChunk;  // fp32 checkpoint rows
    L.bar = o;   o += 8 * kFoldStages;
    o = a16(o);
    L.sC = o;    o += a16(TQ * N * ib);          // raw C of the queries        [TQ][N]
    L.sBr = o;   o += a16(R * N * ib);           // raw B ring of the group     [R][N]
    L.sBn = o;   o += a16(TQ * N * ib);          // raw B of the call's tokens  [TQ][N]
    L.sxr = o;   o += a16(HC * R * P * ib);      // raw x ring of the heads     [HC][R][P]
    L.sxn = o;   o += a16(TQ * HC * P * ib);     // raw x of the call's tokens  [TQ][HC][P]
    L.dring = o; o += a16(HC * pad4(R) * 4);     // dt ring rows                [HC][Rs]
    L.dtn = o;   o += a16(TQ * HC * 4);          // dt of the call's tokens     [TQ][HC]
    L.sA = o;    o += a16(HC * 4);               // A of the heads              [HC]
    L.sD = o;    o += a16(HC * 4);               // D of the heads              [HC]
    L.U = o;     o += a16(HC * W * P * 4);       // fold weights x rows         [HC][L0][P]
    L.Bf = o;    o += a16(W * N * 4);            // committed B as fp32         [L0][N]
    L.scoef = o; o += a16(HC * TQ * TQ * 4);     // coefficients of the call's tokens [HC][TQ][TQ]
    L.sdec = o;  o += a16(HC * TQ * 4);          // decay of the fresh copy     [HC][TQ]
    L.sfdec = o; o += a16(HC * 4);               // decay of the folded checkpoint [HC]
    L.sCf = o;   o += a16(TQ * N * 4);           // C as fp32                   [TQ][N]
    L.sdot = o;  o += a16(HC * P * TQ * 4);      // fresh copy . C per row      [HC*P][TQ]
    L.si = o;    o += 32;
    L.bytes = o;
    return L;
}

template <int N, int RK, int TQ, bool BF>
__global__ void __launch_bounds__(kThreads, 3) m2_fold_kernel(const M2Args a, const M2FoldLay Ly) {
    constexpr int Q = N / 4;              // column quads per row
    constexpr int RG = kThreads / Q;      // row groups per stage
    constexpr int FC = kFoldChunk / (N * 4);  // fp32 rows per stage (= 4 * RG)
    constexpr int IB = BF ? 2 : 4;
    constexpr int kLamChunks = 3;         // entries per head: L0 + T <= W + 8 <= 72 = at most 3 warps of lanes
    static_assert(FC == 4 * RG, "each thread owns 4 consecutive rows of a stage");
    static_assert(Q >= 4, "quad_rows_sum pairs lanes at Q/2 and Q/4");
    extern __shared__ __align__(128) uint8_t smraw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, P = a.P, W = a.W, R = a.R, T = a.T, G = a.G, HC = a.HC;
    const int hpg = H / G;
    float *stg = reinterpret_cast<float *>(smraw + Ly.stage);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smraw + Ly.bar);
    uint8_t *sC = smraw + Ly.sC, *sBr = smraw + Ly.sBr, *sBn = smraw + Ly.sBn;
    uint8_t *sxr = smraw + Ly.sxr, *sxn = smraw + Ly.sxn;
    float *dring = reinterpret_cast<float *>(smraw + Ly.dring);
    float *dtn = reinterpret_cast<float *>(smraw + Ly.dtn);
    float *sA = reinterpret_cast<float *>(smraw + Ly.sA);
    float *sD = reinterpret_cast<float *>(smraw + Ly.sD);
    float *U = reinterpret_cast<float *>(smraw + Ly.U);
    float *Bf = reinterpret_cast<float *>(smraw + Ly.Bf);
    float *scoef = reinterpret_cast<float *>(smraw + Ly.scoef);
    float *sdec = reinterpret_cast<float *>(smraw + Ly.sdec);
    float *sfdec = reinterpret_cast<float *>(smraw + Ly.sfdec);
    float *sCf = reinterpret_cast<float *>(smraw + Ly.sCf);
    float *sdot = reinterpret_cast<float *>(smraw + Ly.sdot);
    int *si = reinterpret_cast<int *>(smraw + Ly.si);
    const int nrows = HC * P;
    const int nst = (nrows + FC - 1) / FC;
    const bool reads = (a.op == OP_DECODE || a.op == OP_VERIFY);
    const bool stream = reads;  // every listed sequence folds: stages run on across items
    const int xrow = P * IB, brow = N * IB, xch = xrow / 16, bch = brow / 16;
    const int Rs = a.Rs;
    const int chunks = G * a.cpg;  // CTA work items per sequence
    auto ldx = [](const uint8_t *p) -> float {
        return BF ? bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(p)) : *reinterpret_cast<const float *>(p);
    };
    auto ld2 = [](const uint8_t *p) -> float2 {  // two consecutive raw inputs
        if (BF) {
            const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
            return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
        }
        return *reinterpret_cast<const float2 *>(p);
    };
    auto ld4 = [](const uint8_t *p) -> float4 {  // four consecutive raw inputs
        if (BF) {
            const uint2 u = *reinterpret_cast<const uint2 *>(p);
            return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                               __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
        }
        return *reinterpret_cast<const float4 *>(p);
    };

    // Work items (sequence, chunk of HC heads of one group): decode/verify fold
    // the sequences the prep kernel listed; flush/export visit every sequence.
    const int nitems = (reads ? min(*a.fold_count, a.B) : a.B) * chunks;
    auto item_seq = [&](int it) { return reads ? a.fold_list[it / chunks] : it / chunks; };
    auto item_h0 = [&](int it) {
        const int chunk = it % chunks, g = chunk / a.cpg;
        return g * hpg + (chunk - g * a.cpg) * HC;
    };
    if (tid == 0) {
        for (int k = 0; k < kFoldStages; ++k) mbar_init(&bar[k], 1);
        mbar_init_fence();
    }
    __syncthreads();
    uint32_t gs = 0;    // checkpoint stages consumed so far: slot gs % kFoldStages, phase (gs / kFoldStages) & 1
    int ncur = 0;       // thread 0: stages of the current item issued
    int nnext = 0;      // thread 0: stages of the next item issued (stream only)
    int64_t cseq = 0, cckpt = 0;  // thread 0: counters of the item about to start

    // Staging of item `it` (sequence bb), all threads, one cp.async group each:
    // the rings, A and the call's C, B, dt (read before the stage loop), and the
    // call's x and D (read by the outputs after it).
    auto stage_main = [&](int it, int bb) {
        const int g = (it % chunks) / a.cpg, h0 = item_h0(it);
        const int64_t row0 = (int64_t)bb * H + h0;
        const uint8_t *src = reinterpret_cast<const uint8_t *>(a.Bbuf) + ((int64_t)(bb * G + g) * R) * brow;
        for (int i = tid; i < R * bch; i += kThreads) cp_async16(sBr + i * 16, src + i * 16);
        const uint8_t *xs = reinterpret_cast<const uint8_t *>(a.xbuf) + (row0 * R * P) * IB;
        for (int i = tid; i < HC * R * xch; i += kThreads) cp_async16(sxr + i * 16, xs + i * 16);
        for (int i = tid; i < HC * Rs / 4; i += kThreads) cp_async16(dring + 4 * i, a.dtbuf + row0 * Rs + 4 * i);
        for (int row = warp; row < T; row += kWarps) {
            const int64_t o = (((int64_t)(bb * T + row) * G + g) * N) * IB;
            for (int k = lane; k < bch; k += 32) {
                cp_async16(sC + row * brow + k * 16, reinterpret_cast<const uint8_t *>(a.Cm) + o + k * 16);
                cp_async16(sBn + row * brow + k * 16, reinterpret_cast<const uint8_t *>(a.Bm) + o + k * 16);
            }
        }
        for (int i = tid; i < T * HC; i += kThreads) {
            const int m = i / HC, hh = i - m * HC;
            cp_async4(dtn + i, a.dt + (int64_t)(bb * T + m) * H + h0 + hh);
        }
        if (tid < HC) cp_async4(sA + tid, a.A + h0 + tid);
        cp_async_commit();
    };
    auto stage_out = [&](int it, int bb) {
        const int h0 = item_h0(it);
        for (int m = warp; m < T; m += kWarps) {  // x of the call's tokens: HC heads are contiguous
            const uint8_t *src = reinterpret_cast<const uint8_t *>(a.x) + (((int64_t)(bb * T + m) * H + h0) * P) * IB;
            for (int k = lane; k < HC * xch; k += 32) cp_async16(sxn + m * HC * xrow + k * 16, src + k * 16);
        }
        if (tid < HC) cp_async4(sD + tid, a.D + h0 + tid);
        cp_async_commit();
    };
    int b_next = 0;
    if (blockIdx.x < nitems) {
        b_next = item_seq(blockIdx.x);
        stage_main(blockIdx.x, b_next);
        if (tid == 0) {
            cseq = a.c.seq_pos[b_next];
            cckpt = a.c.ckpt_pos[b_next];
        }
    }

    for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        const int b = b_next;
        const int nxt = item + gridDim.x;
        if (nxt < nitems) b_next = item_seq(nxt);  // first used after the item's first barrier
        const int chunk = item % chunks;
        const int h0 = item_h0(item);
        const int64_t row0 = (int64_t)b * H + h0;
        const int64_t tile0 = row0 * P * N;

        // Thread 0 keeps up to kFoldStages stages in flight: the current item's, then
        // (stream) the next item's.  `consumed` stages have been waited for.
        auto issue = [&](bool next, int c) {
            const int r0 = c * FC, r1 = min(nrows, r0 + FC);
            const uint32_t bytes = (uint32_t)((r1 - r0) * N * 4);
            const uint32_t s = gs + (next ? nst : 0) + c;
            const int k = s % kFoldStages;
            const float *src = next ? a.ckpt + ((int64_t)b_next * H + item_h0(nxt)) * P * N : a.ckpt + tile0;
            mbar_arrive_expect_tx(&bar[k], bytes);
            bulk_g2s(stg + k * (FC * N), src + (int64_t)r0 * N, bytes, &bar[k]);
        };
        auto top_up = [&](uint32_t consumed) {
            while (gs + ncur + nnext < consumed + kFoldStages) {
                if (ncur < nst)
                    issue(false, ncur++);
                else if (stream && nxt < nitems && nnext < nst)
                    issue(true, nnext++);
                else
                    break;
            }
        };

        // 1. The item's x and D; what the counters say (fetched during the
        //    previous item); the staged rings must have landed.
        stage_out(item, b);
        SeqState ss{};
        if (tid == 0) {
            if (stream) top_up(gs);
            ss.seq = cseq;
            ss.ckpt = cckpt;
            const int L0 = (int)(ss.seq - ss.ckpt);
            ss.ok = (ss.ckpt >= 0 && L0 >= 0 && L0 <= W) ? 1 : 0;
            const int fold = ss.ok && (reads ? (L0 + T > W) : (L0 > 0));
            si[0] = fold;
            si[1] = L0;
            si[3] = (int)(ss.ckpt % R);
            if (!ss.ok && !reads && chunk == 0) report(a.c.err, DEV_BAD_COUNTERS, b, h0, L0);
            if (!stream && fold) top_up(gs);
        }
        cp_async_wait_group<1>();  // this item's rings (its x and D may still be in flight)
        __syncthreads();
        const bool fold = si[0] != 0;
        // (stream && !fold: counters the prep kernel reported as bad; the item's
        //  stages are only drained.)
        const int L0 = fold ? si[1] : 0, ckmod = si[3];
        auto slot_of = [&](int e) { const int s = ckmod + e; return s >= R ? s - R : s; };
        auto dt_of = [&](int hh, int e) -> float {
            return e < L0 ? dring[hh * Rs + slot_of(e)] : dtn[(e - L0) * HC + hh];
        };

        // 2. Per head (kWarps / HC warps each): prefix sums of dt*A, fold weights,
        //    decays, the fold-weighted x rows U and the call's own coefficients;
        //    then B of the committed entries and C as fp32.
        if (fold) {
            const int nE = L0 + T;
            const int wph = kWarps / HC;
            const int hh = warp / wph, part = warp - hh * wph;
            if (hh < HC) {
                const float Ah = sA[hh];
                float lamr[kLamChunks], sur[kLamChunks];
                float carry = 0.f;
#pragma unroll
                for (int ch = 0; ch < kLamChunks; ++ch) {
                    lamr[ch] = 0.f;
                    sur[ch] = 0.f;
                    if (ch * 32 < nE) {  // warp-uniform
                        const int e = ch * 32 + lane;
                        float v = e < nE ? dt_of(hh, e) * Ah : 0.f;
                        v = warp_incl_scan(v) + carry;
                        lamr[ch] = v;
                        carry = __shfl_sync(0xffffffffu, v, 31);
                    }
                }
                auto lam_at = [&](int e) -> float {  // e warp-uniform
                    const float v = e < 32 ? lamr[0] : (e < 64 ? lamr[1] : lamr[2]);
                    return __shfl_sync(0xffffffffu, v, e & 31);
                };
                const float lam_f = lam_at(L0 - 1);
#pragma unroll
                for (int ch = 0; ch < kLamChunks; ++ch) {
                    const int e = ch * 32 + lane;
                    if (e < L0) sur[ch] = expf(lam_f - lamr[ch]) * (a.dt_scales ? dt_of(hh, e) : 1.f);
                    if (part == 0 && reads && e >= L0 && e < nE) sdec[hh * TQ + (e - L0)] = expf(lamr[ch] - lam_f);
                }
                if (part == 0 && lane == 0) sfdec[hh] = expf(lam_f);
                for (int e = part; e < L0; e += wph) {  // U[hh][e][p] = weight_e x_e[p]
                    const float w = __shfl_sync(0xffffffffu, e < 32 ? sur[0] : (e < 64 ? sur[1] : sur[2]), e & 31);
                    const uint8_t *xr = sxr + ((hh * R + slot_of(e)) * P) * IB;
                    float2 *Ur = reinterpret_cast<float2 *>(U + (hh * L0 + e) * P);
                    for (int p2 = lane; p2 < P / 2; p2 += 32) {
                        const float2 xv = ld2(xr + 2 * p2 * IB);
                        Ur[p2] = make_float2(w * xv.x, w * xv.y);
                    }
                }
                if (reads) {  // coefficients of the call's own tokens against the fresh checkpoint
                    for (int pr = part; pr < T * T; pr += wph) {
                        const int m = pr / T, j = pr - m * T;  // entry L0 + j, query m
                        if (j > m) continue;                   // warp-uniform
                        float d = 0.f;
                        for (int n = lane; n < N; n += 32) d = fmaf(ldx(sBn + (j * N + n) * IB), ldx(sC + (m * N + n) * IB), d);
                        d = group_sum<32>(d);
                        const float lm = lam_at(L0 + m), lj = lam_at(L0 + j);
                        if (lane == 0)
                            scoef[(hh * TQ + m) * TQ + j] = expf(lm - lj) * d * (a.dt_scales ? dtn[j * HC + hh] : 1.f);
                    }
                }
            }
            for (int i = tid; i < L0 * (N / 4); i += kThreads) {
                const int e = i / (N / 4), n4 = i - e * (N / 4);
                *reinterpret_cast<float4 *>(Bf + e * N + 4 * n4) = ld4(sBr + (slot_of(e) * N + 4 * n4) * IB);
            }
            if (reads)
                for (int i = tid; i < T * N; i += kThreads) sCf[i] = ldx(sC + i * IB);
        }
        __syncthreads();
        // The rings are free: fetch the next item's, and its counters.
        if (nxt < nitems) {
            stage_main(nxt, b_next);
            if (tid == 0) {
                cseq = a.c.seq_pos[b_next];
                cckpt = a.c.ckpt_pos[b_next];
            }
        } else {
            cp_async_commit();  // an empty group keeps the group count uniform
        }
        if (!fold && !stream) {
            if (tid == 0 && a.op == OP_FLUSH)  // nothing to fold; the CTA still arrives
                arrive_and_publish(a.c, b, chunks, -1, -1, -1, 0);
            cp_async_wait_group<1>();  // this item's x and D have landed before they are restaged
            __syncthreads();
            continue;
        }

        // 3. Stages of checkpoint rows: fold, store checkpoint and read copy, dot with C.
        const int q = tid % Q, rg = tid / Q;
        int failed = -1;  // stage whose copy never landed
        for (int c = 0; c < nst; ++c) {
            const uint32_t s = gs + c;
            const int k = s % kFoldStages;
            const bool got = mbar_wait(&bar[k], (s / kFoldStages) & 1);
            const int gr0 = c * FC + 4 * rg;  // first of this thread's 4 rows (one head: P % 4 == 0)
            const bool valid = fold && gr0 < nrows;
            const int hh = valid ? gr0 / P : 0, p0 = gr0 - hh * P;
            float4 v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (valid) {
                const float *tf = stg + k * (FC * N) + (4 * rg) * N + 4 * q;
                const float dc = sfdec[hh];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    v[i] = *reinterpret_cast<const float4 *>(tf + i * N);
                    v[i].x *= dc; v[i].y *= dc; v[i].z *= dc; v[i].w *= dc;
                }
                const float *Ur = U + (hh * L0) * P + p0;
                const float *Br = Bf + 4 * q;
                // Rank-L0 update on packed pairs: row i's columns (x, y) and (z, w)
                // each take one .f32x2 FMA per entry with u_i broadcast to both halves.
                unsigned long long vp[4][2];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    vp[i][0] = f2_pack(v[i].x, v[i].y);
                    vp[i][1] = f2_pack(v[i].z, v[i].w);
                }
#pragma unroll 4
                for (int e = 0; e < L0; ++e) {
                    const float4 u = *reinterpret_cast<const float4 *>(Ur + e * P);
                    const float4 bb = *reinterpret_cast<const float4 *>(Br + e * N);
                    const unsigned long long b01 = f2_pack(bb.x, bb.y), b23 = f2_pack(bb.z, bb.w);
                    const float uv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const unsigned long long ui = f2_pack(uv[i], uv[i]);
                        vp[i][0] = f2_fma(ui, b01, vp[i][0]);
                        vp[i][1] = f2_fma(ui, b23, vp[i][1]);
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    f2_unpack(vp[i][0], v[i].x, v[i].y);
                    f2_unpack(vp[i][1], v[i].z, v[i].w);
                }
            }
            // Every thread has its rows (the stage buffer is free again), and
            // every thread learns whether any wait gave up.
            if (__syncthreads_or(!got)) {
                failed = c;
                break;
            }
            if (tid == 0) top_up(s + 1);
            if (!fold) continue;  // CTA-uniform
            float4 rd[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int gr = gr0 + i;
                const int64_t el = tile0 + (int64_t)(valid ? gr : 0) * N + 4 * q;
                rd[i] = v[i];
                if (a.op == OP_EXPORT) {
                    if (valid) *reinterpret_cast<float4 *>(a.out + el) = v[i];
                    continue;
                }
                if (valid) *reinterpret_cast<float4 *>(a.ckpt + el) = v[i];
                if (RK == SK_BF16) {
                    if (valid) rd[i] = store_quad<SK_BF16>(a.rc, el, v[i], 0.f, 0.f);
                } else if (RK == SK_FP8) {
                    float am = fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w)));
                    am = group_max<Q>(am);
                    const float sc = fp8_scale(am);
                    if (valid) {
                        rd[i] = store_quad<SK_FP8>(a.rc, el, v[i], 0.f, sc);
                        if (q == 0) a.rc_scale[row0 * P + gr] = sc;
                    }
                }
            }
            if (reads) {
#pragma unroll
                for (int m = 0; m < TQ; ++m) {
                    const float4 Cq = *reinterpret_cast<const float4 *>(sCf + m * N + 4 * q);
                    float d[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) d[i] = rd[i].x * Cq.x + rd[i].y * Cq.y + rd[i].z * Cq.z + rd[i].w * Cq.w;
                    const float sum = quad_rows_sum<Q>(d[0], d[1], d[2], d[3], q);
                    const int r = 2 * ((q & (Q / 2)) != 0) + ((q & (Q / 4)) != 0);
                    if (valid && m < T && (q & (Q / 4 - 1)) == 0) sdot[(gr0 + r) * TQ + m] = sum;
                }
            }
        }
        if (failed >= 0) {
            // A checkpoint copy never landed: report, let the copies still in
            // flight (this item's from the failed stage on, the next item's
            // already issued) land, bounded, and stop.
            if (tid == 0) {
                report(a.c.err, DEV_PIPE_TIMEOUT, b, h0, 0);
                for (int c = failed; c < ncur; ++c)
                    mbar_wait(&bar[(gs + c) % kFoldStages], ((gs + c) / kFoldStages) & 1);
                for (int c = 0; c < nnext; ++c)
                    mbar_wait(&bar[(gs + nst + c) % kFoldStages], ((gs + nst + c) / kFoldStages) & 1);
            }
            cp_async_wait_all();
            return;
        }
        gs += nst;
        if (tid == 0) {
            ncur = nnext;
            nnext = 0;
        }
        cp_async_wait_group<1>();  // this item's x and D (the next item's rings may be in flight)
        if (reads && fold) {
            __syncthreads();
            // Outputs of the folded sequence: the fresh copy plus the call's own tokens.
            for (int i = tid; i < T * nrows; i += kThreads) {
                const int m = i / nrows, r2 = i - m * nrows;
                const int hh = r2 / P, p = r2 - hh * P;
                float yv = sdec[hh * TQ + m] * sdot[r2 * TQ + m];
                const float *cf = scoef + (hh * TQ + m) * TQ;
                const uint8_t *xs = sxn + (hh * P + p) * IB;  // token j at xs + j * HC * xrow
                for (int j = 0; j <= m; ++j) yv = fmaf(cf[j], ldx(xs + j * HC * xrow), yv);
                yv = fmaf(sD[hh], ldx(xs + m * HC * xrow), yv);
                a.y[((int64_t)(b * T + m) * H + h0 + hh) * P + p] = yv;
            }
        }
        if (tid == 0 && a.op == OP_FLUSH)  // flush publishes the sequence's counters here
            arrive_and_publish(a.c, b, chunks, -1, ss.seq, -1, 1);
        __syncthreads();  // shared memory is restaged by the next item
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

// Eager decode (T = 1) with two heads of one group per CTA: both heads' state
// rows are requested before anything else and the group's B and C are staged
// once, so each CTA keeps 2 x P x N state elements in flight and its prologue is
// shared by two heads.  Per element it computes exactly what m2_eager_kernel
// computes (the same operations in the same order).  Requires P <= 8 rows per
// thread x (kThreads / (N / 4)) and an even number of heads per group.
template <int N, int SK>
__global__ void __launch_bounds__(kThreads, SK == SK_FP8 ? 2 : 4) m2_eager_decode2_kernel(const M2Args a) {
    constexpr int TPR4 = N / 4;
    constexpr int RPP4 = kThreads / TPR4;
    constexpr int RB = 8;
    extern __shared__ __align__(16) float smem[];
    const int tid = threadIdx.x;
    const int H = a.H, P = a.P, G = a.G;
    const int bh0 = 2 * blockIdx.x;
    const int b = bh0 / H, h0 = bh0 - b * H;
    const int g = h0 / (H / G);
    float *sx = smem;                 // [2][P]
    float *sB = sx + pad4(2 * P);     // [N]
    float *sC = sB + pad4(N);         // [N]
    float *sdot = sC + pad4(N);       // [2][P]
    float *sa = sdot + pad4(2 * P);   // [2] decay
    float *ss = sa + 4;               // [2] input scale
    void *state = (SK == SK_F32) ? (void *)a.ckpt : a.rc;

    const int c4 = tid % TPR4, q0 = tid / TPR4;
    float4 st[2][RB];
    float scl[2][RB];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = q0 + k * RPP4;
            const int64_t row = (int64_t)(bh0 + hh) * P + r;
            st[hh][k] = (r < P) ? load_quad<SK>(state, row * N + 4 * c4) : make_float4(0.f, 0.f, 0.f, 0.f);
            scl[hh][k] = (SK == SK_FP8 && r < P) ? __ldg(a.rc_scale + row) : 1.f;
        }

    // No other CTA of an eager launch reads the counters, so the CTA of the
    // sequence's first heads rewrites them alone (no arrival count, no fence).
    if (tid == 0 && h0 == 0) {
        const int64_t s1 = a.c.seq_pos[b] + 1;
        a.c.seq_pos[b] = s1;
        a.c.ckpt_pos[b] = s1;
    }
    for (int i = tid; i < 2 * P; i += kThreads) sx[i] = ld_in(a.x, (int64_t)(b * H + h0) * P + i, a.in_bf16);
    for (int i = tid; i < N; i += kThreads) {
        const int64_t src = ((int64_t)b * G + g) * N + i;
        sB[i] = ld_in(a.Bm, src, a.in_bf16);
        sC[i] = ld_in(a.Cm, src, a.in_bf16);
    }
    if (tid < 2) {
        const float dtv = a.dt[(int64_t)b * H + h0 + tid];
        sa[tid] = expf(dtv * a.A[h0 + tid]);
        ss[tid] = a.dt_scales ? dtv : 1.f;
    }
    __syncthreads();

    const float4 Bq = reinterpret_cast<const float4 *>(sB)[c4];
    const float4 Cq = reinterpret_cast<const float4 *>(sC)[c4];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const float am = sa[hh], sc_in = ss[hh];
        const int64_t tile0 = (int64_t)(bh0 + hh) * P * N;
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = q0 + k * RPP4;
            const bool valid = r < P;
            const int64_t el = tile0 + (int64_t)(valid ? r : 0) * N + 4 * c4;
            float4 v = st[hh][k];
            if (SK == SK_FP8) { v.x *= scl[hh][k]; v.y *= scl[hh][k]; v.z *= scl[hh][k]; v.w *= scl[hh][k]; }
            const float w = sc_in * (valid ? sx[hh * P + r] : 0.f);
            v.x = fmaf(am, v.x, w * Bq.x); v.y = fmaf(am, v.y, w * Bq.y);
            v.z = fmaf(am, v.z, w * Bq.z); v.w = fmaf(am, v.w, w * Bq.w);
            float d = v.x * Cq.x + v.y * Cq.y + v.z * Cq.z + v.w * Cq.w;
            d = group_sum<TPR4>(d);
            if (c4 == 0 && valid) sdot[hh * P + r] = d;  // output from the fp32 value
            float sc = 1.f;
            if (SK == SK_FP8) {
                const float amx = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
                sc = fp8_scale(group_max<TPR4>(amx));
                if (valid && c4 == 0) a.rc_scale[(int64_t)(bh0 + hh) * P + r] = sc;
            }
            if (valid) store_quad<SK>(state, el, v, 0.f, sc);
        }
    }
    __syncthreads();
    for (int i = tid; i < 2 * P; i += kThreads)
        a.y[(int64_t)(b * H + h0) * P + i] = sdot[i] + a.D[h0 + i / P] * sx[i];
}

// Eager decode (T = 1) of an fp32 state as one stream: a persistent grid whose
// CTAs walk the heads (b, h) gridDim apart.  Each head's P x N fp32 tile arrives
// by one bulk copy into one of kEagerStages shared-memory stages, issued
// kEagerStages - 1 heads ahead, so a CTA keeps up to two tiles in flight while it
// updates the third; the update itself is what m2_eager_kernel computes (the
// same operations in the same order), read from shared memory and written back
// with 128-bit stores.  A head's x row, its group's B and C and its dt, A and D
// are loaded into registers one head ahead.  Waits are bounded.
constexpr int kEagerStages = 3;
template <int N>
__global__ void __launch_bounds__(kThreads, 2) m2_eager_stream_kernel(const M2Args a) {
    constexpr int TPR4 = N / 4;            // threads per state row (one float4 each)
    constexpr int RPP4 = kThreads / TPR4;  // rows per pass
    extern __shared__ __align__(128) uint8_t esm[];
    const int tid = threadIdx.x;
    const int H = a.H, P = a.P, G = a.G;
    const int hpg = H / G;
    const int nitems = a.B * H;
    const int tile = P * N;  // floats
    float *stg = reinterpret_cast<float *>(esm);                 // [kEagerStages][P][N]
    float *sx = stg + kEagerStages * tile;                        // [2][P]
    float *sB = sx + 2 * pad4(P);                                 // [2][N]
    float *sC = sB + 2 * N;                                       // [2][N]
    float *sdot = sC + 2 * N;                                     // [P]
    float *ssc = sdot + pad4(P);                                  // [2][4]: decay, input scale, D
    uint64_t *bar = reinterpret_cast<uint64_t *>(ssc + 8);        // [kEagerStages]
    const int c4 = tid % TPR4, q0 = tid / TPR4;

    if (tid == 0) {
        for (int k = 0; k < kEagerStages; ++k) mbar_init(&bar[k], 1);
        mbar_init_fence();
    }
    __syncthreads();
    auto issue = [&](int li) {  // thread 0: the tile of the CTA's li-th head into stage li % kEagerStages
        const int it = blockIdx.x + li * gridDim.x;
        if (it >= nitems) return;
        const int k = li % kEagerStages;
        mbar_arrive_expect_tx(&bar[k], (uint32_t)(tile * 4));
        bulk_g2s(stg + k * tile, a.ckpt + (int64_t)it * tile, (uint32_t)(tile * 4), &bar[k]);
    };
    if (tid == 0)
        for (int li = 0; li < kEagerStages - 1; ++li) issue(li);

    // The small inputs of head `it`, in registers: x[tid], B[tid], C[tid]; threads
    // 0..2 hold the decay, the input scale and D.
    float rx = 0.f, rB = 0.f, rC = 0.f, rs = 0.f;
    auto load_small = [&](int it) {
        if (it >= nitems) return;
        const int b = it / H, h = it - b * H, g = h / hpg;
        if (tid < P) rx = ld_in(a.x, (int64_t)it * P + tid, a.in_bf16);
        if (tid < N) {
            const int64_t src = ((int64_t)b * G + g) * N + tid;
            rB = ld_in(a.Bm, src, a.in_bf16);
            rC = ld_in(a.Cm, src, a.in_bf16);
        }
        if (tid == 0) rs = expf(a.dt[it] * a.A[h]);
        if (tid == 1) rs = a.dt_scales ? a.dt[it] : 1.f;
        if (tid == 2) rs = a.D[h];
    };
    load_small(blockIdx.x);

    int li = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
        const int b = it / H, h = it - b * H;
        const int k = li % kEagerStages, sl = li & 1;
        // This head's small inputs to shared memory; the next head's into registers.
        if (tid < P) sx[sl * pad4(P) + tid] = rx;
        if (tid < N) {
            sB[sl * N + tid] = rB;
            sC[sl * N + tid] = rC;
        }
        if (tid < 3) ssc[sl * 4 + tid] = rs;
        load_small(it + gridDim.x);
        if (tid == 0) {
            issue(li + kEagerStages - 1);  // its stage was freed at the end of the previous head
            if (h == 0) {  // no other CTA of an eager launch reads the sequence's counters
                const int64_t s1 = a.c.seq_pos[b] + 1;
                a.c.seq_pos[b] = s1;
                a.c.ckpt_pos[b] = s1;
            }
        }
        const bool got = mbar_wait(&bar[k], (uint32_t)((li / kEagerStages) & 1));
        if (__syncthreads_or(!got)) {
            if (tid == 0) {
                report(a.c.err, DEV_PIPE_TIMEOUT, b, h, 0);
                for (int j = 0; j < kEagerStages; ++j)  // copies still in flight land (bounded) before exit
                    if (it + j * (int)gridDim.x < nitems)
                        mbar_wait(&bar[(li + j) % kEagerStages], (uint32_t)(((li + j) / kEagerStages) & 1));
            }
            return;
        }
        const float am = ssc[sl * 4], sc_in = ssc[sl * 4 + 1];
        const float4 Bq = reinterpret_cast<const float4 *>(sB + sl * N)[c4];
        const float4 Cq = reinterpret_cast<const float4 *>(sC + sl * N)[c4];
        const float *st = stg + k * tile;
        float *dst = a.ckpt + (int64_t)it * tile;
        for (int r = q0; r < P; r += RPP4) {
            float4 v = *reinterpret_cast<const float4 *>(st + r * N + 4 * c4);
            const float w = sc_in * sx[sl * pad4(P) + r];
            v.x = fmaf(am, v.x, w * Bq.x); v.y = fmaf(am, v.y, w * Bq.y);
            v.z = fmaf(am, v.z, w * Bq.z); v.w = fmaf(am, v.w, w * Bq.w);
            float d = v.x * Cq.x + v.y * Cq.y + v.z * Cq.z + v.w * Cq.w;
            d = group_sum<TPR4>(d);
            if (c4 == 0) sdot[r] = d;  // output from the fp32 value
            *reinterpret_cast<float4 *>(dst + r * N + 4 * c4) = v;
        }
        __syncthreads();  // the stage is free again and every row's dot is in sdot
        if (tid < P) a.y[(int64_t)it * P + tid] = sdot[tid] + ssc[sl * 4 + 2] * sx[sl * pad4(P) + tid];
    }
}

inline size_t m2_eager_stream_smem(int P, int N) {
    return sizeof(float) * ((size_t)kEagerStages * P * N + 2 * pad4(P) + 4 * N + pad4(P) + 8) +
           sizeof(uint64_t) * kEagerStages;
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
enum M2Kernel : int { M2_EAGER = 0, M2_PREP = 1, M2_FOLD = 2 };

template <int N, int TQ>
inline cudaError_t launch_prep_t(const M2Args &a, size_t smem, cudaStream_t st) {
    auto k = a.in_bf16 ? m2_prep_kernel<N, TQ, true> : m2_prep_kernel<N, TQ, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<dim3(a.H / a.HC, a.B), kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

// The flush kernel is persistent: min(work items, resident CTAs) CTAs.
template <int N, int RK, int TQ>
inline cudaError_t launch_fold_t(const M2Args &a, const M2FoldLay &lay, int num_sms, cudaStream_t st) {
    auto k = a.in_bf16 ? m2_fold_kernel<N, RK, TQ, true> : m2_fold_kernel<N, RK, TQ, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.bytes);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kThreads, lay.bytes);
    if (e != cudaSuccess) return e;
    const int items = a.B * (a.H / a.HC);
    const int grid = items < num_sms * (occ > 0 ? occ : 1) ? items : num_sms * (occ > 0 ? occ : 1);
    k<<<grid, kThreads, lay.bytes, st>>>(a, lay);
    return cudaGetLastError();
}

template <int N, int SK, int TQ>
inline cudaError_t launch_eager_t(const M2Args &a, size_t smem, cudaStream_t st) {
    constexpr int kRows = 8 * (kThreads / (N / 4));  // state rows one pass of the two-head kernel covers
    const size_t ssm = m2_eager_stream_smem(a.P, N);
    if (SK == SK_F32 && TQ == 1 && a.op == OP_DECODE && a.T == 1 && a.P <= kThreads && ssm <= 112 * 1024) {
        auto ks = m2_eager_stream_kernel<N>;
        cudaError_t e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssm);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 0, occ = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, ks, kThreads, ssm)) != cudaSuccess) return e;
        const int items = a.B * a.H, cap = sms * (occ > 0 ? occ : 1);
        ks<<<items < cap ? items : cap, kThreads, ssm, st>>>(a);
        return cudaGetLastError();
    }
    if (TQ == 1 && a.op == OP_DECODE && a.T == 1 && (a.H / a.G) % 2 == 0 && a.P <= kRows) {
        auto k2 = m2_eager_decode2_kernel<N, SK>;
        const int smem2 = (int)sizeof(float) * (2 * pad4(2 * a.P) + 2 * pad4(N) + 8);
        cudaError_t e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
        if (e != cudaSuccess) return e;
        k2<<<a.B * a.H / 2, kThreads, smem2, st>>>(a);
        return cudaGetLastError();
    }
    auto k = m2_eager_kernel<N, SK, TQ>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<a.B * a.H, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int N, int TQ>
inline cudaError_t dispatch_rk(int which, int rk, const M2Args &a, const M2FoldLay &lay, size_t smem, int num_sms,
                               cudaStream_t st) {
    if (which == M2_PREP) return launch_prep_t<N, TQ>(a, smem, st);
    switch (rk) {
        case SK_F32:
            return which == M2_EAGER ? launch_eager_t<N, SK_F32, TQ>(a, smem, st)
                                     : launch_fold_t<N, SK_F32, TQ>(a, lay, num_sms, st);
        case SK_BF16:
            return which == M2_EAGER ? launch_eager_t<N, SK_BF16, TQ>(a, smem, st)
                                     : launch_fold_t<N, SK_BF16, TQ>(a, lay, num_sms, st);
        default:
            return which == M2_EAGER ? launch_eager_t<N, SK_FP8, TQ>(a, smem, st)
                                     : launch_fold_t<N, SK_FP8, TQ>(a, lay, num_sms, st);
    }
}

// Per-dstate entry points; each instantiation lives in its own translation unit.
// which: M2Kernel; lay: flush kernel shared memory (M2_FOLD); smem: the others'.
template <int N>
cudaError_t m2_dispatch_n(int which, int rk, int TQ, const M2Args &a, const M2FoldLay &lay, size_t smem,
                          int num_sms, cudaStream_t st) {
    if (TQ == 1) return dispatch_rk<N, 1>(which, rk, a, lay, smem, num_sms, st);
    if (TQ == 4) return dispatch_rk<N, 4>(which, rk, a, lay, smem, num_sms, st);
    return dispatch_rk<N, 8>(which, rk, a, lay, smem, num_sms, st);
}

}  // namespace rssm
