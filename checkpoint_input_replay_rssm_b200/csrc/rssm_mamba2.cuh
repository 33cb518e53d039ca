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
// the host.  Entry slots of x: E = W + TQ; committed entries sit right-aligned
// before slot W and the call's own tokens at W..W+T-1, so logical entry e is
// slot (W - L0) + e.  The group's B ring is staged whole (R <= W + 8 rows).
struct M2PrepLay {
    int fold, bar, sC, sBr, sBn, sx, dring, dtn, sd, slam, scoef, sdec, su, sfdec, sCf, sdot, si, bytes;
};
inline M2PrepLay m2_prep_lay(int HC, int P, int N, int W, int TQ, int ib) {
    const int E = W + TQ;
    M2PrepLay L{};
    int o = 0;
    L.fold = o;  o += 2 * kFoldChunk;            // fp32 checkpoint rows, two stages
    L.bar = o;   o += 16;                        // their mbarriers
    L.sC = o;    o += a16(TQ * N * ib);          // raw C of the queries     [TQ][N]
    L.sBr = o;   o += a16((W + 8) * N * ib);     // raw B ring of the group  [R][N]
    L.sBn = o;   o += a16(TQ * N * ib);          // raw B of the call's tokens [TQ][N]
    L.sx = o;    o += a16(HC * E * P * ib);      // raw x of the entries     [HC][E][P]
    L.dring = o; o += a16(HC * dt_row_max_bytes(W));  // dt ring rows        [HC][Rs]
    L.dtn = o;   o += a16(TQ * HC * 4);          // dt of the call's tokens  [TQ][HC]
    L.sd = o;    o += a16(TQ * E * 4);           // B_e . C_m                [TQ][E]
    L.slam = o;  o += a16(HC * E * 4);           // prefix sums of dt*A      [HC][E]
    L.scoef = o; o += a16(HC * TQ * E * 4);      // replay coefficients      [HC][TQ][E]
    L.sdec = o;  o += a16(HC * TQ * 4);          // decay of S^ C            [HC][TQ]
    L.su = o;    o += a16(HC * E * 4);           // fold weights             [HC][E]
    L.sfdec = o; o += a16(HC * 4);               // decay of the folded checkpoint [HC]
    L.sCf = o;   o += a16(TQ * N * 4);           // C as fp32                [TQ][N]
    L.sdot = o;  o += a16(HC * P * TQ * 4);      // fresh copy . C per row   [HC*P][TQ]
    L.si = o;    o += 32;
    L.bytes = o;
    return L;
}

struct M2Args {
    int B, H, P, G, W, R, Rs, T, op, in_bf16, dt_scales;  // Rs: dt ring row length
    int HC, cpg;        // heads per prep CTA (divides H / G); prep CTAs per group
    M2PrepLay lay;      // prep kernel shared memory
    int4 *seqinfo;      // per sequence, for the read kernel: {L0, ring slot of entry 0, folded, 0}
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
// Prep / flush kernel: decode (T = 1), verify (T = K), flush and export (T = 0).
//
// One CTA per (group chunk of HC heads, sequence b).  In one round trip it reads
// the sequence's counters and stages the group's whole B ring, the heads' dt
// ring rows and the call's tokens; then B_e . C_m once for the group and, per
// head (one warp each), the prefix sums Lam of dt*A and the coefficients.
//   * no fold: the replay coefficients
//       coef[m][e] = e^{Lam_{L0+m} - Lam_e} (B_e . C_m) s_e,   dec[m] = e^{Lam_{L0+m}}
//     go to the read kernel;
//   * fold (len + T > W, or flush/export): the committed entries are folded into
//     the fp32 checkpoint, S_c <- e^{Lam_{L0-1}} S_c + sum_e e^{Lam_{L0-1} - Lam_e} s_e x_e B_e^T.
//     Thread 0 starts bulk copies of the checkpoint rows (16 KiB stages, two in
//     flight) as soon as it has read the counters; the CTA stores the result
//     with the requantised read copy (or writes it out, for export) and, for
//     decode/verify, computes the outputs from the fresh copy itself.
// Last it appends the call's tokens to the ring, and thread 0 registers the
// CTA's arrival; the last CTA of the sequence publishes the counters.
// ---------------------------------------------------------------------------
template <int N, int RK, int TQ, bool BF>
__global__ void __launch_bounds__(kThreads, 3) m2_prep_kernel(const M2Args a) {
    constexpr int TPR4 = N / 4;           // lanes per row, fp32 quad mapping
    constexpr int RPP4 = kThreads / TPR4;
    constexpr int FC = kFoldChunk / (N * 4);  // fp32 rows per fold stage
    constexpr int FH = FC / RPP4;         // rows per thread per stage (= 4)
    constexpr int FB = 4;                 // buffered B entries held in registers per block
    constexpr int IB = BF ? 2 : 4;
    static_assert(FH * RPP4 == FC, "fold stage is FH rows per thread");
    extern __shared__ __align__(128) uint8_t smraw[];
    const M2PrepLay &Ly = a.lay;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, P = a.P, W = a.W, R = a.R, T = a.T, G = a.G, HC = a.HC;
    const int hpg = H / G;
    const int b = blockIdx.y;
    const int g = blockIdx.x / a.cpg, hc = blockIdx.x - g * a.cpg;
    const int h0 = g * hpg + hc * HC;
    const int E = W + TQ;
    float *fbuf = reinterpret_cast<float *>(smraw + Ly.fold);
    uint64_t *fbar = reinterpret_cast<uint64_t *>(smraw + Ly.bar);
    uint8_t *sC = smraw + Ly.sC, *sBr = smraw + Ly.sBr, *sBn = smraw + Ly.sBn, *sx = smraw + Ly.sx;
    float *dring = reinterpret_cast<float *>(smraw + Ly.dring);
    float *dtn = reinterpret_cast<float *>(smraw + Ly.dtn);
    float *sd = reinterpret_cast<float *>(smraw + Ly.sd);
    float *slam = reinterpret_cast<float *>(smraw + Ly.slam);
    float *scoef = reinterpret_cast<float *>(smraw + Ly.scoef);
    float *sdec = reinterpret_cast<float *>(smraw + Ly.sdec);
    float *su = reinterpret_cast<float *>(smraw + Ly.su);
    float *sfdec = reinterpret_cast<float *>(smraw + Ly.sfdec);
    float *sCf = reinterpret_cast<float *>(smraw + Ly.sCf);
    float *sdot = reinterpret_cast<float *>(smraw + Ly.sdot);
    int *si = reinterpret_cast<int *>(smraw + Ly.si);
    const int64_t row0 = (int64_t)b * H + h0;
    const int64_t tile0 = row0 * P * N;
    const int nrows = HC * P;
    const int nfc = (nrows + FC - 1) / FC;  // fold stages
    const bool reads = (a.op == OP_DECODE || a.op == OP_VERIFY);
    const int xrow = P * IB, brow = N * IB, xch = xrow / 16, bch = brow / 16;
    const int Rs = a.Rs;
    auto ldx = [](const uint8_t *p) -> float {
        return BF ? bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(p)) : *reinterpret_cast<const float *>(p);
    };
    auto fold_issue = [&](int c) {  // thread 0: stage c of the checkpoint rows into buffer c & 1
        const int r0 = c * FC, r1 = min(nrows, r0 + FC);
        const uint32_t bytes = (uint32_t)((r1 - r0) * N * 4);
        mbar_arrive_expect_tx(&fbar[c & 1], bytes);
        bulk_g2s(fbuf + (c & 1) * (FC * N), a.ckpt + tile0 + (int64_t)r0 * N, bytes, &fbar[c & 1]);
    };

    // 1. Counters (thread 0; starts the fold's checkpoint copies when one is due)
    //    and everything that does not depend on them, at once.
    SeqState ss{};
    if (tid == 0) {
        ss = read_counters(a.c, b, W);
        const int L0 = (int)(ss.seq - ss.ckpt);
        int flush = 0;
        if (ss.ok) flush = (a.op == OP_FLUSH || a.op == OP_EXPORT) ? (L0 > 0) : (L0 + T > W);
        si[0] = ss.ok;
        si[1] = ss.ok ? L0 : 0;
        si[2] = flush;
        si[3] = (int)(ss.ckpt % R);
        si[4] = (int)(ss.seq % R);
        if (flush) {
            mbar_init(&fbar[0], 1);
            mbar_init(&fbar[1], 1);
            mbar_init_fence();
            fold_issue(0);
            if (nfc > 1) fold_issue(1);
        }
        // seqinfo: {ring entries the read kernel replays, ring slot of entry 0,
        // folded here, counters valid} -- the read kernel also publishes the
        // sequence's new counters from it
        if (!ss.ok) {
            if (blockIdx.x == 0) report(a.c.err, DEV_BAD_COUNTERS, b, h0, L0);
            if (reads && blockIdx.x == 0) a.seqinfo[b] = make_int4(0, 0, 1, 0);  // nothing to read or publish
        } else if (reads && blockIdx.x == 0) {
            a.seqinfo[b] = make_int4(flush ? 0 : L0, (int)(ss.ckpt % R), flush, 1);
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
        for (int k = lane; k < xch; k += 32) cp_async16(sx + (hh * E + W + m) * xrow + k * 16, src + k * 16);
    }
    for (int i = tid; i < T * HC; i += kThreads) {
        const int m = i / HC, hh = i - m * HC;
        dtn[m * HC + hh] = a.dt[(int64_t)(b * T + m) * H + h0 + hh];
    }
    cp_async_wait_all();
    __syncthreads();
    if (!si[0]) return;  // counters corrupted: reported, sequence skipped, no arrival
    const int L0 = si[1], flush = si[2], ckmod = si[3], spmod = si[4];
    const int base = W - L0, nE = L0 + T;
    const int e0 = flush ? L0 : 0;  // first entry the outputs replay
    auto slot_of = [&](int e) { const int s = ckmod + e; return s >= R ? s - R : s; };
    auto B_of = [&](int e) -> const uint8_t * {  // B of logical entry e
        return e < L0 ? sBr + slot_of(e) * brow : sBn + (e - L0) * brow;
    };
    auto dt_of = [&](int hh, int e) -> float {
        return e < L0 ? dring[hh * Rs + slot_of(e)] : dtn[(e - L0) * HC + hh];
    };
    if (flush) {  // the heads' buffered x, needed only to fold
        const int n1 = min(L0, R - ckmod);
        for (int row = warp; row < 2 * HC; row += kWarps) {
            const int hh = row >> 1, second = row & 1;
            const int cnt = second ? L0 - n1 : n1;
            const uint8_t *src = reinterpret_cast<const uint8_t *>(a.xbuf) +
                                 (((row0 + hh) * R + (second ? 0 : ckmod)) * P) * IB;
            uint8_t *dst = sx + (hh * E + base + (second ? n1 : 0)) * xrow;
            for (int k = lane; k < cnt * xch; k += 32) cp_async16(dst + k * 16, src + k * 16);
        }
    }

    // 2. B_e . C_m once for the group (warps), C as fp32.
    if (reads) {
        for (int pr = warp; pr < T * nE; pr += kWarps) {
            const int m = pr / nE, e = pr - m * nE;
            if (e > L0 + m || e < e0) continue;  // warp-uniform
            const uint8_t *Bp = B_of(e), *Cp = sC + m * brow;
            float d = 0.f;
            for (int n = lane; n < N; n += 32) d = fmaf(ldx(Bp + n * IB), ldx(Cp + n * IB), d);
            d = group_sum<32>(d);
            if (lane == 0) sd[m * E + e] = d;
        }
        for (int i = tid; i < T * N; i += kThreads) sCf[i] = ldx(sC + i * IB);
    }
    __syncthreads();

    // 3. Per head (one warp): prefix sums of dt*A, coefficients, decays.
    for (int hh = warp; hh < HC; hh += kWarps) {
        const float Ah = a.A[h0 + hh];
        float *lam = slam + hh * E + base;
        float carry = 0.f;
        for (int k0 = 0; k0 < nE; k0 += 32) {
            const int e = k0 + lane;
            float v = (e < nE) ? dt_of(hh, e) * Ah : 0.f;
            v = warp_incl_scan(v) + carry;
            if (e < nE) lam[e] = v;
            carry = __shfl_sync(0xffffffffu, v, 31);
        }
        __syncwarp();
        const float lam_f = (flush && L0 > 0) ? lam[L0 - 1] : 0.f;
        for (int e = lane; e < nE; e += 32) {
            const float se = a.dt_scales ? dt_of(hh, e) : 1.f;
            if (reads) {
#pragma unroll
                for (int m = 0; m < TQ; ++m) {
                    if (m >= T || e > L0 + m || e < e0) continue;
                    const float cf = expf(lam[L0 + m] - lam[e]) * sd[m * E + e] * se;
                    if (flush) scoef[(hh * TQ + m) * E + e] = cf;
                    else a.coef[((row0 + hh) * a.TQmax + m) * a.Emax + e] = cf;
                }
            }
            if (flush && e < L0) su[hh * E + e] = expf(lam_f - lam[e]) * se;
        }
        if (lane == 0) sfdec[hh] = flush ? expf(lam_f) : 1.f;
        if (reads && lane < T) {
            const float dcy = expf(lam[L0 + lane] - lam_f);
            if (flush) sdec[hh * TQ + lane] = dcy;
            else a.dec[(row0 + hh) * a.TQmax + lane] = dcy;
        }
    }

    if (flush) {
        cp_async_wait_all();
        __syncthreads();
        // 4. Fold, one staged 16 KiB block of checkpoint rows at a time (the next
        //    one in flight): FH rows per thread, FB buffered B entries per block
        //    in registers; store the checkpoint and the requantised copy, and dot
        //    the fresh copy with C.
        const int c4 = tid % TPR4, q0 = tid / TPR4;
        bool timed_out = false;
        for (int c = 0; c < nfc; ++c) {
            const bool got = mbar_wait(&fbar[c & 1], (c >> 1) & 1);
            if (__syncthreads_or(!got)) {
                timed_out = true;
                break;
            }
            const float *tf = fbuf + (c & 1) * (FC * N);
            float4 v[FH];
            int gr[FH];
#pragma unroll
            for (int k = 0; k < FH; ++k) {
                const int rl = q0 + k * RPP4;
                gr[k] = c * FC + rl;
                v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (gr[k] < nrows) {
                    v[k] = *reinterpret_cast<const float4 *>(tf + rl * N + 4 * c4);
                    const float dc = sfdec[gr[k] / P];
                    v[k].x *= dc; v[k].y *= dc; v[k].z *= dc; v[k].w *= dc;
                }
            }
            for (int eb = 0; eb < L0; eb += FB) {
                float4 Bq[FB];
#pragma unroll
                for (int j = 0; j < FB; ++j) {
                    const uint8_t *Br = B_of(eb + j) + 4 * c4 * IB;
                    Bq[j] = (eb + j < L0) ? make_float4(ldx(Br), ldx(Br + IB), ldx(Br + 2 * IB), ldx(Br + 3 * IB))
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int k = 0; k < FH; ++k) {
                    if (gr[k] >= nrows) continue;
                    const int hh = gr[k] / P, p = gr[k] - hh * P;
                    const uint8_t *xr = sx + (hh * E + base + eb) * xrow + p * IB;
                    const float *uw = su + hh * E + eb;
#pragma unroll
                    for (int j = 0; j < FB; ++j) {
                        if (eb + j < L0) {
                            const float w = uw[j] * ldx(xr + j * xrow);
                            v[k].x = fmaf(w, Bq[j].x, v[k].x); v[k].y = fmaf(w, Bq[j].y, v[k].y);
                            v[k].z = fmaf(w, Bq[j].z, v[k].z); v[k].w = fmaf(w, Bq[j].w, v[k].w);
                        }
                    }
                }
            }
            __syncthreads();  // every thread has its rows of this stage in registers
            if (tid == 0 && c + 2 < nfc) fold_issue(c + 2);
#pragma unroll
            for (int k = 0; k < FH; ++k) {
                const bool valid = gr[k] < nrows;
                const int64_t el = tile0 + (int64_t)(valid ? gr[k] : 0) * N + 4 * c4;
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
                        if (c4 == 0) a.rc_scale[row0 * P + gr[k]] = sc;
                    }
                }
                if (reads) {
#pragma unroll
                    for (int m = 0; m < TQ; ++m) {
                        const float4 Cq = *reinterpret_cast<const float4 *>(sCf + m * N + 4 * c4);
                        float d = rd.x * Cq.x + rd.y * Cq.y + rd.z * Cq.z + rd.w * Cq.w;
                        d = group_sum<TPR4>(d);
                        if (c4 == 0 && valid && m < T) sdot[gr[k] * TQ + m] = d;
                    }
                }
            }
        }
        if (timed_out) {  // a checkpoint copy never landed: reported, sequence left as it was
            if (tid == 0) report(a.c.err, DEV_PIPE_TIMEOUT, b, h0, 0);
            return;
        }
        if (reads) {
            __syncthreads();
            // Outputs of the folded sequence: the fresh copy plus the call's own tokens.
            for (int i = tid; i < T * nrows; i += kThreads) {
                const int m = i / nrows, r2 = i - m * nrows;
                const int hh = r2 / P, p = r2 - hh * P;
                float yv = sdec[hh * TQ + m] * sdot[r2 * TQ + m];
                const float *cf = scoef + (hh * TQ + m) * E;
                const uint8_t *xs = sx + (hh * E + base) * xrow + p * IB;
                for (int e = e0; e <= L0 + m; ++e) yv = fmaf(cf[e], ldx(xs + e * xrow), yv);
                yv = fmaf(a.D[h0 + hh], ldx(sx + (hh * E + W + m) * xrow + p * IB), yv);
                a.y[((int64_t)(b * T + m) * H + h0 + hh) * P + p] = yv;
            }
        }
    }

    // 5. Append the call's tokens to the ring (slots seq_pos + m mod R).
    if (reads) {
        for (int row = warp; row < T * HC; row += kWarps) {
            const int m = row / HC, hh = row - m * HC;
            const int slot = spmod + m >= R ? spmod + m - R : spmod + m;
            uint8_t *dst = reinterpret_cast<uint8_t *>(a.xbuf) + (((row0 + hh) * R + slot) * P) * IB;
            const uint8_t *src = sx + (hh * E + W + m) * xrow;
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
    // 6. Flush: this CTA read the counters long ago; its arrival lets the last CTA
    //    of the sequence publish them.  (Decode and verify publish from the read
    //    kernel, which runs after every prep CTA has read them.)
    if (tid == 0 && a.op == OP_FLUSH)
        arrive_and_publish(a.c, b, G * a.cpg, -1, flush ? ss.seq : -1, -1, flush);
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
    auto k = a.in_bf16 ? m2_prep_kernel<N, RK, TQ, true> : m2_prep_kernel<N, RK, TQ, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<dim3(a.H / a.HC, a.B), kThreads, smem, st>>>(a);
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

// Per-dstate entry points; each instantiation lives in its own translation unit.
template <int N>
cudaError_t m2_dispatch_n(bool eager, int rk, int TQ, const M2Args &a, size_t smem, cudaStream_t st) {
    return dispatch_tq<N>(eager, rk, TQ, a, smem, st);
}

}  // namespace rssm
