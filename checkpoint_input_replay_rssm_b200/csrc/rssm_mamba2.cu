// rssm_mamba2.cu -- host launcher of the Mamba-2 kernels (rssm_mamba2.cuh); the
// kernel instantiations for each dstate are compiled in rssm_mamba2_n*.cu.
#include "rssm_mamba2.cuh"

namespace rssm {

extern template cudaError_t m2_dispatch_n<16>(int, int, int, const M2Args &, const M2FoldLay &, size_t, int, cudaStream_t);
extern template cudaError_t m2_dispatch_n<32>(int, int, int, const M2Args &, const M2FoldLay &, size_t, int, cudaStream_t);
extern template cudaError_t m2_dispatch_n<64>(int, int, int, const M2Args &, const M2FoldLay &, size_t, int, cudaStream_t);
extern template cudaError_t m2_dispatch_n<128>(int, int, int, const M2Args &, const M2FoldLay &, size_t, int, cudaStream_t);

static int tq_of(int T) { return T <= 1 ? 1 : (T <= 4 ? 4 : 8); }
static int in_bytes(const rssm_config &cf) { return cf.input_dtype == RSSM_BF16 ? 2 : 4; }

// Heads per prep CTA: up to the whole group (its B . C is computed once per CTA),
// within 48 KiB of shared memory so that many CTAs stay resident.
static int m2_prep_heads(const rssm_config &cf, int TQ) {
    const int hpg = cf.nheads / cf.ngroups;
    for (int hc = 16; hc > 1; --hc)
        if (hpg % hc == 0 && m2_prep_lay(hc, cf.headdim, cf.dstate, cf.window, TQ, in_bytes(cf)).bytes <= 48 * 1024)
            return hc;
    return 1;
}

// Heads per flush CTA: up to 8 heads of one group, within 75 KiB of shared
// memory so that three CTAs share an SM; a single head may take more.  On the
// 128-head layer three CTAs of 4 heads with two 16 KiB stages each folded in
// 0.63 ms per call, two CTAs of 4 heads with three stages in 0.75 ms, three
// CTAs of 2 heads in 0.70 ms: independent CTAs hide each other's prologue and
// store phases better than a deeper stage ring within one CTA.
static int ring_slots(const rssm_config &cf) { return cf.window + (cf.max_draft > 1 ? cf.max_draft : 1); }
static int m2_fold_heads(const rssm_config &cf, int TQ) {
    const int hpg = cf.nheads / cf.ngroups;
    for (int hc = 8; hc > 1; --hc)
        if (hpg % hc == 0 &&
            m2_fold_lay(hc, cf.headdim, cf.dstate, cf.window, ring_slots(cf), TQ, in_bytes(cf)).bytes <= 76800)
            return hc;
    return 1;
}

size_t mamba2_smem_bytes(const rssm_config &cf, int T) {
    const int TQ = tq_of(T), P = cf.headdim, N = cf.dstate;
    if (cf.mode == RSSM_EAGER)
        return sizeof(float) * ((size_t)2 * pad4(TQ * P) + 2 * pad4(TQ * N) + 2 * pad4(TQ));
    const size_t prep = m2_prep_lay(m2_prep_heads(cf, TQ), P, N, cf.window, TQ, in_bytes(cf)).bytes;
    const size_t fold = m2_fold_lay(m2_fold_heads(cf, TQ), P, N, cf.window, ring_slots(cf), TQ, in_bytes(cf)).bytes;
    return prep > fold ? prep : fold;
}

static cudaError_t dispatch(int which, int N, int rk, int TQ, const M2Args &a, const M2FoldLay &lay, size_t smem,
                            int num_sms, cudaStream_t st) {
    switch (N) {
        case 16: return m2_dispatch_n<16>(which, rk, TQ, a, lay, smem, num_sms, st);
        case 32: return m2_dispatch_n<32>(which, rk, TQ, a, lay, smem, num_sms, st);
        case 64: return m2_dispatch_n<64>(which, rk, TQ, a, lay, smem, num_sms, st);
        default: return m2_dispatch_n<128>(which, rk, TQ, a, lay, smem, num_sms, st);
    }
}

// Replay decode/verify: prep kernel, flush kernel (only when some sequence's
// buffer may be too full for the call's tokens: len_ub + T > W), replay-read
// kernel.  Flush/export: the
// flush kernel over every sequence.  Eager: one kernel.
cudaError_t mamba2_launch(Ctx &h, int op, int T, const rssm_inputs *in, float *y, float *out, cudaStream_t st,
                          const Handoff *ho_in) {
    const Handoff ho = ho_in ? *ho_in : h.handoff();
    M2Args a{};
    const rssm_config &cf = h.cfg;
    const int TQ = tq_of(T), ib = in_bytes(cf);
    a.B = cf.batch; a.H = cf.nheads; a.P = cf.headdim; a.G = cf.ngroups; a.W = cf.window;
    a.R = (int)h.lay.ring; a.Rs = (int)h.lay.ring_stride; a.T = T; a.op = op; a.in_bf16 = ib == 2;
    a.dt_scales = cf.dt_scales_input;
    if (ho.seqinfo) {
        a.seqinfo = ho.seqinfo;
        a.fold_count = ho.fold_count;
        a.fold_list = ho.fold_list;
        a.dec = ho.dec;
        a.coef = ho.coef;
        a.TQmax = ho.tq_max;
        a.Emax = (cf.window + a.TQmax + 3) & ~3;
    }
    a.c = h.counters();
    a.A = (const float *)h.at(h.lay.A_off); a.D = (const float *)h.at(h.lay.D_off);
    a.ckpt = h.lay.ckpt_bytes ? (float *)h.at(h.lay.ckpt_off) : nullptr;
    a.rc = h.lay.rc_bytes ? h.at(h.lay.rc_off) : nullptr;
    a.rc_scale = h.lay.rc_scale_bytes ? (float *)h.at(h.lay.rc_scale_off) : nullptr;
    a.xbuf = h.lay.xbuf_bytes ? h.at(h.lay.xbuf_off) : nullptr;
    a.Bbuf = h.lay.bbuf_bytes ? h.at(h.lay.bbuf_off) : nullptr;
    a.dtbuf = h.lay.sbuf_bytes ? (float *)h.at(h.lay.sbuf_off) : nullptr;
    a.snap = h.lay.snap_bytes ? h.at(h.lay.snap_off) : nullptr;
    if (a.snap && cf.state_dtype == RSSM_FP8E4M3) {
        const size_t elems = (size_t)cf.batch * cf.nheads * cf.headdim * cf.dstate;
        a.snap_scale = (float *)((uint8_t *)a.snap + (size_t)cf.max_draft * elems);
    }
    if (in) { a.x = in->x; a.dt = in->dt; a.Bm = in->Bm; a.Cm = in->Cm; }
    a.y = y; a.out = out;
    const int N = cf.dstate, rk = cf.state_dtype;
    M2FoldLay flay{};

    if (cf.mode == RSSM_EAGER) {
        h.launches += 1;
        return dispatch(M2_EAGER, N, rk, TQ, a, flay, mamba2_smem_bytes(cf, T), h.num_sms, st);
    }
    const int fHC = m2_fold_heads(cf, TQ);
    flay = m2_fold_lay(fHC, cf.headdim, N, cf.window, (int)h.lay.ring, TQ, ib);
    M2Args f = a;  // flush kernel arguments
    f.HC = fHC;
    f.cpg = (cf.nheads / cf.ngroups) / fHC;
    if (!(op == OP_DECODE || op == OP_VERIFY)) {  // flush / export
        h.launches += 1;
        cudaError_t e = dispatch(M2_FOLD, N, rk, TQ, f, flay, 0, h.num_sms, st);
        if (e == cudaSuccess && op == OP_FLUSH) h.len_lb = h.len_ub = 0;
        return e;
    }
    const bool fold = h.len_ub + T > cf.window;
    a.fold_launched = fold;
    a.HC = m2_prep_heads(cf, TQ);
    a.cpg = (cf.nheads / cf.ngroups) / a.HC;
    a.lay = m2_prep_lay(a.HC, cf.headdim, N, cf.window, TQ, ib);
    h.launches += 1;
    cudaError_t e = dispatch(M2_PREP, N, rk, TQ, a, flay, (size_t)a.lay.bytes, h.num_sms, st);
    if (e == cudaSuccess && fold) {
        h.launches += 1;
        e = dispatch(M2_FOLD, N, rk, TQ, f, flay, 0, h.num_sms, st);
    }
    if (e == cudaSuccess && h.split_event) e = cudaEventRecord(h.split_event, st);
    if (e == cudaSuccess) {
        // replay read: C of the group ([B][T][G][N]) is the query, x the buffered entries
        const int G = cf.ngroups;
        h.launches += 1;
        e = launch_read(h, op, T, in->Cm, ib == 2, cf.nheads / G, (int64_t)T * G * N, N, (int64_t)G * N, in->x,
                        (const float *)h.at(h.lay.D_off), y, ho, st, !fold, !h.split_event);
    }
    if (e != cudaSuccess) {  // leave no stale work list behind
        cudaMemsetAsync(ho.fold_count, 0, sizeof(int), st);
        return e;
    }
    update_len_bounds(h, op, T);
    return cudaSuccess;
}

}  // namespace rssm
