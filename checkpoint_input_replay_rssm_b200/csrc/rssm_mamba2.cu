// rssm_mamba2.cu -- host launcher of the Mamba-2 kernels (rssm_mamba2.cuh); the
// kernel instantiations for each dstate are compiled in rssm_mamba2_n*.cu.
#include "rssm_mamba2.cuh"

namespace rssm {

extern template cudaError_t m2_dispatch_n<16>(bool, int, int, const M2Args &, size_t, cudaStream_t);
extern template cudaError_t m2_dispatch_n<32>(bool, int, int, const M2Args &, size_t, cudaStream_t);
extern template cudaError_t m2_dispatch_n<64>(bool, int, int, const M2Args &, size_t, cudaStream_t);
extern template cudaError_t m2_dispatch_n<128>(bool, int, int, const M2Args &, size_t, cudaStream_t);

static int tq_of(int T) { return T <= 1 ? 1 : (T <= 4 ? 4 : 8); }

// Replay pipeline shape: heads per item HC (dividing the heads of a group),
// stages NS and CTAs per SM.  Two CTAs per SM (two producers, sixteen consumer
// warps) when two stages fit 110 KiB each; otherwise one CTA with up to 4 stages
// in 200 KiB.  Items prefer 2 heads, then 1, then 4.
struct M2Pipe { int HC, NS, per_sm; size_t smem; };
static M2Pipe m2_pipe(const rssm_config &cf, int TQ) {
    const int hpg = cf.nheads / cf.ngroups, ib = cf.input_dtype == RSSM_BF16 ? 2 : 4;
    const int rcb = cf.state_dtype == RSSM_F32 ? 4 : (cf.state_dtype == RSSM_BF16 ? 2 : 1);
    auto total = [&](int hc, int ns) {
        return m2_smem_total(ns, hc, cf.headdim, cf.dstate, cf.window, TQ, ib, rcb);
    };
    for (int hc : {4, 2, 1}) {
        if (hpg % hc != 0) continue;
        for (int ns = 3; ns >= 2; --ns)
            if (total(hc, ns) <= 110 * 1024) return {hc, ns, 2, (size_t)total(hc, ns)};
    }
    for (int min_ns : {3, 1}) {
        for (int hc : {2, 1, 4}) {
            if (hpg % hc != 0) continue;
            for (int ns = 4; ns >= min_ns; --ns)
                if (total(hc, ns) <= 200 * 1024) return {hc, ns, 1, (size_t)total(hc, ns)};
        }
    }
    return {1, 1, 1, (size_t)total(1, 1)};
}

size_t mamba2_smem_bytes(const rssm_config &cf, int T) {
    const int TQ = tq_of(T), P = cf.headdim, N = cf.dstate;
    if (cf.mode == RSSM_EAGER)
        return sizeof(float) * ((size_t)2 * pad4(TQ * P) + 2 * pad4(TQ * N) + 2 * pad4(TQ));
    return m2_pipe(cf, TQ).smem;
}

cudaError_t mamba2_launch(const Ctx &h, int op, int T, const rssm_inputs *in, float *y, float *out,
                          cudaStream_t st) {
    M2Args a{};
    const rssm_config &cf = h.cfg;
    a.B = cf.batch; a.H = cf.nheads; a.P = cf.headdim; a.G = cf.ngroups; a.W = cf.window;
    a.R = (int)h.lay.ring; a.Rs = (int)h.lay.ring_stride; a.T = T; a.op = op; a.in_bf16 = cf.input_dtype == RSSM_BF16;
    a.dt_scales = cf.dt_scales_input;
    const M2Pipe pp = m2_pipe(cf, tq_of(T));
    a.HC = pp.HC;
    a.NS = pp.NS;
    {
        const int items = cf.batch * (cf.nheads / pp.HC);
        const int ctas = pp.per_sm * h.num_sms;
        a.grid = items < ctas ? items : ctas;
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
    const bool eager = cf.mode == RSSM_EAGER;
    const int TQ = tq_of(T);
    const size_t smem = mamba2_smem_bytes(cf, T);
    switch (cf.dstate) {
        case 16: return m2_dispatch_n<16>(eager, cf.state_dtype, TQ, a, smem, st);
        case 32: return m2_dispatch_n<32>(eager, cf.state_dtype, TQ, a, smem, st);
        case 64: return m2_dispatch_n<64>(eager, cf.state_dtype, TQ, a, smem, st);
        default: return m2_dispatch_n<128>(eager, cf.state_dtype, TQ, a, smem, st);
    }
}

}  // namespace rssm
