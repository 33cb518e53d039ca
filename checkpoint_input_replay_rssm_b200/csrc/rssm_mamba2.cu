// rssm_mamba2.cu -- host launcher of the Mamba-2 kernels (rssm_mamba2.cuh); the
// kernel instantiations for each dstate are compiled in rssm_mamba2_n*.cu.
#include "rssm_mamba2.cuh"

namespace rssm {

extern template cudaError_t m2_dispatch_n<16>(bool, int, int, const M2Args &, size_t, cudaStream_t);
extern template cudaError_t m2_dispatch_n<32>(bool, int, int, const M2Args &, size_t, cudaStream_t);
extern template cudaError_t m2_dispatch_n<64>(bool, int, int, const M2Args &, size_t, cudaStream_t);
extern template cudaError_t m2_dispatch_n<128>(bool, int, int, const M2Args &, size_t, cudaStream_t);

static int tq_of(int T) { return T <= 1 ? 1 : (T <= 4 ? 4 : 8); }

// Heads per prep CTA: up to 8 heads of one group (the group's B . C is computed
// once per CTA), within 160 KiB of shared memory.
static int m2_prep_heads(const rssm_config &cf, int TQ) {
    const int hpg = cf.nheads / cf.ngroups, ib = cf.input_dtype == RSSM_BF16 ? 2 : 4;
    for (int hc = 8; hc > 1; --hc)
        if (hpg % hc == 0 && m2_prep_lay(hc, cf.headdim, cf.dstate, cf.window, TQ, ib).bytes <= 150 * 1024)
            return hc;
    return 1;
}

size_t mamba2_smem_bytes(const rssm_config &cf, int T) {
    const int TQ = tq_of(T), P = cf.headdim, N = cf.dstate;
    if (cf.mode == RSSM_EAGER)
        return sizeof(float) * ((size_t)2 * pad4(TQ * P) + 2 * pad4(TQ * N) + 2 * pad4(TQ));
    const int ib = cf.input_dtype == RSSM_BF16 ? 2 : 4;
    return (size_t)m2_prep_lay(m2_prep_heads(cf, TQ), P, N, cf.window, TQ, ib).bytes;
}

cudaError_t mamba2_launch(const Ctx &h, int op, int T, const rssm_inputs *in, float *y, float *out,
                          cudaStream_t st) {
    M2Args a{};
    const rssm_config &cf = h.cfg;
    a.B = cf.batch; a.H = cf.nheads; a.P = cf.headdim; a.G = cf.ngroups; a.W = cf.window;
    a.R = (int)h.lay.ring; a.Rs = (int)h.lay.ring_stride; a.T = T; a.op = op; a.in_bf16 = cf.input_dtype == RSSM_BF16;
    a.dt_scales = cf.dt_scales_input;
    a.HC = m2_prep_heads(cf, tq_of(T));
    a.cpg = (cf.nheads / cf.ngroups) / a.HC;
    a.lay = m2_prep_lay(a.HC, cf.headdim, cf.dstate, cf.window, tq_of(T), cf.input_dtype == RSSM_BF16 ? 2 : 4);
    if (h.lay.seqinfo_bytes) {
        a.seqinfo = (int4 *)h.at(h.lay.seqinfo_off);
        a.dec = (float *)h.at(h.lay.dec_off);
        a.coef = (float *)h.at(h.lay.coef_off);
        a.TQmax = (int)h.lay.tq_max;
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
    const bool eager = cf.mode == RSSM_EAGER;
    const int TQ = tq_of(T);
    const size_t smem = mamba2_smem_bytes(cf, T);
    cudaError_t e;
    switch (cf.dstate) {
        case 16: e = m2_dispatch_n<16>(eager, cf.state_dtype, TQ, a, smem, st); break;
        case 32: e = m2_dispatch_n<32>(eager, cf.state_dtype, TQ, a, smem, st); break;
        case 64: e = m2_dispatch_n<64>(eager, cf.state_dtype, TQ, a, smem, st); break;
        default: e = m2_dispatch_n<128>(eager, cf.state_dtype, TQ, a, smem, st); break;
    }
    if (e != cudaSuccess || eager || !(op == OP_DECODE || op == OP_VERIFY)) return e;
    if (h.split_event) {
        e = cudaEventRecord(h.split_event, st);
        if (e != cudaSuccess) return e;
    }
    // replay read: C of the group ([B][T][G][N]) is the query, x the buffered entries
    const int G = cf.ngroups;
    return launch_read(h, op, T, in->Cm, cf.input_dtype == RSSM_BF16, cf.nheads / G, (int64_t)T * G * cf.dstate,
                       cf.dstate, (int64_t)G * cf.dstate, in->x, (const float *)h.at(h.lay.D_off), y, st);
}

}  // namespace rssm
