// rssm_gdn.cu -- host launcher of the Gated DeltaNet kernels (rssm_gdn.cuh); the
// kernel instantiations for each dstate are compiled in rssm_gdn_n*.cu.
#include "rssm_gdn.cuh"

namespace rssm {

extern template cudaError_t g_dispatch_n<16>(bool, int, int, const GArgs &, size_t, cudaStream_t);
extern template cudaError_t g_dispatch_n<32>(bool, int, int, const GArgs &, size_t, cudaStream_t);
extern template cudaError_t g_dispatch_n<64>(bool, int, int, const GArgs &, size_t, cudaStream_t);
extern template cudaError_t g_dispatch_n<128>(bool, int, int, const GArgs &, size_t, cudaStream_t);

static int gtq_of(int T) { return T <= 1 ? 1 : (T <= 4 ? 4 : 8); }

size_t gdn_smem_bytes(const rssm_config &cf, int T) {
    return sizeof(float) * gdn_smem_floats(cf.headdim, cf.dstate, cf.window, gtq_of(T));
}

cudaError_t gdn_launch(const Ctx &h, int op, int T, const rssm_inputs *in, float *y, float *out,
                       cudaStream_t st) {
    GArgs a{};
    const rssm_config &cf = h.cfg;
    a.B = cf.batch; a.H = cf.nheads; a.P = cf.headdim; a.W = cf.window;
    a.R = (int)h.lay.ring; a.Rs = (int)h.lay.ring_stride; a.T = T; a.op = op; a.in_bf16 = cf.input_dtype == RSSM_BF16;
    a.c = h.counters();
    a.ckpt = h.lay.ckpt_bytes ? (float *)h.at(h.lay.ckpt_off) : nullptr;
    a.rc = h.lay.rc_bytes ? h.at(h.lay.rc_off) : nullptr;
    a.rc_scale = h.lay.rc_scale_bytes ? (float *)h.at(h.lay.rc_scale_off) : nullptr;
    a.vbuf = h.lay.xbuf_bytes ? h.at(h.lay.xbuf_off) : nullptr;
    a.kbuf = h.lay.bbuf_bytes ? h.at(h.lay.bbuf_off) : nullptr;
    a.abuf = h.lay.sbuf_bytes ? (float *)h.at(h.lay.sbuf_off) : nullptr;
    a.bbuf = h.lay.tbuf_bytes ? (float *)h.at(h.lay.tbuf_off) : nullptr;
    a.snap = h.lay.snap_bytes ? h.at(h.lay.snap_off) : nullptr;
    if (a.snap && cf.state_dtype == RSSM_FP8E4M3) {
        const size_t elems = (size_t)cf.batch * cf.nheads * cf.headdim * cf.dstate;
        a.snap_scale = (float *)((uint8_t *)a.snap + (size_t)cf.max_draft * elems);
    }
    if (in) { a.q = in->q; a.k = in->k; a.v = in->v; a.alpha = in->alpha; a.beta = in->beta; }
    a.y = y; a.out = out;
    const bool eager = cf.mode == RSSM_EAGER;
    const int TQ = gtq_of(T);
    const size_t smem = gdn_smem_bytes(cf, T);
    switch (cf.dstate) {
        case 16: return g_dispatch_n<16>(eager, cf.state_dtype, TQ, a, smem, st);
        case 32: return g_dispatch_n<32>(eager, cf.state_dtype, TQ, a, smem, st);
        case 64: return g_dispatch_n<64>(eager, cf.state_dtype, TQ, a, smem, st);
        default: return g_dispatch_n<128>(eager, cf.state_dtype, TQ, a, smem, st);
    }
}

}  // namespace rssm
