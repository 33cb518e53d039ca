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
    return sizeof(float) * gdn_smem_floats(cf.headdim, cf.dstate, cf.window, gtq_of(T), cf.kind == RSSM_KDA,
                                           cf.input_dtype == RSSM_BF16 ? 2 : 4);
}

cudaError_t gdn_launch(Ctx &h, int op, int T, const rssm_inputs *in, float *y, float *out, cudaStream_t st,
                       const Handoff *ho_in) {
    GArgs a{};
    const rssm_config &cf = h.cfg;
    a.B = cf.batch; a.H = cf.nheads; a.P = cf.headdim; a.W = cf.window;
    a.R = (int)h.lay.ring; a.Rs = (int)h.lay.ring_stride; a.T = T; a.op = op; a.in_bf16 = cf.input_dtype == RSSM_BF16;
    a.kda = cf.kind == RSSM_KDA;
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
    const int TQ = gtq_of(T), N = cf.dstate;
    const size_t smem = gdn_smem_bytes(cf, T);
    auto v1 = [&](const GArgs &g) -> cudaError_t {
        h.launches += 1;
        switch (N) {
            case 16: return g_dispatch_n<16>(eager, cf.state_dtype, TQ, g, smem, st);
            case 32: return g_dispatch_n<32>(eager, cf.state_dtype, TQ, g, smem, st);
            case 64: return g_dispatch_n<64>(eager, cf.state_dtype, TQ, g, smem, st);
            default: return g_dispatch_n<128>(eager, cf.state_dtype, TQ, g, smem, st);
        }
    };
    if (eager || !(op == OP_DECODE || op == OP_VERIFY)) {
        cudaError_t e = v1(a);
        if (e == cudaSuccess && !eager && op == OP_FLUSH) h.len_lb = h.len_ub = 0;
        return e;
    }
    // Replay decode/verify: the prep kernel (swept queries, coefficients,
    // appends), the fold-only kernel when some buffer may be too full for the
    // call's tokens, then the shared replay-read kernel.
    const Handoff ho = ho_in ? *ho_in : h.handoff();
    a.seqinfo = ho.seqinfo; a.dec = ho.dec; a.coef = ho.coef; a.query = ho.query;
    a.TQmax = ho.tq_max;
    a.Emax = (cf.window + a.TQmax + 3) & ~3;
    const bool fold = h.len_ub + T > cf.window;
    a.fold_launched = fold;
    const int wb = gdn_prep_warp_bytes(N, cf.window, TQ, a.in_bf16 ? 2 : 4, a.kda);
    a.prep_heads = (96 * 1024) / wb;
    if (a.prep_heads > kWarps) a.prep_heads = kWarps;
    if (a.prep_heads < 1) a.prep_heads = 1;
    h.launches += 1;
    cudaError_t e;
    switch (N) {
        case 16: e = g_prep_dispatch_n<16>(TQ, a, st); break;
        case 32: e = g_prep_dispatch_n<32>(TQ, a, st); break;
        case 64: e = g_prep_dispatch_n<64>(TQ, a, st); break;
        default: e = g_prep_dispatch_n<128>(TQ, a, st); break;
    }
    if (e == cudaSuccess && fold) {
        GArgs f = a;
        f.fold_only = 1;
        e = v1(f);
    }
    if (e == cudaSuccess && h.split_event) e = cudaEventRecord(h.split_event, st);
    if (e == cudaSuccess) {
        // swept queries r ([B][H][TQmax][N], fp32) against the read copy; x = v
        h.launches += 1;
        e = launch_read(h, op, T, ho.query, 0, 1, (int64_t)cf.nheads * a.TQmax * N, (int64_t)a.TQmax * N, N, in->v,
                        nullptr, y, ho, st, !fold, !h.split_event);
    }
    if (e != cudaSuccess) {
        cudaMemsetAsync(ho.fold_count, 0, sizeof(int), st);
        return e;
    }
    update_len_bounds(h, op, T);
    return cudaSuccess;
}

}  // namespace rssm
