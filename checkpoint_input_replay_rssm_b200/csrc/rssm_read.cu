// rssm_read.cu -- host launcher of the replay-read kernel (rssm_read.cuh).
#include "rssm_read.cuh"

#include "rssm_internal.h"

namespace rssm {

extern template cudaError_t read_dispatch_n<16>(int, int, const ReadArgs &, size_t, cudaStream_t);
extern template cudaError_t read_dispatch_n<32>(int, int, const ReadArgs &, size_t, cudaStream_t);
extern template cudaError_t read_dispatch_n<64>(int, int, const ReadArgs &, size_t, cudaStream_t);
extern template cudaError_t read_dispatch_n<128>(int, int, const ReadArgs &, size_t, cudaStream_t);

static int tq_of_read(int T) { return T <= 1 ? 1 : (T <= 4 ? 4 : 8); }

// Heads per read CTA: about 128 KiB of read copy per CTA, the heads sharing one
// query row when a query row serves several heads (Mamba-2 groups).  A CTA
// streams its rows in rounds of 8 x 16 bytes per thread, each half of a round
// reissued as soon as it has been dotted, and its small operands' round trips
// overlap the stream; on the 128-head layer 32 KiB gave 0.65 of peak bandwidth, 64 KiB
// 0.76, 128 KiB 0.81, 256 KiB 0.48 (too few CTAs for the SMs).  Shapes with
// small heads are also held to 64 KiB of shared memory at the largest query
// count (the buffered entries and coefficients grow with the heads).
static int read_tqm(const rssm_config &cf) { return cf.max_draft > 1 ? cf.max_draft : 1; }
static int read_ep(const rssm_config &cf) { return (cf.window + read_tqm(cf) + 3) & ~3; }

int read_heads_per_cta(const rssm_config &cf) {
    const int rcb = cf.state_dtype == RSSM_F32 ? 4 : (cf.state_dtype == RSSM_BF16 ? 2 : 1);
    const int ib = cf.input_dtype == RSSM_BF16 ? 2 : 4;
    const int qg = cf.kind == RSSM_MAMBA2 ? cf.nheads / cf.ngroups : 1;
    const int unit = qg > 1 ? qg : cf.nheads;  // heads a CTA may span
    int want = (128 * 1024) / (cf.headdim * cf.dstate * rcb);
    if (want < 1) want = 1;
    int hc = 1;
    for (int d = 2; d <= unit && d <= want; ++d)
        if (unit % d == 0 && cf.nheads % d == 0 &&
            read_lay(d, cf.headdim, cf.dstate, cf.window, tq_of_read(read_tqm(cf)), ib, read_ep(cf)).bytes <=
                64 * 1024)
            hc = d;
    return hc;
}

size_t read_smem_bytes(const rssm_config &cf, int T) {
    const int ib = cf.input_dtype == RSSM_BF16 ? 2 : 4;
    return (size_t)read_lay(read_heads_per_cta(cf), cf.headdim, cf.dstate, cf.window, tq_of_read(T), ib,
                            read_ep(cf)).bytes;
}

cudaError_t launch_read(const Ctx &h, int op, int T, const void *Q, int q_bf16, int q_group, int64_t q_stride_b,
                        int64_t q_stride_row, int64_t q_stride_m, const void *xnew, const float *D,
                        float *y, const Handoff &ho, cudaStream_t st, bool early, bool pdl) {
    const rssm_config &cf = h.cfg;
    ReadArgs r{};
    r.B = cf.batch; r.H = cf.nheads; r.P = cf.headdim; r.R = (int)h.lay.ring; r.W = cf.window;
    r.T = T; r.HC = read_heads_per_cta(cf); r.in_bf16 = cf.input_dtype == RSSM_BF16;
    r.q_group = q_group; r.q_bf16 = q_bf16;
    r.q_stride_b = q_stride_b; r.q_stride_row = q_stride_row; r.q_stride_m = q_stride_m;
    r.Q = Q;
    r.rc = cf.state_dtype == RSSM_F32 ? h.at(h.lay.ckpt_off) : h.at(h.lay.rc_off);
    r.rc_scale = h.lay.rc_scale_bytes ? (const float *)h.at(h.lay.rc_scale_off) : nullptr;
    r.xring = h.at(h.lay.xbuf_off);
    r.xnew = xnew;
    r.D = D;
    r.seqinfo = ho.seqinfo;
    r.dec = ho.dec;
    r.coef = ho.coef;
    r.TQmax = ho.tq_max;
    r.Emax = (cf.window + r.TQmax + 3) & ~3;
    r.y = y;
    r.c = h.counters();
    r.fold_count = ho.fold_count;
    r.op = op;
    r.early = early ? 1 : 0;
    r.pdl = (early && pdl) ? 1 : 0;
    r.q_ready = (Q != (const void *)ho.query) ? 1 : 0;  // Mamba-2: the call's C; GDN / KDA: the swept queries
    const int TQ = tq_of_read(T);
    r.lay = read_lay(r.HC, cf.headdim, cf.dstate, cf.window, TQ, cf.input_dtype == RSSM_BF16 ? 2 : 4, r.Emax);
    const size_t smem = read_smem_bytes(cf, T);
    switch (cf.dstate) {
        case 16: return read_dispatch_n<16>(cf.state_dtype, TQ, r, smem, st);
        case 32: return read_dispatch_n<32>(cf.state_dtype, TQ, r, smem, st);
        case 64: return read_dispatch_n<64>(cf.state_dtype, TQ, r, smem, st);
        default: return read_dispatch_n<128>(cf.state_dtype, TQ, r, smem, st);
    }
}

}  // namespace rssm
