// rssm_static_scratch.cu -- rssm_decode_static_scratch: the replay decode with
// its per-call scratch kept in one file-scope device array instead of the
// handle's workspace.
//
// Who needs it: callers that cannot allocate device memory on the decode path --
// an engine whose memory pool is fixed before the model is loaded, or a step
// captured once and replayed, where a cudaMalloc would stall every stream of the
// device or is not allowed at all -- and that give each layer memory for its
// state only, decoding the layers one after another on one stream.  Every
// replay decode passes a per-call hand-off from its prep kernel to its flush
// and read kernels (per-sequence ring info, the flush work list, the replay
// decays and coefficients, and for Gated DeltaNet / KDA the swept queries:
// about 2.8 MB for a 256-sequence, 128-head Mamba-2 layer with window 16 and
// 4.7 MB for a 256-sequence, 32-head, d_k 128 GDN layer), rewritten by every
// call and dead between calls.  Here every layer shares one such array, part of
// the loaded module: nothing is allocated, at run time or at set-up.
//
// The method itself (the pages on checkpointed input replay) has no such entry
// point; it computes exactly what rssm_decode computes, with the same kernels.
//
// Limits and sharing:
//   - the hand-off of one decode call must fit kStaticScratchBytes (8 MiB);
//     larger layers are refused with RSSM_EINVAL before anything is enqueued;
//   - all calls on a device share the array and each call leaves its contents
//     behind: calls whose kernels can overlap (several streams, several host
//     threads) race on it and must not be issued concurrently;
//   - the first call on a device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current and keeps it for the life
//     of the process: make that first call before any stream capture, and do not
//     use the entry point again on a device after cudaDeviceReset.
#include <mutex>
#include <string>

#include "rssm_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = 8u << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_handoff_scratch[kStaticScratchBytes];

std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

// Offsets of one decode call's hand-off (one query per call) inside the array;
// the swept queries only for the delta-rule layers.
struct Carve {
    size_t seqinfo, fold, dec, coef, query, total;
};
Carve carve(const rssm_config &c) {
    const size_t B = c.batch, H = c.nheads, N = c.dstate;
    const size_t Emax = ((size_t)c.window + 1 + 3) & ~(size_t)3;  // window + 1 entries, padded to 4
    Carve k{};
    size_t o = 0;
    k.seqinfo = o; o = up256(o + B * 16);
    k.fold = o;    o = up256(o + 16 + B * 4);  // count, 3 pad words, list[B]
    k.dec = o;     o = up256(o + B * H * 4);
    k.coef = o;    o = up256(o + B * H * Emax * 4);
    k.query = o;
    if (c.kind != RSSM_MAMBA2) o = up256(o + B * H * N * 4);
    k.total = o;
    return k;
}

// Device address of the array on the current device (looked up once per device).
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev >= 0 && dev < kMaxDevices && g_addr[dev]) {
        *out = g_addr[dev];
        return cudaSuccess;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_handoff_scratch);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) g_addr[dev] = p;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" RSSM_API rssm_status rssm_decode_static_scratch(rssm_handle hh, const rssm_inputs *in, float *y) {
    using namespace rssm;
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    if (h->cfg.mode != RSSM_REPLAY)
        return api_fail(h, RSSM_EINVAL, "decode_static_scratch: only REPLAY layers have a per-call hand-off");
    if (h->pending) return api_fail(h, RSSM_ESTATE, "decode while a verify is pending (commit first)");
    if (!api_inputs_ok(h, in) || !y)
        return api_fail(h, RSSM_EINVAL,
                        "missing or misaligned input/output pointer (device arrays must be 16-byte aligned)");
    const Carve k = carve(h->cfg);
    if (k.total > kStaticScratchBytes)
        return api_fail(h, RSSM_EINVAL,
                        "decode_static_scratch: the hand-off needs " + std::to_string(k.total) +
                            " bytes; the static array holds " + std::to_string(kStaticScratchBytes) +
                            " (needed: batch * 20 + 16 + batch * nheads * 4 * (1 + round_up4(window + 1)) bytes,"
                            " plus batch * nheads * dstate * 4 for a delta-rule layer, each region padded to 256"
                            " bytes)");
    void *base = nullptr;
    cudaError_t e = scratch_address(&base);
    if (e != cudaSuccess) return api_cuda_fail(h, e, "decode_static_scratch: cudaGetSymbolAddress");
    uint8_t *p = (uint8_t *)base;
    Handoff ho{};
    ho.seqinfo = (int4 *)(p + k.seqinfo);
    ho.fold_count = (int *)(p + k.fold);
    ho.fold_list = ho.fold_count + 4;
    ho.dec = (float *)(p + k.dec);
    ho.coef = (float *)(p + k.coef);
    ho.query = h->cfg.kind == RSSM_MAMBA2 ? nullptr : (float *)(p + k.query);
    ho.tq_max = 1;
    // The work-list length must start at zero; the read kernel leaves it zero,
    // but a call refused or failed half-way on another handle may not have.
    e = cudaMemsetAsync(ho.fold_count, 0, sizeof(int), h->stream);
    if (e == cudaSuccess)
        e = h->cfg.kind == RSSM_MAMBA2 ? mamba2_launch(*h, OP_DECODE, 1, in, y, nullptr, h->stream, &ho)
                                       : gdn_launch(*h, OP_DECODE, 1, in, y, nullptr, h->stream, &ho);
    return e == cudaSuccess ? RSSM_OK : api_cuda_fail(h, e, "decode_static_scratch launch");
}
