// rssm_static_scratch.cu -- rssm_decode_static_scratch: the replay decode with
// its per-call hand-off (prep kernel -> flush and read kernels) kept in one
// file-scope device array instead of the handle's workspace.
//
// Who needs it: a caller that budgets device memory per layer for the layer's
// state alone and runs the layers' decodes one after another on one stream.
// Each handle's workspace carries its own hand-off region (for a 256-sequence,
// 128-head, window-16 layer about 2.7 MB), rewritten by every call and dead
// between calls; such a caller wants the hand-off of every layer in one shared
// array that the library owns and that needs no allocation, at run time or at
// set-up: the array is part of the loaded module.
//
// The method itself (the pages on checkpointed input replay) has no such entry
// point; it computes exactly what rssm_decode computes, with the same kernels.
//
// Limits and sharing:
//   - the hand-off of one decode call must fit kStaticScratchBytes; larger
//     layers are refused with RSSM_EINVAL before anything is enqueued;
//   - all calls on a device share the array: calls whose kernels can overlap
//     (several streams, several host threads) race on it and must not be
//     issued concurrently;
//   - the first call on a device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current; a caller that records
//     its calls into a stream capture makes one call before capturing.
#include <mutex>
#include <string>

#include "rssm_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_handoff_scratch[kStaticScratchBytes];

std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

// Offsets of the decode hand-off (one query per call) inside the array.
struct Carve {
    size_t seqinfo, fold, dec, coef, total;
};
Carve carve(const rssm_config &c) {
    const size_t B = c.batch, H = c.nheads;
    const size_t Emax = ((size_t)c.window + 1 + 3) & ~(size_t)3;
    Carve k{};
    size_t o = 0;
    k.seqinfo = o; o = up256(o + B * 16);
    k.fold = o;    o = up256(o + 16 + B * 4);  // count, 3 pad words, list[B]
    k.dec = o;     o = up256(o + B * H * 4);
    k.coef = o;    o = up256(o + B * H * Emax * 4);
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
    if (h->cfg.mode != RSSM_REPLAY || h->cfg.kind != RSSM_MAMBA2)
        return api_fail(h, RSSM_EINVAL, "decode_static_scratch: only REPLAY Mamba-2 layers have a hand-off");
    if (h->pending) return api_fail(h, RSSM_ESTATE, "decode while a verify is pending (commit first)");
    if (!api_inputs_ok(h, in) || !y)
        return api_fail(h, RSSM_EINVAL,
                        "missing or misaligned input/output pointer (device arrays must be 16-byte aligned)");
    const Carve k = carve(h->cfg);
    if (k.total > kStaticScratchBytes)
        return api_fail(h, RSSM_EINVAL,
                        "decode_static_scratch: the hand-off needs " + std::to_string(k.total) +
                            " bytes; the static array holds " + std::to_string(kStaticScratchBytes) +
                            " (batch * nheads * (window + 4) * 4 bytes must stay below it)");
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
    ho.tq_max = 1;
    // The work-list length must start at zero; the read kernel leaves it zero,
    // but a call refused or failed half-way on another handle may not have.
    e = cudaMemsetAsync(ho.fold_count, 0, sizeof(int), h->stream);
    if (e == cudaSuccess) e = mamba2_launch(*h, OP_DECODE, 1, in, y, nullptr, h->stream, &ho);
    return e == cudaSuccess ? RSSM_OK : api_cuda_fail(h, e, "decode_static_scratch launch");
}
