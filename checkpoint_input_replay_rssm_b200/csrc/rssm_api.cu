// rssm_api.cu -- the C ABI (include/rssm.h): validation, workspace layout,
// handle life cycle and the host side of every call.  All device work is
// enqueued on the handle's stream; nothing here allocates device memory.
#include <stdio.h>
#include <string.h>

#include <new>

#include "rssm_internal.h"

using rssm::Ctx;

namespace {

thread_local std::string g_create_error;

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

bool validate(const rssm_config *c, std::string *why) {
    char buf[256];
    auto fail = [&](const char *m) { if (why) *why = m; return false; };
    if (!c) return fail("config is NULL");
    if (c->kind != RSSM_MAMBA2 && c->kind != RSSM_GDN && c->kind != RSSM_KDA)
        return fail("kind must be MAMBA2, GDN or KDA");
    if (c->mode != RSSM_REPLAY && c->mode != RSSM_EAGER) return fail("mode must be REPLAY or EAGER");
    if (c->state_dtype < RSSM_F32 || c->state_dtype > RSSM_FP8E4M3) return fail("bad state_dtype");
    if (c->input_dtype != RSSM_F32 && c->input_dtype != RSSM_BF16) return fail("input_dtype must be F32 or BF16");
    if (c->batch < 1 || c->nheads < 1) return fail("batch and nheads must be >= 1");
    if ((int64_t)c->batch * c->nheads > 0x7fffffffLL) return fail("batch * nheads too large");
    if (c->headdim < 8 || c->headdim > 256 || c->headdim % 8 != 0)
        return fail("headdim must be a multiple of 8 in 8..256");
    if (c->dstate != 16 && c->dstate != 32 && c->dstate != 64 && c->dstate != 128)
        return fail("dstate must be 16, 32, 64 or 128");
    if (c->kind == RSSM_MAMBA2 && (c->ngroups < 1 || c->nheads % c->ngroups != 0))
        return fail("ngroups must be >= 1 and divide nheads");
    if (c->window < 1 || c->window > 64) return fail("window must be in 1..64");
    if (c->max_draft < 0 || c->max_draft > 8 || c->max_draft > c->window) {
        snprintf(buf, sizeof buf, "max_draft must be in 0..min(8, window) (got %d)", c->max_draft);
        if (why) *why = buf;
        return false;
    }
    if (c->dt_scales_input != 0 && c->dt_scales_input != 1) return fail("dt_scales_input must be 0 or 1");
    if (c->kind != RSSM_MAMBA2 && c->dt_scales_input) return fail("dt_scales_input is Mamba-2 only");
    return true;
}

void layout(const rssm_config *c, rssm_workspace_layout *L) {
    memset(L, 0, sizeof *L);
    const size_t B = c->batch, H = c->nheads, P = c->headdim, N = c->dstate;
    const size_t G = c->kind == RSSM_MAMBA2 ? (size_t)c->ngroups : H;
    const size_t elems = B * H * P * N;
    const size_t sb = c->state_dtype == RSSM_F32 ? 4 : (c->state_dtype == RSSM_BF16 ? 2 : 1);
    const size_t ib = c->input_dtype == RSSM_BF16 ? 2 : 4;
    const bool fp8 = c->state_dtype == RSSM_FP8E4M3;
    const bool replay = c->mode == RSSM_REPLAY;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
    L->error_off = take(8 * sizeof(int32_t));
    L->seq_pos_off = take(B * 8);
    L->ckpt_pos_off = take(B * 8);
    L->pending_off = take(B * 4);
    L->flush_count_off = take(B * 4);
    L->arrive_off = take(B * 4);
    L->A_off = take(H * 4);
    L->D_off = take(H * 4);
    L->ring = (size_t)c->window + (size_t)(c->max_draft > 1 ? c->max_draft : 1);
    const size_t R = L->ring;
    L->ring_stride = (R + 3) & ~(size_t)3;
    const size_t Rs = L->ring_stride;
    if (replay || c->state_dtype == RSSM_F32) {
        L->ckpt_bytes = elems * 4;
        L->ckpt_off = take(L->ckpt_bytes);
    }
    if (c->state_dtype != RSSM_F32) {
        L->rc_bytes = elems * sb;
        L->rc_off = take(L->rc_bytes);
    }
    if (fp8) {
        L->rc_scale_bytes = B * H * P * 4;
        L->rc_scale_off = take(L->rc_scale_bytes);
    }
    if (replay) {
        L->xbuf_bytes = B * H * R * P * ib;
        L->xbuf_off = take(L->xbuf_bytes);
        L->bbuf_bytes = B * G * R * N * ib;
        L->bbuf_off = take(L->bbuf_bytes);
        L->sbuf_bytes = c->kind == RSSM_KDA ? B * H * R * N * 4 : B * H * Rs * 4;
        L->sbuf_off = take(L->sbuf_bytes);
        if (c->kind != RSSM_MAMBA2) {
            L->tbuf_bytes = B * H * Rs * 4;
            L->tbuf_off = take(L->tbuf_bytes);
        }
        // prep -> read hand-off, rewritten by every decode/verify
        const size_t TQm = (size_t)(c->max_draft > 1 ? c->max_draft : 1);
        L->tq_max = TQm;
        L->seqinfo_bytes = B * 16 + 16 + ((B * 4 + 15) & ~(size_t)15);
        L->seqinfo_off = take(L->seqinfo_bytes);
        L->dec_bytes = B * H * TQm * 4;
        L->dec_off = take(L->dec_bytes);
        L->coef_bytes = B * H * TQm * (((size_t)c->window + TQm + 3) & ~(size_t)3) * 4;
        L->coef_off = take(L->coef_bytes);
        if (c->kind != RSSM_MAMBA2) {
            L->query_bytes = B * H * TQm * N * 4;
            L->query_off = take(L->query_bytes);
        }
    } else if (c->max_draft > 0) {
        L->snap_bytes = (size_t)c->max_draft * (elems * sb + (fp8 ? B * H * P * 4 : 0));
        L->snap_off = take(L->snap_bytes);
    }
    L->total_bytes = off;
}

rssm_status fail(Ctx *h, rssm_status st, const std::string &m) {
    if (h) h->err = m;
    return st;
}

rssm_status cuda_fail(Ctx *h, cudaError_t e, const char *what) {
    std::string m = std::string(what) + ": " + cudaGetErrorString(e);
    return fail(h, RSSM_ECUDA, m);
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }

bool inputs_ok(const Ctx *h, const rssm_inputs *in) {
    if (!in) return false;
    if (h->cfg.kind == RSSM_MAMBA2)
        return in->x && in->dt && in->Bm && in->Cm && aligned16(in->x) && aligned16(in->Bm) &&
               aligned16(in->Cm);
    return in->q && in->k && in->v && in->alpha && in->beta && aligned16(in->q) &&
           aligned16(in->k) && aligned16(in->v) && (h->cfg.kind != RSSM_KDA || aligned16(in->alpha));
}

cudaError_t launch_kind(Ctx *h, int op, int T, const rssm_inputs *in, float *y, float *out) {
    if (h->cfg.kind == RSSM_MAMBA2) return rssm::mamba2_launch(*h, op, T, in, y, out, h->stream);
    return rssm::gdn_launch(*h, op, T, in, y, out, h->stream);
}

}  // namespace

namespace rssm {
rssm_status api_fail(Ctx *h, rssm_status st, const std::string &m) { return fail(h, st, m); }
rssm_status api_cuda_fail(Ctx *h, cudaError_t e, const char *what) { return cuda_fail(h, e, what); }
bool api_inputs_ok(const Ctx *h, const rssm_inputs *in) { return inputs_ok(h, in); }
}  // namespace rssm

extern "C" {

size_t rssm_workspace_bytes(const rssm_config *cfg) {
    if (!validate(cfg, nullptr)) return 0;
    rssm_workspace_layout L;
    layout(cfg, &L);
    return L.total_bytes;
}

rssm_status rssm_workspace_layout_of(const rssm_config *cfg, rssm_workspace_layout *out) {
    std::string why;
    if (!out) return RSSM_EINVAL;
    if (!validate(cfg, &why)) return RSSM_EINVAL;
    layout(cfg, out);
    return RSSM_OK;
}

// Largest dynamic shared memory any kernel of this configuration asks for
// (decode and verify query counts; flush and export use the decode layout).
static size_t smem_need(const rssm_config &c) {
    size_t need = 0;
    const int Ts[2] = {1, c.max_draft > 1 ? c.max_draft : 1};
    for (int T : Ts) {
        const size_t k = c.kind == RSSM_MAMBA2 ? rssm::mamba2_smem_bytes(c, T) : rssm::gdn_smem_bytes(c, T);
        if (k > need) need = k;
        if (c.mode == RSSM_REPLAY) {
            const size_t r = rssm::read_smem_bytes(c, T);
            if (r > need) need = r;
        }
    }
    return need;
}

rssm_status rssm_create(const rssm_config *cfg, void *workspace, size_t workspace_bytes,
                        void *stream, rssm_handle *out) {
    std::string why;
    if (!out) { g_create_error = "out is NULL"; return RSSM_EINVAL; }
    *out = nullptr;
    if (!validate(cfg, &why)) { g_create_error = why; return RSSM_EINVAL; }
    rssm_workspace_layout L;
    layout(cfg, &L);
    if (!workspace) { g_create_error = "workspace is NULL"; return RSSM_EINVAL; }
    if (((uintptr_t)workspace & 255) != 0) { g_create_error = "workspace must be 256-byte aligned"; return RSSM_EINVAL; }
    if (workspace_bytes < L.total_bytes) { g_create_error = "workspace too small"; return RSSM_EINVAL; }
    Ctx *h = new (std::nothrow) Ctx();
    if (!h) { g_create_error = "out of host memory"; return RSSM_EINVAL; }
    h->cfg = *cfg;
    h->lay = L;
    h->ws = (uint8_t *)workspace;
    h->ws_bytes = workspace_bytes;
    h->stream = (cudaStream_t)stream;
    int dev = 0, sms = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess && sms > 0) h->num_sms = sms;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess && optin > 0) {
        const size_t need = smem_need(*cfg);
        if (need > (size_t)optin) {
            g_create_error = "this shape's kernels need " + std::to_string(need) +
                             " bytes of shared memory per CTA; the device allows " + std::to_string(optin);
            delete h;
            return RSSM_EINVAL;
        }
    }
    if (e == cudaSuccess) e = cudaMemsetAsync(h->ws, 0, L.total_bytes, h->stream);
    if (e != cudaSuccess) {
        g_create_error = std::string("zeroing the workspace: ") + cudaGetErrorString(e);
        delete h;
        return RSSM_ECUDA;
    }
    *out = (rssm_handle)h;
    return RSSM_OK;
}

rssm_status rssm_destroy(rssm_handle hh) {
    delete (Ctx *)hh;
    return RSSM_OK;
}

rssm_status rssm_set_stream(rssm_handle hh, void *stream) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    h->stream = (cudaStream_t)stream;
    return RSSM_OK;
}

rssm_status rssm_set_params(rssm_handle hh, const float *A, const float *D) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    if (h->cfg.kind != RSSM_MAMBA2) return fail(h, RSSM_EINVAL, "set_params is for Mamba-2 layers");
    if (!A || !D) return fail(h, RSSM_EINVAL, "A and D must be device pointers");
    const size_t bytes = (size_t)h->cfg.nheads * sizeof(float);
    cudaError_t e = cudaMemcpyAsync(h->at(h->lay.A_off), A, bytes, cudaMemcpyDeviceToDevice, h->stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(h->at(h->lay.D_off), D, bytes, cudaMemcpyDeviceToDevice, h->stream);
    return e == cudaSuccess ? RSSM_OK : cuda_fail(h, e, "set_params");
}

rssm_status rssm_import_state(rssm_handle hh, const float *S) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    if (!S) return fail(h, RSSM_EINVAL, "S is NULL");
    if (h->pending) return fail(h, RSSM_ESTATE, "import while a verify is pending");
    cudaError_t e = rssm::launch_import(*h, S, h->stream);
    if (h->lay.rc_bytes) h->launches += 1;
    if (e == cudaSuccess)
        e = cudaMemsetAsync(h->at(h->lay.seq_pos_off), 0, h->lay.A_off - h->lay.seq_pos_off, h->stream);
    h->len_lb = h->len_ub = 0;
    return e == cudaSuccess ? RSSM_OK : cuda_fail(h, e, "import_state");
}

rssm_status rssm_export_state(rssm_handle hh, float *S_out) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    if (!S_out) return fail(h, RSSM_EINVAL, "S_out is NULL");
    cudaError_t e;
    if (h->cfg.mode == RSSM_REPLAY) {
        // Fold the committed buffered entries on the way out; sequences with an
        // empty buffer are copied from the checkpoint first.
        const size_t bytes = h->lay.ckpt_bytes;
        e = cudaMemcpyAsync(S_out, h->at(h->lay.ckpt_off), bytes, cudaMemcpyDeviceToDevice, h->stream);
        if (e == cudaSuccess) e = launch_kind(h, rssm::OP_EXPORT, 0, nullptr, nullptr, S_out);
    } else {
        h->launches += 1;
        e = rssm::launch_export_eager(*h, S_out, h->stream);
    }
    return e == cudaSuccess ? RSSM_OK : cuda_fail(h, e, "export_state");
}

rssm_status rssm_decode(rssm_handle hh, const rssm_inputs *in, float *y) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    if (h->pending) return fail(h, RSSM_ESTATE, "decode while a verify is pending (commit first)");
    if (!inputs_ok(h, in) || !y) return fail(h, RSSM_EINVAL, "missing or misaligned input/output pointer (device arrays must be 16-byte aligned)");
    cudaError_t e = launch_kind(h, rssm::OP_DECODE, 1, in, y, nullptr);
    return e == cudaSuccess ? RSSM_OK : cuda_fail(h, e, "decode launch");
}

rssm_status rssm_verify(rssm_handle hh, int32_t K, const rssm_inputs *in, float *y) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    if (h->pending) return fail(h, RSSM_ESTATE, "verify while a verify is pending (commit first)");
    if (K < 1 || K > h->cfg.max_draft || K > h->cfg.window)
        return fail(h, RSSM_EINVAL, "K must be in 1..min(max_draft, window)");
    if (!inputs_ok(h, in) || !y) return fail(h, RSSM_EINVAL, "missing or misaligned input/output pointer (device arrays must be 16-byte aligned)");
    cudaError_t e = launch_kind(h, rssm::OP_VERIFY, K, in, y, nullptr);
    if (e != cudaSuccess) return cuda_fail(h, e, "verify launch");
    h->pending = K;
    return RSSM_OK;
}

rssm_status rssm_commit(rssm_handle hh, const int32_t *accept_len) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    if (!h->pending) return fail(h, RSSM_ESTATE, "commit with nothing pending");
    if (!accept_len) return fail(h, RSSM_EINVAL, "accept_len is NULL");
    h->launches += 1;
    cudaError_t e = rssm::launch_commit(*h, accept_len, h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "commit launch");
    h->pending = 0;
    return RSSM_OK;
}

rssm_status rssm_flush(rssm_handle hh) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    if (h->pending) return fail(h, RSSM_ESTATE, "flush while a verify is pending (commit first)");
    if (h->cfg.mode != RSSM_REPLAY) return RSSM_OK;
    cudaError_t e = launch_kind(h, rssm::OP_FLUSH, 0, nullptr, nullptr, nullptr);
    return e == cudaSuccess ? RSSM_OK : cuda_fail(h, e, "flush launch");
}

rssm_status rssm_read_counters(rssm_handle hh, int64_t *seq_pos, int64_t *ckpt_pos,
                               int32_t *pending, int32_t *flush_count) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    const size_t B = h->cfg.batch;
    cudaError_t e = cudaSuccess;
    if (seq_pos && e == cudaSuccess)
        e = cudaMemcpyAsync(seq_pos, h->at(h->lay.seq_pos_off), B * 8, cudaMemcpyDeviceToHost, h->stream);
    if (ckpt_pos && e == cudaSuccess)
        e = cudaMemcpyAsync(ckpt_pos, h->at(h->lay.ckpt_pos_off), B * 8, cudaMemcpyDeviceToHost, h->stream);
    if (pending && e == cudaSuccess)
        e = cudaMemcpyAsync(pending, h->at(h->lay.pending_off), B * 4, cudaMemcpyDeviceToHost, h->stream);
    if (flush_count && e == cudaSuccess)
        e = cudaMemcpyAsync(flush_count, h->at(h->lay.flush_count_off), B * 4, cudaMemcpyDeviceToHost, h->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(h->stream);
    return e == cudaSuccess ? RSSM_OK : cuda_fail(h, e, "read_counters");
}

rssm_status rssm_status_word(rssm_handle hh, int32_t *info) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    int32_t w[4] = {0, 0, 0, 0};
    cudaError_t e = cudaMemcpyAsync(w, h->at(h->lay.error_off), sizeof w, cudaMemcpyDeviceToHost, h->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "status_word");
    if (info) memcpy(info, w, sizeof w);
    if (w[0] != 0) {
        char buf[128];
        snprintf(buf, sizeof buf, "device error %d (sequence %d, head %d, value %d)", w[0], w[1], w[2], w[3]);
        return fail(h, RSSM_EDEVICE, buf);
    }
    return RSSM_OK;
}

rssm_status rssm_clear_status(rssm_handle hh) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    cudaError_t e = cudaMemsetAsync(h->at(h->lay.error_off), 0, 8 * sizeof(int32_t), h->stream);
    return e == cudaSuccess ? RSSM_OK : cuda_fail(h, e, "clear_status");
}

rssm_status rssm_set_split_event(rssm_handle hh, void *event) {
    Ctx *h = (Ctx *)hh;
    if (!h) return RSSM_EINVAL;
    h->split_event = (cudaEvent_t)event;
    return RSSM_OK;
}

int64_t rssm_launch_count(rssm_handle hh) {
    Ctx *h = (Ctx *)hh;
    return h ? h->launches : -1;
}

const char *rssm_last_error(rssm_handle hh) {
    Ctx *h = (Ctx *)hh;
    return h ? h->err.c_str() : g_create_error.c_str();
}

}  // extern "C"
