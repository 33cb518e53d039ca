/*
 * rssm.h -- C ABI of librssm: replay-based SSM-layer decode state on one B200.
 *
 * The operation (ReplaySSM, "cache SSM inputs, not state"): a layer's recurrent
 * state is kept as a checkpoint plus a buffer of the most recent inputs; each
 * token's output is computed from the checkpoint and the buffer without
 * writing state, and the checkpoint is rewritten only when the buffer is full
 * (blog.thibaultmonteiro.fr, "Tenir le journal plutot que le solde";
 * irisproject.cloud, "L'astuce du checkpoint et du tampon"; aikraft.ru,
 * "Reshenie ReplaySSM": the checkpoint is stored once per window).  A
 * low-precision copy of the checkpoint serves the reads while the fp32
 * checkpoint takes the recurrent updates, so the copy's rounding never feeds
 * back (irisproject.cloud, "Deux precisions pour le prix d'une").  Speculative
 * drafts are appended to the buffer and rejection only moves the buffer
 * pointer (irisproject.cloud, "Un retour en arriere qui devient trivial").
 * The same calls also drive an eager read-modify-write baseline, the
 * per-token state rewrite the reports start from (blog.thibaultmonteiro.fr,
 * "La fiche qu'on reecrit a chaque token").
 *
 * Layer recurrences, per sequence b and head h (S is headdim x dstate for
 * Mamba-2, d_v x d_k for Gated DeltaNet and KDA; rows contiguous along dstate / d_k):
 *   Mamba-2:  S_t = exp(dt_t A_h) S_{t-1} + (s_t x_t) B_t^T,  y_t = S_t C_t + D_h x_t,
 *             s_t = dt_t when cfg.dt_scales_input else 1; B, C shared by the
 *             nheads/ngroups heads of a group.
 *   GDN:      S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t.
 *   KDA:      S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t.
 *
 * Conventions shared by every call:
 *   - The library allocates no device memory.  The caller owns the workspace
 *     (rssm_workspace_bytes) and every input/output buffer; none is retained
 *     after a call returns except the workspace, which belongs to the handle.
 *   - Every call enqueues its kernels on the handle's CUDA stream and returns
 *     without synchronising, except rssm_read_counters and rssm_status_word,
 *     which synchronise that stream.
 *   - Pointers named "device" must be device (or managed) memory; "host"
 *     pointers are ordinary host memory.  All device arrays are dense,
 *     row-major, and 16-byte aligned.
 *   - Misuse the host can see (bad sizes, null pointers, a decode while a
 *     verify is pending, ...) returns an error code synchronously and enqueues
 *     nothing.  Inconsistencies only the device can see (an accept length out
 *     of range, a corrupted counter) set the workspace's error word, which
 *     rssm_status_word reports; kernels never trap.
 *   - On any non-OK return, rssm_last_error(h) describes the failure.
 */
#ifndef RSSM_H
#define RSSM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RSSM_API __attribute__((visibility("default")))
#else
#define RSSM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RSSM_OK = 0,
    RSSM_EINVAL = 1,  /* invalid argument or configuration */
    RSSM_ESTATE = 2,  /* call not allowed in the handle's current state */
    RSSM_ECUDA = 3,   /* a CUDA runtime call failed (launch, copy, sync) */
    RSSM_EDEVICE = 4  /* the device error word is set (rssm_status_word) */
} rssm_status;

/* MAMBA2: S_t = exp(dt_t A_h) S_{t-1} + x_t B_t^T, y_t = S_t C_t + D_h x_t.
 * GDN (Gated DeltaNet): S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t.
 * KDA (Kimi Delta Attention): GDN with a gate per key channel,
 *      S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t
 * (the three layer kinds of the hybrid models on blog.thibaultmonteiro.fr, "Des couches
 * rapides sur le papier"; the page names KDA without a formula, and the one above is the
 * plainest reading: the GDN update with the scalar gate made a diagonal). */
typedef enum { RSSM_MAMBA2 = 0, RSSM_GDN = 1, RSSM_KDA = 2 } rssm_kind;

/* REPLAY: checkpoint + read copy + input buffer.  EAGER: one state, read and
 * rewritten every token (the baseline); with state_dtype BF16 or FP8E4M3 this is
 * the single shared low-precision state the dual-precision scheme is compared to. */
typedef enum { RSSM_REPLAY = 0, RSSM_EAGER = 1 } rssm_mode;

typedef enum { RSSM_F32 = 0, RSSM_BF16 = 1, RSSM_FP8E4M3 = 2 } rssm_dtype;

/* Device error codes written to the first word of the error block. */
typedef enum {
    RSSM_DEV_OK = 0,
    RSSM_DEV_BAD_ACCEPT = 1,  /* accept_len[b] < 0 or > pending[b]; treated as 0 */
    RSSM_DEV_BAD_COUNTERS = 2, /* seq_pos - ckpt_pos outside [0, window], or a fold due that the
                                  host did not schedule (counters changed outside the API);
                                  sequence skipped */
    RSSM_DEV_PIPE_TIMEOUT = 3  /* a bulk copy into shared memory did not complete within 2 s;
                                  the kernel stopped and the sequence was left as it was */
} rssm_device_error;

typedef struct {
    int32_t kind;        /* rssm_kind */
    int32_t mode;        /* rssm_mode */
    int32_t state_dtype; /* REPLAY: read-copy dtype (F32 = no copy, outputs read the fp32
                            checkpoint).  EAGER: dtype the single state is stored in.
                            FP8E4M3 uses one fp32 scale per state row (amax / 448). */
    int32_t input_dtype; /* F32 | BF16: dtype of x, B, C (Mamba-2) or q, k, v (GDN, KDA);
                            the buffer stores them as given.  dt, alpha, beta are fp32. */
    int32_t batch;       /* sequences B >= 1 */
    int32_t nheads;      /* heads H >= 1 */
    int32_t headdim;     /* P: Mamba-2 headdim, GDN/KDA d_v; a multiple of 8 in 8..256 */
    int32_t dstate;      /* N: Mamba-2 dstate, GDN/KDA d_k; one of 16, 32, 64, 128 */
    int32_t ngroups;     /* Mamba-2: G >= 1 dividing H (B/C per group).  GDN, KDA: ignored */
    int32_t window;      /* W: buffer window, 1..64 */
    int32_t max_draft;   /* largest K accepted by rssm_verify, 0..8 and <= W */
    int32_t dt_scales_input; /* Mamba-2 only: 1 = input term dt_t x_t B_t^T, 0 = x_t B_t^T */
} rssm_config;

/* Byte offsets (from the workspace base) and sizes of every workspace region;
 * a size of 0 means the region is absent in this configuration. */
typedef struct {
    size_t error_off;                    /* int32[8]: code, b, h, value; [4] is kernel-internal */
    size_t seq_pos_off, ckpt_pos_off;    /* int64[B] each                          */
    size_t pending_off, flush_count_off; /* int32[B] each                          */
    size_t arrive_off;                   /* int32[B] (kernel-internal, kept at 0)  */
    size_t A_off, D_off;                 /* fp32[H] each (Mamba-2)                 */
    size_t ckpt_off, ckpt_bytes;         /* fp32[B][H][P][N]: checkpoint (REPLAY) or the
                                            state (EAGER, F32)                     */
    size_t rc_off, rc_bytes;             /* state_dtype[B][H][P][N]: read copy (REPLAY) or
                                            the state (EAGER, BF16/FP8)            */
    size_t rc_scale_off, rc_scale_bytes; /* fp32[B][H][P] (FP8 only)               */
    size_t ring;                         /* R = window + max(max_draft, 1) slots   */
    size_t ring_stride;                  /* R rounded up to a multiple of 4: row length of the
                                            fp32 scalar rings below (16-byte rows) */
    size_t xbuf_off, xbuf_bytes;         /* Mamba-2 x[B][H][R][P]; GDN/KDA v[B][H][R][P] (input_dtype) */
    size_t bbuf_off, bbuf_bytes;         /* Mamba-2 B[B][G][R][N]; GDN/KDA k[B][H][R][N] (input_dtype) */
    size_t sbuf_off, sbuf_bytes;         /* Mamba-2 dt[B][H][ring_stride]; GDN alpha[B][H][ring_stride];
                                            KDA alpha[B][H][R][N] (fp32)                              */
    size_t tbuf_off, tbuf_bytes;         /* GDN/KDA beta[B][H][ring_stride] (fp32)                 */
    size_t snap_off, snap_bytes;         /* EAGER: max_draft snapshots of the state (+ scales)      */
    /* REPLAY: hand-off from the prep kernel to the flush and read kernels within one call */
    size_t tq_max;                       /* max(max_draft, 1): queries per call            */
    size_t seqinfo_off, seqinfo_bytes;   /* int32[B][4] per sequence, then the flush kernel's
                                            work list: int32 count, 3 pad, int32[B] (padded) */
    size_t dec_off, dec_bytes;           /* fp32[B][H][tq_max]                             */
    size_t coef_off, coef_bytes;         /* fp32[B][H][tq_max][window + tq_max, padded to 4] */
    size_t query_off, query_bytes;       /* GDN/KDA: fp32[B][H][tq_max][dstate] swept queries */
    size_t total_bytes;
} rssm_workspace_layout;

/* Per-token inputs.  T = 1 for rssm_decode, T = K for rssm_verify.  All device. */
typedef struct {
    const void *x;      /* Mamba-2 [B][T][H][P] input_dtype */
    const float *dt;    /* Mamba-2 [B][T][H] fp32 (already softplus-ed, > 0 expected) */
    const void *Bm;     /* Mamba-2 [B][T][G][N] input_dtype */
    const void *Cm;     /* Mamba-2 [B][T][G][N] input_dtype */
    const void *q;      /* GDN/KDA [B][T][H][N] input_dtype */
    const void *k;      /* GDN/KDA [B][T][H][N] input_dtype */
    const void *v;      /* GDN/KDA [B][T][H][P] input_dtype */
    const float *alpha; /* GDN [B][T][H] fp32; KDA [B][T][H][N] fp32, 16-byte aligned */
    const float *beta;  /* GDN/KDA [B][T][H] fp32 */
} rssm_inputs;

typedef struct rssm_ctx *rssm_handle;

/* Workspace size in bytes for cfg (0 if cfg is invalid).  Host only, no CUDA call. */
RSSM_API size_t rssm_workspace_bytes(const rssm_config *cfg);

/* Fill *out with the workspace regions for cfg.  Host only, no CUDA call. */
RSSM_API rssm_status rssm_workspace_layout_of(const rssm_config *cfg, rssm_workspace_layout *out);

/* Create a handle over a caller-owned device workspace of at least
 * rssm_workspace_bytes(cfg) bytes, 256-byte aligned.  `stream` is a cudaStream_t
 * (NULL = legacy default stream).  Enqueues zeroing of the counters, error word and
 * buffers; the state is zero until rssm_import_state.  The handle (host memory) is
 * freed by rssm_destroy; the workspace stays the caller's.  RSSM_EINVAL (nothing
 * enqueued) for an invalid cfg, a NULL, misaligned or too small workspace, or a
 * shape whose kernels need more shared memory per CTA than the current device
 * allows (large headdim x window x max_draft with fp32 inputs); the reason is in
 * rssm_last_error(NULL). */
RSSM_API rssm_status rssm_create(const rssm_config *cfg, void *workspace, size_t workspace_bytes,
                        void *stream, rssm_handle *out);
RSSM_API rssm_status rssm_destroy(rssm_handle h);
RSSM_API rssm_status rssm_set_stream(rssm_handle h, void *stream);

/* Mamba-2 per-head parameters: A[H] (negative), D[H]; device fp32, copied. */
RSSM_API rssm_status rssm_set_params(rssm_handle h, const float *A, const float *D);

/* Install state S (device fp32 [B][H][P][N]) as the committed state: the
 * checkpoint becomes S and its read copy is requantised from it (the fp32
 * checkpoint is the reference the low-precision copy is derived from;
 * irisproject.cloud, "Deux precisions pour le prix d'une"), the buffer empties,
 * counters reset.  Not allowed while a verify is pending (RSSM_ESTATE). */
RSSM_API rssm_status rssm_import_state(rssm_handle h, const float *S);

/* Write the committed state (checkpoint with the committed buffered entries
 * folded in -- the journal replayed onto the balance, blog.thibaultmonteiro.fr,
 * "Tenir le journal plutot que le solde"; for EAGER the dequantised state) to
 * S_out (device fp32 [B][H][P][N]).  Does not change the handle.  Allowed
 * while a verify is pending: pending drafts are not part of the committed state. */
RSSM_API rssm_status rssm_export_state(rssm_handle h, float *S_out);

/* One decode token for every sequence: folds a full buffer into the checkpoint
 * first where needed (len + 1 > W), appends the token, writes y (device fp32
 * [B][1][H][P]) from the read copy and the buffered inputs without writing
 * state, and commits the token (blog.thibaultmonteiro.fr, "Tenir le journal
 * plutot que le solde"; aikraft.ru, "Reshenie ReplaySSM").  RSSM_ESTATE while a
 * verify is pending. */
RSSM_API rssm_status rssm_decode(rssm_handle h, const rssm_inputs *in, float *y);

/* rssm_decode with the call's scratch in one library-owned static device array
 * of 8 MiB instead of the handle's workspace, for callers that cannot allocate
 * device memory on the decode path (a memory pool fixed before the model loads,
 * a captured step where an allocation would stall or is not allowed) and that
 * decode their layers one after another on one stream.  The scratch is the prep
 * kernel's per-call hand-off to the flush and read kernels.  The pages on
 * checkpointed input replay have no counterpart; the results equal
 * rssm_decode's.  Allocates nothing.  REPLAY layers only (EAGER: RSSM_EINVAL).
 * Refused (RSSM_EINVAL, nothing enqueued) when the hand-off -- batch * 20 + 16 +
 * batch * nheads * 4 * (1 + round_up4(window + 1)) bytes, plus
 * batch * nheads * dstate * 4 for GDN/KDA, each region padded to 256 bytes --
 * exceeds the array.  All calls on a device share the array and leave their
 * contents in it, so calls that may run concurrently (several streams or
 * threads) race.  The first call on a device looks up the array's address and
 * keeps it for the life of the process: make that call before any stream
 * capture, and do not use this entry point on a device again after
 * cudaDeviceReset. */
RSSM_API rssm_status rssm_decode_static_scratch(rssm_handle h, const rssm_inputs *in, float *y);

/* Prompt prefill of a Mamba-2 layer, the step before replay decode: for every
 * sequence b and head h, run the prompt's T tokens through the recurrence from
 * the state S0 and write every token's output and the fp32 state after the
 * prompt -- the checkpoint a decode starts from, to be installed with
 * rssm_import_state.  The prompt is processed in chunks of 128 tokens: within a
 * chunk the outputs come from the chunk's own inputs through the decayed pairwise
 * products C_t . B_s plus the state at the chunk's start, and the state moves to
 * the next chunk by one decay and a rank-128 update (the checkpoint + buffered
 * inputs algebra of the replay read, the chunk being the buffer;
 * blog.thibaultmonteiro.fr, "Tenir le journal plutot que le solde").  The pages
 * describe no prefill; the result is the eager recurrence's
 * (y_t = S_t C_t + D x_t) to fp32 accuracy: the products run on the tensor cores
 * with bf16 operands, the fp32 ones split into two bf16 parts.
 *   cfg:   batch, nheads, ngroups as for rssm_config; headdim P in {32, 64, 96};
 *          dstate must be 128; T >= 1 prompt tokens; dt_scales_input 0 or 1.
 *   A, D:  device fp32 [H].  S0: device fp32 [B][H][P][N], or NULL for a zero state.
 *   in:    x [B][T][H][P] bf16, dt [B][T][H] fp32, Bm, Cm [B][T][G][N] bf16 (device,
 *          16-byte aligned; the other fields are ignored).
 *   y:     device fp32 [B][T][H][P] (16-byte aligned).  S_out: device fp32 [B][H][P][N]
 *          (may not alias S0).
 *   dev_error: device int32[4] or NULL; {RSSM_DEV_PIPE_TIMEOUT, b, h, 0} is written
 *          there if a tensor-core wait gives up (2 s), and that head's S_out is not written.
 *   stream: cudaStream_t (NULL = legacy default stream).
 * Enqueues one kernel and returns; allocates nothing.  RSSM_EINVAL (nothing
 * enqueued) for NULL pointers, unsupported sizes or misaligned arrays. */
typedef struct {
    int32_t batch, nheads, headdim, dstate, ngroups;
    int32_t T;               /* prompt tokens >= 1 */
    int32_t dt_scales_input; /* 1 = input term dt_t x_t B_t^T, 0 = x_t B_t^T */
} rssm_prefill_config;
RSSM_API rssm_status rssm_mamba2_prefill(const rssm_prefill_config *cfg, const float *A, const float *D,
                                         const float *S0, const rssm_inputs *in, float *y, float *S_out,
                                         int32_t *dev_error, void *stream);

/* Speculative verify of K drafts (1 <= K <= max_draft, K <= W) for every
 * sequence: folds where len + K > W, appends the drafts uncommitted and writes
 * y (device fp32 [B][K][H][P]), draft m seeing the committed tokens and drafts
 * 0..m (the drafts go into the input buffer like any token; irisproject.cloud,
 * "Un retour en arriere qui devient trivial").  The checkpoint is not otherwise
 * touched.  Must be followed by rssm_commit before the next decode, verify or
 * flush (RSSM_ESTATE otherwise); RSSM_EINVAL for K out of range. */
RSSM_API rssm_status rssm_verify(rssm_handle h, int32_t K, const rssm_inputs *in, float *y);

/* Accept the first accept_len[b] drafts of the pending verify (device int32
 * [B]); the rest are dropped by not advancing the buffer pointer (REPLAY; a
 * rejection is a pointer that does not move, irisproject.cloud, "Un retour en
 * arriere qui devient trivial") or by not copying their snapshot (EAGER).
 * 0 <= accept_len[b] <= K is required; an out-of-range value is treated as 0
 * and sets RSSM_DEV_BAD_ACCEPT.  RSSM_ESTATE if no verify is pending. */
RSSM_API rssm_status rssm_commit(rssm_handle h, const int32_t *accept_len);

/* Fold every committed buffered entry into the checkpoint and requantise the
 * read copy (REPLAY; EAGER: no-op).  Decode and verify fold on their own when
 * a buffer is full (the checkpoint is rewritten only then,
 * blog.thibaultmonteiro.fr, "Tenir le journal plutot que le solde"); this call
 * forces it, e.g. before a state export.  RSSM_ESTATE while a verify is pending. */
RSSM_API rssm_status rssm_flush(rssm_handle h);

/* Copy the per-sequence counters to host arrays (each may be NULL); synchronises. */
RSSM_API rssm_status rssm_read_counters(rssm_handle h, int64_t *seq_pos, int64_t *ckpt_pos,
                               int32_t *pending, int32_t *flush_count);

/* Synchronise and read the device error word into info[4] (may be NULL):
 * {code, sequence, head, value}.  Returns RSSM_EDEVICE if code != 0. */
RSSM_API rssm_status rssm_status_word(rssm_handle h, int32_t *info);
/* Enqueue clearing of the device error word. */
RSSM_API rssm_status rssm_clear_status(rssm_handle h);

/* Measurement hook: when `event` (a cudaEvent_t) is not NULL, every REPLAY
 * decode/verify records it on the handle's stream between its two kernels (the
 * prep/flush kernel and the replay-read kernel), so a caller can time them
 * apart.  NULL (the default) records nothing. */
RSSM_API rssm_status rssm_set_split_event(rssm_handle h, void *event);

/* Number of kernels this handle has enqueued so far (running total). */
RSSM_API int64_t rssm_launch_count(rssm_handle h);

/* Description of the last failure on h (h == NULL: of the last failed create). */
RSSM_API const char *rssm_last_error(rssm_handle h);

#ifdef __cplusplus
}
#endif
#endif /* RSSM_H */
