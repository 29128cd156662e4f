/*
 * dlm.h -- C ABI of the B200 (sm_100a) diffusion-LM noising-plus-loss library.
 *
 * One training step of a native diffusion language model, between the clean
 * token ids of a batch and the gradient of the loss with respect to the
 * model's logits (or its hidden states and output head):
 *
 *   dlm_sample_t             per-sequence (or per-document) time t and mask
 *                            probability p
 *   dlm_corrupt              seeded corruption of the clean ids
 *   dlm_loss_fwd_bwd         inverse-time weighted CE over the vocabulary at
 *                            the corrupted positions, forward + backward, from
 *                            materialised bf16 logits (dlm_loss_fwd_bwd_ex:
 *                            with the uniform-noise objective options)
 *   dlm_linear_loss_fwd_bwd  the same loss from hidden states and a linear
 *                            output head, logits never materialised
 *                            (dlm_linear_loss_fwd_bwd_ex: aligned or shifted
 *                            targets; dlm_linear_loss_uniform_fwd_bwd: the
 *                            uniform-noise loss with its encoder term)
 *   dlm_decision_loss_fwd_bwd  typed-decision losses at label slots
 *                            (candidate-restricted CE, full-vocabulary CE,
 *                            Brier), forward + backward
 *
 * The method (page title, section):
 *   "LLaDA-8B-MDLM-LoRA", Training table, row "Objective": t ~ U(0,1) per
 *       sequence, mask probability p = (1 - 1e-3) t + 1e-3, cross-entropy on
 *       masked tokens divided by p.
 *   "Native diffusion language-model training", model table: absorbing mask
 *       with aligned logits (Nemotron) or shifted logits (Dream); uniform token
 *       noise with a causal encoder (DiffusionGemma).  "Packed training":
 *       documents stay isolated; positions restart at document boundaries.
 *       "Adapters, merging and inference": Cut Cross Entropy computes the
 *       full-vocabulary CE from hidden states without materialising logits,
 *       aligned targets, plain linear head.
 *   "diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning notes: total =
 *       diffusion CE + encoder_loss_weight * encoder AR CE; canvas positions
 *       replaced by uniform-random vocabulary ids at rate t ~ U(eps, 1).
 *
 * Conventions for every call
 *   - All array arguments are DEVICE pointers owned by the caller, except the
 *     dlm_layout_t structs themselves (host memory, read during the call).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronise, except dlm_get_device_status.
 *   - The library allocates no device memory.  Scratch comes from a caller
 *     workspace of at least dlm_*_workspace_size() bytes, 256-byte aligned
 *     (1024-byte aligned for the dlm_linear_* calls).  A *_workspace_size()
 *     call returns 0 for arguments its loss call would refuse.
 *     A workspace may be reused by calls ordered on one stream; calls that
 *     overlap on the GPU need separate workspaces.
 *   - Host-checkable errors return before anything is enqueued.  Errors that
 *     depend on device data (an id outside [0, vocab), a non-monotone
 *     cu_seqlens, a bounded wait that ran out) set bits in a device status
 *     word; the affected rows are treated as unscored and the call still
 *     completes.  Read the word with dlm_get_device_status.
 *   - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *   - Requires compute capability 10.0 (B200); other devices get
 *     DLM_ERR_UNSUPPORTED.
 */
#ifndef DLM_H_
#define DLM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of this ABI are the only ones the shared library exports. */
#if defined(__GNUC__)
#define DLM_API __attribute__((visibility("default")))
#else
#define DLM_API
#endif

typedef enum dlm_status {
    DLM_OK = 0,
    DLM_ERR_INVALID_ARGUMENT = 1,
    DLM_ERR_UNSUPPORTED = 2,
    DLM_ERR_WORKSPACE_TOO_SMALL = 3,
    DLM_ERR_CUDA = 4
} dlm_status_t;

/* noise process */
enum { DLM_ABSORBING = 0, DLM_UNIFORM = 1 };
/* logit alignment: row i scores token i, or token i+1 of the same unit */
enum { DLM_ALIGNED = 0, DLM_SHIFTED = 1 };

/* bits of the device status word */
#define DLM_DEV_BAD_TOKEN_ID   0x1u  /* a scored target id outside [0, vocab)      */
#define DLM_DEV_BAD_LAYOUT     0x2u  /* cu_seqlens not 0..n_tokens non-decreasing  */
#define DLM_DEV_WAIT_TIMEOUT   0x4u  /* a bounded on-chip wait gave up             */
#define DLM_DEV_BAD_LABEL      0x8u  /* a malformed typed-decision label           */

/* Opaque CUDA stream (ABI-compatible with cudaStream_t / CUstream). */
typedef struct CUstream_st *dlm_stream_t;

/* How tokens are grouped into units (the thing t is drawn for).
 *   Dense:  cu_seqlens == NULL; n_units sequences of seq_len tokens each,
 *           token i of the flattened [n_units, seq_len] array is position
 *           i % seq_len of unit i / seq_len.  n_tokens = n_units * seq_len.
 *   Packed: cu_seqlens = [n_units + 1] int32 document offsets (device),
 *           cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_units] = n_tokens;
 *           seq_len is ignored.  Positions restart at each document start.
 *   pad_mask: [n_tokens] uint8 (device), 1 = padding, or NULL.  Pads are
 *           never corrupted, never scored, and not counted in N.
 * Limits: n_units < 2^24, positions < 2^31, n_tokens < 2^31. */
typedef struct dlm_layout {
    int32_t n_units;
    int32_t seq_len;
    int64_t n_tokens;
    const int32_t *cu_seqlens;
    const uint8_t *pad_mask;
} dlm_layout_t;

/* Human-readable name of a status code (static string, never NULL). */
DLM_API const char *dlm_status_string(dlm_status_t status);

/* Text of the last CUDA error this library saw on the calling host thread
 * (a DLM_ERR_CUDA return), or "" if none.  Static/thread-local storage owned
 * by the library; valid until the next failing call on the same thread. */
DLM_API const char *dlm_last_cuda_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
DLM_API int dlm_version(void);

/* ------------------------------------------------------------------------
 * dlm_sample_t -- time and mask probability per unit.
 *   "LLaDA-8B-MDLM-LoRA", Training table, row "Objective" (absorbing):
 *       t = u,                 p = (1 - eps) t + eps
 *   "diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning notes (uniform):
 *       t = (1 - eps) u + eps, p = t
 * u = k / 2^24 where k = top 24 bits of SplitMix64 output number
 * (counter + 1) from state `seed`, counter = unit << 32 (stream 0);
 * fp32 arithmetic with one rounding per operation (c1 = 1 - eps first).
 * t, p: [n_units] float (device, written).  mode: DLM_ABSORBING|DLM_UNIFORM.
 * eps in [0, 1).  n_units = 0 is a no-op.
 * ---------------------------------------------------------------------- */
DLM_API dlm_status_t dlm_sample_t(uint64_t seed, int32_t n_units, int32_t mode, float eps,
                          float *t, float *p, dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_corrupt -- seeded corruption of clean ids ("LLaDA-8B-MDLM-LoRA",
 * Training table, row "Objective"; "diffusiongemma-26B-A4B-it-ALWAYS-THINK",
 * Finetuning notes; "Native diffusion language-model training", Packed
 * training).  Per non-pad token at position `pos` of unit `u`:
 *   corrupted = (float)(h1 >> 40) < p[u] * 2^24       (strict, exact fp32)
 *   h1 = SplitMix64(seed, counter = 1 << 56 | u << 32 | pos)
 *   absorbing: noisy = mask_id
 *   uniform:   noisy = ((h2 >> 32) * vocab) >> 32,  h2 with stream 2 in place
 *              of 1 -- a uniform id in [0, vocab), may equal the clean id.
 * Pads keep their id and are never corrupted.  Uncorrupted tokens keep their
 * clean id.  For uniform noise pass the canvas tokens only.
 *   clean_ids [n_tokens] int32, p [n_units] float (from dlm_sample_t),
 *   noisy_ids [n_tokens] int32 (written), corrupted [n_tokens] uint8 (written,
 *   0/1), dev_status: a device uint32 that gets DLM_DEV_BAD_LAYOUT or'ed in
 *   if cu_seqlens is inconsistent (may be NULL).
 * mask_id is only read for absorbing noise; vocab only for uniform noise.
 * ---------------------------------------------------------------------- */
DLM_API dlm_status_t dlm_corrupt(const dlm_layout_t *layout, const int32_t *clean_ids,
                         const float *p, int32_t mode, int32_t mask_id, int32_t vocab,
                         uint64_t seed, int32_t *noisy_ids, uint8_t *corrupted,
                         uint32_t *dev_status, dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_loss_fwd_bwd -- weighted CE over the vocabulary, forward + backward,
 * from materialised bf16 logits.
 *
 * Rows and targets (diffusion term, one logits row per token of `layout`):
 *   row i scores token j = i (DLM_ALIGNED) or j = i + 1 of the same unit
 *   (DLM_SHIFTED; a unit's last row is unscored); j must be non-pad.
 *   absorbing: only corrupted j are scored, weight w = 1 / (p[unit] * N),
 *              N = number of non-pad tokens of `layout`.
 *   uniform:   every such j is scored, w = 1 / (number of scored rows).
 * Encoder AR term (uniform only, enc_logits != NULL): one row per token of
 *   `enc_layout`; row i scores enc_ids[i+1] of the same unit (non-pad),
 *   w = enc_ar_weight / (number of such rows).  enc_layout.n_units must equal
 *   layout.n_units (unit u of the canvas is unit u of the encoder sequence).
 * Per scored row r with target y:  ce_r = logsumexp(x_r) - x_r[y] over the
 *   full vocabulary (mask-id column included).
 * Outputs:
 *   loss[0]          = sum_r w_r ce_r                               (float)
 *   unit_loss[u]     = the same sum over unit u's rows (may be NULL)
 *   dlogits[r, v]    = grad_scale * w_r * (softmax(x_r)_v - [v == y_r]) on
 *                      scored rows, exactly 0 on every other row; bf16, same
 *                      layout as logits; every element of [rows, vocab] is
 *                      written (columns vocab..ld-1 are not touched).
 *   enc_dlogits      = the same for the encoder rows.
 * logits: [layout.n_tokens rows, ld] bf16, row stride ld >= vocab elements.
 * enc_logits: [enc_layout.n_tokens, enc_ld] bf16.  clean_ids / enc_ids:
 * int32 clean ids.  corrupted: from dlm_corrupt (absorbing; ignored for
 * uniform).  p: [n_units] from dlm_sample_t (absorbing; ignored for uniform).
 * Reductions run in a fixed order: results are bitwise reproducible.
 * Fast path when vocab, ld, enc_ld are multiples of 8 and the logits /
 * dlogits pointers are 16-byte aligned; any other shape takes a slower
 * general kernel with the same results.
 * ---------------------------------------------------------------------- */
DLM_API size_t dlm_loss_workspace_size(const dlm_layout_t *layout, const dlm_layout_t *enc_layout);

DLM_API dlm_status_t dlm_loss_fwd_bwd(const dlm_layout_t *layout, const uint16_t *logits, int64_t ld,
                              int32_t vocab, const int32_t *clean_ids, const uint8_t *corrupted,
                              const float *p, int32_t mode, int32_t align,
                              const dlm_layout_t *enc_layout, const uint16_t *enc_logits,
                              int64_t enc_ld, const int32_t *enc_ids, float enc_ar_weight,
                              float grad_scale, float *loss, float *unit_loss,
                              uint16_t *dlogits, uint16_t *enc_dlogits,
                              void *workspace, size_t workspace_bytes, dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_loss_fwd_bwd_ex -- dlm_loss_fwd_bwd with objective options for uniform
 * noise ("Native diffusion language-model training", Objective and
 * recurrence options: DiffusionGemma's Rhine objectives use time weighting
 * inv_one_minus_t with objective_reduction example_mean; rhine_weight_clip
 * caps the 1 / (1 - t) weights).
 *
 * For mode == DLM_UNIFORM the weight of a scored canvas row of unit u becomes
 *   w = f_u / (number of scored canvas rows)           DLM_REDUCE_TOKEN_MEAN
 *   w = f_u / (B' * n_u)                               DLM_REDUCE_EXAMPLE_MEAN
 * with n_u the scored canvas rows of unit u, B' the units that have any, and
 *   f_u = 1                                            DLM_TIME_WEIGHT_NONE
 *   f_u = min(1 / (1 - t_u), weight_clip)              DLM_TIME_WEIGHT_INV_ONE_MINUS_T
 * (no cap when weight_clip <= 0; t_u = p[u], the uniform-noise time from
 * dlm_sample_t, which p must then hold).  The encoder AR term is unchanged.
 * options == NULL, or every field at its default, is dlm_loss_fwd_bwd.
 * Non-default time weighting or reduction with absorbing noise, or time
 * weighting without p, return DLM_ERR_INVALID_ARGUMENT; so does
 * options->struct_size < 16.
 * ---------------------------------------------------------------------- */
#define DLM_TIME_WEIGHT_NONE 0
#define DLM_TIME_WEIGHT_INV_ONE_MINUS_T 1
#define DLM_REDUCE_TOKEN_MEAN 0
#define DLM_REDUCE_EXAMPLE_MEAN 1

typedef struct {
    uint32_t struct_size;      /* sizeof(dlm_loss_options_t) */
    int32_t time_weighting;    /* DLM_TIME_WEIGHT_* */
    float weight_clip;         /* cap of 1 / (1 - t); <= 0: none */
    int32_t reduction;         /* DLM_REDUCE_* */
    int32_t keep_unscored_rows;/* 1: rows of dlogits / enc_dlogits that are not
                                  scored are left as they are instead of being
                                  zeroed (for a caller that keeps them zero);
                                  any noise mode.  Read only when struct_size
                                  covers it (older 16-byte structs: 0). */
} dlm_loss_options_t;

DLM_API dlm_status_t dlm_loss_fwd_bwd_ex(const dlm_layout_t *layout, const uint16_t *logits, int64_t ld,
                                 int32_t vocab, const int32_t *clean_ids, const uint8_t *corrupted,
                                 const float *p, int32_t mode, int32_t align,
                                 const dlm_layout_t *enc_layout, const uint16_t *enc_logits,
                                 int64_t enc_ld, const int32_t *enc_ids, float enc_ar_weight,
                                 float grad_scale, const dlm_loss_options_t *options, float *loss,
                                 float *unit_loss, uint16_t *dlogits, uint16_t *enc_dlogits,
                                 void *workspace, size_t workspace_bytes, dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_loss_fwd_bwd_static -- dlm_loss_fwd_bwd without a caller workspace.
 * No counterpart on the pages: this entry point exists for callers that are
 * not allowed to call cudaMalloc (code handed only its input and output
 * buffers by a host program that owns all device memory, e.g. a plugin in
 * another framework or a process held to a fixed memory pool), and that
 * therefore cannot provide the workspace dlm_loss_fwd_bwd takes.
 *
 * Same arguments and results as dlm_loss_fwd_bwd, minus the workspace.  The
 * scratch is a fixed device array of DLM_STATIC_SCRATCH_BYTES inside this
 * library, held by every GPU that loads the library until the process exits;
 * the call allocates nothing.  A problem whose dlm_loss_workspace_size()
 * exceeds DLM_STATIC_SCRATCH_BYTES is refused with
 * DLM_ERR_WORKSPACE_TOO_SMALL before anything is enqueued (2 MiB fits about
 * 100,000 logits rows, diffusion plus encoder, over a few thousand units).
 * Every call looks up the array's device address in the context current on
 * the calling thread (no address is cached, so non-primary contexts and a
 * device reset between calls are safe).  The first call in a context also
 * loads this library's device code there; make that first call before any
 * stream capture.  All calls share the one array: calls that overlap on the GPU (on
 * different streams, or from different host threads without ordering) race
 * and corrupt each other's results; order them on one stream.  Each call
 * re-initialises what it needs, so contents left by an earlier call are
 * harmless.  The device status word of these calls is not readable from
 * outside (use dlm_loss_fwd_bwd with a workspace when you need it).
 * ---------------------------------------------------------------------- */
#define DLM_STATIC_SCRATCH_BYTES (2u << 20)

DLM_API dlm_status_t dlm_loss_fwd_bwd_static(const dlm_layout_t *layout, const uint16_t *logits,
                              int64_t ld, int32_t vocab, const int32_t *clean_ids,
                              const uint8_t *corrupted, const float *p, int32_t mode, int32_t align,
                              const dlm_layout_t *enc_layout, const uint16_t *enc_logits,
                              int64_t enc_ld, const int32_t *enc_ids, float enc_ar_weight,
                              float grad_scale, float *loss, float *unit_loss,
                              uint16_t *dlogits, uint16_t *enc_dlogits, dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_linear_loss_fwd_bwd -- the absorbing, aligned loss above with
 * logits = hidden @ weight^T formed tile by tile on the tensor cores and never
 * written to memory ("Native diffusion language-model training", Adapters,
 * merging and inference: Cut Cross Entropy, plain linear head, aligned).
 *   hidden [n_tokens, d_model] bf16 row-major; weight [vocab, d_model] bf16
 *   row-major.  Logits are formed in fp32 from the bf16 inputs.
 *   d_hidden [n_tokens, d_model] bf16 (written; rows of unscored tokens = 0).
 *   d_weight [vocab, d_model] bf16 (written), or NULL to skip it.
 *   loss / unit_loss as for dlm_loss_fwd_bwd (unit_loss may be NULL).
 * Requires d_model % 64 == 0 and vocab % 8 == 0, 16-byte aligned pointers,
 * a 1024-byte aligned workspace and fewer than 2^31 - 256 tokens; otherwise
 * DLM_ERR_INVALID_ARGUMENT before anything is enqueued.
 * ---------------------------------------------------------------------- */
DLM_API size_t dlm_linear_loss_workspace_size(const dlm_layout_t *layout, int32_t d_model,
                                      int32_t vocab);

DLM_API dlm_status_t dlm_linear_loss_fwd_bwd(const dlm_layout_t *layout, const uint16_t *hidden,
                                     const uint16_t *weight, int32_t d_model, int32_t vocab,
                                     const int32_t *clean_ids, const uint8_t *corrupted,
                                     const float *p, float grad_scale, float *loss,
                                     float *unit_loss, uint16_t *d_hidden, uint16_t *d_weight,
                                     void *workspace, size_t workspace_bytes,
                                     dlm_stream_t stream);

/* dlm_linear_loss_fwd_bwd_ex -- the same with the alignment as an argument:
 * DLM_ALIGNED as above, or DLM_SHIFTED (row i, i.e. hidden state i, scores
 * token i + 1 of the same unit; a unit's last row is unscored -- the rows
 * and weights of dlm_loss_fwd_bwd with DLM_SHIFTED).  The page describes
 * Cut Cross Entropy for aligned targets only; the shifted form carries the
 * unfused loss's Dream alignment over.  Any other align returns
 * DLM_ERR_INVALID_ARGUMENT. */
DLM_API dlm_status_t dlm_linear_loss_fwd_bwd_ex(const dlm_layout_t *layout, const uint16_t *hidden,
                                        const uint16_t *weight, int32_t d_model, int32_t vocab,
                                        const int32_t *clean_ids, const uint8_t *corrupted,
                                        const float *p, int32_t align, float grad_scale,
                                        float *loss, float *unit_loss, uint16_t *d_hidden,
                                        uint16_t *d_weight, void *workspace, size_t workspace_bytes,
                                        dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_linear_loss_uniform_fwd_bwd -- the uniform-noise loss of
 * dlm_loss_fwd_bwd (DLM_UNIFORM) from hidden states and a linear output
 * head, logits never materialised: the DiffusionGemma objective
 * ("diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning notes: canvas CE +
 * encoder_loss_weight * encoder AR CE) through the Cut Cross Entropy form of
 * "Native diffusion language-model training", Adapters, merging and
 * inference.  The page describes that form for absorbing noise and aligned
 * targets only; this call carries the unfused uniform loss over unchanged.
 *   Canvas term: every non-pad canvas target is scored (row i scores token
 *     i, or token i + 1 of the same unit with DLM_SHIFTED), w = 1 / (number
 *     of scored canvas rows), logits = hidden @ weight^T.
 *   Encoder term (enc_layout != NULL): row i of enc_hidden scores enc_ids[i+1]
 *     of the same unit (non-pad), w = enc_ar_weight / (number of such rows),
 *     logits = enc_hidden @ weight^T with the same head.
 *   hidden [layout.n_tokens, d_model], enc_hidden [enc_layout.n_tokens,
 *   d_model], weight [vocab, d_model]: bf16 row-major.  clean_ids
 *   [layout.n_tokens] (the canvas targets), enc_ids [enc_layout.n_tokens].
 *   No corrupted mask or p: uniform noise scores every canvas position.
 *   d_hidden, d_enc_hidden: bf16, same shapes as hidden / enc_hidden
 *   (written; rows with no target = 0).  d_weight [vocab, d_model] bf16, the
 *   sum of both terms' contributions (written), or NULL to skip it.
 *   enc_layout.n_units must equal layout.n_units (unit u of the canvas is
 *   unit u of the encoder sequence); unit_loss[u] sums both terms of unit u.
 *   Requires d_model % 64 == 0, vocab % 8 == 0, 16-byte aligned pointers and
 *   fewer than 2^31 - 256 rows in total; otherwise DLM_ERR_INVALID_ARGUMENT
 *   before anything is enqueued.  Ids outside [0, vocab) set DLM_DEV_BAD_TOKEN_ID in
 *   the device status word; their rows are skipped.
 * Workspace: dlm_linear_loss_uniform_workspace_size(layout, enc_layout,
 * d_model, vocab) bytes, 1024-byte aligned (enc_layout may be NULL).
 * ---------------------------------------------------------------------- */
DLM_API size_t dlm_linear_loss_uniform_workspace_size(const dlm_layout_t *layout,
                                              const dlm_layout_t *enc_layout,
                                              int32_t d_model, int32_t vocab);

DLM_API dlm_status_t dlm_linear_loss_uniform_fwd_bwd(const dlm_layout_t *layout,
                                             const uint16_t *hidden,
                                             const dlm_layout_t *enc_layout,
                                             const uint16_t *enc_hidden, const int32_t *enc_ids,
                                             const uint16_t *weight, int32_t d_model,
                                             int32_t vocab, const int32_t *clean_ids,
                                             int32_t align, float enc_ar_weight, float grad_scale,
                                             float *loss, float *unit_loss, uint16_t *d_hidden,
                                             uint16_t *d_enc_hidden, uint16_t *d_weight,
                                             void *workspace, size_t workspace_bytes,
                                             dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_get_device_status -- copy the device status word of a loss workspace
 * (first 4 bytes) to *host_status after the work queued on `stream`;
 * synchronises `stream`.  Each dlm_loss_fwd_bwd / dlm_linear_loss_fwd_bwd
 * call clears the word first, so it reports that call.
 * ---------------------------------------------------------------------- */
DLM_API dlm_status_t dlm_get_device_status(const void *workspace, uint32_t *host_status,
                                   dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_test_skip_device_check -- test hook, off by default; not for use in
 * training.  With enabled = 1 every call skips its check for a B200 and goes
 * straight on to its CUDA calls.  On a host without a usable device those
 * calls fail, and each entry point must turn the failure into
 * DLM_ERR_CUDA with a message (dlm_last_cuda_error) instead of crashing:
 * this is how the library's CUDA error paths are tested without a GPU.  On a
 * host with a device, enabling it lets a call launch its kernels on whatever
 * device is current (sm_100a code only runs on a B200).  enabled = 0 restores
 * the check; any other value returns DLM_ERR_INVALID_ARGUMENT.  The setting
 * is process-wide.
 * ---------------------------------------------------------------------- */
DLM_API dlm_status_t dlm_test_skip_device_check(int32_t enabled);

/* ------------------------------------------------------------------------
 * dlm_selftest_bounded_wait -- exercise the library's failure detection on
 * the device.  Every on-chip wait of the kernels above (mbarrier phases of
 * the TMA / tensor-core pipelines) gives up after a time limit, records
 * DLM_DEV_WAIT_TIMEOUT in the status word and lets the kernel end, so a
 * broken pipeline cannot hang the GPU.  This call launches one thread that
 * waits, through the same bounded wait, on a barrier phase that nothing ever
 * completes, with a limit of `limit_ns` nanoseconds (1 .. 1e10): on return of
 * the kernel *dev_status (device uint32) has DLM_DEV_WAIT_TIMEOUT or'ed in and
 * the CUDA context is still usable.  (The pages describe failure handling
 * only at the level of the training loop; this is the library's own check.)
 * ---------------------------------------------------------------------- */
DLM_API dlm_status_t dlm_selftest_bounded_wait(uint64_t limit_ns, uint32_t *dev_status,
                                               dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_decision_loss_fwd_bwd -- typed-decision losses at label slots,
 * forward + backward ("Native diffusion language-model training",
 * Typed-decision training: candidate-restricted CE, full-vocabulary CE and a
 * 0.1 Brier term; Labels: hard / dist / set labels, labels.label_softmax,
 * hard_label_smoothing; Adapters, merging and inference: the restricted-label
 * and Brier terms are computed over the allowed answers).
 *
 * A label slot is the canvas position of one question's answer; its logits
 * row z covers the whole vocabulary, and its question has K (1..128)
 * distinct answer tokens a_0..a_{K-1} in canonical order.  With r = softmax
 * of the K candidate logits, P = softmax over the vocabulary, q the CE
 * target and y the Brier target over the K answers:
 *   CE_res  = -sum_k q_k log r_k             (label_softmax RESTRICTED, BOTH)
 *   CE_full = -sum_k q_k log P(a_k)          (label_softmax FULL, BOTH)
 *   Brier   = sum_k (r_k - y_k)^2, times brier_weight (0.1 on the page)
 *   loss    = (1 / n_slots) * sum over slots of its terms
 * Targets by label kind (label_kind[i]; label_val holds one float per
 * answer, at cand_off[i] .. cand_off[i+1]-1):
 *   DLM_LABEL_HARD: val = 1 at the gold answer, 0 elsewhere.  y = val,
 *       q = (1 - hard_label_smoothing) val + hard_label_smoothing / K.
 *   DLM_LABEL_DIST: val = the probabilities (finite, >= 0).  q = y = val.
 *   DLM_LABEL_SET:  val = 1 for each allowed answer, 0 elsewhere (at least
 *       one 1).  q = y = val / (number of allowed answers).
 * Arguments (device pointers unless stated):
 *   logits [n_rows, ld] bf16; slot_rows [n_slots] int64: the logits row of
 *       each slot, or NULL for row i = slot i (logits computed at the label
 *       slots only; then n_rows >= n_slots).  ld >= vocab.
 *   cand_off [n_slots + 1] int32 (offsets into cand_ids and label_val,
 *       non-decreasing, within 0..n_cands), cand_ids [n_cands] int32 answer
 *       token ids, label_kind [n_slots] int32, label_val [n_cands] float.
 *   grad_scale g: the gradient written is g * d loss / d z.
 *   loss [1] float (written); slot_loss [n_slots] float: each slot's
 *       contribution (its terms / n_slots; sums to loss), or NULL.
 *   dlogits [n_slots, ld_out] bf16 (row i = slot i; columns 0..vocab-1
 *       written, the rest untouched); ld_out >= vocab.
 *   workspace: at least dlm_decision_workspace_size(n_slots, vocab) bytes,
 *       256-byte aligned; its status word is read by dlm_get_device_status.
 * Errors: n_slots outside 0..DLM_DECISION_MAX_SLOTS, vocab <= 0, a bad
 * label_softmax, a negative or non-finite brier_weight, smoothing outside
 * [0, 1], a non-finite grad_scale, a null pointer, ld / ld_out < vocab,
 * n_rows < 1 (or < n_slots without slot_rows), n_cands < 0 or a workspace
 * that is not 256-byte aligned return DLM_ERR_INVALID_ARGUMENT, and a
 * workspace smaller than dlm_decision_workspace_size() returns
 * DLM_ERR_WORKSPACE_TOO_SMALL, before anything is enqueued.  On the device, a slot whose row is outside
 * [0, n_rows) or whose answer offsets leave 0..n_cands sets
 * DLM_DEV_BAD_LAYOUT; an answer id outside [0, vocab) sets
 * DLM_DEV_BAD_TOKEN_ID; K outside 1..128, repeated answer ids, an unknown
 * kind or a malformed label set DLM_DEV_BAD_LABEL; such a slot adds 0 to the
 * loss (the mean still divides by n_slots) and its dlogits row is all
 * zeros.  n_slots = 0 writes
 * loss = 0.  The 16-byte load path needs ld and ld_out multiples of 8 and
 * 16-byte aligned logits and dlogits; other shapes take a scalar path.
 * Not built: full_ce_weighting: dft (the page gives no formula).
 * ---------------------------------------------------------------------- */
#define DLM_LABEL_HARD 0
#define DLM_LABEL_DIST 1
#define DLM_LABEL_SET 2
#define DLM_LABEL_SOFTMAX_RESTRICTED 1
#define DLM_LABEL_SOFTMAX_FULL 2
#define DLM_LABEL_SOFTMAX_BOTH 3
#define DLM_DECISION_MAX_ANSWERS 128
#define DLM_DECISION_MAX_SLOTS 65535

DLM_API size_t dlm_decision_workspace_size(int32_t n_slots, int32_t vocab);

DLM_API dlm_status_t dlm_decision_loss_fwd_bwd(int32_t n_slots, const uint16_t *logits, int64_t n_rows,
                                       int64_t ld, int32_t vocab, const int64_t *slot_rows,
                                       const int32_t *cand_off, int64_t n_cands, const int32_t *cand_ids,
                                       const int32_t *label_kind, const float *label_val,
                                       int32_t label_softmax, float brier_weight,
                                       float hard_label_smoothing, float grad_scale, float *loss,
                                       float *slot_loss, uint16_t *dlogits, int64_t ld_out,
                                       void *workspace, size_t workspace_bytes, dlm_stream_t stream);

/* ------------------------------------------------------------------------
 * dlm_scale_bf16 -- x[r, c] *= *scale in place for r < rows, c < cols (bf16,
 * row stride ld >= cols), where scale is a DEVICE float: the upstream
 * gradient of a scalar loss, applied by an autograd backward to a gradient
 * the loss call has already written with grad_scale = 1.  When *scale is
 * exactly 1 (loss.backward() on the loss itself) the kernel reads it and
 * returns without touching x, so the host never needs to read the scalar.
 * Otherwise each element is rounded to bf16 again after the product (one
 * more rounding than passing the factor as grad_scale to the loss call).
 * The pages have no counterpart: this serves the autograd wrappers of the
 * Python binding.  rows or cols = 0 is a no-op; a negative size, ld < cols
 * or a null pointer return DLM_ERR_INVALID_ARGUMENT.
 * ---------------------------------------------------------------------- */
DLM_API dlm_status_t dlm_scale_bf16(uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                    const float *scale, dlm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DLM_H_ */
