/*
 * gpt2step -- one GPT-2 training step (forward, backward, global-norm clip and
 * AdamW) on a single B200, as a C ABI.
 *
 * The step is the one fixed by "Pretraining and adapting a language model on a
 * dependency-free stack" (arXiv 2609.28568):
 *   §4.1 (Fig. 1)  GPT-2 decoder: pre-LayerNorm blocks with residuals around
 *                  attention and MLP, tied input/output embeddings, vocabulary
 *                  padded to a multiple of 128 with the softmax over real ids
 *                  only, N(0, 0.02) init with residual-writing projections
 *                  scaled by 1/sqrt(2L);
 *   §4.3           bf16 activations; fp32 master weights, gradients, optimizer
 *                  state, LayerNorm statistics and loss; AdamW (0.9, 0.95),
 *                  eps 1e-8, weight decay 0.1 on 2-D weights only; gradients
 *                  clipped to global norm 1.0; linear warmup then cosine decay;
 *   §4.4           gradient accumulation over micro-batches.
 *
 * Conventions for every call below:
 *   - Pointers named *_dev are device pointers, *_host are host pointers.
 *   - Every call returns a gpt2_status (0 = GPT2_OK). Calls never abort; after a
 *     data error (bad token id, non-finite loss or norm) the model stays usable.
 *   - All device work is enqueued on the stream given to gpt2_create, in call
 *     order. A call that writes a host result synchronises that stream first
 *     and then reports any error the device recorded since the last such call.
 *   - Not thread-safe per model; distinct models are independent.
 */
#ifndef GPT2STEP_H
#define GPT2STEP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gpt2_status {
  GPT2_OK = 0,
  GPT2_ERR_ARG = 1,          /* invalid argument, unsupported shape, short arena    */
  GPT2_ERR_CUDA = 2,         /* a CUDA runtime/driver call failed                   */
  GPT2_ERR_TOKEN_RANGE = 3,  /* a token or target id outside [0, vocab_real)         */
  GPT2_ERR_NONFINITE = 4,    /* loss or gradient norm not finite; step not applied   */
  GPT2_ERR_STATE = 5,        /* call out of order (e.g. clip_adamw with no fwd_bwd)  */
  GPT2_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up (kernel bug)      */
} gpt2_status;

/* Model and optimiser configuration. Field names follow GPT-2 and §4.1/§4.3. */
typedef struct gpt2_config {
  int32_t n_layer, n_head, n_embd, seq_len;   /* L, H, C, T                                  */
  int32_t vocab_real, vocab_padded;           /* V; 0 => round V up to a multiple of 128     */
  int32_t micro_batch, grad_accum;            /* B per fwd_bwd call; accum is informational   */
  float max_lr, min_lr;                       /* schedule end points (§4.3: 6e-4 -> 0)        */
  int32_t warmup_steps, total_steps;          /* §4.3: 700 warmup of 18,865                   */
  float beta1, beta2, eps, weight_decay, grad_clip; /* 0.9, 0.95, 1e-8, 0.1, 1.0               */
} gpt2_config;

typedef struct gpt2_model gpt2_model; /* opaque */

/* Which state array gpt2_read / gpt2_write address (GPT2_WEIGHTS_BF16, the
 * bf16 copy the tensor cores read, only through gpt2_state_device_ptr). */
enum { GPT2_PARAMS = 0, GPT2_GRADS = 1, GPT2_ADAM_M = 2, GPT2_ADAM_V = 3, GPT2_WEIGHTS_BF16 = 4 };

/* Bytes of device memory the caller must provide to gpt2_create for this
 * configuration (fp32 params, grads, m, v; bf16 weight copy; saved activations;
 * logits; workspaces). Returns 0 for an invalid configuration. Supported shapes:
 * n_embd a multiple of 128 with head size 32 or 64, seq_len a multiple of 64
 * (at most 4096), vocab_padded a multiple of 128. */
size_t gpt2_arena_bytes(const gpt2_config* cfg);

/* Create a model inside the caller's arena (device memory, at least
 * gpt2_arena_bytes(cfg) bytes, 1024-byte aligned; owned by the caller and
 * required to outlive gpt2_destroy). Parameters are initialised on the device
 * from `seed` (§4.1: N(0, 0.02), residual-writing projections x 1/sqrt(2L),
 * LayerNorm gains 1, biases 0, padded vocabulary rows 0) with Philox4x32-10
 * (Salmon et al., SC'11), stream k = parameter kind k, Box-Muller normals.
 * Gradients and Adam moments start at 0. `cuda_stream` is a cudaStream_t
 * (NULL = legacy default stream). On success *out receives the model. */
int gpt2_create(const gpt2_config* cfg, uint64_t seed, void* dev_arena, size_t arena_bytes,
                void* cuda_stream, gpt2_model** out);

/* Release host-side state. The arena is untouched and stays owned by the caller. */
void gpt2_destroy(gpt2_model* model);

/* One micro-step: forward and backward on tokens_dev / targets_dev (device,
 * int32, [micro_batch, seq_len] row-major, ids in [0, vocab_real); read-only,
 * only during the enqueued work). Gradients of this micro-batch's mean loss are
 * ADDED to the fp32 gradient buffers. If loss_out is non-NULL the stream is
 * synchronised and the micro-batch mean loss is written there; with NULL the
 * call is fully asynchronous. */
int gpt2_fwd_bwd(gpt2_model* model, const int32_t* tokens_dev, const int32_t* targets_dev,
                 float* loss_out);

/* Optimizer step `step` (0-based; lr from the warmup + cosine schedule).
 * Averages the accumulated gradients over the number of fwd_bwd calls since
 * the last step, clips them to global norm grad_clip, applies AdamW with bias
 * correction at t = step + 1, refreshes the bf16 weight copy and zeroes the
 * gradients. If the norm or any accumulated loss is not finite, the weights and
 * moments are left unchanged (the gradients are still cleared) and the next
 * synchronising call returns GPT2_ERR_NONFINITE. grad_norm_out (optional,
 * synchronises) receives the pre-clip norm. GPT2_ERR_STATE if no fwd_bwd ran
 * since the last step. */
int gpt2_clip_adamw(gpt2_model* model, int32_t step, float* grad_norm_out);

/* Mean loss of the last completed optimizer step (mean over its micro-steps)
 * and its pre-clip gradient norm. Synchronises. Either pointer may be NULL. */
int gpt2_last_step_stats(gpt2_model* model, float* mean_loss_out, float* grad_norm_out);

/* Held-out loss: forward only, no gradients touched, mean over
 * batch * seq_len positions. tokens_dev / targets_dev are device int32
 * [batch, seq_len]; batch may exceed micro_batch (processed in chunks).
 * Synchronises and writes *loss_out. */
int gpt2_eval_loss(gpt2_model* model, const int32_t* tokens_dev, const int32_t* targets_dev,
                   int32_t batch, float* loss_out);

/* A whole optimizer step from HOST buffers: for each of n_micro micro-batches,
 * copy tokens/targets (int32 [n_micro, micro_batch, seq_len], pinned or
 * pageable host memory) to the device, run fwd_bwd, then clip_adamw(step).
 * Synchronises; writes the mean loss and pre-clip norm (either may be NULL). */
int gpt2_train_step_host(gpt2_model* model, const int32_t* tokens_host, const int32_t* targets_host,
                         int32_t n_micro, int32_t step, float* mean_loss_out,
                         float* grad_norm_out);

/* Per-position losses (fp32, [micro_batch * seq_len]) of the last fwd_bwd,
 * copied to host_dst (n must equal micro_batch * seq_len). Synchronises. */
int gpt2_token_losses(gpt2_model* model, float* host_dst, int64_t n);

/* Learning rate the schedule gives for `step` (host arithmetic only). */
float gpt2_lr(const gpt2_model* model, int32_t step);

/* The same schedule from a configuration alone, no model or GPU needed
 * (§4.3: linear warmup over warmup_steps to max_lr, then a cosine to min_lr at
 * total_steps; step is 0-based, warmup gives max_lr * (step + 1) / warmup_steps,
 * steps past total_steps stay at min_lr). Returns -1 for a NULL config. */
double gpt2_schedule_lr(const gpt2_config* cfg, int32_t step);

/* Number of CUDA kernels this model has launched so far (host-side count). */
int64_t gpt2_kernel_launches(const gpt2_model* model);

/* Per-class timing of the model's own kernels with CUDA events recorded on its
 * stream around each launch group. gpt2_profile_enable(model, 1) synchronises,
 * clears the totals and starts recording; 0 stops. gpt2_profile_read
 * synchronises and returns, for class `cls` (0 .. gpt2_profile_num_classes()-1,
 * named by gpt2_profile_class_name), the summed device time in ms, the number
 * of launch groups, and their summed algorithmic work: FLOPs for "gemm" and the
 * attention classes, bytes of HBM traffic for the others. */
int gpt2_profile_enable(gpt2_model* model, int on);
int gpt2_profile_num_classes(void);
const char* gpt2_profile_class_name(int cls);
int gpt2_profile_read(gpt2_model* model, int cls, double* ms, int64_t* launches, double* work);

/* Human-readable name of a status code (static string). */
const char* gpt2_status_string(int status);

/* Introspection: the named tensors (148 for 12 blocks: wte, wpe, 12 per block,
 * ln_f weight and bias), with GPT-2 names such as "h.10.ln_2.weight". */
int gpt2_num_tensors(const gpt2_model* model);
/* name: static string owned by the model; shape: up to 2 dims; ndim 1 or 2. */
int gpt2_tensor_info(const gpt2_model* model, int idx, const char** name, int64_t shape[2],
                     int* ndim);
/* Copy tensor idx of state array `what` to / from host fp32 memory (element
 * count = product of its shape). Synchronises. Writing PARAMS also refreshes
 * that tensor's bf16 copy. */
int gpt2_read(gpt2_model* model, int what, int idx, float* host_dst);
int gpt2_write(gpt2_model* model, int what, int idx, const float* host_src);

/* Device address and length (elements: fp32, or bf16 for GPT2_WEIGHTS_BF16)
 * of the whole state array `what` inside the caller's arena, for collectives
 * over it: data-parallel ranks ("Pretraining and adapting a language model on
 * a dependency-free stack", §4.4, three cards) average GPT2_GRADS across ranks
 * between their last gpt2_fwd_bwd and gpt2_clip_adamw, on the model's stream.
 * Valid while the model lives; no copy, no synchronisation. Writing
 * GPT2_PARAMS through it does not refresh the bf16 copy (use gpt2_write).
 *
 * Flat layout (the same for every array): region 0 = [0, P1) holds the 1-D
 * parameters (LayerNorm gains and biases, linear biases); [P1, P) holds the
 * 2-D weights in buckets, in the order the backward pass finishes their
 * gradients: one bucket per block from the last block to the first, then
 * {wpe, wte}. Tensors start 64-element aligned; each bucket is zero-padded to
 * a multiple of 7,680 elements, so it splits into equal shards that are
 * multiples of 64 elements for any world size dividing 120. Gaps stay zero. */
int gpt2_state_device_ptr(gpt2_model* model, int what, void** dev_ptr, int64_t* count);

/* ---- sharded optimizer step (data parallelism in the ZeRO-1 form) ----------
 * §4.4 averages the gradients across cards once per optimizer step. In the
 * sharded form each rank reduce-scatters (averages) the 2-D buckets so that it
 * holds the averaged gradient of one shard of every bucket, all-reduces region
 * 0, updates region 0 and its shards only, and all-gathers the bf16 weights of
 * every bucket. The fp32 masters and Adam moments outside a rank's shards are
 * then stale and unused (the forward and backward read the 2-D weights only
 * through the bf16 copy and region 0 in fp32). */

/* Number of 2-D buckets (n_layer + 1). */
int gpt2_num_buckets(const gpt2_model* model);

/* Element range [begin, end) of bucket b (0 .. gpt2_num_buckets - 1, in the
 * order their gradients become final), or of region 0 for b = -1. */
int gpt2_bucket_range(const gpt2_model* model, int b, int64_t* begin, int64_t* end);

/* Register one cudaEvent_t per bucket (n == gpt2_num_buckets; n == 0 clears).
 * Every gpt2_fwd_bwd then records event b on the model's stream as soon as
 * bucket b's gradients are final for that micro-step (the last event also
 * marks region 0), so that a collective on another stream can start on a
 * bucket while the backward works on the earlier blocks. The events stay the
 * caller's; they must outlive the registration. */
int gpt2_set_bucket_events(gpt2_model* model, void* const* events, int n);

/* Enqueue on the model's stream: *dev_out (a device double) = the sum of
 * squares of the accumulated gradients over the element ranges
 * ranges[2i] .. ranges[2i+1] (n_ranges <= 64, bounds multiples of 64 inside
 * the flat array). */
int gpt2_grad_sumsq(gpt2_model* model, const int64_t* ranges, int n_ranges, double* dev_out);

/* The update of gpt2_clip_adamw restricted to the given element ranges, with
 * the global norm taken from *dev_sumsq (device double: the sum of squares of
 * the accumulated gradients over the whole model, e.g. gpt2_grad_sumsq's
 * partials summed across ranks): norm = sqrt(*dev_sumsq) / micro-steps, clip
 * scale min(1, clip / norm), AdamW with the schedule's lr(step) on params, m, v
 * and the bf16 copy inside the ranges; then ALL gradients are cleared and the
 * micro-step count restarts. GPT2_ERR_STATE without a micro-step since the
 * last update; *grad_norm_out (may be NULL) synchronises, as in
 * gpt2_clip_adamw. */
int gpt2_clip_adamw_ranges(gpt2_model* model, int32_t step, const int64_t* ranges, int n_ranges,
                           const double* dev_sumsq, float* grad_norm_out);

/* Total parameter count: real vocabulary rows only (124,439,808 for GPT-2
 * 124M, §4.1) when padded == 0, all stored rows when padded != 0. */
int64_t gpt2_num_params(const gpt2_config* cfg, int padded);

#ifdef __cplusplus
}
#endif
#endif /* GPT2STEP_H */
