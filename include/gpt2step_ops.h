/*
 * gpt2step_ops -- the individual steps of the GPT-2 training step, one call
 * each, on caller-owned device buffers. They are the kernels gpt2_fwd_bwd and
 * gpt2_clip_adamw run, exposed so that each step can be checked on its own.
 *
 * Common conventions:
 *   - "bf16" buffers hold IEEE bfloat16 values (2 bytes), row-major, with the
 *     row stride equal to the row length and 16-byte aligned base pointers.
 *   - fp32 buffers are float, row-major.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream); every call only
 *     enqueues work and returns GPT2_OK, GPT2_ERR_ARG (unsupported shape or NULL
 *     pointer, nothing enqueued) or GPT2_ERR_CUDA (launch failure).
 *   - `dev_err` is a device int the caller zeroes; kernels OR flags into it
 *     (1 = token id out of range, 4 = a bounded device wait timed out).
 *   - Workspaces are caller-owned device memory of at least the size the
 *     matching *_workspace query returns; their contents on entry do not matter.
 *
 * Section references are to "Pretraining and adapting a language model on a
 * dependency-free stack" (arXiv 2609.28568) unless noted.
 */
#ifndef GPT2STEP_OPS_H
#define GPT2STEP_OPS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Linear layer forward (§4.1 Fig. 1: QKV, attention and MLP projections, tied
 * head). out[M,N] = inp[M,K] . w[N,K]^T (+ bias[N]) (+ resid[M,N]); all bf16
 * except bias (fp32, may be NULL unless resid is given). Requires N % 32 == 0,
 * K % 64 == 0. Runs on the tcgen05 tensor cores with fp32 accumulation. */
int gpt2op_linear_fwd(const void* inp, const void* w, const float* bias, const void* resid, void* out, int M,
                      int N, int K, int* dev_err, void* stream);

/* MLP fc + GELU (tanh approximation): pre = inp . w^T + bias, gelu = GELU(pre);
 * both written as bf16 [M,N]. */
int gpt2op_linear_fwd_gelu(const void* inp, const void* w, const float* bias, void* pre_out, void* gelu_out, int M,
                           int N, int K, int* dev_err, void* stream);

/* Input gradient of a linear layer: din[M,K] = dout[M,N] . w[N,K], optionally
 * multiplied elementwise by GELU'(gelu_pre[M,K]) (gelu_pre may be NULL).
 * Requires K % 64 == 0 and N % 64 == 0. */
int gpt2op_linear_dgrad(const void* dout, const void* w, const void* gelu_pre, void* din, int M, int N, int K,
                        int* dev_err, void* stream);

/* Weight gradient: dw[N,K] (fp32) += dout[M,N]^T . inp[M,K]. `splits` > 1
 * divides the M reduction across CTAs (fp32 atomic accumulation); 0 chooses
 * automatically. Requires N % 64 == 0, K % 64 == 0, M % 64 == 0. */
int gpt2op_linear_wgrad(const void* dout, const void* inp, float* dw, int M, int N, int K, int splits, int* dev_err,
                        void* stream);

/* Both gradients of a linear layer in one launch (§4.1 Fig. 1 backward; the
 * form gpt2_fwd_bwd uses for every block's four linear layers):
 *   din[M,K] = dout[M,N] . w[N,K]  (times GELU'(gelu_pre[M,K]) if gelu_pre is
 *              not NULL; then colsum, if not NULL, fp32 [K], += the column sums
 *              of the stored bf16 din -- the MLP fc bias gradient)
 *   dw[N,K] (fp32) += dout[M,N]^T . inp[M,K]
 * The weight-gradient tiles follow the input-gradient tiles in one persistent
 * tile list; the M reduction of dw is split across CTAs (fp32 atomics) by a
 * host-side estimate of the busiest SM pair's finish time. Requires M >= 256,
 * M % 64 == 0, N % 256 == 0, K % 256 == 0; other shapes return GPT2_ERR_ARG.
 * *splits_out (may be NULL) receives the dw reduction split chosen. */
int gpt2op_linear_bwd(const void* dout, const void* w, const void* inp, const void* gelu_pre, void* din, float* dw,
                      float* colsum, int M, int N, int K, int* splits_out, int* dev_err, void* stream);

/* Bias gradient: db[N] (fp32) += sum over rows of dout[M,N] (bf16). N % 8 == 0.
 * With a workspace: a deterministic two-pass column sum. With workspace NULL:
 * one launch whose strips add into db by fp32 atomics (the form gpt2_fwd_bwd
 * uses; db 16-byte aligned; the order of the additions, and so the last bits,
 * may vary between runs). */
size_t gpt2op_bias_grad_workspace(int M, int N);
int gpt2op_bias_grad(const void* dout, float* db, int M, int N, void* workspace, size_t ws_bytes, void* stream);

/* LayerNorm forward over rows of C (§4.1 pre-LN blocks, §4.3 fp32 statistics):
 * y = (x - mean) * rstd * w + b with eps 1e-5 and biased variance; x, y bf16
 * [rows, C]; w, b fp32 [C]; mean, rstd fp32 [rows]. C in {128, 256, 384, 512,
 * 768, 1024, 1536, 2048}. */
int gpt2op_layernorm_fwd(const void* x, const float* w, const float* b, void* y, float* mean, float* rstd, int rows,
                         int C, void* stream);

/* LayerNorm backward: dx = LN'(dy) (+ dresid, the residual-stream gradient, may
 * be NULL; dx may alias dresid); dw, db (fp32 [C]) += column sums of dy * xhat
 * and dy. With a workspace the column sums are combined in a fixed order by a
 * second launch (deterministic). With workspace NULL each CTA adds its sums
 * into dw and db by fp32 vector atomics in the same launch (the form
 * gpt2_fwd_bwd uses; dw, db 16-byte aligned; the last bits may vary between
 * runs). */
size_t gpt2op_layernorm_bwd_workspace(int rows, int C);
int gpt2op_layernorm_bwd(const void* dy, const void* x, const float* mean, const float* rstd, const float* w,
                         const void* dresid, void* dx, float* dw, float* db, int rows, int C, void* workspace,
                         size_t ws_bytes, void* stream);

/* LayerNorm backward for callers that cannot allocate device memory: the same
 * operation, arguments and results as gpt2op_layernorm_bwd, without the
 * workspace. The pages have no counterpart; it exists for code that must not
 * call cudaMalloc, e.g. a plugin whose host application owns every device
 * allocation through its own budgeted pool, or a thread that may not block on
 * the implicit device synchronisation an allocation can cause.
 * Its scratch is one fixed array inside the library, of
 * gpt2op_layernorm_bwd_noalloc_max_bytes() = 2,424,832 bytes, that every GPU
 * which loads the library keeps until the process exits. A call fits exactly
 * when gpt2op_layernorm_bwd_workspace(rows, C) is at most that size (the
 * workspace is 8 * C bytes per CTA; a CTA takes 8 / 12 / 8 / 4 rows for C <= 512 /
 * 768 / 1024 / larger, up to 296 / 148 / 148 / 296 CTAs, so any row count fits
 * for C <= 1024); a call needing more returns GPT2_ERR_ARG before touching the
 * GPU. The first call on a device looks up the array's device address and
 * should come before any stream capture. All calls share the array: calls that
 * overlap on the GPU race. */
size_t gpt2op_layernorm_bwd_noalloc_max_bytes(void);
int gpt2op_layernorm_bwd_noalloc(const void* dy, const void* x, const float* mean, const float* rstd, const float* w,
                                 const void* dresid, void* dx, float* dw, float* db, int rows, int C, void* stream);

/* Causal multi-head attention forward (grow_a_language_model_intro, activities
 * 5-6: softmax(Q K^T / sqrt(hd)) V with a causal mask). qkv bf16 [B,T,3C]
 * (q | k | v, heads contiguous), out bf16 [B,T,C], lse fp32 [B,H,T] (natural
 * log-sum-exp of the scaled scores). hd in {32, 64}, T % 64 == 0. T % 128 == 0
 * runs on tcgen05 (scores and output accumulated in tensor memory); other
 * shapes on mma.sync. */
int gpt2op_attention_fwd(const void* qkv, void* out, float* lse, int B, int T, int H, int hd, int* dev_err,
                         void* stream);

/* Attention backward from the saved output and lse: dqkv bf16 [B,T,3C].
 * T % 128 == 0 (and H <= 64) runs on tcgen05, other shapes on mma.sync. The
 * workspace (fp32 dQ accumulator [B*T, C] followed by 32 bytes per query and
 * head of per-query terms) must be 16-byte aligned; its contents on entry do
 * not matter. Concurrent calls must not share a workspace.
 * dbias, if not NULL (fp32 [3C], 16-byte aligned, else GPT2_ERR_ARG): += the
 * gradient of a bias added to qkv, i.e. the column sums of dqkv over the B*T
 * rows. On tcgen05 they are formed from exact identities: the q third sums dQ
 * in fp32 before rounding, the v third sums dO (each causal softmax row sums
 * to one, so dV's column sums equal dO's), the k third gets nothing (its
 * gradient is exactly zero: a shift shared by a query's scores cancels in the
 * softmax). On mma.sync the column sums of the stored bf16 dqkv are added
 * (fp32 atomics; the k third then holds rounding-level values). */
size_t gpt2op_attention_bwd_workspace(int B, int T, int H, int hd);
int gpt2op_attention_bwd(const void* qkv, const void* out, const void* dout, const float* lse, void* dqkv,
                         float* dbias, int B, int T, int H, int hd, void* workspace, size_t ws_bytes, int* dev_err,
                         void* stream);

/* Vocabulary-masked softmax cross-entropy, forward and backward fused (§4.1:
 * softmax over the V real ids only). logits bf16 [N,Vp] are overwritten in
 * place with dz = (softmax - onehot(target)) * dscale for columns < V and
 * exactly 0 for columns >= V; losses fp32 [N] = lse - z[target]. A target
 * outside [0, V) gives loss 0, no one-hot term, and flag 1 in dev_err. */
int gpt2op_softmax_ce(void* logits, const int32_t* targets, float* losses, int N, int V, int Vp, float dscale,
                      int* dev_err, void* stream);

/* The tied lm_head and the softmax-CE as one op ("Pretraining and adapting a
 * language model on a dependency-free stack" §4.1: logits = ln_f output x wte^T,
 * softmax over the V real ids). h bf16 [N,C] and wte bf16 [Vp,C] row-major;
 * logits bf16 [N,Vp] (caller-owned, 16-byte aligned) receive the logits, then,
 * when write_grad is non-zero, are overwritten with dz exactly as
 * gpt2op_softmax_ce does; losses fp32 [N]. When the GEMM runs on CTA pairs
 * (N >= 256 rows and 256-wide tiles chosen, as for the model's logits), its
 * epilogue also writes each row's running (max, sum of 2^) over every 128
 * columns of the stored bf16 logits into the workspace, so the cross-entropy
 * reads the logits once (not at all for losses alone); otherwise the two-pass
 * kernel runs. The workspace (gpt2op_lm_head_ce_workspace bytes, 8-byte
 * aligned, contents on entry irrelevant) is required either way. Errors as
 * gpt2op_softmax_ce; a missing, short or misaligned workspace returns
 * GPT2_ERR_ARG before any launch. */
size_t gpt2op_lm_head_ce_workspace(int N, int Vp);
int gpt2op_lm_head_ce(const void* h, const void* wte, const int32_t* targets, void* logits, float* losses, int N,
                      int C, int V, int Vp, float dscale, int write_grad, void* workspace, size_t ws_bytes,
                      int* dev_err, void* stream);

/* The loss of the tied lm_head without its logits ever being stored (the
 * evaluation form of gpt2op_lm_head_ce; §4.1 tied head, softmax over the V real
 * ids): the GEMM's epilogue keeps, per row, only the (max, sum) partials of the
 * bf16-rounded logits over ids < V and the target's logit, and losses fp32 [N] =
 * lse - z[target]. No gradient. h bf16 [N,C], wte bf16 [Vp,C]; N >= 256 (the
 * CTA-pair GEMM; smaller N returns GPT2_ERR_ARG); workspace as
 * gpt2op_lm_head_ce_workspace. A target outside [0, V) gives loss 0 and flag 1. */
int gpt2op_lm_head_loss(const void* h, const void* wte, const int32_t* targets, float* losses, int N, int C, int V,
                        int Vp, void* workspace, size_t ws_bytes, int* dev_err, void* stream);

/* Cross-entropy with an ignore index per target (the loss taken only on chosen
 * positions, e.g. the answers of question/answer text; "Pretraining and
 * adapting a language model on a dependency-free stack" trains its adapter that
 * way). The pages have no kernel for it: this is the vocabulary-masked
 * softmax-CE above where rows whose target equals ignore_index (any value but
 * INT_MIN) get loss 0 and a gradient of exactly 0 and raise no error. dscale is
 * the caller's, normally 1 / (number of kept rows) for the mean over kept rows. */
int gpt2op_softmax_ce_masked(void* logits, const int32_t* targets, float* losses, int N, int V, int Vp,
                             int ignore_index, float dscale, int* dev_err, void* stream);

/* Token + position embedding: out[b,t,:] = wte[tok[b,t],:] + wpe[t,:] (bf16).
 * Ids outside [0, V) read row 0 and set flag 1 in dev_err. */
int gpt2op_embedding_fwd(const int32_t* tokens, const void* wte, const void* wpe, void* out, int B, int T, int C,
                         int V, int* dev_err, void* stream);

/* Embedding backward: dwte[tok,:] += dx, dwpe[t,:] += sum_b dx (fp32). Rows with
 * the same id within a block of 64 positions are summed in position order and
 * added into dwte once by fp32 vector atomics (dwte 16-byte aligned; the last
 * bits may vary between runs); ids outside [0, V) are skipped. */
int gpt2op_embedding_bwd(const int32_t* tokens, const void* dx, float* dwte, float* dwpe, int B, int T, int C, int V,
                         void* stream);

/* Self-test of the bounded device wait that every mbarrier wait of this
 * library uses (no counterpart on the pages: it checks the library's own
 * failure handling). One CTA waits on a shared-memory barrier that nothing
 * completes, gives up after limit_ns (1 ms .. 5 s) of %globaltimer time,
 * records flag 4 in dev_err (a device int the caller zeroes) and returns, so
 * the context stays usable. The call synchronises `stream` and returns the
 * status the step's calls map that word to: GPT2_ERR_TIMEOUT when the wait
 * ran out, GPT2_OK if it did not, GPT2_ERR_ARG for a limit out of range. */
int gpt2op_wait_selftest(int64_t limit_ns, int* dev_err, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* GPT2STEP_OPS_H */
