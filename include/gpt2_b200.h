/*
 * gpt2_b200.h -- C ABI of a B200-native (sm_100a) GPT-2 training step.
 *
 * The step is the one on the pages "Karpathy's Zero to Hero, Lecture 9: Reproduce GPT-2
 * (124M) -- notes, code and timestamps" (cited below as L9, by section) and the
 * "reproduce-gpt2" README (RG2): the forward and backward pass of a pre-LayerNorm
 * decoder-only Transformer with a tied wte / lm_head, the cross-entropy loss, gradient
 * accumulation over micro-steps, the global-norm gradient clip and the AdamW update.
 *
 * Conventions of every call:
 *   - Return value: GPT2_OK (0) or one of the negative GPT2_ERR_* codes.  No C++
 *     exception crosses this boundary.  gpt2_last_error() gives a one-line message.
 *   - Work is enqueued on the context's CUDA stream (gpt2_set_stream) and is
 *     asynchronous unless a call says it synchronises.
 *   - Device-side checks (token ids, target ids, bounded waits inside kernels) never
 *     trap: they record a code that the next synchronising call reports as
 *     GPT2_ERR_TOKEN / GPT2_ERR_TARGET / GPT2_ERR_TIMEOUT.
 *   - The library owns all parameters, gradients, optimizer state and activations.
 *     Buffers passed in are owned by the caller.
 */
#ifndef GPT2_B200_H
#define GPT2_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPT2_OK 0
#define GPT2_ERR_ARG (-1)      /* null pointer or invalid value */
#define GPT2_ERR_OOM (-2)      /* device allocation failed */
#define GPT2_ERR_CUDA (-3)     /* a CUDA runtime call failed */
#define GPT2_ERR_SHAPE (-4)    /* B > max_batch, T > block_size, unsupported size */
#define GPT2_ERR_TOKEN (-5)    /* an input id outside [0, vocab_size) */
#define GPT2_ERR_TARGET (-6)   /* a target outside [0, vocab_size) and not -1 */
#define GPT2_ERR_TIMEOUT (-7)  /* a bounded device wait gave up */
#define GPT2_ERR_STATE (-8)    /* call out of order (e.g. backward without forward) */

#define GPT2_FP32 0            /* parity mode: fp32 storage and fp32 (SIMT) arithmetic */
#define GPT2_BF16 1            /* bf16 GEMM / attention operands, fp32 accumulation, fp32
                                  residual stream, LN statistics, softmax, loss, grads,
                                  AdamW state and master weights (L9 "1:36:50 – 1:48:25";
                                  RG2 "Training-efficiency optimizations") */

/* Model and run configuration (L9 "28:07 – 41:44": GPTConfig; "2:06:39 – 2:14:58":
 * the vocabulary padded to 50304; "2:34:49 – 2:46:43": gradient accumulation).
 * Constraints: n_embd % n_head == 0, head size in {16, 32, 64}, n_embd a multiple of 32
 * and at most 1024, vocab_size <= padded_vocab_size < 131072, max_batch * block_size
 * <= 131072. */
typedef struct {
  int n_layer;            /* 12 for GPT-2 124M */
  int n_embd;             /* 768 */
  int n_head;             /* 12 */
  int block_size;         /* 1024: the longest T */
  int vocab_size;         /* 50257: ids and targets live in [0, vocab_size) */
  int padded_vocab_size;  /* 50304: rows of wte, columns of the logits */
  int max_batch;          /* largest B a forward call may use */
  int grad_accum_steps;   /* k: backward scales gradients by 1/k */
  int precision;          /* GPT2_FP32 or GPT2_BF16 */
} gpt2_config;

typedef struct gpt2_ctx gpt2_ctx;

/* Allocates all device state on the current device and initialises the parameters
 * (L9 "1:13:27 – 1:22:16"; RG2 "Initialization"): N(0, 0.02) for wte, wpe and Linear
 * weights, 0.02 / sqrt(2 n_layer) for attn.c_proj and mlp.c_proj weights, zero biases,
 * LayerNorm weight 1 and bias 0; wte/lm_head is one tensor drawn once.  The normal draws
 * are counter based: tensor t (0-based, canonical order below) uses state_t = SplitMix64
 * output t of `seed`; its element e is float(std * sqrt(-2 ln u1) cos(2 pi u2)) with
 * u1 = 1 - (r_2e >> 11) 2^-53, u2 = (r_2e+1 >> 11) 2^-53, r_j the j-th SplitMix64 output
 * of state_t.  On failure *out is set to NULL. */
int gpt2_create(const gpt2_config* cfg, uint64_t seed, gpt2_ctx** out);
void gpt2_destroy(gpt2_ctx* ctx);

/* Use `cuda_stream` (a cudaStream_t, e.g. a PyTorch stream) for all later work; NULL
 * selects the library's own stream. */
int gpt2_set_stream(gpt2_ctx* ctx, void* cuda_stream);

/* Launch the forward and backward passes as CUDA graphs (default: on, unless the
 * environment variable GPT2_B200_GRAPHS is "0" when the context is created).  For each
 * (pass, B, T) the first call runs its kernels directly, the second captures them into a
 * graph on the context stream, and later calls replay that graph, which removes the
 * per-kernel launch gaps.  The graph holds the context's buffers and the launch decisions
 * of that shape; results are identical to direct launches.  If a capture fails the context
 * falls back to direct launches.  Calls made while profiling run directly. */
int gpt2_set_graphs(gpt2_ctx* ctx, int enable);

/* Forward pass and mean cross-entropy (L9 "Code you'll write": GPT.forward; "52:38 –
 * 1:06:18": F.cross_entropy on flattened logits).
 * tokens, targets: DEVICE int32 [B, T] row-major, caller-owned, read during the call's
 *   stream work (they are copied inside the library, so they may be reused once the
 *   stream passes this call).  targets may be NULL (no loss); -1 marks an ignored target.
 * The softmax covers all padded_vocab_size columns.  loss = mean over non-ignored rows,
 * NOT divided by grad_accum_steps.  loss_out: HOST float; if non-NULL the call
 * synchronises and also reports device-side errors; if NULL nothing is read back.
 * Errors: GPT2_ERR_SHAPE if B > max_batch, T > block_size or B*T == 0. */
int gpt2_forward(gpt2_ctx* ctx, const int32_t* tokens, const int32_t* targets, int B, int T, float* loss_out);

/* Same as gpt2_forward with HOST token / target buffers: they are copied to the device
 * on the context stream (pinned host memory makes the copy asynchronous). */
int gpt2_forward_host(gpt2_ctx* ctx, const int32_t* tokens, const int32_t* targets, int B, int T,
                      float* loss_out);

/* Backward pass of the last forward (which must have had targets): adds the gradients
 * of loss / grad_accum_steps to the gradient buffers (L9 "2:34:49 – 2:46:43").  The tied
 * wte receives the lm_head and the embedding gradients (L9 "1:06:18 – 1:13:27").
 * Gradients are deterministic: no floating-point atomics.  GPT2_ERR_STATE without a
 * preceding forward with targets. */
int gpt2_backward(gpt2_ctx* ctx);

/* The flat f32 gradient buffer on the device (gpt2_num_params floats in the canonical
 * order below), owned by the context and valid until gpt2_destroy.  A caller may read or
 * rewrite it on the context stream between the last gpt2_backward of a step and
 * gpt2_adamw_step: data-parallel training averages it across ranks there, once per
 * optimizer step (L9 "2:59:25 – 3:10:20 Synchronizing gradients and losses": the
 * all-reduce averages every gradient, and only on the last micro-step).  Fills
 * *device_ptr and *n; GPT2_ERR_ARG for a null argument. */
int gpt2_get_grad_buffer(gpt2_ctx* ctx, float** device_ptr, int64_t* n);

/* Sets every gradient to zero (optimizer.zero_grad(), L9 "52:38 – 1:06:18"). */
int gpt2_zero_grad(gpt2_ctx* ctx);

/* One optimizer step (L9 "Code you'll write": one optimizer step; "2:14:58 – 2:25:57";
 * "2:25:57 – 2:34:49"):  norm = sqrt(sum of all squared gradients, the tied tensor once);
 * s = min(1, clip / (norm + 1e-6)); for every tensor with g = s * grad:
 *   p *= 1 - lr * wd (only tensors with >= 2 dims: wte, wpe and the Linear weights);
 *   m = beta1 m + (1 - beta1) g;  v = beta2 v + (1 - beta2) g^2;
 *   p -= lr * (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps),  t = 1, 2, ...
 * grad_norm_out: HOST float for the pre-clip norm; non-NULL synchronises. */
int gpt2_adamw_step(gpt2_ctx* ctx, float lr, float beta1, float beta2, float eps, float weight_decay, float clip,
                    float* grad_norm_out);

/* Learning rate at step `it` (L9 "Code you'll write": get_lr; "2:14:58 – 2:25:57"):
 * max_lr * (it + 1) / warmup_steps for it < warmup_steps; min_ratio * max_lr for
 * it > max_steps; otherwise min + 0.5 (1 + cos(pi r)) (max - min) with
 * r = (it - warmup_steps) / (max_steps - warmup_steps).  Host function, double math. */
double gpt2_lr_cosine(int64_t it, double max_lr, int64_t warmup_steps, int64_t max_steps, double min_ratio);

/* Next-token sampling ("Karpathy's Zero to Hero, Lecture 9: Reproduce GPT-2 (124M)" notes,
 * "28:07 – 41:44 Loading the weights and generating text": the last position's logits,
 * softmax, the 50 most probable tokens kept and renormalised, one token drawn; "3:22:33 –
 * 3:28:16 Validation loss and sampling during training": the draw has its own seeded
 * generator, so the uniforms are the caller's).  For each i < n, row rows[i] of the last
 * forward's logits (token positions b*T + t, columns [0, vocab_size)): the k largest
 * logits, ties to the lower id, in descending order; their softmax; out[i] = the first of
 * them whose cumulative probability exceeds u[i] (u[i] clamped into [0, 1)).  If out_topk
 * is non-NULL it receives the n x min(k, vocab_size) kept ids in that order.
 * rows (int32 [n]), u (f32 [n]), out, out_topk: DEVICE buffers, caller-owned; the call is
 * asynchronous on the context stream.  A forward without targets is the inference and
 * validation path (validation loss: a forward with targets and no backward).
 * Errors: GPT2_ERR_STATE unless the last call that touched the logits was a forward (a
 * backward overwrites them with their gradient); GPT2_ERR_SHAPE for n <= 0 or k outside
 * [1, GPT2_SAMPLE_MAX_K].  A row outside [0, B*T) of the last forward gives out[i] = -1 and
 * GPT2_ERR_ARG at the next synchronising call. */
#define GPT2_SAMPLE_MAX_K 1024
int gpt2_sample_top_k(gpt2_ctx* ctx, const int32_t* rows, const float* u, int n, int k, int32_t* out,
                      int32_t* out_topk);

/* Number of CUDA kernels this library has launched in this process so far. */
int64_t gpt2_kernel_launches(void);

/* ---- inspection, parity and checkpoint (all synchronous, HOST buffers) ----
 * Flat parameter order ("canonical"): wte [Vp, C], wpe [T, C], then per layer l:
 * ln_1.weight [C], ln_1.bias [C], attn.c_attn.weight [3C, C], attn.c_attn.bias [3C],
 * attn.c_proj.weight [C, C], attn.c_proj.bias [C], ln_2.weight [C], ln_2.bias [C],
 * mlp.c_fc.weight [4C, C], mlp.c_fc.bias [4C], mlp.c_proj.weight [C, 4C],
 * mlp.c_proj.bias [C]; then ln_f.weight [C], ln_f.bias [C].  Weights are [out, in]. */
int64_t gpt2_num_params(const gpt2_ctx* ctx);
int gpt2_get_params(gpt2_ctx* ctx, float* host_dst);
int gpt2_set_params(gpt2_ctx* ctx, const float* host_src);   /* also refreshes bf16 copies */
int gpt2_get_grads(gpt2_ctx* ctx, float* host_dst);
int gpt2_get_optimizer_state(gpt2_ctx* ctx, float* m_dst, float* v_dst, int64_t* t_out);
int gpt2_set_optimizer_state(gpt2_ctx* ctx, const float* m_src, const float* v_src, int64_t t);
/* From the last forward with targets: per-row argmax over all padded columns (ties to
 * the lowest index) [B*T] int32; per-row log-sum-exp [B*T] float. */
int gpt2_get_argmax(gpt2_ctx* ctx, int32_t* host_dst);
int gpt2_get_lse(gpt2_ctx* ctx, float* host_dst);
/* Loss of the last forward with targets (synchronises). */
int gpt2_get_loss(gpt2_ctx* ctx, float* loss_out);
/* Waits for the context stream and reports device-side errors. */
int gpt2_synchronize(gpt2_ctx* ctx);
const char* gpt2_last_error(const gpt2_ctx* ctx);

/* ---- single operations on caller buffers (DEVICE pointers, caller-owned), for tests
 * of one kernel against a reference.  They run on `stream` (a cudaStream_t or NULL) and
 * do not synchronise. ---- */

/* bf16 tensor-core GEMM (tcgen05, TMA-fed):
 *   D[m, n] = sum_k A(m, k) B(n, k),  m < M, n < N, k < K
 *   A(m, k) = A[m*lda + k] if a_mn_major == 0 else A[k*lda + m]   (bf16)
 *   B(n, k) = B[n*ldb + k] if b_mn_major == 0 else B[k*ldb + n]   (bf16)
 * epilogue 0: C(bf16)[m*ldc + n] = alpha D + bias[n];  1: C(f32) = alpha D + bias;
 *          2: C(f32) += alpha D.  bias (f32 [N]) may be NULL.  Pointers 16-byte aligned,
 * lda, ldb, ldc multiples of 8; (a_mn_major, b_mn_major) = (1, 0) is not supported.
 * workspace (f32, ws_floats) may be NULL; with it, epilogue 2 may split K. */
int gpt2op_gemm_bf16(void* stream, int M, int N, int K, const void* A, int64_t lda, int a_mn_major, const void* B,
                     int64_t ldb, int b_mn_major, void* C, int64_t ldc, int epilogue, const float* bias, float alpha,
                     float* workspace, int64_t ws_floats);

/* The fused epilogues of the Transformer block on the same GEMM (D, layouts and alignment as
 * for gpt2op_gemm_bf16).  "Karpathy's Zero to Hero, Lecture 9" notes, "Code you'll write"
 * (the pre-norm Block adds each sublayer's output to the residual stream; the MLP applies
 * the tanh GELU) and "1:48:25 – 2:00:19 torch.compile and the GPU memory hierarchy" (the
 * elementwise work fused with the kernel that produces its input):
 *   epilogue 3 (residual):  C(f32)[m*ldc + n] = aux(f32)[m*ld_aux + n] + alpha D + bias[n]
 *   epilogue 4 (GELU):      u = alpha D + bias[n];  aux_out(bf16)[m*ld_aux_out + n] = gelu_tanh'(u);
 *                           C(bf16)[m*ldc + n] = gelu_tanh(u)
 *   epilogue 5 (GELU grad): C(bf16)[m*ldc + n] = alpha D * aux(bf16)[m*ld_aux + n]
 *                           (aux: the gelu_tanh'(u) epilogue 4 kept, so the backward of the MLP
 *                           multiplies by it instead of evaluating tanh again)
 * bias (f32 [N]) may be NULL for 3 and 4 and is ignored by 5.  aux / aux_out are device
 * buffers the caller owns, 16-byte aligned, with ld_aux / ld_aux_out multiples of 8
 * elements; aux may equal C for epilogue 3 (an in-place residual update).  GELU uses the
 * hardware tanh approximation (results rounded to bf16).  GPT2_ERR_ARG for a null operand,
 * an unknown epilogue or a bias / aux / aux_out that is not 16-byte aligned; GPT2_ERR_CUDA if
 * a launch or tensor-map encode fails. */
int gpt2op_gemm_bf16_fused(void* stream, int M, int N, int K, const void* A, int64_t lda, int a_mn_major,
                           const void* B, int64_t ldb, int b_mn_major, void* C, int64_t ldc, int epilogue,
                           const float* bias, float alpha, const void* aux, int64_t ld_aux, void* aux_out,
                           int64_t ld_aux_out);

/* Causal attention forward over qkv [B*T, 3C] (q | k | v, head h at columns h*hd..):
 * out [B*T, C], lse [B, H, T] float.  precision selects fp32 or bf16 qkv/out. */
int gpt2op_attention_fwd(void* stream, int precision, const void* qkv, void* out, float* lse, int B, int T, int H,
                         int head_dim);
/* Its backward: dqkv [B*T, 3C] from dout [B*T, C]; Dbuf float [B, H, T] is scratch.
 * Both: the bf16 tensor-core path (head_dim 64) needs qkv, out, dout and dqkv 16-byte
 * aligned and returns GPT2_ERR_ARG otherwise; GPT2_ERR_SHAPE for an unsupported head_dim. */
int gpt2op_attention_bwd(void* stream, int precision, const void* qkv, const void* out, const void* dout,
                         const float* lse, float* Dbuf, void* dqkv, int B, int T, int H, int head_dim);

/* The same backward with no scratch argument and no device allocation.  The pages have
 * no counterpart: it is an interface for callers that cannot allocate (a C caller with no
 * allocator of its own, or one whose device memory a caching allocator has reserved
 * up front and that cannot afford the device-wide synchronisation of cudaFree).
 * D = rowsum(dO * O) goes to one fixed f32 array of GPT2OP_NOALLOC_ATTN_MAX_ROWS entries
 * (1 MiB) compiled into the library, one per device.
 *   - Arguments, layouts and results are those of gpt2op_attention_bwd minus Dbuf.
 *   - GPT2_ERR_SHAPE if B, T, H or head_dim <= 0 or B*H*T > GPT2OP_NOALLOC_ATTN_MAX_ROWS;
 *     this check runs before any CUDA call.  GPT2_ERR_ARG for a null pointer or an
 *     unknown precision.
 *   - The first call on each device looks up the array's address (cudaGetSymbolAddress)
 *     and caches it; make that first call before any stream capture begins.
 *   - Nothing needs to start at zero: the call writes every row sum before reading it.
 *   - The array is shared by all callers in the process: calls whose executions overlap
 *     on one device (different streams, concurrent host threads) race on it. */
#define GPT2OP_NOALLOC_ATTN_MAX_ROWS 262144
int gpt2op_attention_bwd_noalloc(void* stream, int precision, const void* qkv, const void* out, const void* dout,
                                 const float* lse, void* dqkv, int B, int T, int H, int head_dim);

/* LayerNorm forward over rows of x (f32 [N, C]): y (bf16 or f32 by precision), mean and
 * rstd (f32 [N]); eps 1e-5, biased variance (nn.LayerNorm defaults). */
int gpt2op_layernorm_fwd(void* stream, int precision, const float* x, const float* w, const float* b, void* y,
                         float* mean, float* rstd, int N, int C);

/* Token and position embedding ("Karpathy's Zero to Hero, Lecture 9: Reproduce GPT-2
 * (124M)" notes, "Code you'll write": the forward pass adds wte[token] and wpe[position]).
 * Forward: x f32 [B*T, C] = wte[tokens[n]] + wpe[n mod T] from f32 tables wte [V, C] and
 * wpe [>= T, C]; tokens int32 [B*T].  An id outside [0, V) embeds as zeros and sets the
 * device error word to GPT2_ERR_TOKEN (read with gpt2op_device_error).
 * Backward: dwte[v] += the sum of the rows of dx0 (f32 [B*T, C]) at positions holding
 * token v, dwpe[t] += sum over b of dx0[b*T + t]; ids are clamped into [0, V).  The sums
 * are deterministic (no atomics; a fixed order that depends only on the ids).  ws is
 * device scratch of gpt2op_embedding_bwd_ws_bytes(B*T, C) bytes, 256-byte aligned; after
 * the call its first B*T uint64 words hold the sort keys token << 32 | position in
 * ascending order.  The f32 tables, x, dx0, dwte, dwpe and ws must be 16-byte aligned.
 * Both: GPT2_ERR_ARG for a null or misaligned pointer; GPT2_ERR_SHAPE unless B, T,
 * C, V > 0, C % 4 == 0, and for the backward B*T <= 131072 and V < 2^20. */
int gpt2op_embedding_fwd(void* stream, const int32_t* tokens, const float* wte, const float* wpe, float* x, int B,
                         int T, int C, int V);
int64_t gpt2op_embedding_bwd_ws_bytes(int N, int C);
int gpt2op_embedding_bwd(void* stream, const int32_t* tokens, const float* dx0, float* dwte, float* dwpe, int B,
                         int T, int C, int V, void* ws);

/* The sampling of gpt2_sample_top_k on caller logits: DEVICE logits [n_rows, ld] (bf16 or
 * f32 by precision), columns [0, V) sampled, ld >= V.  Same rows / u / out / out_topk
 * contract; a row outside [0, n_rows) gives out[i] = -1 and sets the device error word to
 * GPT2_ERR_ARG (read with gpt2op_device_error).  GPT2_ERR_SHAPE for n, n_rows or V <= 0,
 * ld < V or k outside [1, GPT2_SAMPLE_MAX_K]; GPT2_ERR_ARG for a null pointer. */
int gpt2op_sample_top_k(void* stream, int precision, const void* logits, int64_t ld, int n_rows,
                        const int32_t* rows, const float* u, int n, int V, int k, int32_t* out, int32_t* out_topk);

/* Fused classifier head (lm_head + softmax + cross-entropy), forward and backward, on
 * caller buffers: h bf16 [N, C] (the final LayerNorm output), W bf16 [V, C] (the tied
 * weight), targets int32 [N] in [0, V) or -1.  Writes loss (f32 scalar, mean over
 * non-ignored rows), lse f32 [N], argmax int32 [N], dh f32 [N, C] = d loss / d h and
 * dW f32 [V, C] += d loss / d W.  logits_ws is bf16 scratch of N * ldl elements with
 * ldl >= V, ldl % 8 == 0 (the bf16 logits, turned into their gradient in place);
 * aux_ws is f32 scratch of at least gpt2op_classifier_aux_floats(N, V) floats. */
int64_t gpt2op_classifier_aux_floats(int N, int V);
int gpt2op_classifier_fwd_bwd(void* stream, const void* h, const void* W, const int32_t* targets, int N, int V, int C,
                              void* logits_ws, int64_t ldl, float* aux_ws, float* loss, float* lse, int32_t* argmax,
                              float* dh, float* dW);

/* ---- per-kernel-class timing with CUDA events on the context stream ----
 * Between gpt2_profile_start and gpt2_profile_stop every launch the context makes is
 * bracketed by two events; stop synchronises and returns, per class, the summed event
 * time (ms), the launch count, and the algorithmic FLOPs and HBM bytes of those launches
 * (arrays of GPT2_PROF_CLASSES entries, any may be NULL). */
#define GPT2_PROF_CLASSES 12
#define GPT2_PROF_GEMM_FWD 0    /* qkv, attn-proj, fc, mlp-proj forward GEMMs */
#define GPT2_PROF_GEMM_BWD 1    /* their dX and dW GEMMs */
#define GPT2_PROF_HEAD_FWD 2    /* lm_head GEMM with the fused softmax partials */
#define GPT2_PROF_HEAD_BWD 3    /* lm_head dh and dwte GEMMs */
#define GPT2_PROF_ATTN_FWD 4
#define GPT2_PROF_ATTN_BWD 5
#define GPT2_PROF_LN_FWD 6
#define GPT2_PROF_LN_BWD 7
#define GPT2_PROF_CE 8          /* softmax finalisation, loss, logit gradient */
#define GPT2_PROF_BIAS 9        /* LayerNorm and bias gradients summed from partial rows */
#define GPT2_PROF_EMBED 10      /* embedding gather and its backward */
#define GPT2_PROF_OPTIM 11      /* global norm and AdamW */
int gpt2_profile_start(gpt2_ctx* ctx);
int gpt2_profile_stop(gpt2_ctx* ctx, double* ms, int64_t* launches, double* flops, double* bytes);

/* Self-test of the bounded waits inside the pipelined kernels (no counterpart on the pages):
 * one kernel in which a single lane and then a whole warp wait on mbarriers that nothing will
 * ever complete, each for at most limit_ns (1 .. 1e9) nanoseconds.  Both waits must give up,
 * record GPT2_ERR_TIMEOUT in the device error word (read it with gpt2op_device_error), let a
 * 16-byte bulk copy from src16 that is still in flight land, and return; status (DEVICE int
 * [2], caller-owned) receives 0 for each wait that gave up, 1 for one that succeeded.  src16:
 * DEVICE, 16-byte aligned, 16 readable bytes.  Asynchronous on `stream`.  GPT2_ERR_ARG for a
 * null or misaligned pointer or a limit outside the range. */
int gpt2op_bounded_wait_selftest(void* stream, int64_t limit_ns, const void* src16, int* status);

/* Reads and clears the device error word of the current device (GPT2_OK if none). */
int gpt2op_device_error(void);

#ifdef __cplusplus
}
#endif
#endif /* GPT2_B200_H */
