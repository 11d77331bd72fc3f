/*
 * gpt2.h -- C ABI of libgpt2.so: one GPT-2 pretraining step on one B200.
 *
 * The step is the one the GPT-2 pages describe: "Criei GPT-2 do zero com uma
 * RTX 4090" (section "Configuração do treinamento": GPT-2 small, micro-batch
 * 16x1024, 32x gradient accumulation, vocabulary padded 50257 -> 50304) and
 * "Pré-treinar um LLM: dados, compute, leis de escala e custo" (opening
 * section: next-token cross-entropy optimised by AdamW; compute section:
 * forward 2N, backward two matmul-sized gradients per layer; memory section:
 * fp32 weight, gradient, m and v).  Model: pre-LayerNorm decoder blocks with
 * learned positions, causal multi-head attention, GELU(tanh) MLP, LM head
 * tied to the token embedding; mean cross-entropy over the B*T positions
 * (those with a target, when some are masked); decoupled-weight-decay AdamW
 * with fp32 master weights.  Around the step: gradient-norm clipping, AdamW
 * over one shard of the flat buffers (data parallelism with sharded optimizer
 * state), and incremental decoding with a key/value cache (prefill, decode
 * step, greedy choice) on the same model.
 *
 * Conventions for every function below
 * - Ownership: the caller allocates and owns every device buffer (the
 *   parameters, gradients, AdamW moments and one workspace).  The library
 *   allocates only its small host-side context in gpt2_create.
 * - Pointers: device pointers unless a parameter says "host".  Buffers must be
 *   16-byte aligned.  Token / target ids are int32, row-major [batch, n_ctx].
 * - Streams: `stream` is a cudaStream_t (NULL = legacy default stream).  Every
 *   call except gpt2_get_status, gpt2_step_host and gpt2_create/destroy is
 *   asynchronous on that stream and returns after enqueueing its kernels.
 * - Errors: 0 on success, a negative GPT2_ERR_* code otherwise.  Argument and
 *   shape errors are detected on the host before anything is enqueued.
 *   Conditions only the device can see (an id outside [0, vocab_real), a
 *   non-finite loss, a bounded device wait that ran out) are latched in a
 *   device word and returned by the next gpt2_get_status.  No kernel traps or
 *   asserts.
 * - Precision: mode 0 computes in bf16 on tensor cores with fp32 accumulation
 *   (activations bf16; master weights, gradients and AdamW state fp32); mode 1
 *   is a correctness mode that computes everything in fp32 on CUDA cores;
 *   mode 2 is mode 0 made bitwise repeatable: the one reduction of mode 0
 *   whose order varies from run to run (the attention backward's fp32 dQ sum
 *   over key blocks) is done in key-block order from per-block partial tiles
 *   (head_dim 64, n_ctx <= 4096; ceil(n_ctx/128) * max_batch * n_ctx * d more
 *   fp32 of workspace; every other reduction of the step is already in a
 *   fixed order).
 *
 * Flat parameter layout (fp32 master, fp32 grad, m, v and the bf16 shadow all
 * share it; offsets in elements):
 *   wte[V,d], wpe[n_ctx,d], then for each layer
 *   ln1_g[d], ln1_b[d], w_qkv[3d,d], b_qkv[3d], w_o[d,d], b_o[d],
 *   ln2_g[d], ln2_b[d], w_fc[4d,d], b_fc[4d], w_mp[d,4d], b_mp[d],
 *   and finally lnf_g[d], lnf_b[d].
 * Weights are [out, in] row-major (y = x W^T + b).  q, k, v are consecutive
 * d-column blocks of the QKV output; head h owns columns [h*hd, (h+1)*hd) of
 * each block, hd = d / n_head.
 */
#ifndef GPT2_B200_H
#define GPT2_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gpt2_ctx gpt2_ctx;

enum {
  GPT2_OK = 0,
  GPT2_ERR_INVALID_ARG = -1,      /* NULL pointer, bad value, misaligned buffer */
  GPT2_ERR_UNSUPPORTED_SHAPE = -2,/* d % 64, vocab_padded % 128, hd not in {16, 64}, ... */
  GPT2_ERR_CUDA = -3,             /* a CUDA runtime/driver call failed */
  GPT2_ERR_BAD_STATE = -4,        /* e.g. gpt2_backward without a preceding forward */
  GPT2_ERR_TOKEN_RANGE = -5,      /* device: an id outside [0, vocab_real) (clamped to 0) */
  GPT2_ERR_NONFINITE = -6,        /* device: loss is NaN or Inf */
  GPT2_ERR_TIMEOUT = -7,          /* device: a bounded pipeline wait ran out */
  GPT2_ERR_WORKSPACE = -8,        /* workspace smaller than gpt2_workspace_bytes */
  GPT2_ERR_TOO_LARGE = -9,        /* problem exceeds the built-in scratch of an allocation-free entry point */
  GPT2_ERR_POSITION_RANGE = -10   /* device: a decode position or prompt length out of range (row 0 / skipped) */
};

typedef struct {
  int n_layer;      /* L */
  int d_model;      /* d, a multiple of 64 */
  int n_head;       /* H; head_dim = d / H must be 16 or 64 */
  int n_ctx;        /* T: sequence length of every batch row; wpe has n_ctx rows */
  int vocab_real;   /* ids must lie in [0, vocab_real) (50257 for GPT-2) */
  int vocab_padded; /* V >= vocab_real, a multiple of 128 (50304); the softmax spans all V */
  int max_batch;    /* largest batch any call will pass */
  int mode;         /* 0 = bf16 tensor-core compute, 1 = fp32 correctness mode, 2 = mode 0, bitwise repeatable */
} gpt2_config;

typedef struct {
  float* master;          /* fp32 [param_count] */
  uint16_t* shadow;       /* bf16 copy of master [param_count]; may be NULL in mode 1 */
  float* grad;            /* fp32 [param_count] */
  float* m;               /* fp32 [param_count], AdamW first moment */
  float* v;               /* fp32 [param_count], AdamW second moment */
  void* workspace;        /* device scratch of workspace_bytes bytes */
  size_t workspace_bytes; /* >= gpt2_workspace_bytes(cfg, cfg->max_batch) */
} gpt2_buffers;

/* Number of parameters (elements) in the flat layout; 0 for an invalid cfg. */
size_t gpt2_param_count(const gpt2_config* cfg);

/* Bytes of workspace needed for micro-batches up to `batch` rows: saved
 * activations of every layer, the bf16 (mode 0) logits/dlogits buffer
 * [batch*n_ctx, V] and backward scratch.  0 for an invalid cfg. */
size_t gpt2_workspace_bytes(const gpt2_config* cfg, int batch);

/* Describe tensor `index` (0-based, in layout order) of the flat layout:
 * its name ("wte", "wpe", "h<l>.<name>", "lnf_g", "lnf_b"), element offset,
 * rows and cols (cols = 1 for vectors).  *name points to static storage
 * valid until the next call.  GPT2_ERR_INVALID_ARG past the last tensor. */
int gpt2_tensor_info(const gpt2_config* cfg, int index, const char** name,
                     size_t* offset, size_t* rows, size_t* cols);

/* Validate cfg and buffers and create a context bound to them.  Zeroes the
 * internal scatter accumulator inside the workspace (synchronously).  The
 * buffers must outlive the context. */
int gpt2_create(const gpt2_config* cfg, const gpt2_buffers* bufs, gpt2_ctx** out);
int gpt2_destroy(gpt2_ctx* ctx);

/* GPT-2 initialisation: every 2-D weight (wte, wpe, w_qkv, w_fc) ~ N(0, 0.02^2)
 * except the two projections into the residual stream (w_o, w_mp) ~
 * N(0, (0.02/sqrt(2L))^2); biases and LayerNorm shifts 0, LayerNorm gains 1.
 * Normal draws: Box-Muller on Philox4x32-10 (Salmon et al., SC'11) keyed by
 * `seed`, counter = element index.  Also zeroes grad, m, v and refreshes
 * the bf16 shadow. */
int gpt2_init_params(gpt2_ctx* ctx, uint64_t seed, void* stream);

/* Re-derive the bf16 shadow from the fp32 master (after the caller wrote the
 * master directly, e.g. when restoring a checkpoint). */
int gpt2_refresh_shadow(gpt2_ctx* ctx, void* stream);

/* Forward pass and loss.  tokens, targets: device int32 [batch, n_ctx]
 * (targets[b,t] is the id at t+1 of the stream, or -1 for a position that
 * takes no part in the loss: the masked loss of instruction tuning, "Criei
 * GPT-2 do zero com uma RTX 4090", section "Usei SFT para fazê-lo
 * conversar").  Writes the mean cross-entropy over the positions with a
 * target (batch*n_ctx of them without -1s) to *loss_dev (device fp32) and
 * keeps the activations (and the dlogits of this batch) in the workspace for
 * gpt2_backward.  The ids are copied into the workspace, so the caller's
 * arrays may be reused as soon as this call's work has run. */
int gpt2_forward_loss(gpt2_ctx* ctx, const int32_t* tokens, const int32_t* targets,
                      int batch, float* loss_dev, void* stream);

/* Backward pass of the last forward: grad = (accumulate ? grad : 0)
 * + grad_scale * d(loss)/d(params).  With k-step gradient accumulation pass
 * grad_scale = 1/k and accumulate = 0 on the first micro-batch, 1 after.
 * GPT2_ERR_BAD_STATE if no forward preceded it. */
int gpt2_backward(gpt2_ctx* ctx, float grad_scale, int accumulate, void* stream);

/* gpt2_backward that finishes the gradients in buckets, for a data-parallel
 * exchange overlapped with the backward ("Pré-treinar um LLM", parallelism
 * paragraph: the gradients are averaged over the data-parallel copies).
 * events: n_events = n_layer + 2 CUDA events (cudaEvent_t) owned by the
 * caller; each is recorded on `stream` as soon as its bucket's gradients are
 * final: events[l] for decoder block l (its weights, biases and LayerNorm
 * parameters, one contiguous range of the flat layout), events[n_layer] for
 * the final LayerNorm, events[n_layer + 1] for wte and wpe (recorded last:
 * the tied wte gradient takes the embedding scatter at the end).  The order
 * of recording is n_layer, n_layer - 1, ..., 0, n_layer + 1.  The gradients
 * equal gpt2_backward's.  GPT2_ERR_INVALID_ARG for a wrong event count or a
 * NULL event. */
int gpt2_backward_bucketed(gpt2_ctx* ctx, float grad_scale, int accumulate, void* const* events, int n_events,
                           void* stream);

/* One AdamW step over the whole flat buffer (decoupled weight decay on the
 * 2-D tensors only; bias-corrected with step counter `step` >= 1):
 *   p <- p (1 - lr wd);  m <- b1 m + (1-b1) g;  v <- b2 v + (1-b2) g^2
 *   p <- p - lr (m / (1-b1^step)) / (sqrt(v / (1-b2^step)) + eps)
 * and refreshes the bf16 shadow. */
int gpt2_adamw_step(gpt2_ctx* ctx, float lr, float beta1, float beta2, float eps,
                    float weight_decay, int step, void* stream);

/* Global L2 norm of the flat gradient buffer, sqrt(sum g^2), into the device
 * fp32 scalar *norm_dev (4-byte aligned; NULL keeps it in the workspace).
 * Two fixed-order reduction passes over a fixed grid, so the value is
 * bitwise repeatable.  The pages do not clip gradients; this and
 * gpt2_adamw_step_clip serve a training loop that does. */
int gpt2_grad_norm(gpt2_ctx* ctx, float* norm_dev, void* stream);

/* gpt2_adamw_step with global-norm gradient clipping first: every gradient is
 * scaled by min(1, max_norm / (||g|| + 1e-6)), ||g|| computed on the device as
 * in gpt2_grad_norm (no host synchronisation).  max_norm = 0 is exactly
 * gpt2_adamw_step; a negative or NaN max_norm is GPT2_ERR_INVALID_ARG.  The
 * gradient buffer itself is left unscaled. */
int gpt2_adamw_step_clip(gpt2_ctx* ctx, float lr, float beta1, float beta2, float eps,
                         float weight_decay, int step, float max_norm, void* stream);

/* gpt2_adamw_step restricted to elements [offset, offset + count) of the flat
 * buffers (master, m, v, the bf16 shadow; grad read there); offset and count
 * are multiples of 4 and the range lies inside the layout, else
 * GPT2_ERR_INVALID_ARG.  Each element gets exactly the update the full call
 * gives it (the weight-decay mask follows the element's tensor).  This is the
 * optimizer step of a rank that owns one shard of the optimizer state
 * (data parallelism with sharded AdamW state: reduce-scatter the gradient,
 * update the own shard, all-gather the weights). */
int gpt2_adamw_step_range(gpt2_ctx* ctx, float lr, float beta1, float beta2, float eps,
                          float weight_decay, int step, size_t offset, size_t count, void* stream);

/* grad <- 0. */
int gpt2_zero_grad(gpt2_ctx* ctx, void* stream);

/* Synchronises `stream`, returns and clears the latched device status
 * (GPT2_OK, GPT2_ERR_TOKEN_RANGE, GPT2_ERR_NONFINITE, GPT2_ERR_TIMEOUT or
 * GPT2_ERR_POSITION_RANGE),
 * or GPT2_ERR_CUDA if the stream reports an error. */
int gpt2_get_status(gpt2_ctx* ctx, void* stream);

/* One whole training step from HOST memory: copies tokens/targets (host,
 * int32 [batch, n_ctx], preferably pinned) to the device, runs forward,
 * backward (grad_scale 1, accumulate 0) and AdamW, copies the loss back into
 * *loss_host and synchronises the stream before returning.  When the context
 * holds a captured micro-step (gpt2_graph_capture) for the same batch with
 * grad_scale 1 and accumulate 0, the ids are copied straight into the
 * graph's inputs and the graph runs instead of the separate launches (same
 * kernels, same results; the loss is read from where the graph writes it). */
int gpt2_step_host(gpt2_ctx* ctx, const int32_t* tokens_host, const int32_t* targets_host,
                   int batch, float* loss_host, float lr, float beta1, float beta2,
                   float eps, float weight_decay, int step, void* stream);

/* Static text for an error code. */
const char* gpt2_strerror(int code);

/* Number of CUDA kernels this library has launched in this process so far
 * (all contexts and entry points); a diagnostic for launch accounting. */
uint64_t gpt2_kernel_launches(void);

/* ------------------------------------------------------------------------
 * Incremental decoding with a key/value cache: the inference forward of the
 * sampling loop ("Criei GPT-2 do zero com uma RTX 4090", sections "Vendo o
 * modelo ficar mais inteligente aos poucos" and "Conversando de verdade com
 * ele": the model continues a prompt one token at a time).  The logits a
 * decode step returns for a row whose token sits at position p are the
 * forward's logits at position p for that row's tokens 0..p; the cache holds
 * every layer's K and V of positions 0..p-1 so that only the new position is
 * computed.  Weights are the ones the forward uses (bf16 shadow in mode 0,
 * fp32 master in mode 1); the cache holds K and V in that dtype, and the
 * residual stream of a step stays fp32.
 *
 * A cache is sized for (batch, max_len): 1 <= batch <= 16, 1 <= max_len <=
 * n_ctx.  Every call on it passes the same batch and max_len, and the
 * buffer's size in bytes (cache_bytes): a call whose (batch, max_len) needs
 * more than cache_bytes is GPT2_ERR_INVALID_ARG before anything is enqueued.
 * It is one caller-owned device buffer of at least gpt2_kv_cache_bytes bytes,
 * 256-byte aligned;
 * layout: per layer l the K plane then the V plane, each [batch][n_head]
 * [max_len][head_dim] (padded to 256 bytes), then the step's fp32 scratch.
 * Positions are per row (device int32 [batch]), so rows may sit at different
 * positions.  A position outside [0, max_len), a prompt length outside
 * [1, max_len] or an id outside [0, vocab_real) latches
 * GPT2_ERR_POSITION_RANGE / GPT2_ERR_TOKEN_RANGE for gpt2_get_status (the
 * row then reads id 0 / position 0 and its cache write is skipped).
 * ---------------------------------------------------------------------- */

/* Bytes of a cache for (batch, max_len); 0 if the configuration or the
 * sizes are invalid. */
size_t gpt2_kv_cache_bytes(const gpt2_config* cfg, int batch, int max_len);

/* Prompt processing: runs the training forward over tokens (device int32
 * [batch, n_ctx]; batch <= max_batch; ids past a row's prompt are any valid
 * id, causality keeps them out of the prompt's results), copies K and V of
 * positions < prompt_len[b] (device int32 [batch]) into the cache, and writes
 * the logits after each row's last prompt token to logits (device fp32
 * [batch, vocab_padded]).  Overwrites the forward's activations (a following
 * gpt2_backward returns GPT2_ERR_BAD_STATE). */
int gpt2_prefill(gpt2_ctx* ctx, void* cache, size_t cache_bytes, int batch, int max_len,
                 const int32_t* tokens, const int32_t* prompt_len, float* logits, void* stream);

/* One decode step: row b feeds tokens[b] (device int32 [batch]) at position
 * pos[b] (device int32 [batch]), writes its K and V into the cache at pos[b],
 * attends to positions 0..pos[b] and writes the next-token logits to logits
 * (device fp32 [batch, vocab_padded]).  tokens and pos are read on the device,
 * so a loop of steps can be captured in one CUDA graph. */
int gpt2_decode_step(gpt2_ctx* ctx, void* cache, size_t cache_bytes, int batch, int max_len,
                     const int32_t* tokens, const int32_t* pos, float* logits, void* stream);

/* Greedy choice: next_tokens[b] = the id v < vocab_real with the largest
 * logits[b, v] (device fp32 [batch, vocab_padded]); the lowest id among equal
 * maxima, the first NaN if a row holds one.  If pos (device int32 [batch]) is
 * not NULL, pos[b] += 1, so next_tokens and pos feed the next decode step.
 * The pages give no sampling rule; greedy is the plainest. */
int gpt2_greedy_next(gpt2_ctx* ctx, const float* logits, int batch, int32_t* next_tokens, int32_t* pos,
                     void* stream);

/* ------------------------------------------------------------------------
 * Single-operation entry points used by the kernel unit tests.  They run the
 * same kernels the step runs, on caller buffers.
 * ---------------------------------------------------------------------- */

/* C[M,N] = alpha * sum_k A(m,k) B(n,k)  (+ beta * C when C is fp32).
 * The linear layers' forward, input-gradient and weight-gradient products of
 * the compute section are all of this form with different operand majorness.
 * A: bf16; a_mn_major = 0 -> stored [M, lda] (k contiguous),
 *                         1 -> stored [K, lda] (m contiguous).
 * B: bf16; b_mn_major = 0 -> stored [N, ldb], 1 -> stored [K, ldb].
 * C: c_fp32 = 0 -> bf16 [M, ldc] (beta ignored); 1 -> fp32 [M, ldc].
 * K must be a multiple of 64; lda, ldb, ldc multiples of 8.
 * workspace (device, may be NULL) holds split-K partial sums for fp32 C;
 * bn (0 = auto, 128 or 256) and splits (0 = auto) override the tiling. */
int gpt2_op_gemm_bf16(const uint16_t* A, int a_mn_major, int lda,
                      const uint16_t* B, int b_mn_major, int ldb,
                      void* C, int c_fp32, int ldc, int M, int N, int K,
                      float alpha, float beta, void* workspace, size_t workspace_bytes,
                      int bn, int splits, void* stream);

/* Causal attention forward on a packed QKV activation: qkv bf16 [B*T, 3*H*hd]
 * -> o bf16 [B*T, H*hd], lse fp32 [B, H, T] (natural-log log-sum-exp of the
 * scaled scores).  hd in {16, 64}. */
int gpt2_op_attention_fwd_bf16(const uint16_t* qkv, uint16_t* o, float* lse,
                               int B, int T, int H, int hd, void* stream);

/* Its backward: given do (bf16 [B*T, H*hd]) writes dqkv (bf16 [B*T, 3*H*hd]).
 * scratch: device fp32, at least B*T*H*hd + B*H*T floats. */
int gpt2_op_attention_bwd_bf16(const uint16_t* qkv, const uint16_t* o, const float* lse,
                               const uint16_t* dout, uint16_t* dqkv, float* scratch,
                               int B, int T, int H, int hd, void* stream);

/* Hang detection.  Every pipeline wait inside the tcgen05 GEMM and attention
 * kernels (a TMA copy, an MMA, a hand-off between warps) gives up after a
 * limit, records GPT2_ERR_TIMEOUT in the device status word (what
 * gpt2_get_status reads, or the status argument of gpt2_op_gemm_bf16_status),
 * lets the copies and MMAs already in flight finish, frees its tensor memory
 * and returns, so the context stays usable.  This sets the limit in
 * nanoseconds on the current device (0 restores the default of 2 s).  This
 * is the library's failure detection: a hung pipeline becomes an error the
 * host reads instead of a hung GPU.  Not stream-ordered: call it with no
 * kernel of the library in flight. */
int gpt2_set_wait_timeout_ns(uint64_t ns);

/* gpt2_op_gemm_bf16 with a device status word: status (device int, 4-byte
 * aligned) is OR-ed with GPT2's device error bits (4 = a pipeline wait timed
 * out). */
int gpt2_op_gemm_bf16_status(const uint16_t* A, int a_mn_major, int lda, const uint16_t* B, int b_mn_major, int ldb,
                             void* C, int c_fp32, int ldc, int M, int N, int K, float alpha, float beta,
                             void* workspace, size_t workspace_bytes, int bn, int splits, int* status,
                             void* stream);

/* Allocation-free variant of gpt2_op_attention_bwd_bf16 (same inputs, same
 * output dqkv, no scratch argument).  The paper has no counterpart: this entry
 * point exists for callers that cannot call cudaMalloc -- a host that gives a
 * plug-in only its input and output buffers, a runtime whose caching
 * allocator already holds the device memory, or a loop that cannot afford
 * cudaMalloc's device synchronisation.  Its scratch (fp32 dQ accumulator and
 * D vector, B*T*H*hd + B*H*T floats) lives in a 16 MiB array compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.  hd < 1 returns GPT2_ERR_INVALID_ARG and an hd other than 16 or 64
 * GPT2_ERR_UNSUPPORTED_SHAPE, as for the scratch-taking call; a supported
 * shape whose scratch exceeds the array returns GPT2_ERR_TOO_LARGE.  Every
 * call made outside a stream capture looks up the array's address in the
 * current context (cudaGetSymbolAddress), so a cudaDeviceReset or another
 * context being current is picked up; inside a capture the address recorded
 * by the last uncaptured call on that device is used, and a capture with no
 * such earlier call returns GPT2_ERR_BAD_STATE.  Make the first call on a
 * device before any stream capture, and call it again (uncaptured) after a
 * cudaDeviceReset before capturing.  All calls share the one array: calls
 * that may overlap on the GPU (unordered streams) race and must not be
 * issued.  It calls no allocator. */
int gpt2_op_attention_bwd_bf16_noalloc(const uint16_t* qkv, const uint16_t* o, const float* lse,
                                       const uint16_t* dout, uint16_t* dqkv,
                                       int B, int T, int H, int hd, void* stream);

/* ---- single HBM-bound steps of the path, for kernel tests and profiling --
 * bf16 activations, row-major, 16-byte aligned; d a multiple of 64 up to
 * 2048 (GPT2_ERR_UNSUPPORTED_SHAPE otherwise).  Asynchronous on `stream`. */

/* LayerNorm forward over M rows of width d ("Pré-treinar um LLM" and the
 * pre-LayerNorm block of GPT-2): per row mean and biased variance, eps 1e-5,
 * y = (x - mean) * rstd * gamma + beta.  x, y bf16 [M, d]; gamma, beta bf16
 * [d]; mean, rstd fp32 [M] (saved for the backward). */
int gpt2_op_layernorm_fwd_bf16(const uint16_t* x, const uint16_t* gamma, const uint16_t* beta, uint16_t* y,
                               float* mean, float* rstd, int M, int d, void* stream);

/* Floats of scratch gpt2_op_layernorm_bwd_bf16 needs (0 for M or d < 1). */
size_t gpt2_op_layernorm_bwd_scratch_floats(int M, int d);

/* Its backward (the chain rule of the forward above): dx (=, or += with
 * accumulate) the input gradient, bf16 [M, d]; dgamma_dbeta fp32 [2d] =
 * (sum over rows of dy * xhat, sum over rows of dy), written.  mean, rstd as
 * the forward saved them.  scratch: device fp32 of at least
 * gpt2_op_layernorm_bwd_scratch_floats(M, d) (GPT2_ERR_WORKSPACE if smaller);
 * the row-block partial sums, added in a fixed order. */
int gpt2_op_layernorm_bwd_bf16(const uint16_t* dy, const uint16_t* x, const float* mean, const float* rstd,
                               const uint16_t* gamma, uint16_t* dx, int accumulate, float* dgamma_dbeta,
                               float* scratch, size_t scratch_floats, int M, int d, void* stream);

/* Floats of scratch gpt2_op_colsum_bf16 needs (0 for M or N < 1). */
size_t gpt2_op_colsum_scratch_floats(int M, int N);

/* Column sums of x (bf16 [M, N], N a multiple of 8): out[n] = sum_m x[m, n]
 * (fp32 [N], written), the bias gradient of a linear layer ("Pré-treinar um
 * LLM", compute section: the backward's gradients of each layer).  Row-block
 * partials in scratch (at least gpt2_op_colsum_scratch_floats(M, N) floats),
 * added in a fixed order. */
int gpt2_op_colsum_bf16(const uint16_t* x, int M, int N, float* out, float* scratch, size_t scratch_floats,
                        void* stream);

/* ---- the tied LM head with its fused softmax cross-entropy, alone --------
 * "Pré-treinar um LLM", memory section: the logits are one vocabulary-sized
 * vector per token; here they never reach HBM in fp32.  The forward GEMM
 * z = x w^T computes, in its epilogue, each row's maximum and sum of exp(z -
 * max) per 128-column part of the vocabulary, stores those exponentials
 * (bf16, [M, V]) in the scratch, and keeps the target logits; a merge kernel
 * forms each row's log-sum-exp, loss_rows[m] = LSE - z[m, target] (0 for
 * target -1) and *loss = their mean over the rows with a target, and
 * rewrites the stored exponentials in place as dz = softmax(z) -
 * onehot(target) (bf16).  The backward's two GEMMs read that dz:
 * dx = (grad_scale / n_valid) dz w (bf16 [M, d], written) and
 * dw (=, or += with accumulate) (grad_scale / n_valid) dz^T x (fp32 [V, d]).
 * x bf16 [M, d], w bf16 [V, d] (256-byte aligned), targets int32 [M] in
 * [0, vocab_real) or -1; V a multiple of 128, d of 64.  The backward reads
 * the scratch the forward wrote (same M, V, targets unchanged).  Device
 * status: the int at scratch offset 0 (bit 1 = a target id out of range,
 * counted as masked; bit 2 = non-finite loss), cleared by each forward. */
size_t gpt2_op_lm_head_ce_scratch_bytes(int M, int V);
int gpt2_op_lm_head_ce_fwd_bf16(const uint16_t* x, const uint16_t* w, const int32_t* targets, int M, int V, int d,
                                int vocab_real, float* loss, float* loss_rows, void* scratch, size_t scratch_bytes,
                                void* stream);
int gpt2_op_lm_head_ce_bwd_bf16(const uint16_t* x, const uint16_t* w, int M, int V, int d, float grad_scale,
                                uint16_t* dx, float* dw, int accumulate, void* scratch, size_t scratch_bytes,
                                void* stream);

/* ------------------------------------------------------------------------
 * The micro-step as a CUDA graph.  A step launches about 300 kernels; issued
 * one by one, the gaps between them cost about 3 % of the step.
 * gpt2_graph_capture records the forward, the loss and the backward of one
 * micro-batch of `batch` rows (grad_scale and accumulate as in gpt2_backward,
 * fixed by the capture; the loss written to loss_dev, a device float, or to
 * the context's own loss word when NULL) into a graph the context owns,
 * replacing an earlier one.  It computes nothing: the kernels are recorded on
 * `stream`, which must be a stream the caller created (not the legacy default
 * stream), and every kernel must have been run once on the device before (one
 * eager step), since their one-time set-up cannot happen inside a capture.
 * gpt2_graph_step copies the step's token and target ids (device int32
 * [batch, n_ctx]) into the graph's own input buffers and launches the graph on
 * `stream`: the same kernels and the same results as gpt2_forward_loss and
 * gpt2_backward with those arguments.  gpt2_adamw_step (or its variants)
 * follows as usual.  The graph's kernels count in gpt2_kernel_launches at each
 * launch.  Errors: INVALID_ARG for a NULL context or stream, or a batch outside
 * [1, max_batch]; BAD_STATE for gpt2_graph_step without a graph; CUDA if the
 * capture fails (no graph is kept).  gpt2_graph_release frees the graph
 * (gpt2_destroy does too). */
int gpt2_graph_capture(gpt2_ctx* ctx, int batch, float grad_scale, int accumulate, float* loss_dev, void* stream);
int gpt2_graph_step(gpt2_ctx* ctx, const int32_t* tokens, const int32_t* targets, void* stream);
int gpt2_graph_release(gpt2_ctx* ctx);

/* One linear layer of a decoder block with the epilogue the step fuses into
 * its GEMM ("Criei GPT-2 do zero", model section: the QKV and attention
 * output projections, the GELU(tanh) MLP and the residual stream;
 * "Pré-treinar um LLM", compute section: one matmul of the forward):
 *   act 0: out = x w^T + bias                       (QKV projection)
 *   act 1: out = x w^T + bias + resid                (attention output / MLP proj)
 *   act 2: u = x w^T + bias; out = GELU(u), out2 = GELU'(u)   (MLP fc; GELU'
 *          is what the backward multiplies the incoming gradient by)
 * GELU(u) = u/2 (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))).  Accumulation in
 * fp32, every output rounded once to bf16.
 * x bf16 [M, K] row-major, w bf16 [N, K] row-major (the layer's weight as
 * stored), bias bf16 [N], resid / out / out2 bf16 [M, N] row-major; all
 * 16-byte aligned.  resid is read only for act 1 and out2 written only for
 * act 2 (both may be NULL otherwise).  K a multiple of 64, N of 8.  Errors:
 * INVALID_ARG for NULL or misaligned buffers, a negative size or an act
 * outside 0..2; UNSUPPORTED_SHAPE for K or N off those multiples. */
int gpt2_op_linear_bf16(const uint16_t* x, const uint16_t* w, const uint16_t* bias, const uint16_t* resid,
                        uint16_t* out, uint16_t* out2, int M, int N, int K, int act, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPT2_B200_H */
