/*
 * ttt.h -- C ABI of libttt: the inner loop of end-to-end test-time training
 * (TTT-E2E) with the E2-TTT closed-form chunk update, on one B200 (sm_100a).
 *
 * Pages (cited by title and section):
 *   [TTT-E2E] "TTT-E2E：端到端测试时训练的长上下文语言建模"
 *   [E2-TTT]  "Rethinking Expressivity and Efficiency in Test-Time Training"
 *   [Review]  "NVIDIA开源TTT-E2E：128K上下文快2.7倍"
 *
 * What one call computes ([TTT-E2E] 内层循环：测试时训练; [E2-TTT] 方法细节,
 * Algorithm 1).  For each sequence, the T hidden rows are cut into chunks of b
 * rows.  For each chunk, in order:
 *   1. forward at the chunk-start fast weights through n_blocks residual
 *      blocks, each  h <- h + S_l(h)  (frozen static MLP, optional) then
 *      h <- h + D_l(h)  (dynamic MLP, fast weights W_l);
 *      GELU:   D(x) = W2 GELU(W1 x);   SwiGLU: D(x) = W3 (SiLU(W1 x) * (W2 x))
 *      ([E2-TTT] 快速权重网络实例化, without the inner LayerNorm; [Review]
 *      dual-MLP paragraph);
 *   2. frozen RMSNorm + LM head, next-token cross-entropy l_t against
 *      tokens[t] ([TTT-E2E] 核心方法);
 *   3. one backward giving the per-token negative gradients G_t of every
 *      dynamic matrix at the chunk-start weights;
 *   4. chunk-end state by Proposition 3.1 ([E2-TTT] 命题3.1):
 *        M_C = btilde_0 M_0 + sum_t eta_t btilde_t G_t
 *        W_C = gtilde_0 W_0 + btilde_0 R_1 M_0 + sum_t eta_t btilde_t R_t G_t
 *      with btilde_t = prod_{i>t} beta_i, gtilde_t = prod_{i>t} gamma_i,
 *      R_t = sum_{i>=t} gtilde_i / btilde_i (evaluated without division).
 * This equals the per-token recursion M_t = beta_t M_{t-1} + eta_t G_t,
 * W_t = gamma_t W_{t-1} + M_t ([E2-TTT] 原始公式) at every chunk end.
 *
 * Conventions shared by every entry point
 *   - Every array argument is a DEVICE pointer on the handle's device,
 *     row-major, float32 unless stated, owned by the caller.  Nothing is
 *     freed or retained by the library after a call returns, except the
 *     frozen-parameter copies a handle owns.
 *   - Enqueued work is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Argument and shape errors are returned
 *     synchronously and launch nothing.  Inside a prefill the aggregation
 *     GEMMs run on a second stream the handle owns, forked from and joined
 *     back into `stream` with events, so the call's work is ordered on
 *     `stream` as a whole.
 *   - Errors found on the device (token out of range, non-finite loss, a
 *     bounded wait that ran out) are recorded in the handle's device status
 *     word and read back with ttt_get_device_status().
 *   - Not thread-safe per handle; different handles are independent.
 *   - Fast-weight packing, per sequence: [n_blocks][m] matrices, each
 *     row-major and contiguous, m = 2 for GELU (W1 [h,d], W2 [d,h]) and 3 for
 *     SwiGLU (W1 gate [h,d], W2 up [h,d], W3 down [d,h]).  The static MLPs use
 *     the same packing without the sequence dimension.
 */
#ifndef TTT_H_
#define TTT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ttt_status {
  TTT_OK = 0,
  TTT_ERR_INVALID_ARG = 1, /* null pointer, bad enum, negative size           */
  TTT_ERR_SHAPE = 2,       /* T % b != 0, b < 1, sizes out of range           */
  TTT_ERR_UNSUPPORTED = 3, /* d, hidden or vocab not a multiple of 16; no GPU  */
  TTT_ERR_WORKSPACE = 4,   /* workspace pointer null or smaller than needed    */
  TTT_ERR_TOKEN_RANGE = 5, /* device: a token outside [0, vocab)               */
  TTT_ERR_NONFINITE = 6,   /* device: a chunk loss is NaN or infinite          */
  TTT_ERR_TIMEOUT = 7,     /* device: a bounded wait ran out of iterations     */
  TTT_ERR_CUDA = 8         /* a CUDA runtime call failed (see ttt_last_error)  */
} ttt_status;

enum { TTT_MLP_GELU = 0, TTT_MLP_SWIGLU = 1 };
enum { TTT_PREC_FP32 = 0, TTT_PREC_BF16 = 1 };
enum { TTT_REDUCE_MEAN = 0, TTT_REDUCE_SUM = 1 };
enum { TTT_RULE_E2TTT = 0, TTT_RULE_LACT = 1 };
enum { TTT_HEAD_LM = 0, TTT_HEAD_RECON = 1 };

/* Model shape.  d, hidden, vocab: multiples of 16, at least 16, and
 * d <= 16384, hidden <= 65536, vocab < 2^26.  n_blocks in [1, 64].
 * precision: TTT_PREC_FP32 = every contraction in float32 on CUDA cores;
 * TTT_PREC_BF16 = contractions on tcgen05 tensor cores with bfloat16
 * operands (round to nearest even) and float32 accumulation, while the
 * state W, M, the residual stream, the softmax and all elementwise work stay
 * float32.  rms_eps: the RMSNorm epsilon (z = g * h / sqrt(mean(h^2)+eps)).
 * loss_reduction: the chunk objective.  TTT_REDUCE_MEAN (default reading):
 * the mean next-token loss over the chunk, as in the first inner-loop sketch
 * of [TTT-E2E] (F.cross_entropy with its default mean); the per-token loss in
 * the recursion is l_t / b, so beta = 0, gamma = 1, eta = alpha is one SGD
 * step on the chunk's mean loss and b = 1 is online SGD.  TTT_REDUCE_SUM:
 * l_t itself (the second sketch's reduction='sum').  The reported chunk loss
 * is the mean either way.
 * update_rule: how a chunk's per-token gradients G_t become the chunk-end
 * state.  TTT_RULE_E2TTT: Proposition 3.1 of [E2-TTT] (命题3.1), the exact
 * chunk end of M_t = beta_t M_{t-1} + eta_t G_t, W_t = gamma_t W_{t-1} + M_t.
 * TTT_RULE_LACT: LaCT's chunk-wise rule as [E2-TTT] states it (高效的逐块
 * 更新机制): G = sum_t eta_t G_t, M_C = (mean_t beta_t) M_0 + G,
 * W_C = W_0 + M_C (gamma unused).
 * head: the self-supervised loss that drives the update.  TTT_HEAD_LM: the
 * frozen RMSNorm + LM head next-token cross-entropy of ttt_prefill.
 * TTT_HEAD_RECON: [E2-TTT]'s own layer, run by ttt_prefill_recon: key/value
 * reconstruction through f_W(x) = x + LN(MLP_W(x)) (快速权重网络实例化; LN
 * without affine parameters, epsilon = rms_eps), loss the mean squared error,
 * outputs f_{W_0}(q_t); requires n_blocks == 1 and has_static == 0, and
 * ignores vocab (lm_head and rms_gain may be NULL at creation). */
typedef struct ttt_config {
  int32_t d;
  int32_t hidden;
  int32_t vocab;
  int32_t n_blocks;
  int32_t mlp;        /* TTT_MLP_GELU or TTT_MLP_SWIGLU */
  int32_t has_static; /* 1: each block has a frozen static MLP before the dynamic one */
  int32_t precision;  /* TTT_PREC_FP32 or TTT_PREC_BF16 */
  int32_t loss_reduction; /* TTT_REDUCE_MEAN or TTT_REDUCE_SUM */
  float rms_eps;
  int32_t update_rule; /* TTT_RULE_E2TTT or TTT_RULE_LACT */
  int32_t head;        /* TTT_HEAD_LM or TTT_HEAD_RECON */
} ttt_config;

typedef struct ttt_handle ttt_handle;

/* Create a handle on the current CUDA device and bind the frozen parameters
 * ([TTT-E2E] 架构设计: frozen final norm and LM head; [Review] dual MLP).
 *   lm_head  [vocab, d]  device float32 (E; logits = z E^T)
 *   rms_gain [d]         device float32 (g)
 *   static_w [n_blocks * m * hidden * d] device float32, packed as above, or
 *            NULL when cfg->has_static == 0 (must be non-NULL otherwise).
 * The handle copies (and for bf16 converts) these; the caller may free them
 * after this call returns.  Synchronous.  *out is set only on TTT_OK. */
ttt_status ttt_create(const ttt_config* cfg, const float* lm_head, const float* rms_gain,
                      const float* static_w, ttt_handle** out);

/* Release the handle and everything it owns (waits for its device work). */
void ttt_destroy(ttt_handle* h);

/* Bytes of device workspace ttt_prefill needs for (batch, T, b).  Host-only. */
ttt_status ttt_workspace_size(const ttt_handle* h, int32_t batch, int32_t T, int32_t b,
                              size_t* bytes);

/* The inner loop over `batch` independent sequences of T tokens, chunk size b
 * ([E2-TTT] Algorithm 1, applied chunk after chunk; [TTT-E2E] 内层循环).
 *   hidden     [batch, T, d]  hidden rows entering the updated blocks
 *   tokens     [batch, T]     int32, tokens[s,t] is the label of hidden row t
 *                             (the caller pre-shifts; every chunk has b terms)
 *   W          [batch * n_blocks * m * hidden * d]  in: W_0, out: final W
 *   M          same shape                            in: M_0, out: final M
 *   eta, beta, gamma [batch, T]  per-token learning rate, momentum, decay
 *                             ([E2-TTT] 原始公式); any finite values accepted
 *   chunk_loss [batch, T/b]   out: mean of the b token losses of each chunk,
 *                             taken at that chunk's start weights
 *   workspace  device scratch of at least ttt_workspace_size() bytes, 256-byte
 *              aligned; its contents are not preserved
 * W and M are updated in place.  hidden, W and M must be 16-byte aligned
 * (TTT_ERR_INVALID_ARG otherwise).  T must be a multiple of b (TTT_ERR_SHAPE
 * otherwise); T == 0 or batch == 0 is a no-op.  hidden, tokens and the
 * scalars must not alias W, M, chunk_loss or the workspace. */
ttt_status ttt_prefill(ttt_handle* h, int32_t batch, int32_t T, int32_t b,
                       const float* hidden, const int32_t* tokens, float* W, float* M,
                       const float* eta, const float* beta, const float* gamma,
                       float* chunk_loss, void* workspace, size_t ws_bytes, void* stream);

/* ttt_prefill on HOST buffers, end to end: the inputs go to the device and the
 * results come back inside the call, which returns once W, M and chunk_loss
 * are in host memory.  Same operation as ttt_prefill ([TTT-E2E] 内层循环:
 * 测试时训练; [E2-TTT] Algorithm 1, Proposition 3.1).
 *   hidden [batch, T, d], tokens [batch, T], eta/beta/gamma [batch, T]:
 *     host arrays, read only.
 *   W0, M0: host arrays (packed as for ttt_prefill), the initial state, read
 *     only; W, M: host arrays receiving the final state (they may be W0 and
 *     M0 themselves).  chunk_loss [batch, T/b]: host, written.
 *   seg_chunks: the sequence is streamed in segments of seg_chunks chunks
 *     (0: about 8 segments); segment s + 1's inputs are copied while segment
 *     s runs, through two device slots.  With attention blocks the whole
 *     sequence is one segment (a chunk reads earlier chunks' keys).  Chunk-end
 *     state is the only carried state, so the result is ttt_prefill's bit for
 *     bit whatever the segment length.
 *   device_buffer: caller-owned device memory of ttt_host_buffer_size() bytes,
 *     256-byte aligned (state, losses, two input slots, the workspace).
 * Copies overlap the compute only from page-locked (pinned) host memory;
 * pageable buffers work but serialise the copies.  Argument errors return
 * without copying or launching; device-side errors go to the status word
 * (ttt_get_device_status).  The call synchronises `stream`. */
ttt_status ttt_host_buffer_size(const ttt_handle* h, int32_t batch, int32_t T, int32_t b, int32_t seg_chunks,
                                size_t* bytes);
ttt_status ttt_prefill_host(ttt_handle* h, int32_t batch, int32_t T, int32_t b, int32_t seg_chunks,
                            const float* hidden, const int32_t* tokens, const float* W0, const float* M0, float* W,
                            float* M, const float* eta, const float* beta, const float* gamma, float* chunk_loss,
                            void* device_buffer, size_t buffer_bytes, void* stream);

/* ttt_prefill without a caller-provided workspace and without allocating:
 * for callers that must not allocate device memory while they run (memory
 * budgeted once at start-up, a host that owns the allocator, or a loop that
 * cannot afford the implicit device synchronisation of cudaMalloc/cudaFree).
 * The pages have no counterpart; this is a deployment variant of ttt_prefill.
 * Same arguments and results as ttt_prefill minus workspace/ws_bytes; the
 * caller still passes every input and output.  Its scratch is a 16 MiB
 * file-scope device array inside the library, held by every GPU that loads
 * the library until the process exits; calls needing more scratch than that
 * (ttt_workspace_size() > 16 MiB) return TTT_ERR_WORKSPACE with the sizes in
 * ttt_last_error().  Launches run directly on `stream` (no CUDA graph).  The
 * first call on a device (and the first after a device reset, which gives the
 * device a new context) looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the one array: calls whose work
 * overlaps on the GPU (other streams, other threads, other handles) race and
 * corrupt each other's results; serialise them.  Nothing in the array needs
 * to start at zero: every buffer is written before it is read in a call, and
 * the call clears its split-K arrival counters itself. */
ttt_status ttt_prefill_noalloc(ttt_handle* h, int32_t batch, int32_t T, int32_t b, const float* hidden,
                               const int32_t* tokens, float* W, float* M, const float* eta, const float* beta,
                               const float* gamma, float* chunk_loss, void* stream);

/* Per-kernel-class record of one profiled prefill. */
typedef struct ttt_kernel_stat {
  char name[24];     /* kernel class, e.g. "agg_update", "mlp_up", "ce_logits_lse" */
  int64_t launches;  /* launches of this class in the call */
  double ms;         /* summed device time, CUDA events around each launch */
  double flops;      /* executed tensor-core FLOPs (2 M N K per GEMM), 0 for row kernels */
  double bytes;      /* algorithmic bytes: each operand, state and output moved once */
} ttt_kernel_stat;

/* The same computation as ttt_prefill (same arguments, same results), run
 * without the CUDA graph and with CUDA events around every launch, for
 * tracing.  Synchronises `stream` before returning.  Fills stats[0..n) with
 * one record per kernel class that ran (at most max_stats). */
ttt_status ttt_prefill_profiled(ttt_handle* h, int32_t batch, int32_t T, int32_t b, const float* hidden,
                                const int32_t* tokens, float* W, float* M, const float* eta, const float* beta,
                                const float* gamma, float* chunk_loss, void* workspace, size_t ws_bytes,
                                void* stream, ttt_kernel_stat* stats, int32_t max_stats, int32_t* n_stats);

/* [E2-TTT]'s own layer over `batch` independent sequences of T tokens, chunk
 * size b, for a handle created with head = TTT_HEAD_RECON (背景知识: TTT建模范式;
 * 快速权重网络实例化; Algorithm 1).  For every chunk, at the chunk-start weights
 * W_0: outputs o_t = f_{W_0}(q_t) and losses L_t = mean_j (f_{W_0}(k_t) - v_t)_j^2
 * with f_W(x) = x + LN(MLP_W(x)); then the chunk update of the handle's rule
 * from the per-token gradients of one backward (loss reduction as for ttt_prefill).
 *   K, V, Q    [batch, T, d]  device float32: keys, values, queries
 *   W, M       [batch * m * hidden * d]  in: W_0, M_0; out: final state (as ttt_prefill)
 *   eta, beta, gamma [batch, T]  per-token scalars
 *   O          [batch, T, d]  out: the outputs o_t
 *   chunk_loss [batch, T/b]   out: mean of the chunk's L_t
 *   workspace  at least ttt_workspace_size() bytes, 256-byte aligned
 * K, V, Q, O, W, M 16-byte aligned; T % b == 0.  A handle with the LM head is
 * TTT_ERR_UNSUPPORTED here (and a reconstruction handle in ttt_prefill). */
ttt_status ttt_prefill_recon(ttt_handle* h, int32_t batch, int32_t T, int32_t b, const float* K, const float* V,
                             const float* Q, float* W, float* M, const float* eta, const float* beta,
                             const float* gamma, float* O, float* chunk_loss, void* workspace, size_t ws_bytes,
                             void* stream);

/* Frozen sliding-window attention in front of every updated block ([TTT-E2E]
 * the sketch's TTTE2EBlock and TTTSelfAttention; 滑动窗口注意力, window k = 8K
 * and chunk b = 1K with k >= b in 关键设计参数).  After this call ttt_prefill
 * runs each block as h <- h + Attn(LN(h)), then the static and dynamic MLPs:
 *   LN(h) = (h - mean) / sqrt(var + ln_eps) * ln_gain + ln_bias
 *   q, k, v = LN(h) Wq^T, Wk^T, Wv^T split into n_heads heads of d / n_heads;
 *   q and k rotated by the rotary embedding (rotate-half form, angle
 *   pos * 10000^(-2i/d_head) at the token's position in the sequence);
 *   softmax(q.k / sqrt(d_head)) over the keys at positions j with
 *   0 <= pos - j < window (causal; earlier chunks' keys and values inside the
 *   window included, as computed when their chunk ran); output o Wo^T.
 * With attention a token's loss depends on earlier tokens' rows, so the
 * update below the top block's attention is formed from the gradients of the
 * K_W- and K_M-weighted chunk losses (sum_t K_t G_t = grad of sum_t K_t l_t).
 *   attn_w  [n_blocks, 4, d, d]  device float32: Wq, Wk, Wv, Wo of each block
 *                                (copied, in the handle's operand precision)
 *   ln_gain, ln_bias [n_blocks, d]  device float32, 16-byte aligned (copied)
 * n_heads = 0 removes the attention.  d % n_heads == 0 and d / n_heads a
 * multiple of 16 (TTT_ERR_SHAPE), window >= 1 and ln_eps > 0
 * (TTT_ERR_INVALID_ARG); the handle's head must be TTT_HEAD_LM
 * (TTT_ERR_UNSUPPORTED).  With attention, ttt_prefill needs b % 8 == 0 and a
 * workspace that holds the keys and values of the whole sequence
 * (ttt_workspace_size reports it); ttt_predict is TTT_ERR_UNSUPPORTED.
 * Synchronous. */
ttt_status ttt_set_attention(ttt_handle* h, int32_t n_heads, int32_t window, const float* attn_w,
                             const float* ln_gain, const float* ln_bias, float ln_eps);

/* Final prediction at fixed fast weights ([TTT-E2E] 持续学习框架, the 预测
 * step: after the inner loop the weights W_T hold the context, and the
 * sequence is scored again with them; the page's inner-loop sketch ends with
 * this forward-only pass).  The forward of ttt_prefill (blocks, frozen
 * RMSNorm, LM head, next-token loss) at W, with no backward and no update:
 *   hidden [batch, T, d]  device float32, 16-byte aligned
 *   tokens [batch, T]     device int32 labels in [0, vocab), as in ttt_prefill
 *   W      [batch, n_blocks, m, h, d]  device float32 fast weights (read
 *                         only), ttt_prefill's layout; 16-byte aligned
 *   group_loss [batch, T/b]  device float32 out: the mean loss of each run of
 *                         b consecutive positions (the loss-by-position curve;
 *                         the mean of all of them is the final loss)
 *   token_loss [batch, T]    device float32 out, or NULL: every token's loss
 *   workspace  at least ttt_workspace_size(h, batch, T, b) bytes, 256-byte aligned
 * b is only the number of rows per sequence in one pass (any divisor of T;
 * a larger b gives larger GEMMs and needs a larger workspace).  Token range
 * errors and non-finite group losses are recorded in the device status word,
 * as in ttt_prefill.  Captured into a CUDA graph per distinct call, like
 * ttt_prefill.  A reconstruction-head handle is TTT_ERR_UNSUPPORTED. */
ttt_status ttt_predict(ttt_handle* h, int32_t batch, int32_t T, int32_t b, const float* hidden,
                       const int32_t* tokens, const float* W, float* group_loss, float* token_loss,
                       void* workspace, size_t ws_bytes, void* stream);

/* The per-token and per-chunk coefficients of a chunk update rule for every
 * chunk, on the device.  rule = TTT_RULE_E2TTT: the scalar kernels of
 * Proposition 3.1 ([E2-TTT] 定义高效后缀乘积与比例和, 命题3.1; computed in the
 * division-free form K_W_t = eta_t sum_{j>=t} (prod_{i=t+1}^{j} beta_i)
 * gtilde_j, float64 inside).  rule = TTT_RULE_LACT: K_W_t = K_M_t = eta_t and
 * the chunk's mean momentum factor ([E2-TTT] 高效的逐块更新机制).
 *   eta, beta, gamma [batch, T]  in
 *   KW, KM [batch, T]            out: E2TTT: eta_t btilde_t R_t and eta_t btilde_t;
 *                                     LaCT: eta_t and eta_t
 *   consts [batch, T/b, 4]       out: (coefficient of W_0 in W_C, of M_0 in M_C,
 *                                     of M_0 in W_C, 0): E2TTT (gtilde_0,
 *                                     btilde_0, btilde_0 R_1, 0); LaCT (1, mean
 *                                     beta, mean beta, 0)
 * T % b == 0 required; an unknown rule is TTT_ERR_INVALID_ARG.  No handle
 * needed; asynchronous on `stream`. */
ttt_status ttt_scalar_kernels(int32_t rule, int32_t batch, int32_t T, int32_t b, const float* eta,
                              const float* beta, const float* gamma, float* KW, float* KM,
                              float* consts, void* stream);

/* Input-dependent update scalars for every token ([E2-TTT] 依赖于输入的动态参数化):
 *   eta_t   = eta_base * sigmoid(w_eta . x_t + b_eta)
 *   beta_t  = sigmoid(w_beta . x_t + b_beta) ^ (1 / tau)
 *   alpha_t = alpha_base * sigmoid(w_alpha . x_t + b_alpha),  gamma_t = 1 - eta_t alpha_t
 *   hidden [batch, T, d]   device float32, x_t (the rows entering the updated
 *                          blocks, as passed to ttt_prefill); 16-byte aligned
 *   heads  [3, d]          device float32 rows w_eta, w_beta, w_alpha; 16-byte aligned
 *   eta, beta, gamma [batch, T]  device float32 out, ready for ttt_prefill
 * The Linear maps carry the biases b_eta, b_beta, b_alpha.  d % 4 == 0 and
 * tau > 0 (finite) are required (TTT_ERR_SHAPE / TTT_ERR_INVALID_ARG
 * otherwise).  Float32 dot products in a fixed order (deterministic).  No
 * handle needed; asynchronous on `stream`. */
ttt_status ttt_scalar_heads(int32_t batch, int32_t T, int32_t d, const float* hidden, const float* heads,
                            float b_eta, float b_beta, float b_alpha, float eta_base, float alpha_base,
                            float tau, float* eta, float* beta, float* gamma, void* stream);

/* The tensor-core GEMM the inner loop is built on, exposed for testing and
 * reuse: D[z] = A[z] B[z]^T for z < batch, i.e.
 *   D[z](m, n) = sum_{k < K} A[z](m, k) * B[z](n, k)
 * with bfloat16 operands (device, 16-byte aligned) and float32 output D
 * (row-major, leading dimension ldd, batch stride strideD, in elements).
 * A(m, k) is at A + z*strideA + (a_kmajor ? m*lda + k : k*lda + m); same for
 * B(n, k).  lda, ldb, strideA, strideB: multiples of 8 elements; strides are
 * nonzero when batch > 1.  workspace (256-byte aligned, >= 1 MiB, or NULL)
 * lets the engine split K across CTA pairs when the output has too few tiles
 * to fill the GPU; its contents are not preserved.  Asynchronous on `stream`. */
ttt_status ttt_gemm_bf16(int32_t M, int32_t N, int32_t K, int32_t batch, const void* A, int64_t lda,
                         int64_t strideA, int32_t a_kmajor, const void* B, int64_t ldb, int64_t strideB,
                         int32_t b_kmajor, float* D, int64_t ldd, int64_t strideD, void* workspace,
                         size_t ws_bytes, void* stream);

/* Synchronise `stream`, return the first device-side error recorded by this
 * handle's kernels since the last call (TTT_OK if none) and clear it. */
ttt_status ttt_get_device_status(ttt_handle* h, void* stream);

/* Self-test of the bounded-wait mechanism every spin loop in the library
 * uses: launches one kernel that waits on a device flag nothing sets, giving
 * up after `spin_limit` polls and recording TTT_ERR_TIMEOUT in the handle's
 * status word.  No fault, no trap; the context stays usable. */
ttt_status ttt_selftest_bounded_wait(ttt_handle* h, uint32_t spin_limit, void* stream);

/* Static description of a status code. */
const char* ttt_status_string(ttt_status s);

/* Text of the last host-side error on this thread ("" if none). */
const char* ttt_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* TTT_H_ */
