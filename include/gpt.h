/*
 * gpt.h - C ABI of the B200 (sm_100a) GPT-2 / nanoGPT causal decoder forward pass.
 *
 * What the library computes is the forward pass the nanoGPT pages describe:
 *   - "nanoGPT 全局流程图" (devpress.csdn.net), §3.2 前向传播: tok_emb + pos_emb, the Blocks,
 *     ln_f, then logits = lm_head(x) and F.cross_entropy(..., ignore_index=-1) when targets
 *     are given, or lm_head(x[:, [-1], :]) and no loss when they are not;
 *   - same page §2.5: the pre-LN Block x = x + attn(ln_1(x)); x = x + mlp(ln_2(x)),
 *     CausalSelfAttention (c_attn C->3C, heads, softmax(mask(q k^T / sqrt(hs))) v, c_proj),
 *     MLP (c_fc C->4C, GELU, c_proj 4C->C), LayerNorm with eps 1e-5;
 *   - same page §2.3: the head is tied to the token embedding (one [V, C] table);
 *   - "nanoGPT 核心代码速查表" (pgsm.cn), 七、关键函数签名: forward(idx, targets=None) ->
 *     (logits, loss).
 *
 * Conventions that hold for every entry point:
 *   - Every pointer is a DEVICE pointer unless stated otherwise.  The caller owns and
 *     allocates every buffer; no entry point allocates or frees device memory.
 *   - Tensors are dense and row-major; shapes are given outermost first.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*, NULL = legacy default
 *     stream) and runs asynchronously, except where GPT_FLAG_SYNC_CHECK asks for a
 *     synchronising error check.
 *   - Every entry point returns an int status: GPT_OK (0) or a negative GPT_ERR_* code.
 *     Argument errors are detected on the host before anything is enqueued.  Device-side
 *     conditions (an out-of-range token id or target, a pipeline wait that exceeded its
 *     time limit) are recorded in a device status word and reported by gpt_check_status()
 *     or by a call made with GPT_FLAG_SYNC_CHECK.  No kernel traps or asserts.
 *   - Results are deterministic: every reduction runs in a fixed order.
 *   - Storage precision: GPT_DTYPE_BF16 stores weights, activations between kernels and
 *     logits in bf16, accumulates in fp32 and keeps the residual stream, LayerNorm
 *     statistics, softmax and cross-entropy in fp32.  GPT_DTYPE_F32 is fp32 throughout.
 */
#ifndef GPT_B200_H
#define GPT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPT_ABI_VERSION 1

/* ---- status codes ------------------------------------------------------------------ */
#define GPT_OK                 0
#define GPT_ERR_NULL          -1  /* a required pointer is NULL */
#define GPT_ERR_BAD_SHAPE     -2  /* inconsistent sizes: T > block_size, C % n_head != 0, ... */
#define GPT_ERR_BAD_ALIGN     -3  /* a pointer is not 16-byte aligned */
#define GPT_ERR_WS_TOO_SMALL  -4  /* workspace_bytes < gpt_workspace_bytes(...) */
#define GPT_ERR_INDEX         -5  /* device: a token id outside [0, V) or a target outside [0, V) and != -1 */
#define GPT_ERR_TIMEOUT       -6  /* device: a pipeline wait exceeded its time limit; results invalid */
#define GPT_ERR_UNSUPPORTED   -7  /* valid request this build does not implement (e.g. bf16 with hs != 64) */
#define GPT_ERR_CUDA          -8  /* a CUDA runtime call failed (launch error, no device, ...) */

/* ---- configuration ------------------------------------------------------------------ */
#define GPT_DTYPE_F32   0
#define GPT_DTYPE_BF16  1

#define GPT_GELU_ERF    0   /* x * Phi(x), nn.GELU()'s default ("nanoGPT架构逐步详解", 4. MLP) */
#define GPT_GELU_TANH   1   /* 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) */

#define GPT_FLAG_SYNC_CHECK 1  /* synchronise `stream` at the end and return the device status */

/* GPTConfig ("nanoGPT 全局流程图", §2.1 模型配置).  Dropout is not a field: it is 0.0 there
 * and the identity in a forward pass. */
typedef struct gpt_config {
    int32_t n_layer;
    int32_t n_head;
    int32_t n_embd;       /* C; head size hs = C / n_head */
    int32_t block_size;   /* rows of wpe; T must not exceed it */
    int32_t vocab_size;   /* V; rows of the tied wte / lm_head table */
    int32_t bias;         /* 1: Linear and LayerNorm layers carry biases; 0: none are read */
    int32_t dtype;        /* GPT_DTYPE_F32 or GPT_DTYPE_BF16 */
    int32_t gelu;         /* GPT_GELU_ERF or GPT_GELU_TANH */
} gpt_config_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* gpt_status_string(int status);

/* GPT_ABI_VERSION of the loaded library. */
int gpt_abi_version(void);

/* The CUDA runtime's message for the last failed CUDA call made by this library on the calling
 * thread (the cause behind a GPT_ERR_CUDA), or "no error".  Static string, never NULL. */
const char* gpt_last_cuda_error(void);

/* Checks a configuration: positive sizes, C % n_head == 0, dtype and gelu in range,
 * and, for GPT_DTYPE_BF16, hs == 64 and C % 8 == 0 (the tensor-core kernels' layout).
 * Returns GPT_OK, GPT_ERR_NULL, GPT_ERR_BAD_SHAPE or GPT_ERR_UNSUPPORTED. */
int gpt_validate_config(const gpt_config_t* cfg);

/* ---- packed weights ------------------------------------------------------------------
 * All parameters live in ONE device buffer of gpt_weights_bytes(cfg) bytes, each tensor at
 * a 256-byte aligned offset, stored in the config's dtype, in this order (the nanoGPT
 * module tree of "nanoGPT 全局流程图" §2.2 and §2.5):
 *   0 wte [V, C]            (also the lm_head weight: tied, §2.3)
 *   1 wpe [block_size, C]
 *   then for each layer l:  ln_1.weight [C], ln_1.bias [C],
 *                           attn.c_attn.weight [3C, C], attn.c_attn.bias [3C],
 *                           attn.c_proj.weight [C, C],  attn.c_proj.bias [C],
 *                           ln_2.weight [C], ln_2.bias [C],
 *                           mlp.c_fc.weight [4C, C],    mlp.c_fc.bias [4C],
 *                           mlp.c_proj.weight [C, 4C],  mlp.c_proj.bias [C]
 *   then ln_f.weight [C], ln_f.bias [C].
 * Linear weights are [out, in] (nn.Linear).  Bias slots exist even when cfg->bias == 0;
 * they are then never read. */
size_t gpt_weights_bytes(const gpt_config_t* cfg);   /* 0 on an invalid config */
int    gpt_weights_count(const gpt_config_t* cfg);   /* 2 + 12 * n_layer + 2, or < 0 */
/* Fills offsets[i] (bytes) and numels[i] (elements) for i < min(n, count).  Either array
 * may be NULL.  Returns the tensor count or a negative status. */
int    gpt_weights_layout(const gpt_config_t* cfg, size_t* offsets, size_t* numels, int n);

/* ---- workspace ----------------------------------------------------------------------
 * Bytes of device scratch gpt_forward / gpt_block need for a [B, T] batch (activations,
 * cross-entropy partials and the device status word).  0 on invalid arguments.  The
 * workspace must be 256-byte aligned; its contents need no initialisation and are
 * overwritten by each call, so calls that share a workspace must be serialised on one
 * stream. */
size_t gpt_workspace_bytes(const gpt_config_t* cfg, int B, int T);

/* Synchronises `stream`, reads and clears the device status word in `workspace`, and
 * returns it (GPT_OK, GPT_ERR_INDEX or GPT_ERR_TIMEOUT), or GPT_ERR_CUDA. */
int gpt_check_status(void* workspace, void* stream);

/* Testing aid with no counterpart in the pages: sets, on the current device, the time after
 * which a pipeline wait inside the tensor-core kernels (a thread waiting for a copy, a product or
 * another warp's result) gives up, in nanoseconds; 0 restores the default of 1 s.  A kernel whose
 * wait gives up records GPT_ERR_TIMEOUT in its status word, lets every copy and product it has
 * already issued finish (those drains keep the default limit), releases its tensor memory and
 * returns; its outputs are then invalid.
 *   force_timeout != 0 makes the causal attention kernel, the product kernels (gpt_linear,
 *   single CTAs for M < 256 and CTA pairs from M = 256) and the single-launch decode step
 *   (gpt_decode_step and gpt_generate in bf16, at its first grid barrier) launched from then on
 *   wait first for an event that never happens, so their time-out path runs on purpose after
 *   `ns`; 0 turns that off.  A decode step that timed out leaves the position where it was.
 * Call it with no kernel of this library running or queued on the device (it copies to the device
 * synchronously).  Returns GPT_OK or GPT_ERR_CUDA. */
int gpt_set_wait_limit_ns(unsigned long long ns, int force_timeout);

/* ---- the forward pass ---------------------------------------------------------------
 * GPT.forward(idx, targets) ("nanoGPT 全局流程图", §3.2; "nanoGPT 代码解析", forward).
 *   weights  packed buffer described above.
 *   idx      int64 [B, T], token ids in [0, V).
 *   targets  int64 [B, T] in [0, V) or -1 (ignored), or NULL.
 *   logits   with targets: [B, T, V]; without: [B, 1, V], the last position only.
 *            bf16 for GPT_DTYPE_BF16, fp32 for GPT_DTYPE_F32.  Must be 16-byte aligned.
 *   loss     fp32 scalar: mean of logsumexp(z) - z[target] over rows whose target != -1;
 *            NaN when every target is -1.  May be NULL.  Untouched when targets == NULL.
 *   row_loss fp32 [B, T]: per-position loss, 0 at ignored positions.  May be NULL.
 *   loss_sum_count  fp64 [2]: {sum of counted row losses, number of counted rows}, the
 *            terms a batch-sharded caller adds across devices.  May be NULL.
 *   Requires 1 <= T <= block_size and B >= 1.  With bf16, the cross-entropy is taken from
 *   the fp32 accumulators, before the logits are rounded for storage.
 * The device status word in `workspace` is cleared at the start of every gpt_forward and
 * gpt_block call.
 * Returns GPT_OK once enqueued (or, with GPT_FLAG_SYNC_CHECK, once finished and checked). */
int gpt_forward(const gpt_config_t* cfg, const void* weights,
                const int64_t* idx, const int64_t* targets, int B, int T,
                void* logits, float* loss, float* row_loss, double* loss_sum_count,
                void* workspace, size_t workspace_bytes, void* stream, int flags);

/* One pre-LN Block in place ("nanoGPT 全局流程图", §2.5 Block.forward):
 *   x = x + attn(ln_1(x)); x = x + mlp(ln_2(x))  for layer `layer` of `weights`.
 *   x  fp32 [B, T, C] (the residual stream is fp32 for both dtypes), updated in place.
 *   workspace as for gpt_forward (gpt_workspace_bytes(cfg, B, T) bytes). */
int gpt_block(const gpt_config_t* cfg, const void* weights, int layer, float* x, int B, int T,
              void* workspace, size_t workspace_bytes, void* stream, int flags);

/* Causal self-attention of one batch of heads ("nanoGPT 全局流程图", §2.5 (B) 步骤3-6;
 * "nanoGPT架构逐步详解", 3. 因果自注意力):
 *   y[b, h, i] = sum_{j <= i} softmax_j(q[b,h,i] . k[b,h,j] / sqrt(hs)) v[b,h,j]
 *   q, k, v, y  [B, nh, T, hs], 16-byte aligned, dtype GPT_DTYPE_BF16 (hs must be 64) or
 *               GPT_DTYPE_F32 (1 <= hs <= 128).
 *   status      optional device int32 (NULL allowed); a pipeline time-out writes
 *               GPT_ERR_TIMEOUT there.  It is never cleared by the library. */
int gpt_attention(const void* q, const void* k, const void* v, void* y,
                  int B, int nh, int T, int hs, int dtype, int32_t* status, void* stream);

/* ---- single kernels of the forward pass (same kernels gpt_forward launches) ----------- */

/* x[b, t, :] = wte[idx[b, t], :] + wpe[t, :]  ("nanoGPT 全局流程图", §3.2 ①).
 *   wte [V, C], wpe [>= T, C] in `dtype`; x fp32 [B, T, C].  An id outside [0, V) reads
 *   row 0 instead and writes GPT_ERR_INDEX to *status (optional device int32). */
int gpt_embed(const void* wte, const void* wpe, const int64_t* idx, float* x,
              int B, int T, int C, int V, int dtype, int32_t* status, void* stream);

/* out = (x - mean) / sqrt(var + 1e-5) * w + b per row, var the population variance
 * ("nanoGPT 全局流程图", §2.5 (A)).  x fp32 [rows, C]; w, b [C] in `dtype` (b may be NULL);
 * out [rows, C] in `dtype`.  C <= 2048 and C % 4 == 0. */
int gpt_layernorm(const float* x, const void* w, const void* b, void* out,
                  int rows, int C, int dtype, void* stream);

#define GPT_EPI_STORE   0  /* out = x W^T + b                       (out in dtype)      */
#define GPT_EPI_GELU    1  /* out = gelu(x W^T + b)                 (out in dtype)      */
#define GPT_EPI_RESID   2  /* out += x W^T + b, out fp32            (residual stream)   */

/* nn.Linear with a fused epilogue: x [M, K], W [N, K] (nn.Linear layout), b [N] or NULL,
 * all in `dtype`; out [M, N] as the epilogue says.  gelu = GPT_GELU_*.  With bf16,
 * K % 8 == 0 and N % 8 == 0.  status: optional device int32 that receives GPT_ERR_TIMEOUT
 * if a pipeline wait of the tensor-core kernel expires (never cleared by the library). */
int gpt_linear(const void* x, const void* W, const void* b, void* out, int M, int N, int K,
               int dtype, int epilogue, int gelu, int32_t* status, void* stream);

/* The inference branch of the head ("nanoGPT 全局流程图", §3.2 ④: with no targets only the last
 * position goes through ln_f and lm_head, logits [B, 1, V]):
 *   logits[b, :] = LayerNorm(x[b * ldx .. b * ldx + C); lnf_w, lnf_b) wte^T
 *   x       fp32 residual rows, row b at element offset b * ldx (for a [B, T, C] residual stream,
 *           pass &x[0, T-1, 0] and ldx = T * C); 16-byte aligned, ldx % 4 == 0.
 *   lnf_w, lnf_b  [C] in `dtype` (lnf_b may be NULL); wte [V, C] in `dtype`, 16-byte aligned.
 *   logits  [B, V] in `dtype` (rows V elements apart).
 *   status  optional device int32 (NULL allowed): GPT_ERR_TIMEOUT if a pipeline wait of the
 *           tensor-core kernel gave up (never cleared by the library).
 *   Requires C % 8 == 0, and C <= 2048 for bf16 (for fp32, min(B, 16) * C * 8 <= 227 KB);
 *   else GPT_ERR_UNSUPPORTED.  One read of wte per 16 rows: the product is bound by HBM.
 *   gpt_forward with targets == NULL runs this on its final residual rows. */
int gpt_lm_head_last(const float* x, long long ldx, const void* lnf_w, const void* lnf_b,
                     const void* wte, int B, int C, int V, int dtype, void* logits, int32_t* status,
                     void* stream);

/* Tied head with fused cross-entropy ("nanoGPT 全局流程图", §3.2 ④ and §3.3):
 *   logits = u wte^T ([rows, V] in `dtype`), then per row logsumexp - logit[target] over all
 *   V columns, averaged over rows whose target != -1 (fixed-order reduction).
 *   u [rows, C] in `dtype` (the ln_f output), wte [V, C], targets int64 [rows].
 *   loss / row_loss / loss_sum_count as in gpt_forward (each may be NULL).
 *   workspace: gpt_lm_head_workspace_bytes(rows, V) bytes, 256-byte aligned; its status word
 *   is read by gpt_check_status(). */
size_t gpt_lm_head_workspace_bytes(int rows, int V);
int gpt_lm_head_loss(const void* u, const void* wte, const int64_t* targets, int rows, int C,
                     int V, int dtype, void* logits, float* loss, float* row_loss,
                     double* loss_sum_count, void* workspace, size_t workspace_bytes,
                     void* stream, int flags);

/* gpt_lm_head_loss without a workspace argument.  The pages have no counterpart: this exists
 * for callers that cannot allocate device memory when they need the loss (a serving process
 * that gave all of its GPU memory to a fixed pool at start-up, a plugin inside another
 * framework whose allocator it may not bypass, a latency-critical loop that cannot pay for
 * cudaMalloc and its implicit device synchronisation).  Arguments and results are those of
 * gpt_lm_head_loss.
 *   Scratch: a static 16 MiB device array inside this library, held by every GPU that uses the
 *   library until the process exits.  A request needing more than that
 *   (gpt_lm_head_workspace_bytes(rows, V) > 16 MiB; about 5,300 rows at V = 50304) returns
 *   GPT_ERR_WS_TOO_SMALL before anything is enqueued.  Nothing is allocated or freed.
 *   The first call on each device looks up the array's device address (cudaGetSymbolAddress)
 *   with that device current and keeps it for the life of the process; make that first call
 *   before any stream capture begins.  cudaDeviceReset (or any other teardown of the device's
 *   primary context) invalidates the kept address: do not call this entry point on a device
 *   after resetting it.
 *   All calls on a device share the array and it keeps the last call's contents (the status
 *   word is cleared at the start of each call): calls whose work overlaps on the GPU race, so
 *   order them on one stream.  With GPT_FLAG_SYNC_CHECK the status word is read from the array.
 *   Without that flag a call whose head product gave up on a bounded wait (GPT_ERR_TIMEOUT in
 *   the status word) still returns GPT_OK, and its loss may then be built from partial sums an
 *   earlier call left in the array: pass GPT_FLAG_SYNC_CHECK where that matters. */
int gpt_lm_head_loss_noalloc(const void* u, const void* wte, const int64_t* targets, int rows,
                             int C, int V, int dtype, void* logits, float* loss, float* row_loss,
                             double* loss_sum_count, void* stream, int flags);

/* ---- generation with a key/value cache ------------------------------------------------
 * "nanoGPT 全局流程图", 第五阶段 生成文本 (GPT.generate); "nanoGPT 核心代码速查表", 七、关键函数签名
 * (generate(idx, max_new_tokens, temperature, top_k) -> tokens).  Each step feeds the last
 * block_size tokens of the sequence to the model, takes the last position's logits, divides
 * them by the temperature, keeps the logits not below the top_k-th largest (every logit at
 * that value is kept), turns them into probabilities with softmax and draws the next token
 * from them.  The cache is this library's incremental form of the same forward ("DummyGPTModel",
 * 扩展方向 names the KV cache as an inference optimisation): while the sequence fits in
 * block_size, a step runs only the newest position against the cached keys and values of the
 * earlier ones, which gives the logits of the full forward up to rounding.
 *
 * KV cache: n_layer x [B, block_size, 2, n_embd] in the configuration's dtype (k of position
 * t in [.., t, 0, :], v in [.., t, 1, :]), gpt_kv_cache_bytes(cfg, B) bytes, 16-byte aligned,
 * owned by the caller.  The draw: with u in [0, 1) supplied by the caller (one per sequence and
 * step), the token is the smallest index i with p_0 + ... + p_i > u * (p_0 + ... + p_{V-1}),
 * p the kept exponentials; random numbers are inputs, never generated here.
 * Decoding entry points require n_embd % 8 == 0 and head size % 8 == 0, <= 128. */
size_t gpt_kv_cache_bytes(const gpt_config_t* cfg, int B);

/* Workspace of gpt_prefill (T <= T_prefill) and gpt_decode_step (any T_prefill >= 1), 256-byte
 * aligned.  The same workspace carries the decode position between calls (device-side, so a
 * captured step can be replayed); do not share it between sequences decoded concurrently. */
size_t gpt_decode_workspace_bytes(const gpt_config_t* cfg, int B, int T_prefill);

/* Forward over idx int64 [B, T] (1 <= T <= block_size) that writes every layer's k and v of
 * positions [0, T) into kv_cache and the logits of position T-1 to logits fp32 [B, V]; sets the
 * decode position to T.  flags: GPT_FLAG_SYNC_CHECK as in gpt_forward. */
int gpt_prefill(const gpt_config_t* cfg, const void* weights, const int64_t* idx, int B, int T,
                void* kv_cache, float* logits, void* workspace, size_t workspace_bytes,
                void* stream, int flags);

/* One new token per sequence, tok[b * ld_tok] (int64), at the decode position p held in the
 * workspace: each layer appends its k, v at p and attends over positions [0, p]; writes the
 * logits fp32 [B, V] of that position and advances p by one.  The cache must hold positions
 * [0, p) from gpt_prefill and earlier steps with the same B.  p must be < block_size: beyond
 * it the step writes nothing to the cache, records GPT_ERR_BAD_SHAPE in the status word and
 * its logits are meaningless (gpt_generate re-runs gpt_prefill on the window instead). */
int gpt_decode_step(const gpt_config_t* cfg, const void* weights, const int64_t* tok,
                    long long ld_tok, int B, void* kv_cache, float* logits, void* workspace,
                    size_t workspace_bytes, void* stream, int flags);

/* The sampling step on logits fp32 [B, V] (V <= 53248: one row is staged in shared memory;
 * GPT_ERR_UNSUPPORTED above that), temperature > 0 (GPT_ERR_BAD_SHAPE otherwise),
 * top_k <= 0 for no top-k filter, u fp32 [B] in [0, 1); writes out[b * ld_out] (int64).  The
 * top-k threshold is taken on the logits before the division (the same order for any
 * positive temperature).  Sums run in a fixed order; the result is deterministic. */
int gpt_sample(const float* logits, int B, int V, float temperature, int top_k, const float* u,
               int64_t* out, long long ld_out, void* stream);

/* GPT.generate: out int64 [B, T0 + max_new_tokens] = idx [B, T0] followed by max_new_tokens
 * drawn tokens; uniforms fp32 [max_new_tokens, B] (step-major).  step_logits: optional fp32
 * [max_new_tokens, B, V] that receives each step's logits before the temperature (NULL to
 * skip).  Step s sees the last min(T0 + s, block_size) tokens: the first step and every step
 * whose sequence is longer than block_size run gpt_prefill on that window (the positions of
 * a cropped window shift, so the cache is rebuilt); the others run gpt_decode_step.
 * workspace: gpt_generate_workspace_bytes(cfg, B, T0, max_new_tokens) bytes. */
size_t gpt_generate_workspace_bytes(const gpt_config_t* cfg, int B, int T0, int max_new_tokens);
int gpt_generate(const gpt_config_t* cfg, const void* weights, const int64_t* idx, int B, int T0,
                 int max_new_tokens, float temperature, int top_k, const float* uniforms,
                 int64_t* out, float* step_logits, void* kv_cache, void* workspace,
                 size_t workspace_bytes, void* stream, int flags);

/* ---- optimizer step -------------------------------------------------------------------
 * "nanoGPT 全局流程图", 3.5 学习率调度, 3.6 梯度裁剪 + 参数更新 and 优化器配置; "nanoGPT 代码解析",
 * configure_optimizers.  One training step's update of every parameter: the gradients are
 * scaled by min(1, max_grad_norm / (||g||_2 + 1e-6)) with ||g||_2 the norm over ALL gradient
 * entries (torch.nn.utils.clip_grad_norm_), then torch.optim.AdamW's update with decoupled weight
 * decay, applied with weight_decay to the tensors of two dimensions (wte, wpe and each layer's
 * four Linear weights) and with none to the rest (biases, LayerNorm weights and biases). */

/* get_lr(it): linear warm-up to learning_rate over warmup_iters, cosine decay to min_lr at
 * lr_decay_iters, min_lr afterwards (the page's curve; its listing stops at the cosine).  The
 * page's values: 6e-4, 6e-5, 2000, 600000.  Host function. */
double gpt_lr_schedule(long long it, double learning_rate, double min_lr, long long warmup_iters,
                       long long lr_decay_iters);

typedef struct gpt_adamw {
    float lr;             /* this step's learning rate (gpt_lr_schedule) */
    float beta1, beta2;   /* 0.9, 0.95 on the page */
    float eps;            /* 1e-8 (torch's default; the page does not set it) */
    float weight_decay;   /* 0.1 on the page; applied to two-dimensional tensors only */
    float max_grad_norm;  /* 1.0 on the page; <= 0 disables clipping */
    int32_t step;         /* optimizer steps taken including this one, >= 1 (bias corrections) */
} gpt_adamw_t;

/* Elements of each flat fp32 optimizer array: gpt_weights_bytes(cfg) / element size of
 * cfg->dtype.  Tensor i of gpt_weights_layout sits at element offset offsets[i] / element size;
 * the padding between tensors, and the bias slots when cfg->bias == 0, are never read or
 * written. */
size_t gpt_param_elems(const gpt_config_t* cfg);
size_t gpt_adamw_workspace_bytes(void);   /* scratch of gpt_adamw_step, 256-byte aligned */

/* params, grads, exp_avg, exp_avg_sq: fp32 [gpt_param_elems(cfg)], 16-byte aligned; params and
 * both moments are updated in place (moments start at zero before step 1).  weights: the packed
 * buffer in cfg->dtype that the forward reads, or NULL; when given, each updated parameter is
 * also written there (rounded to bf16 for GPT_DTYPE_BF16).  grad_norm: optional device float
 * that receives ||g||_2 before clipping.  Sums run in a fixed order: results are deterministic.
 * GPT_ERR_BAD_SHAPE for step < 1, negative or non-finite lr, betas outside [0, 1), eps <= 0,
 * negative weight_decay.  flags: GPT_FLAG_SYNC_CHECK synchronises the stream before returning. */
int gpt_adamw_step(const gpt_config_t* cfg, float* params, const float* grads, float* exp_avg,
                   float* exp_avg_sq, void* weights, const gpt_adamw_t* hp, float* grad_norm,
                   void* workspace, size_t workspace_bytes, void* stream, int flags);

/* ---- backward pieces ------------------------------------------------------------------
 * "nanoGPT 全局流程图", 3.4 反向传播 (loss.backward(): the chain rule from the mean cross-entropy
 * back to every parameter).  These are the steps of the backward pass that are not matrix
 * products; each is the derivative of the forward operation named, in fp32 unless stated, with
 * every reduction in a fixed order (deterministic). */

/* d(loss)/d(logits) for the mean cross-entropy over rows whose target is not -1:
 * dlogits[r, v] = (softmax(logits[r])[v] - [v == targets[r]]) / n, 0 for ignored rows, n the
 * counted rows read from loss_sum_count[1] (the {sum, count} pair gpt_forward writes; device
 * fp64).  logits / dlogits [rows, V] in `dtype`; the softmax is taken over all V columns.  A target
 * outside [0, V) and != -1 gives a zero row and GPT_ERR_INDEX in *status (optional). */
int gpt_cross_entropy_backward(const void* logits, const int64_t* targets, const double* loss_sum_count,
                               int rows, int V, int dtype, void* dlogits, int32_t* status, void* stream);

/* LayerNorm backward (eps 1e-5, population variance): y = xhat w + b.  dy, x, dx fp32 [rows, C]
 * (C <= 4096); w [C] in `dtype`.  dx = rstd (dxhat - mean(dxhat) - xhat mean(dxhat xhat)) with
 * dxhat = dy w, added to dx when accumulate != 0.  dw = sum over rows of dy xhat and db = sum of
 * dy (fp32 [C]; db may be NULL), added when accumulate_wb != 0.  workspace: the column partials,
 * gpt_layernorm_backward_workspace_bytes(rows, C) bytes, 256-byte aligned. */
size_t gpt_layernorm_backward_workspace_bytes(int rows, int C);
int gpt_layernorm_backward(const float* dy, const float* x, const void* w, int rows, int C, int dtype,
                           float* dx, int accumulate, float* dw, float* db, int accumulate_wb,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Bias gradient of a Linear layer: db[c] (+)= sum over rows of dy[r, c]; dy [rows, C] in
 * `dtype`, db fp32 [C].  workspace: gpt_bias_grad_workspace_bytes(rows, C) bytes. */
size_t gpt_bias_grad_workspace_bytes(int rows, int C);
int gpt_bias_grad(const void* dy, int rows, int C, int dtype, float* db, int accumulate,
                  void* workspace, size_t workspace_bytes, void* stream);

/* GELU backward: dpre = dh * gelu'(pre) elementwise (n elements); dh fp32, pre and dpre in
 * `dtype`; gelu = GPT_GELU_ERF (Phi(z) + z phi(z)) or GPT_GELU_TANH (the tanh form's derivative). */
int gpt_gelu_backward(const float* dh, const void* pre, long long n, int dtype, int gelu, void* dpre,
                      void* stream);

/* Embedding backward ("全局流程图" §3.2 ①: x = wte[idx] + wpe[t]): dwte[v] += sum of dx[b, t] over
 * the positions with idx[b, t] = v, in position order; dwpe[t] += sum over the batch of dx[b, t].
 * idx int64 [B, T], dx fp32 [B, T, C], dwte fp32 [V, C], dwpe fp32 [>= T, C].  B * T <= 16384 (the
 * positions are ordered by token inside one CTA).  workspace: gpt_embedding_backward_workspace_bytes
 * bytes.  An id outside [0, V) is skipped and GPT_ERR_INDEX written to *status (optional). */
size_t gpt_embedding_backward_workspace_bytes(int B, int T);
int gpt_embedding_backward(const int64_t* idx, const float* dx, int B, int T, int C, int V, float* dwte,
                           float* dwpe, void* workspace, size_t workspace_bytes, int32_t* status,
                           void* stream);

/* Causal attention as gpt_attention, also writing lse [B, nh, T] fp32: for each query row,
 * log2 of sum_j 2^(s_ij log2(e) / sqrt(hs)) with s_ij = q_i . k_j — the row's log-sum-exp in
 * base-2 units of the scaled score, which lets the backward recompute the probabilities. */
int gpt_attention_train(const void* q, const void* k, const void* v, void* y, float* lse, int B, int nh,
                        int T, int hs, int dtype, int32_t* status, void* stream);

/* Backward of causal attention ("全局流程图" 3.4 applied to §2.5 (B)): with p_ij recomputed from
 * q, k and lse, D_i = dout_i . o_i and dS_ij = p_ij (dout_i . v_j - D_i) for j <= i,
 *   dq_i = sum_j dS_ij k_j / sqrt(hs),  dk_j = sum_i dS_ij q_i / sqrt(hs),  dv_j = sum_i p_ij dout_i.
 * All [B, nh, T, hs] in `dtype` (o = the forward's y, lse from gpt_attention_train); hs 32 or 64;
 * fp32 accumulation.  bf16 with hs 64 and 16-byte aligned operands runs two tensor-core kernels
 * (dK/dV per 128-key tile, dQ per 128-query tile; P and dS rounded to bf16 as MMA operands);
 * everything else runs SIMT kernels.  Results are bit-reproducible (fixed summation order).
 * workspace: gpt_attention_backward_workspace_bytes(B, nh, T) bytes, 256-byte aligned (D and a
 * padded copy of lse).  status: optional device int32 that receives GPT_ERR_TIMEOUT if a pipeline
 * wait of the tensor-core kernels expires (as gpt_linear). */
size_t gpt_attention_backward_workspace_bytes(int B, int nh, int T);
int gpt_attention_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                           const float* lse, void* dq, void* dk, void* dv, int B, int nh, int T, int hs,
                           int dtype, void* workspace, size_t workspace_bytes, int32_t* status,
                           void* stream);

/* Backward of nn.Linear y = x W^T + b ("nanoGPT 全局流程图", 3.4 反向传播):
 *   dx = dy W       fp32 [rows, n_in], overwritten
 *   dW += dy^T x    fp32 [n_out, n_in], accumulated
 * dy [rows, n_out], x [rows, n_in], W [n_out, n_in] (nn.Linear layout), dense, in `dtype`.  bf16: the
 * tensor-core GEMM reads dy, x and W where they are, as MN-major operands wherever the product
 * needs a transpose (no copies); n_out and n_in multiples of 8, pointers 16-byte aligned.  fp32:
 * transposed copies in workspace feed the SIMT GEMM.  workspace:
 * gpt_linear_backward_workspace_bytes(rows, n_out, n_in, dtype) bytes (256 for bf16), 256-byte
 * aligned.  The bias gradient is gpt_bias_grad of dy.  status: as gpt_linear. */
size_t gpt_linear_backward_workspace_bytes(int rows, int n_out, int n_in, int dtype);
int gpt_linear_backward(const void* dy, const void* x, const void* W, int rows, int n_out, int n_in, int dtype,
                        float* dx, float* dW, void* workspace, size_t workspace_bytes, int32_t* status,
                        void* stream);

/* out[c * ld_out + r] = in[r * ld_in + c] for r < rows, c < cols, converting between bf16 and fp32
 * (the operand layouts of the backward's products). */
int gpt_transpose(const void* in, int in_dtype, long long ld_in, void* out, int out_dtype,
                  long long ld_out, int rows, int cols, void* stream);

/* ---- the training step ----------------------------------------------------------------
 * "nanoGPT 全局流程图" 3.2-3.4: forward with targets, then loss.backward().  gpt_forward_train runs
 * gpt_forward's computation and keeps what the backward needs in `acts`
 * (gpt_train_activation_bytes(cfg, B, T) bytes, 256-byte aligned; per layer the residual input,
 * both LayerNorm outputs, q/k/v, the attention output and its per-row log-sum-exp, the c_fc
 * pre-activation (bf16: GELU's derivative there, all the backward needs of it) and the GELU
 * output; then the final residual, ln_f's output, the logits, each row's logsumexp (bf16: from
 * the head's fp32 accumulators; the backward's d(logits) then takes one pass) and the
 * {sum of row losses, counted rows} pair).  loss: device fp32 scalar.  workspace: as gpt_forward.
 * gpt_backward adds loss_scale * d(loss)/d(parameter) to grads (fp32, the flat element layout of
 * gpt_param_elems; zero it before the first micro-batch), reading acts; the tied head's and the
 * embedding's contributions to wte are both added.  The mean is over the counted rows in acts'
 * {sum, count} pair (at byte offset gpt_train_loss_terms_offset): a data-parallel caller sums the
 * pair over its ranks before the backward, so each rank's gradient is its share of the global
 * mean and a SUM all-reduce of grads gives the whole batch's gradient.  loss_scale: 1, or 1/K for
 * K accumulated micro-batches (the page's loss / gradient_accumulation_steps); must be > 0.
 * workspace: gpt_backward_workspace_bytes.
 * Head size 32 or 64; for bf16, B * T % 8 == 0; B * T <= 16384.  Linear layers' backward products
 * are gpt_linear_backward's (bf16: tensor-core GEMM on MN-major operands, no transposed copies);
 * the attention backward is gpt_attention_backward's (bf16, head size 64: tensor cores). */
size_t gpt_train_activation_bytes(const gpt_config_t* cfg, int B, int T);
size_t gpt_backward_workspace_bytes(const gpt_config_t* cfg, int B, int T);
int gpt_forward_train(const gpt_config_t* cfg, const void* weights, const int64_t* idx,
                      const int64_t* targets, int B, int T, void* acts, size_t acts_bytes, float* loss,
                      void* workspace, size_t workspace_bytes, void* stream, int flags);
size_t gpt_train_loss_terms_offset(const gpt_config_t* cfg, int B, int T);
int gpt_backward(const gpt_config_t* cfg, const void* weights, const int64_t* idx, const int64_t* targets,
                 int B, int T, const void* acts, size_t acts_bytes, float* grads, float loss_scale,
                 void* workspace, size_t workspace_bytes, void* stream, int flags,
                 void* const* bucket_events);

/* Gradient buckets for overlapping a data-parallel gradient reduction with the backward ("nanoGPT
 * 全局流程图" 3.4 and the per-GPU batch of "nanoGPT 核心代码速查表" 七): n_layer + 1 element ranges
 * [starts[i], stops[i]) of the flat fp32 gradient array, in the order gpt_backward finishes them:
 * bucket i < n_layer holds every parameter of layer n_layer - 1 - i (bucket 0 also ln_f's), bucket
 * n_layer holds wte and wpe (complete only after the embedding's gradient, the last step).  Together
 * they cover the array once.  gpt_backward's bucket_events (NULL, or n_layer + 1 cudaEvent_t handles,
 * entries may be NULL): event i is recorded on `stream` right after the last kernel that writes
 * bucket i, so another stream may wait on it and reduce that range while the backward goes on.
 * Returns n_layer + 1 (filling at most n entries; either array may be NULL) or a negative status. */
int gpt_grad_buckets(const gpt_config_t* cfg, size_t* starts, size_t* stops, int n);

#ifdef __cplusplus
}
#endif

#endif /* GPT_B200_H */
