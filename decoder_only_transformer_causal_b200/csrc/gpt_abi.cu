// The C ABI declared in include/gpt.h: argument validation, the packed-weight layout, the
// workspace plan and the launch sequence of the forward pass.  All work runs in the
// kernels of this library; nothing here computes on the host.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "internal.h"

#define GPT_API extern "C" __attribute__((visibility("default")))

namespace gpt {

namespace {
thread_local cudaError_t g_last_cuda_error = cudaSuccess;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return GPT_OK;
    g_last_cuda_error = e;
    return GPT_ERR_CUDA;
}

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    static int cached[64] = {0};
    if (dev < 0 || dev >= 64) dev = 0;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

int opt_in_smem(const void* kern, size_t bytes, size_t (&opted)[kMaxDevices]) {
    int dev = 0;
    int rc = cuda_status(cudaGetDevice(&dev));
    if (rc) return rc;
    if (dev >= 0 && dev < kMaxDevices && bytes <= opted[dev]) return GPT_OK;
    rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)));
    if (rc) return rc;
    if (dev >= 0 && dev < kMaxDevices) opted[dev] = bytes;
    return GPT_OK;
}

// ------------------------------------------------------------------ TMA descriptors
namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

int encode(CUtensorMap* m, const void* base, cuuint32_t rank, const cuuint64_t* dims, const cuuint64_t* strides,
           const cuuint32_t* box, CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
           CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
    if (reinterpret_cast<uintptr_t>(base) & 15) return GPT_ERR_BAD_ALIGN;
    for (cuuint32_t i = 0; i + 1 < rank; ++i)
        if (strides[i] & 15) return GPT_ERR_BAD_ALIGN;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return GPT_ERR_CUDA;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, dt, rank, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GPT_OK : GPT_ERR_CUDA;
}
}  // namespace

int make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    return encode(m, base, 2, dims, strides, box);
}

int make_tmap_2d_sw64(CUtensorMap* m, const void* base, bool fp32, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    return encode(m, base, 2, dims, strides, box,
                  fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_64B);
}

int make_tmap_bf16_4d(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides_bytes[3],
                      const uint32_t box[4]) {
    const cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
    const cuuint64_t s[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
    const cuuint32_t b[4] = {box[0], box[1], box[2], box[3]};
    return encode(m, base, 4, d, s, b);
}

}  // namespace gpt

using namespace gpt;

namespace {

constexpr int kTensorsPerLayer = 12;
enum {
    W_LN1_W = 0, W_LN1_B, W_ATTN_W, W_ATTN_B, W_PROJ_W, W_PROJ_B,
    W_LN2_W, W_LN2_B, W_FC_W, W_FC_B, W_FC2_W, W_FC2_B
};

size_t a256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The fused last-position head: the tensor-core kernel for bf16 (C <= 2048), the LayerNorm-prologue
// GEMV for fp32, which stages up to 16 rows of the normalised input and its fp32 source in shared
// memory.
bool head_last_supported(int C, int B, int dtype) {
    if (dtype == GPT_DTYPE_BF16) return head_last_tc_supported(C);
    return C % 8 == 0 && gemv_smem_bytes(B, C, dtype, true) <= 227u * 1024u;
}

int launch_head_last(const float* x, long long ldx, const void* lnw, const void* lnb, const void* wte, int B, int C,
                     int V, int dtype, void* logits, int32_t* status, cudaStream_t s) {
    if (dtype == GPT_DTYPE_BF16)
        return launch_head_last_bf16(x, ldx, static_cast<const bf16*>(lnw), static_cast<const bf16*>(lnb),
                                     static_cast<const bf16*>(wte), B, C, V, static_cast<bf16*>(logits), V, status, s);
    return launch_gemv(kGemvEpiStore, true, dtype, x, ldx, lnw, lnb, wte, nullptr, logits, V, B, V, C, 0, nullptr,
                       nullptr, C, 1, 0, s);
}

int elem_size(const gpt_config_t* c) { return c->dtype == GPT_DTYPE_BF16 ? 2 : 4; }

int validate(const gpt_config_t* c) {
    if (!c) return GPT_ERR_NULL;
    if (c->n_layer < 0 || c->n_head <= 0 || c->n_embd <= 0 || c->block_size <= 0 || c->vocab_size <= 0)
        return GPT_ERR_BAD_SHAPE;
    if (c->n_embd % c->n_head) return GPT_ERR_BAD_SHAPE;
    if (c->dtype != GPT_DTYPE_F32 && c->dtype != GPT_DTYPE_BF16) return GPT_ERR_BAD_SHAPE;
    if (c->gelu != GPT_GELU_ERF && c->gelu != GPT_GELU_TANH) return GPT_ERR_BAD_SHAPE;
    if (c->n_embd % 4) return GPT_ERR_UNSUPPORTED;       // 16-byte rows in the row kernels
    if (c->n_embd > 2048) return GPT_ERR_UNSUPPORTED;    // LayerNorm keeps a row in registers
    const int hs = c->n_embd / c->n_head;
    if (c->dtype == GPT_DTYPE_BF16) {
        if (hs != 64) return GPT_ERR_UNSUPPORTED;        // tensor-core attention tile
        if (c->n_embd % 8) return GPT_ERR_UNSUPPORTED;   // 16-byte TMA rows
    } else if (hs > 128) {
        return GPT_ERR_UNSUPPORTED;
    }
    return GPT_OK;
}

// Offsets (bytes) and element counts of the packed weights, in the documented order.
int layout(const gpt_config_t* c, size_t* offs, size_t* numels, int n) {
    const size_t C = c->n_embd, V = c->vocab_size, bs = c->block_size, es = elem_size(c);
    const int count = 2 + kTensorsPerLayer * c->n_layer + 2;
    size_t off = 0;
    int k = 0;
    auto put = [&](size_t numel) {
        if (k < n) {
            if (offs) offs[k] = off;
            if (numels) numels[k] = numel;
        }
        off += a256(numel * es);
        ++k;
    };
    put(V * C);
    put(bs * C);
    for (int l = 0; l < c->n_layer; ++l) {
        put(C); put(C);
        put(3 * C * C); put(3 * C);
        put(C * C); put(C);
        put(C); put(C);
        put(4 * C * C); put(4 * C);
        put(4 * C * C); put(C);
    }
    put(C);
    put(C);
    (void)count;
    return k;
}

size_t weights_total(const gpt_config_t* c) {
    const size_t C = c->n_embd, V = c->vocab_size, bs = c->block_size, es = elem_size(c);
    size_t per_layer = a256(C * es) * 6 + a256(3 * C * C * es) + a256(3 * C * es) + a256(C * C * es) +
                       a256(4 * C * C * es) + a256(4 * C * es) + a256(4 * C * C * es);
    return a256(V * C * es) + a256(bs * C * es) + per_layer * c->n_layer + 2 * a256(C * es);
}

// Pointers into the packed weight buffer, computed from the same layout as layout().
struct Weights {
    const uint8_t* base;
    const gpt_config_t* c;
    size_t head, layer_bytes, in_layer[kTensorsPerLayer], tail;
    const void* wte() const { return base; }
    const void* wpe() const { return base + a256(static_cast<size_t>(c->vocab_size) * c->n_embd * elem_size(c)); }
    const void* layer(int l, int which) const { return base + head + layer_bytes * l + in_layer[which]; }
    const void* bias(int l, int which) const { return c->bias ? layer(l, which) : nullptr; }
    const void* lnf_w() const { return base + tail; }
    const void* lnf_b() const {
        return c->bias ? base + tail + a256(static_cast<size_t>(c->n_embd) * elem_size(c)) : nullptr;
    }
};

struct Plan {
    size_t ctrl, x, u, qkv, y, h, part, tlogit, rowloss, total;
    int n_part;
};

Plan plan_ws(const gpt_config_t* c, long long B, long long T) {
    Plan P{};
    const size_t N = static_cast<size_t>(B * T), C = c->n_embd, es = elem_size(c);
    size_t off = 0;
    P.ctrl = off; off += 256;
    P.x = off; off += a256(N * C * 4);
    P.u = off; off += a256(N * C * es);
    P.qkv = off; off += a256(N * 3 * C * es);
    P.y = off; off += a256(N * C * es);
    P.h = off; off += a256(N * 4 * C * es);
    P.n_part = c->dtype == GPT_DTYPE_BF16 ? gemm_ce_parts(c->vocab_size) : 0;
    P.part = off; off += a256(N * static_cast<size_t>(P.n_part) * 8);
    P.tlogit = off; off += a256(N * 4);
    P.rowloss = off; off += a256(N * 4);
    P.total = off;
    return P;
}

int32_t* status_word(void* ws) { return static_cast<int32_t*>(ws); }

int sync_and_read_status(void* ws, cudaStream_t s) {
    int rc = cuda_status(cudaStreamSynchronize(s));
    if (rc) return rc;
    int32_t st = 0;
    rc = cuda_status(cudaMemcpy(&st, ws, sizeof(st), cudaMemcpyDeviceToHost));
    if (rc) return rc;
    rc = cuda_status(cudaMemset(ws, 0, sizeof(st)));
    if (rc) return rc;
    return st;
}

#define GPT_TRY(expr)               \
    do {                            \
        int _rc = (expr);           \
        if (_rc != GPT_OK) return _rc; \
    } while (0)

// One pre-LN Block ("nanoGPT 全局流程图", §2.5): x += attn(ln_1(x)); x += mlp(ln_2(x)).
// With kv_layer set, the layer's k and v of positions [0, T) are also copied into that cache
// ([B, block_size, 2C]) for incremental decoding.
int run_block(const gpt_config_t* c, const Weights& W, int l, float* x, int B, int T, uint8_t* ws,
              const Plan& P, cudaStream_t s, void* kv_layer = nullptr) {
    const int C = c->n_embd, nh = c->n_head, hs = C / nh;
    const int N = B * T;
    int32_t* status = status_word(ws);
    void* u = ws + P.u;
    void* qkv = ws + P.qkv;
    void* y = ws + P.y;
    void* h = ws + P.h;
    GPT_TRY(launch_layernorm(x, W.layer(l, W_LN1_W), W.bias(l, W_LN1_B), u, N, C, c->dtype, s));
    if (c->dtype == GPT_DTYPE_BF16) {
        const bf16* ub = static_cast<const bf16*>(u);
        bf16* qkvb = static_cast<bf16*>(qkv);
        GPT_TRY(launch_gemm_bf16(ub, C, static_cast<const bf16*>(W.layer(l, W_ATTN_W)), C,
                                 static_cast<const bf16*>(W.bias(l, W_ATTN_B)), qkv, 3LL * C, N, 3 * C, C,
                                 GPT_EPI_STORE, c->gelu, nullptr, status, s));
        if (kv_layer) GPT_TRY(launch_kv_store(qkv, kv_layer, B, T, C, 2, c->block_size, s));
        AttnLayout L{};
        L.q = qkvb;
        L.k = qkvb + C;
        L.v = qkvb + 2 * C;
        L.sb = 3LL * C * T;
        L.sh = hs;
        L.st = 3LL * C;
        L.y = static_cast<bf16*>(y);
        L.y_sb = static_cast<long long>(C) * T;
        L.y_sh = hs;
        L.y_st = C;
        GPT_TRY(launch_attention_bf16(L, B, nh, T, status, s));
        GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(y), C, static_cast<const bf16*>(W.layer(l, W_PROJ_W)), C,
                                 static_cast<const bf16*>(W.bias(l, W_PROJ_B)), x, C, N, C, C, GPT_EPI_RESID,
                                 c->gelu, nullptr, status, s));
        GPT_TRY(launch_layernorm(x, W.layer(l, W_LN2_W), W.bias(l, W_LN2_B), u, N, C, c->dtype, s));
        GPT_TRY(launch_gemm_bf16(ub, C, static_cast<const bf16*>(W.layer(l, W_FC_W)), C,
                                 static_cast<const bf16*>(W.bias(l, W_FC_B)), h, 4LL * C, N, 4 * C, C,
                                 GPT_EPI_GELU, c->gelu, nullptr, status, s));
        GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(h), 4LL * C, static_cast<const bf16*>(W.layer(l, W_FC2_W)),
                                 4LL * C, static_cast<const bf16*>(W.bias(l, W_FC2_B)), x, C, N, C, 4 * C,
                                 GPT_EPI_RESID, c->gelu, nullptr, status, s));
    } else {
        const float* uf = static_cast<const float*>(u);
        float* qkvf = static_cast<float*>(qkv);
        GPT_TRY(launch_linear_f32(uf, C, static_cast<const float*>(W.layer(l, W_ATTN_W)),
                                  static_cast<const float*>(W.bias(l, W_ATTN_B)), qkvf, 3LL * C, N, 3 * C, C,
                                  GPT_EPI_STORE, c->gelu, s));
        if (kv_layer) GPT_TRY(launch_kv_store(qkv, kv_layer, B, T, C, 4, c->block_size, s));
        AttnLayoutF32 L{};
        L.q = qkvf;
        L.k = qkvf + C;
        L.v = qkvf + 2 * C;
        L.sb = 3LL * C * T;
        L.sh = hs;
        L.st = 3LL * C;
        L.y = static_cast<float*>(y);
        L.y_sb = static_cast<long long>(C) * T;
        L.y_sh = hs;
        L.y_st = C;
        GPT_TRY(launch_attention_f32(L, B, nh, T, hs, s));
        GPT_TRY(launch_linear_f32(static_cast<const float*>(y), C, static_cast<const float*>(W.layer(l, W_PROJ_W)),
                                  static_cast<const float*>(W.bias(l, W_PROJ_B)), x, C, N, C, C, GPT_EPI_RESID,
                                  c->gelu, s));
        GPT_TRY(launch_layernorm(x, W.layer(l, W_LN2_W), W.bias(l, W_LN2_B), u, N, C, c->dtype, s));
        GPT_TRY(launch_linear_f32(uf, C, static_cast<const float*>(W.layer(l, W_FC_W)),
                                  static_cast<const float*>(W.bias(l, W_FC_B)), static_cast<float*>(h), 4LL * C, N,
                                  4 * C, C, GPT_EPI_GELU, c->gelu, s));
        GPT_TRY(launch_linear_f32(static_cast<const float*>(h), 4LL * C, static_cast<const float*>(W.layer(l, W_FC2_W)),
                                  static_cast<const float*>(W.bias(l, W_FC2_B)), x, C, N, C, 4 * C, GPT_EPI_RESID,
                                  c->gelu, s));
    }
    return GPT_OK;
}

void fill_weights(Weights& W, const gpt_config_t* c, const void* base) {
    W.base = static_cast<const uint8_t*>(base);
    W.c = c;
    size_t offs[2 + kTensorsPerLayer + 2];
    gpt_config_t one = *c;
    one.n_layer = 1;
    layout(&one, offs, nullptr, 2 + kTensorsPerLayer + 2);
    W.head = offs[2];
    for (int i = 0; i < kTensorsPerLayer; ++i) W.in_layer[i] = offs[2 + i] - W.head;
    W.layer_bytes = offs[2 + kTensorsPerLayer] - W.head;
    W.tail = W.head + W.layer_bytes * static_cast<size_t>(c->n_layer);
}

int check_common(const gpt_config_t* c, const void* weights, int B, int T, void* ws, size_t ws_bytes,
                 Plan* P) {
    GPT_TRY(validate(c));
    if (!weights || !ws) return GPT_ERR_NULL;
    if (B < 1 || T < 1 || T > c->block_size) return GPT_ERR_BAD_SHAPE;
    if (static_cast<long long>(B) * T > 0x7fffffffLL / 4 / c->n_embd) return GPT_ERR_UNSUPPORTED;
    if (!aligned(weights, 256) || !aligned(ws, 256)) return GPT_ERR_BAD_ALIGN;
    *P = plan_ws(c, B, T);
    if (ws_bytes < P->total) return GPT_ERR_WS_TOO_SMALL;
    return GPT_OK;
}

// ------------------------------------------------------------------ incremental decoding
// Workspace of the decoding entry points.  The state that lives across calls, and the buffers
// whose size does not depend on the prefill length, come first at fixed offsets (the control
// block with the status word at byte 0 and the decode position at byte 4, the attention merge
// counters, the split-attention partials, fp32 logits [B, V], a token window [B, block_size]);
// then the forward plan for a prefill of up to T_pref positions, whose buffers also hold the
// one-row-per-sequence activations of a decode step.  A prefill and the decode steps after it
// may therefore size the workspace for different T_pref.
struct DecodePlan {
    Plan P;
    size_t counter, part, logits, window, total;
};

DecodePlan plan_decode(const gpt_config_t* c, int B, int T_pref) {
    DecodePlan D;
    const int hs = c->n_embd / c->n_head;
    size_t off = 256;
    D.counter = off; off += a256(static_cast<size_t>(B) * c->n_head * 4);
    D.part = off; off += a256(decode_attn_part_floats(B, c->n_head, hs, c->block_size) * 4);
    D.logits = off; off += a256(static_cast<size_t>(B) * c->vocab_size * 4);
    D.window = off; off += a256(static_cast<size_t>(B) * c->block_size * 8);
    // the forward plan shares the control block at 0; its buffers move past the fixed region
    Plan P = plan_ws(c, B, T_pref);
    const size_t shift = off - 256;
    for (size_t* f : {&P.x, &P.u, &P.qkv, &P.y, &P.h, &P.part, &P.tlogit, &P.rowloss, &P.total}) *f += shift;
    D.P = P;
    D.total = P.total;
    return D;
}

int* pos_word(void* ws) { return reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + 4); }

size_t kv_layer_bytes(const gpt_config_t* c, int B) {
    return static_cast<size_t>(B) * c->block_size * 2 * c->n_embd * elem_size(c);
}

int validate_decode(const gpt_config_t* c) {
    GPT_TRY(validate(c));
    const int hs = c->n_embd / c->n_head;
    if ((c->n_embd % 8) || (hs % 8) || hs > 128) return GPT_ERR_UNSUPPORTED;
    return GPT_OK;
}

int check_decode(const gpt_config_t* c, const void* weights, int B, const void* kv, void* ws, size_t ws_bytes,
                 int T_pref, DecodePlan* D) {
    GPT_TRY(validate_decode(c));
    if (!weights || !kv || !ws) return GPT_ERR_NULL;
    if (B < 1 || T_pref < 1 || T_pref > c->block_size) return GPT_ERR_BAD_SHAPE;
    if (static_cast<long long>(B) * c->block_size > 0x7fffffffLL / 4 / c->n_embd) return GPT_ERR_UNSUPPORTED;
    if (B > 65535 / c->n_head) return GPT_ERR_UNSUPPORTED;
    if (!aligned(weights, 256) || !aligned(ws, 256) || !aligned(kv, 16)) return GPT_ERR_BAD_ALIGN;
    *D = plan_decode(c, B, T_pref);
    if (ws_bytes < D->total) return GPT_ERR_WS_TOO_SMALL;
    return GPT_OK;
}

// Forward over idx [B, T] (contiguous) that fills every layer's cache at positions [0, T),
// then logits fp32 [B, V] of position T-1 at row stride ldl, and sets the decode position to T.
int prefill_impl(const gpt_config_t* c, const Weights& W, const int64_t* idx, int B, int T, uint8_t* kv,
                 float* logits, long long ldl, uint8_t* ws, const DecodePlan& D, cudaStream_t s) {
    const int C = c->n_embd, V = c->vocab_size, N = B * T;
    const Plan& P = D.P;
    int32_t* status = status_word(ws);
    float* x = reinterpret_cast<float*>(ws + P.x);
    void* u = ws + P.u;
    GPT_TRY(launch_embed(W.wte(), W.wpe(), idx, x, B, T, C, V, c->dtype, status, s));
    for (int l = 0; l < c->n_layer; ++l)
        GPT_TRY(run_block(c, W, l, x, B, T, ws, P, s, kv + kv_layer_bytes(c, B) * l));
    GPT_TRY(launch_layernorm(x, W.lnf_w(), W.lnf_b(), u, N, C, c->dtype, s));
    const uint8_t* ulast = static_cast<const uint8_t*>(u) + static_cast<size_t>(T - 1) * C * elem_size(c);
    GPT_TRY(launch_gemv(3, false, c->dtype, ulast, static_cast<long long>(T) * C, nullptr, nullptr, W.wte(), nullptr,
                        logits, ldl, B, V, C, c->gelu == GPT_GELU_TANH, nullptr, nullptr, C, c->block_size, 0, s));
    return launch_decode_reset(pos_word(ws), T, reinterpret_cast<int*>(ws + D.counter), B * c->n_head, s);
}

// One token per sequence (tok[b * ld_tok]) at the decode position p: every layer appends its
// k, v at p and attends over positions [0, p]; logits fp32 [B, V] at row stride ldl; p += 1.
int decode_step_impl(const gpt_config_t* c, const Weights& W, const int64_t* tok, long long ld_tok, int B,
                     uint8_t* kv, float* logits, long long ldl, uint8_t* ws, const DecodePlan& D, cudaStream_t s) {
    const int C = c->n_embd, V = c->vocab_size, nh = c->n_head, hs = C / nh, bs = c->block_size;
    const int dt = c->dtype, gt = c->gelu == GPT_GELU_TANH;
    const Plan& P = D.P;
    int32_t* status = status_word(ws);
    int* pos = pos_word(ws);
    float* x = reinterpret_cast<float*>(ws + P.x);
    void* q = ws + P.qkv;
    void* y = ws + P.y;
    void* h = ws + P.h;
    float* part = reinterpret_cast<float*>(ws + D.part);
    int* counter = reinterpret_cast<int*>(ws + D.counter);
    if (decode_persistent_supported(dt, B, C, hs, V, c->bias)) {
        // the whole step in one cooperative launch with grid barriers between its phases
        long long off[kTensorsPerLayer];
        for (int i = 0; i < kTensorsPerLayer; ++i) off[i] = static_cast<long long>(W.in_layer[i]);
        return launch_decode_persistent(W.wte(), W.wpe(), W.layer(0, 0), static_cast<long long>(W.layer_bytes), off,
                                        c->bias, W.lnf_w(), W.lnf_b(), tok, ld_tok, kv,
                                        static_cast<long long>(kv_layer_bytes(c, B) / 2), logits, ldl, pos, x, q, y,
                                        h, part, counter,
                                        static_cast<int>(decode_attn_part_floats(1, 1, hs, bs) / (hs + 2)),
                                        reinterpret_cast<unsigned*>(ws + 8), status, B, C, nh, V, c->n_layer, bs, gt,
                                        s);
    }
    GPT_TRY(launch_embed_pos(W.wte(), W.wpe(), tok, ld_tok, pos, x, B, C, V, bs, dt, status, s));
    for (int l = 0; l < c->n_layer; ++l) {
        uint8_t* kvl = kv + kv_layer_bytes(c, B) * l;
        // q, k, v = c_attn(ln_1(x)); k, v appended to the cache at the position
        GPT_TRY(launch_gemv(4, true, dt, x, C, W.layer(l, W_LN1_W), W.bias(l, W_LN1_B), W.layer(l, W_ATTN_W),
                            W.bias(l, W_ATTN_B), q, C, B, 3 * C, C, gt, kvl, pos, C, bs, 0, s));
        GPT_TRY(launch_decode_attention(dt, q, kvl, pos, part, counter, y, B, nh, hs, bs, s));
        GPT_TRY(launch_gemv(2, false, dt, y, C, nullptr, nullptr, W.layer(l, W_PROJ_W), W.bias(l, W_PROJ_B), x, C,
                            B, C, C, gt, nullptr, nullptr, C, bs, 0, s));
        GPT_TRY(launch_gemv(1, true, dt, x, C, W.layer(l, W_LN2_W), W.bias(l, W_LN2_B), W.layer(l, W_FC_W),
                            W.bias(l, W_FC_B), h, 4LL * C, B, 4 * C, C, gt, nullptr, nullptr, C, bs, 0, s));
        GPT_TRY(launch_gemv(2, false, dt, h, 4LL * C, nullptr, nullptr, W.layer(l, W_FC2_W), W.bias(l, W_FC2_B), x,
                            C, B, C, 4 * C, gt, nullptr, nullptr, C, bs, 0, s));
    }
    // logits = ln_f(x) wte^T; the same kernel advances the position
    return launch_gemv(3, true, dt, x, C, W.lnf_w(), W.lnf_b(), W.wte(), nullptr, logits, ldl, B, V, C, gt, nullptr,
                       pos, C, bs, 1, s);
}

// The widest prefill gpt_generate runs: the prompt (cropped to the window), or a full window
// once the sequence outgrows it.
int generate_prefill_len(const gpt_config_t* c, int T0, int max_new_tokens) {
    const long long longest = static_cast<long long>(T0) + (max_new_tokens > 0 ? max_new_tokens - 1 : 0);
    return longest > c->block_size ? c->block_size : T0;
}

int check_sample_args(int B, int V, float temperature, const float* logits, const float* u, const int64_t* out) {
    if (!logits || !u || !out) return GPT_ERR_NULL;
    if (B < 1 || V < 1) return GPT_ERR_BAD_SHAPE;
    if (!(temperature > 0.f) || !isfinite(temperature)) return GPT_ERR_BAD_SHAPE;
    if (V > sample_max_vocab()) return GPT_ERR_UNSUPPORTED;
    return GPT_OK;
}

}  // namespace

// =================================================================== exported ABI
GPT_API const char* gpt_status_string(int status) {
    switch (status) {
        case GPT_OK: return "ok";
        case GPT_ERR_NULL: return "a required pointer is NULL";
        case GPT_ERR_BAD_SHAPE: return "inconsistent sizes";
        case GPT_ERR_BAD_ALIGN: return "pointer not aligned";
        case GPT_ERR_WS_TOO_SMALL: return "workspace too small";
        case GPT_ERR_INDEX: return "token id or target out of range";
        case GPT_ERR_TIMEOUT: return "device pipeline wait timed out";
        case GPT_ERR_UNSUPPORTED: return "unsupported configuration";
        case GPT_ERR_CUDA: return "CUDA runtime error";
        default: return "unknown status";
    }
}

GPT_API int gpt_abi_version(void) { return GPT_ABI_VERSION; }

GPT_API const char* gpt_last_cuda_error(void) {
    return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

GPT_API int gpt_validate_config(const gpt_config_t* cfg) { return validate(cfg); }

GPT_API size_t gpt_weights_bytes(const gpt_config_t* cfg) {
    if (validate(cfg) != GPT_OK) return 0;
    return weights_total(cfg);
}

GPT_API int gpt_weights_count(const gpt_config_t* cfg) {
    const int rc = validate(cfg);
    if (rc != GPT_OK) return rc;
    return 2 + kTensorsPerLayer * cfg->n_layer + 2;
}

GPT_API int gpt_weights_layout(const gpt_config_t* cfg, size_t* offsets, size_t* numels, int n) {
    const int rc = validate(cfg);
    if (rc != GPT_OK) return rc;
    return layout(cfg, offsets, numels, n < 0 ? 0 : n);
}

GPT_API size_t gpt_workspace_bytes(const gpt_config_t* cfg, int B, int T) {
    if (validate(cfg) != GPT_OK || B < 1 || T < 1 || T > cfg->block_size) return 0;
    return plan_ws(cfg, B, T).total;
}

GPT_API int gpt_set_wait_limit_ns(unsigned long long ns, int force_timeout) {
    GPT_TRY(set_wait_limit_attention(ns, force_timeout));
    GPT_TRY(set_wait_limit_gemm(ns, force_timeout));
    GPT_TRY(set_wait_limit_head(ns, force_timeout));
    GPT_TRY(set_wait_limit_decode(ns, force_timeout));
    return set_wait_limit_attention_bwd(ns, force_timeout);
}

GPT_API int gpt_check_status(void* workspace, void* stream) {
    if (!workspace) return GPT_ERR_NULL;
    return sync_and_read_status(workspace, static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_forward(const gpt_config_t* cfg, const void* weights, const int64_t* idx, const int64_t* targets,
                        int B, int T, void* logits, float* loss, float* row_loss, double* loss_sum_count,
                        void* workspace, size_t workspace_bytes, void* stream, int flags) {
    Plan P;
    GPT_TRY(check_common(cfg, weights, B, T, workspace, workspace_bytes, &P));
    if (!idx || !logits) return GPT_ERR_NULL;
    if (!aligned(logits, 16)) return GPT_ERR_BAD_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Weights W;
    fill_weights(W, cfg, weights);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* status = status_word(ws);
    const int C = cfg->n_embd, V = cfg->vocab_size, N = B * T;
    float* x = reinterpret_cast<float*>(ws + P.x);
    void* u = ws + P.u;

    GPT_TRY(cuda_status(cudaMemsetAsync(status, 0, sizeof(int32_t), s)));
    GPT_TRY(launch_embed(W.wte(), W.wpe(), idx, x, B, T, C, V, cfg->dtype, status, s));
    for (int l = 0; l < cfg->n_layer; ++l) GPT_TRY(run_block(cfg, W, l, x, B, T, ws, P, s));

    if (!targets && head_last_supported(C, B, cfg->dtype)) {
        // Inference branch: only the last position's logits, [B, 1, V] (§3.2 ④): ln_f of the B
        // last residual rows fused into one HBM-bound pass over wte (per 16 rows).
        GPT_TRY(launch_head_last(x + static_cast<long long>(T - 1) * C, static_cast<long long>(T) * C, W.lnf_w(),
                                 W.lnf_b(), W.wte(), B, C, V, cfg->dtype, logits, status, s));
        if (flags & GPT_FLAG_SYNC_CHECK) return sync_and_read_status(ws, s);
        return GPT_OK;
    }
    GPT_TRY(launch_layernorm(x, W.lnf_w(), W.lnf_b(), u, N, C, cfg->dtype, s));

    if (targets) {
        float* rl = row_loss ? row_loss : reinterpret_cast<float*>(ws + P.rowloss);
        if (cfg->dtype == GPT_DTYPE_BF16) {
            CeArgs ce{targets, reinterpret_cast<float2*>(ws + P.part), reinterpret_cast<float*>(ws + P.tlogit),
                      P.n_part};
            GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(u), C, static_cast<const bf16*>(W.wte()), C, nullptr,
                                     logits, V, N, V, C, 3 /* EPI_CE */, cfg->gelu, &ce, status, s));
            GPT_TRY(launch_ce_rows_from_parts(ce.part, P.n_part, ce.tlogit, targets, N, V, rl, status, s));
        } else {
            GPT_TRY(launch_linear_f32(static_cast<const float*>(u), C, static_cast<const float*>(W.wte()), nullptr,
                                      static_cast<float*>(logits), V, N, V, C, GPT_EPI_STORE, cfg->gelu, s));
            GPT_TRY(launch_ce_rows_from_logits(static_cast<const float*>(logits), targets, N, V, rl, status, s));
        }
        GPT_TRY(launch_loss_finalize(rl, targets, N, V, loss, loss_sum_count, s));
    } else {
        // Inference branch for widths the fused head above does not take: ln_f over every row,
        // then the product of the last rows.
        const long long lda = static_cast<long long>(T) * C;
        if (cfg->dtype == GPT_DTYPE_BF16) {
            const bf16* ulast = static_cast<const bf16*>(u) + static_cast<long long>(T - 1) * C;
            GPT_TRY(launch_gemm_bf16(ulast, lda, static_cast<const bf16*>(W.wte()), C, nullptr, logits, V, B, V, C,
                                     GPT_EPI_STORE, cfg->gelu, nullptr, status, s));
        } else {
            const float* ulast = static_cast<const float*>(u) + static_cast<long long>(T - 1) * C;
            GPT_TRY(launch_linear_f32(ulast, lda, static_cast<const float*>(W.wte()), nullptr,
                                      static_cast<float*>(logits), V, B, V, C, GPT_EPI_STORE, cfg->gelu, s));
        }
    }
    if (flags & GPT_FLAG_SYNC_CHECK) return sync_and_read_status(ws, s);
    return GPT_OK;
}

GPT_API int gpt_lm_head_last(const float* x, long long ldx, const void* lnf_w, const void* lnf_b, const void* wte,
                             int B, int C, int V, int dtype, void* logits, int32_t* status, void* stream) {
    if (!x || !lnf_w || !wte || !logits) return GPT_ERR_NULL;
    if (B < 1 || C < 1 || V < 1 || ldx < C) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (!head_last_supported(C, B, dtype)) return GPT_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || (ldx % 4) || !aligned(wte, 16)) return GPT_ERR_BAD_ALIGN;
    return launch_head_last(x, ldx, lnf_w, lnf_b, wte, B, C, V, dtype, logits, status,
                            static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_block(const gpt_config_t* cfg, const void* weights, int layer, float* x, int B, int T,
                      void* workspace, size_t workspace_bytes, void* stream, int flags) {
    Plan P;
    GPT_TRY(check_common(cfg, weights, B, T, workspace, workspace_bytes, &P));
    if (!x) return GPT_ERR_NULL;
    if (layer < 0 || layer >= cfg->n_layer) return GPT_ERR_BAD_SHAPE;
    if (!aligned(x, 16)) return GPT_ERR_BAD_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Weights W;
    fill_weights(W, cfg, weights);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    GPT_TRY(cuda_status(cudaMemsetAsync(status_word(ws), 0, sizeof(int32_t), s)));
    GPT_TRY(run_block(cfg, W, layer, x, B, T, ws, P, s));
    if (flags & GPT_FLAG_SYNC_CHECK) return sync_and_read_status(ws, s);
    return GPT_OK;
}

GPT_API int gpt_attention(const void* q, const void* k, const void* v, void* y, int B, int nh, int T, int hs,
                          int dtype, int32_t* status, void* stream) {
    if (!q || !k || !v || !y) return GPT_ERR_NULL;
    if (B < 0 || nh < 0 || T < 0 || hs <= 0) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(y, 16)) return GPT_ERR_BAD_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long sh = static_cast<long long>(T) * hs, sb = sh * nh;
    if (dtype == GPT_DTYPE_BF16) {
        if (hs != 64) return GPT_ERR_UNSUPPORTED;
        AttnLayout L{static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v), sb, sh, hs,
                     static_cast<bf16*>(y), sb, sh, hs};
        return launch_attention_bf16(L, B, nh, T, status, s);
    }
    if (hs > 128) return GPT_ERR_UNSUPPORTED;
    AttnLayoutF32 L{static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), sb, sh, hs,
                    static_cast<float*>(y), sb, sh, hs};
    return launch_attention_f32(L, B, nh, T, hs, s);
}

GPT_API int gpt_embed(const void* wte, const void* wpe, const int64_t* idx, float* x, int B, int T, int C, int V,
                      int dtype, int32_t* status, void* stream) {
    if (!wte || !wpe || !idx || !x) return GPT_ERR_NULL;
    if (B < 0 || T < 0 || C <= 0 || V <= 0 || (C % 4)) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (!aligned(wte, 16) || !aligned(wpe, 16) || !aligned(x, 16)) return GPT_ERR_BAD_ALIGN;
    return launch_embed(wte, wpe, idx, x, B, T, C, V, dtype, status, static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_layernorm(const float* x, const void* w, const void* b, void* out, int rows, int C, int dtype,
                          void* stream) {
    if (!x || !w || !out) return GPT_ERR_NULL;
    if (rows < 0 || C <= 0 || (C % 4)) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(out, 16) || (b && !aligned(b, 16))) return GPT_ERR_BAD_ALIGN;
    return launch_layernorm(x, w, b, out, rows, C, dtype, static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_linear(const void* x, const void* W, const void* b, void* out, int M, int N, int K, int dtype,
                       int epilogue, int gelu, int32_t* status, void* stream) {
    if (!x || !W || !out) return GPT_ERR_NULL;
    if (M < 0 || N <= 0 || K <= 0) return GPT_ERR_BAD_SHAPE;
    if (epilogue != GPT_EPI_STORE && epilogue != GPT_EPI_GELU && epilogue != GPT_EPI_RESID) return GPT_ERR_BAD_SHAPE;
    if (gelu != GPT_GELU_ERF && gelu != GPT_GELU_TANH) return GPT_ERR_BAD_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == GPT_DTYPE_BF16) {
        if ((K % 8) || (N % 8)) return GPT_ERR_UNSUPPORTED;
        if (!aligned(x, 16) || !aligned(W, 16) || !aligned(out, 16) || (b && !aligned(b, 16))) return GPT_ERR_BAD_ALIGN;
        return launch_gemm_bf16(static_cast<const bf16*>(x), K, static_cast<const bf16*>(W), K,
                                static_cast<const bf16*>(b), out, N, M, N, K, epilogue, gelu, nullptr, status, s);
    }
    if (dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    return launch_linear_f32(static_cast<const float*>(x), K, static_cast<const float*>(W),
                             static_cast<const float*>(b), static_cast<float*>(out), N, M, N, K, epilogue, gelu, s);
}

GPT_API size_t gpt_lm_head_workspace_bytes(int rows, int V) {
    if (rows < 1 || V < 1) return 0;
    const size_t n = rows;
    return 256 + a256(n * static_cast<size_t>(gemm_ce_parts(V)) * 8) + a256(n * 4) + a256(n * 4);
}

GPT_API int gpt_lm_head_loss(const void* u, const void* wte, const int64_t* targets, int rows, int C, int V,
                             int dtype, void* logits, float* loss, float* row_loss, double* loss_sum_count,
                             void* workspace, size_t workspace_bytes, void* stream, int flags) {
    if (!u || !wte || !targets || !logits || !workspace) return GPT_ERR_NULL;
    if (rows < 1 || C <= 0 || V <= 0) return GPT_ERR_BAD_SHAPE;
    if (workspace_bytes < gpt_lm_head_workspace_bytes(rows, V)) return GPT_ERR_WS_TOO_SMALL;
    if (!aligned(workspace, 256) || !aligned(u, 16) || !aligned(wte, 16) || !aligned(logits, 16))
        return GPT_ERR_BAD_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* status = status_word(ws);
    const size_t n = rows;
    const int n_part = gemm_ce_parts(V);
    float2* part = reinterpret_cast<float2*>(ws + 256);
    float* tlogit = reinterpret_cast<float*>(ws + 256 + a256(n * n_part * 8));
    float* rl_ws = reinterpret_cast<float*>(ws + 256 + a256(n * n_part * 8) + a256(n * 4));
    float* rl = row_loss ? row_loss : rl_ws;
    GPT_TRY(cuda_status(cudaMemsetAsync(status, 0, sizeof(int32_t), s)));
    if (dtype == GPT_DTYPE_BF16) {
        if ((C % 8) || (V % 8)) return GPT_ERR_UNSUPPORTED;
        CeArgs ce{targets, part, tlogit, n_part};
        GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(u), C, static_cast<const bf16*>(wte), C, nullptr, logits, V,
                                 rows, V, C, 3 /* EPI_CE */, GPT_GELU_ERF, &ce, status, s));
        GPT_TRY(launch_ce_rows_from_parts(part, n_part, tlogit, targets, rows, V, rl, status, s));
    } else if (dtype == GPT_DTYPE_F32) {
        GPT_TRY(launch_linear_f32(static_cast<const float*>(u), C, static_cast<const float*>(wte), nullptr,
                                  static_cast<float*>(logits), V, rows, V, C, GPT_EPI_STORE, GPT_GELU_ERF, s));
        GPT_TRY(launch_ce_rows_from_logits(static_cast<const float*>(logits), targets, rows, V, rl, status, s));
    } else {
        return GPT_ERR_BAD_SHAPE;
    }
    GPT_TRY(launch_loss_finalize(rl, targets, rows, V, loss, loss_sum_count, s));
    if (flags & GPT_FLAG_SYNC_CHECK) return sync_and_read_status(ws, s);
    return GPT_OK;
}

// ------------------------------------------------------------------ generation (decode.cu)
GPT_API size_t gpt_kv_cache_bytes(const gpt_config_t* cfg, int B) {
    if (validate_decode(cfg) != GPT_OK || B < 1) return 0;
    return kv_layer_bytes(cfg, B) * cfg->n_layer;
}

GPT_API size_t gpt_decode_workspace_bytes(const gpt_config_t* cfg, int B, int T_prefill) {
    if (validate_decode(cfg) != GPT_OK || B < 1 || T_prefill < 1 || T_prefill > cfg->block_size) return 0;
    return plan_decode(cfg, B, T_prefill).total;
}

GPT_API size_t gpt_generate_workspace_bytes(const gpt_config_t* cfg, int B, int T0, int max_new_tokens) {
    if (validate_decode(cfg) != GPT_OK || B < 1 || T0 < 1 || max_new_tokens < 0) return 0;
    return plan_decode(cfg, B, generate_prefill_len(cfg, T0, max_new_tokens)).total;
}

GPT_API int gpt_prefill(const gpt_config_t* cfg, const void* weights, const int64_t* idx, int B, int T,
                        void* kv_cache, float* logits, void* workspace, size_t workspace_bytes, void* stream,
                        int flags) {
    DecodePlan D;
    GPT_TRY(check_decode(cfg, weights, B, kv_cache, workspace, workspace_bytes, T, &D));
    if (!idx || !logits) return GPT_ERR_NULL;
    if (!aligned(logits, 16)) return GPT_ERR_BAD_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Weights W;
    fill_weights(W, cfg, weights);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    GPT_TRY(cuda_status(cudaMemsetAsync(status_word(ws), 0, sizeof(int32_t), s)));
    GPT_TRY(prefill_impl(cfg, W, idx, B, T, static_cast<uint8_t*>(kv_cache), logits, cfg->vocab_size, ws, D, s));
    if (flags & GPT_FLAG_SYNC_CHECK) return sync_and_read_status(ws, s);
    return GPT_OK;
}

GPT_API int gpt_decode_step(const gpt_config_t* cfg, const void* weights, const int64_t* tok, long long ld_tok, int B,
                            void* kv_cache, float* logits, void* workspace, size_t workspace_bytes, void* stream,
                            int flags) {
    DecodePlan D;
    GPT_TRY(check_decode(cfg, weights, B, kv_cache, workspace, workspace_bytes, 1, &D));
    if (!tok || !logits) return GPT_ERR_NULL;
    if (!aligned(logits, 16)) return GPT_ERR_BAD_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Weights W;
    fill_weights(W, cfg, weights);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    GPT_TRY(decode_step_impl(cfg, W, tok, ld_tok, B, static_cast<uint8_t*>(kv_cache), logits, cfg->vocab_size, ws,
                             D, s));
    if (flags & GPT_FLAG_SYNC_CHECK) return sync_and_read_status(ws, s);
    return GPT_OK;
}

GPT_API int gpt_sample(const float* logits, int B, int V, float temperature, int top_k, const float* u, int64_t* out,
                       long long ld_out, void* stream) {
    GPT_TRY(check_sample_args(B, V, temperature, logits, u, out));
    return launch_sample(logits, V, B, V, temperature, top_k, u, out, ld_out, static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_generate(const gpt_config_t* cfg, const void* weights, const int64_t* idx, int B, int T0,
                         int max_new_tokens, float temperature, int top_k, const float* uniforms, int64_t* out,
                         float* step_logits, void* kv_cache, void* workspace, size_t workspace_bytes, void* stream,
                         int flags) {
    GPT_TRY(validate_decode(cfg));
    if (!idx || !out || (max_new_tokens > 0 && !uniforms)) return GPT_ERR_NULL;
    if (B < 1 || T0 < 1 || max_new_tokens < 0) return GPT_ERR_BAD_SHAPE;
    if (static_cast<long long>(T0) + max_new_tokens > 0x7fffffffLL) return GPT_ERR_BAD_SHAPE;
    if (max_new_tokens > 0 && (!(temperature > 0.f) || !isfinite(temperature))) return GPT_ERR_BAD_SHAPE;
    if (max_new_tokens > 0 && cfg->vocab_size > sample_max_vocab()) return GPT_ERR_UNSUPPORTED;
    DecodePlan D;
    GPT_TRY(check_decode(cfg, weights, B, kv_cache, workspace, workspace_bytes,
                         generate_prefill_len(cfg, T0, max_new_tokens), &D));
    if (step_logits && !aligned(step_logits, 16)) return GPT_ERR_BAD_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Weights W;
    fill_weights(W, cfg, weights);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* kv = static_cast<uint8_t*>(kv_cache);
    int64_t* window = reinterpret_cast<int64_t*>(ws + D.window);
    const int V = cfg->vocab_size, bs = cfg->block_size;
    const long long ld = static_cast<long long>(T0) + max_new_tokens;
    GPT_TRY(cuda_status(cudaMemsetAsync(status_word(ws), 0, sizeof(int32_t), s)));
    GPT_TRY(launch_copy_tokens(idx, T0, out, ld, B, T0, s));
    for (int st = 0; st < max_new_tokens; ++st) {
        const long long n = static_cast<long long>(T0) + st;  // current length
        float* lg = step_logits ? step_logits + static_cast<size_t>(st) * B * V : reinterpret_cast<float*>(ws + D.logits);
        if (st == 0 || n > bs) {
            // the model sees the last min(n, block_size) tokens; once the sequence is longer than
            // the window every position shifts, so the cache is rebuilt from the window
            const int Tw = static_cast<int>(n < bs ? n : bs);
            GPT_TRY(launch_copy_tokens(out + (n - Tw), ld, window, Tw, B, Tw, s));
            GPT_TRY(prefill_impl(cfg, W, window, B, Tw, kv, lg, V, ws, D, s));
        } else {
            GPT_TRY(decode_step_impl(cfg, W, out + (n - 1), ld, B, kv, lg, V, ws, D, s));
        }
        GPT_TRY(launch_sample(lg, V, B, V, temperature, top_k, uniforms + static_cast<size_t>(st) * B, out + n, ld, s));
    }
    if (flags & GPT_FLAG_SYNC_CHECK) return sync_and_read_status(ws, s);
    return GPT_OK;
}

// ------------------------------------------------------------------ optimizer step (optim.cu)
GPT_API double gpt_lr_schedule(long long it, double learning_rate, double min_lr, long long warmup_iters,
                               long long lr_decay_iters) {
    if (it < warmup_iters) return learning_rate * static_cast<double>(it + 1) / static_cast<double>(warmup_iters + 1);
    if (it > lr_decay_iters) return min_lr;
    const double decay_ratio =
        static_cast<double>(it - warmup_iters) / static_cast<double>(lr_decay_iters - warmup_iters);
    const double coeff = 0.5 * (1.0 + cos(3.14159265358979323846 * decay_ratio));
    return min_lr + coeff * (learning_rate - min_lr);
}

GPT_API size_t gpt_param_elems(const gpt_config_t* cfg) {
    if (validate(cfg) != GPT_OK) return 0;
    return weights_total(cfg) / elem_size(cfg);
}

GPT_API size_t gpt_adamw_workspace_bytes(void) { return adamw_workspace_bytes(); }

GPT_API int gpt_adamw_step(const gpt_config_t* cfg, float* params, const float* grads, float* exp_avg,
                           float* exp_avg_sq, void* weights, const gpt_adamw_t* hp, float* grad_norm,
                           void* workspace, size_t workspace_bytes, void* stream, int flags) {
    GPT_TRY(validate(cfg));
    if (!params || !grads || !exp_avg || !exp_avg_sq || !hp || !workspace) return GPT_ERR_NULL;
    if (hp->step < 1 || !(hp->lr >= 0.f) || !isfinite(hp->lr) || !(hp->beta1 >= 0.f && hp->beta1 < 1.f) ||
        !(hp->beta2 >= 0.f && hp->beta2 < 1.f) || !(hp->eps > 0.f) || !(hp->weight_decay >= 0.f) ||
        !isfinite(hp->max_grad_norm))
        return GPT_ERR_BAD_SHAPE;
    if (workspace_bytes < adamw_workspace_bytes()) return GPT_ERR_WS_TOO_SMALL;
    if (!aligned(params, 16) || !aligned(grads, 16) || !aligned(exp_avg, 16) || !aligned(exp_avg_sq, 16) ||
        !aligned(workspace, 256) || (weights && !aligned(weights, 256)) || (grad_norm && !aligned(grad_norm, 4)))
        return GPT_ERR_BAD_ALIGN;
    const int count = 2 + kTensorsPerLayer * cfg->n_layer + 2;
    if (count > kOptMaxTensors) return GPT_ERR_UNSUPPORTED;
    static thread_local OptTable tab;  // ~25 KB: not on the stack
    size_t offs[kOptMaxTensors], numels[kOptMaxTensors];
    layout(cfg, offs, numels, count);
    const long long ch = opt_chunk_elems();
    long long chunks = 0;
    int n = 0;
    for (int i = 0; i < count; ++i) {
        // configure_optimizers: decay iff the tensor has two dimensions (wte, wpe, the four
        // Linear weights of a layer).  Without biases (cfg->bias == 0) the bias slots are not
        // parameters: they are skipped like padding.
        bool two_d = i < 2, is_bias = i == count - 1;
        if (i >= 2 && i < 2 + kTensorsPerLayer * cfg->n_layer) {
            const int j = (i - 2) % kTensorsPerLayer;
            two_d = j == W_ATTN_W || j == W_PROJ_W || j == W_FC_W || j == W_FC2_W;
            is_bias = j == W_LN1_B || j == W_ATTN_B || j == W_PROJ_B || j == W_LN2_B || j == W_FC_B || j == W_FC2_B;
        }
        if (is_bias && !cfg->bias) continue;
        tab.off[n] = static_cast<long long>(offs[i] / elem_size(cfg));
        tab.numel[n] = static_cast<long long>(numels[i]);
        if (tab.numel[n] % 4) return GPT_ERR_UNSUPPORTED;  // float4 rows
        tab.decay[n] = two_d ? 1 : 0;
        tab.chunk0[n] = chunks;
        chunks += (tab.numel[n] + ch - 1) / ch;
        ++n;
    }
    tab.n = n;
    tab.chunk0[n] = chunks;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    GPT_TRY(launch_adamw(tab, cfg->dtype, params, grads, exp_avg, exp_avg_sq, weights, hp->lr, hp->beta1, hp->beta2,
                         hp->eps, hp->weight_decay, hp->step, hp->max_grad_norm, grad_norm, workspace, s));
    if (flags & GPT_FLAG_SYNC_CHECK) return cuda_status(cudaStreamSynchronize(s));
    return GPT_OK;
}

// ------------------------------------------------------------------ backward pieces (backward.cu)
GPT_API int gpt_cross_entropy_backward(const void* logits, const int64_t* targets, const double* loss_sum_count,
                                       int rows, int V, int dtype, void* dlogits, int32_t* status, void* stream) {
    if (!logits || !targets || !loss_sum_count || !dlogits) return GPT_ERR_NULL;
    if (rows < 0 || V <= 0) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (rows == 0) return GPT_OK;
    return launch_ce_backward(logits, dtype, targets, loss_sum_count, dlogits, rows, V, status,
                              static_cast<cudaStream_t>(stream));
}

GPT_API size_t gpt_layernorm_backward_workspace_bytes(int rows, int C) {
    if (rows < 1 || C < 1) return 0;
    return a256(static_cast<size_t>(layernorm_backward_parts(rows, C)) * 2 * C * 4);
}

GPT_API int gpt_layernorm_backward(const float* dy, const float* x, const void* w, int rows, int C, int dtype,
                                   float* dx, int accumulate, float* dw, float* db, int accumulate_wb, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    if (!dy || !x || !w || !dx || !dw || !workspace) return GPT_ERR_NULL;
    if (rows < 1 || C < 1 || C > 4096) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (workspace_bytes < gpt_layernorm_backward_workspace_bytes(rows, C)) return GPT_ERR_WS_TOO_SMALL;
    if (!aligned(workspace, 256)) return GPT_ERR_BAD_ALIGN;
    return launch_layernorm_backward(dy, x, w, dtype, dx, accumulate, dw, db, accumulate_wb,
                                     static_cast<float*>(workspace), rows, C, static_cast<cudaStream_t>(stream));
}

GPT_API size_t gpt_bias_grad_workspace_bytes(int rows, int C) {
    if (rows < 1 || C < 1) return 0;
    return a256(static_cast<size_t>(colsum_parts(rows)) * C * 4);
}

GPT_API int gpt_bias_grad(const void* dy, int rows, int C, int dtype, float* db, int accumulate, void* workspace,
                          size_t workspace_bytes, void* stream) {
    if (!dy || !db || !workspace) return GPT_ERR_NULL;
    if (rows < 1 || C < 1 || rows > 65535 * 128) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (workspace_bytes < gpt_bias_grad_workspace_bytes(rows, C)) return GPT_ERR_WS_TOO_SMALL;
    if (!aligned(workspace, 256)) return GPT_ERR_BAD_ALIGN;
    return launch_colsum(dy, dtype, rows, C, db, accumulate, static_cast<float*>(workspace),
                         static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_gelu_backward(const float* dh, const void* pre, long long n, int dtype, int gelu, void* dpre,
                              void* stream) {
    if (!dh || !pre || !dpre) return GPT_ERR_NULL;
    if (n < 0) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (gelu != GPT_GELU_ERF && gelu != GPT_GELU_TANH) return GPT_ERR_BAD_SHAPE;
    if (n == 0) return GPT_OK;
    return launch_gelu_backward(dh, pre, dtype, dpre, n, gelu == GPT_GELU_TANH, static_cast<cudaStream_t>(stream));
}

GPT_API size_t gpt_embedding_backward_workspace_bytes(int B, int T) {
    if (B < 1 || T < 1 || static_cast<long long>(B) * T > embed_backward_max_rows()) return 0;
    return a256(static_cast<size_t>(B) * T * 8);
}

GPT_API int gpt_embedding_backward(const int64_t* idx, const float* dx, int B, int T, int C, int V, float* dwte,
                                   float* dwpe, void* workspace, size_t workspace_bytes, int32_t* status,
                                   void* stream) {
    if (!idx || !dx || !dwte || !dwpe || !workspace) return GPT_ERR_NULL;
    if (B < 1 || T < 1 || C < 1 || V < 1) return GPT_ERR_BAD_SHAPE;
    if (static_cast<long long>(B) * T > embed_backward_max_rows()) return GPT_ERR_UNSUPPORTED;
    if (workspace_bytes < gpt_embedding_backward_workspace_bytes(B, T)) return GPT_ERR_WS_TOO_SMALL;
    if (!aligned(workspace, 256)) return GPT_ERR_BAD_ALIGN;
    return launch_embed_backward(idx, dx, B, T, C, V, dwte, dwpe, static_cast<unsigned long long*>(workspace), status,
                                 static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ attention for training (train.cu)
GPT_API int gpt_attention_train(const void* q, const void* k, const void* v, void* y, float* lse, int B, int nh, int T,
                                int hs, int dtype, int32_t* status, void* stream) {
    if (!q || !k || !v || !y || !lse) return GPT_ERR_NULL;
    if (B < 0 || nh < 0 || T < 0 || hs <= 0) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(y, 16)) return GPT_ERR_BAD_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long sh = static_cast<long long>(T) * hs, sb = sh * nh;
    if (dtype == GPT_DTYPE_BF16) {
        if (hs != 64) return GPT_ERR_UNSUPPORTED;
        AttnLayout L{static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v), sb, sh, hs,
                     static_cast<bf16*>(y), sb, sh, hs, lse};
        return launch_attention_bf16(L, B, nh, T, status, s);
    }
    if (hs > 128) return GPT_ERR_UNSUPPORTED;
    AttnLayoutF32 L{static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), sb, sh, hs,
                    static_cast<float*>(y), sb, sh, hs, lse};
    return launch_attention_f32(L, B, nh, T, hs, s);
}

GPT_API size_t gpt_attention_backward_workspace_bytes(int B, int nh, int T) {
    if (B < 1 || nh < 1 || T < 1) return 0;
    return a256(attn_bwd_scratch_bytes(B, nh, T));
}

GPT_API int gpt_attention_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                   const float* lse, void* dq, void* dk, void* dv, int B, int nh, int T, int hs,
                                   int dtype, void* workspace, size_t workspace_bytes, int32_t* status,
                                   void* stream) {
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return GPT_ERR_NULL;
    if (B < 0 || nh < 0 || T < 0 || hs <= 0) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (hs != 32 && hs != 64) return GPT_ERR_UNSUPPORTED;
    if (workspace_bytes < gpt_attention_backward_workspace_bytes(B, nh, T)) return GPT_ERR_WS_TOO_SMALL;
    const long long sh = static_cast<long long>(T) * hs, sb = sh * nh;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* D = static_cast<float*>(workspace);
    if (dtype == GPT_DTYPE_BF16) {
        AttnBwdLayout<bf16> L{static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v),
                              sb, sh, hs, static_cast<const bf16*>(o), static_cast<const bf16*>(dout), sb, sh, hs,
                              static_cast<bf16*>(dq), static_cast<bf16*>(dk), static_cast<bf16*>(dv), lse};
        return launch_attention_backward(&L, nullptr, B, nh, T, hs, D, status, s);
    }
    AttnBwdLayout<float> L{static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), sb,
                           sh, hs, static_cast<const float*>(o), static_cast<const float*>(dout), sb, sh, hs,
                           static_cast<float*>(dq), static_cast<float*>(dk), static_cast<float*>(dv), lse};
    return launch_attention_backward(nullptr, &L, B, nh, T, hs, D, status, s);
}

GPT_API size_t gpt_linear_backward_workspace_bytes(int rows, int n_out, int n_in, int dtype) {
    if (rows < 1 || n_out < 1 || n_in < 1) return 0;
    if (dtype == GPT_DTYPE_BF16) return 256 + a256(gemm_acc_split_bytes(n_out, n_in, rows));
    if (dtype != GPT_DTYPE_F32) return 0;
    const size_t r = rows, o = n_out, i = n_in;
    return 256 + a256(i * o * 4) + a256(o * r * 4) + a256(i * r * 4);
}

GPT_API int gpt_linear_backward(const void* dy, const void* x, const void* W, int rows, int n_out, int n_in, int dtype,
                                float* dx, float* dW, void* workspace, size_t workspace_bytes, int32_t* status,
                                void* stream) {
    if (!dy || !x || !W || !dx || !dW || !workspace) return GPT_ERR_NULL;
    if (rows < 0 || n_out <= 0 || n_in <= 0) return GPT_ERR_BAD_SHAPE;
    if (dtype != GPT_DTYPE_BF16 && dtype != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    if (rows == 0) return GPT_OK;
    if (workspace_bytes < gpt_linear_backward_workspace_bytes(rows, n_out, n_in, dtype)) return GPT_ERR_WS_TOO_SMALL;
    if (!aligned(workspace, 256) || !aligned(dx, 16) || !aligned(dW, 16)) return GPT_ERR_BAD_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == GPT_DTYPE_BF16) {
        if ((n_out % 8) || (n_in % 8)) return GPT_ERR_UNSUPPORTED;
        if (!aligned(dy, 16) || !aligned(x, 16) || !aligned(W, 16)) return GPT_ERR_BAD_ALIGN;
        const bf16* y = static_cast<const bf16*>(dy);
        // dx = dy W: dy K-major, W stored [n_out = K, n_in = N] (MN-major B), stored (not added)
        GPT_TRY(launch_gemm_bf16_bwd(y, n_out, false, static_cast<const bf16*>(W), n_in, true, dx, n_in, rows, n_in,
                                     n_out, GEMM_BWD_STORE_F32, nullptr, 0, 0, status, s));
        // dW += dy^T x: dy stored [rows = K, n_out = M], x stored [rows = K, n_in = N] (both MN-major)
        return launch_gemm_bf16_acc(y, n_out, true, static_cast<const bf16*>(x), n_in, true, dW, n_in, n_out, n_in,
                                    rows, status, s, reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + 256));
    }
    GPT_TRY(cuda_status(cudaMemsetAsync(dx, 0, static_cast<size_t>(rows) * n_in * 4, s)));
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const size_t r = rows, o = n_out, i = n_in;
    float* wT = reinterpret_cast<float*>(ws + 256);
    float* yT = reinterpret_cast<float*>(ws + 256 + a256(i * o * 4));
    float* xT = reinterpret_cast<float*>(ws + 256 + a256(i * o * 4) + a256(o * r * 4));
    GPT_TRY(launch_transpose(W, GPT_DTYPE_F32, n_in, wT, GPT_DTYPE_F32, n_out, n_out, n_in, s));
    GPT_TRY(launch_linear_f32(static_cast<const float*>(dy), n_out, wT, nullptr, dx, n_in, rows, n_in, n_out,
                              GPT_EPI_RESID, GPT_GELU_ERF, s));
    GPT_TRY(launch_transpose(dy, GPT_DTYPE_F32, n_out, yT, GPT_DTYPE_F32, rows, rows, n_out, s));
    GPT_TRY(launch_transpose(x, GPT_DTYPE_F32, n_in, xT, GPT_DTYPE_F32, rows, rows, n_in, s));
    return launch_linear_f32(yT, rows, xT, nullptr, dW, n_in, n_out, n_in, rows, GPT_EPI_RESID, GPT_GELU_ERF, s);
}

GPT_API int gpt_transpose(const void* in, int in_dtype, long long ld_in, void* out, int out_dtype, long long ld_out,
                          int rows, int cols, void* stream) {
    if (!in || !out) return GPT_ERR_NULL;
    if (rows < 0 || cols < 0 || ld_in < cols || ld_out < rows) return GPT_ERR_BAD_SHAPE;
    for (int d : {in_dtype, out_dtype})
        if (d != GPT_DTYPE_BF16 && d != GPT_DTYPE_F32) return GPT_ERR_BAD_SHAPE;
    return launch_transpose(in, in_dtype, ld_in, out, out_dtype, ld_out, rows, cols, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ training step: forward + backward
namespace {

// Activations the backward needs, per layer and at the end (N = B * T rows, E = storage type).
struct ActPlan {
    size_t x_in, u1, qkv, y, lse, x_mid, u2, pre, h, layer;  // offsets within a layer's block
    size_t final_off, x_f, u_f, logits, sum_count, row_lse, total;
};

ActPlan plan_acts(const gpt_config_t* c, long long B, long long T) {
    ActPlan A{};
    const size_t N = static_cast<size_t>(B * T), C = c->n_embd, es = elem_size(c);
    size_t off = 0;
    A.x_in = off; off += a256(N * C * 4);
    A.u1 = off; off += a256(N * C * es);
    A.qkv = off; off += a256(N * 3 * C * es);
    A.y = off; off += a256(N * C * es);
    A.lse = off; off += a256(static_cast<size_t>(B) * c->n_head * T * 4);
    A.x_mid = off; off += a256(N * C * 4);
    A.u2 = off; off += a256(N * C * es);
    A.pre = off; off += a256(N * 4 * C * es);
    A.h = off; off += a256(N * 4 * C * es);
    A.layer = off;
    size_t f = A.layer * c->n_layer;
    A.final_off = f;
    A.x_f = f; f += a256(N * C * 4);
    A.u_f = f; f += a256(N * C * es);
    A.logits = f; f += a256(N * static_cast<size_t>(c->vocab_size) * es);
    A.sum_count = f; f += 256;
    A.row_lse = f; f += a256(N * 4);  // bf16: each row's logsumexp from the head's fp32 accumulators
    A.total = f;
    return A;
}

// Scratch of the backward pass.
struct BwdPlan {
    size_t splitk;
    size_t ctrl, dz, dzT, wT, gE, gT, aT, d1, dx, dpre, dqkv, dy, D, parts, sort, total;
};

BwdPlan plan_bwd(const gpt_config_t* c, long long B, long long T) {
    BwdPlan P{};
    const size_t N = static_cast<size_t>(B * T), C = c->n_embd, V = c->vocab_size, es = elem_size(c);
    size_t off = 0;
    P.ctrl = off; off += 256;
    // Transposed copies of the Linear layers' operands: fp32 only (bf16 hands the GEMM the stored
    // matrices as MN-major operands).
    const size_t tr = c->dtype == GPT_DTYPE_BF16 ? 0 : 1;
    P.dz = off; off += a256(N * V * es);
    P.dzT = off; off += a256(tr * N * V * es);
    P.wT = off; off += a256(tr * std::max(V * C, 4 * C * C) * es);
    P.gE = off; off += a256(N * 4 * C * es);
    P.gT = off; off += a256(tr * N * 4 * C * es);
    P.aT = off; off += a256(tr * N * 4 * C * es);
    P.d1 = off; off += a256(N * 4 * C * 4);
    P.dx = off; off += a256(N * C * 4);
    P.dpre = off; off += a256(N * 4 * C * es);
    P.dqkv = off; off += a256(N * 3 * C * es);
    P.dy = off; off += a256(N * C * es);
    P.D = off; off += a256(attn_bwd_scratch_bytes(B, c->n_head, T));
    const size_t lnp = static_cast<size_t>(layernorm_backward_parts(static_cast<int>(N), static_cast<int>(C))) * 3 * C;
    const size_t csp = static_cast<size_t>(colsum_parts(static_cast<int>(N))) * 4 * C;
    // per-band column sums: db_fc's from the DGELU product, db_attn's from the attention backward
    const size_t bands = std::max((N + 31) / 32 * 4 * C, static_cast<size_t>(B * ((T + 31) / 32)) * 3 * C);
    P.parts = off; off += a256(std::max({lnp, csp, bands}) * 4);
    P.sort = off; off += a256(N * 8);
    // split-K partial products of the weight-gradient GEMMs (bf16)
    size_t sk = 0;
    if (c->dtype == GPT_DTYPE_BF16) {
        const int n = static_cast<int>(N), e = static_cast<int>(C);
        sk = std::max({gemm_acc_split_bytes(3 * e, e, n), gemm_acc_split_bytes(e, e, n), gemm_acc_split_bytes(4 * e, e, n),
                       gemm_acc_split_bytes(e, 4 * e, n), gemm_acc_split_bytes(static_cast<int>(V), e, n)});
    }
    P.splitk = off; off += a256(sk);
    P.total = off;
    return P;
}

int check_train(const gpt_config_t* c, const void* weights, const int64_t* idx, const int64_t* targets, int B, int T,
                const void* acts, size_t acts_bytes, ActPlan* A) {
    GPT_TRY(validate(c));
    if (!weights || !idx || !targets || !acts) return GPT_ERR_NULL;
    if (B < 1 || T < 1 || T > c->block_size) return GPT_ERR_BAD_SHAPE;
    const int hs = c->n_embd / c->n_head;
    if (hs != 32 && hs != 64) return GPT_ERR_UNSUPPORTED;
    const long long N = static_cast<long long>(B) * T;
    if (c->dtype == GPT_DTYPE_BF16 && (N % 8)) return GPT_ERR_UNSUPPORTED;  // K of the weight-gradient products
    if (N > embed_backward_max_rows()) return GPT_ERR_UNSUPPORTED;
    if (N * std::max<long long>(c->vocab_size, 4LL * c->n_embd) > 0x7fffffffLL) return GPT_ERR_UNSUPPORTED;
    if (!aligned(weights, 256) || !aligned(acts, 256)) return GPT_ERR_BAD_ALIGN;
    *A = plan_acts(c, B, T);
    if (acts_bytes < A->total) return GPT_ERR_WS_TOO_SMALL;
    return GPT_OK;
}

// out[M, N] (fp32) += A[M, K] B[N, K]^T with A, B dense (row strides lda, ldb) in the config dtype.
int gemm_acc(const gpt_config_t* c, const void* A, long long lda, const void* Bm, long long ldb, float* out,
             long long ldo, int M, int N, int K, int32_t* status, cudaStream_t s) {
    if (c->dtype == GPT_DTYPE_BF16)
        return launch_gemm_bf16(static_cast<const bf16*>(A), lda, static_cast<const bf16*>(Bm), ldb, nullptr, out, ldo,
                                M, N, K, GPT_EPI_RESID, c->gelu, nullptr, status, s);
    if (ldb != K) return GPT_ERR_UNSUPPORTED;
    return launch_linear_f32(static_cast<const float*>(A), lda, static_cast<const float*>(Bm), nullptr, out, ldo, M, N,
                             K, GPT_EPI_RESID, c->gelu, s);
}

}  // namespace

GPT_API size_t gpt_train_activation_bytes(const gpt_config_t* cfg, int B, int T) {
    if (validate(cfg) != GPT_OK || B < 1 || T < 1 || T > cfg->block_size) return 0;
    return plan_acts(cfg, B, T).total;
}

GPT_API size_t gpt_backward_workspace_bytes(const gpt_config_t* cfg, int B, int T) {
    if (validate(cfg) != GPT_OK || B < 1 || T < 1 || T > cfg->block_size) return 0;
    return plan_bwd(cfg, B, T).total;
}

GPT_API int gpt_forward_train(const gpt_config_t* cfg, const void* weights, const int64_t* idx, const int64_t* targets,
                              int B, int T, void* acts, size_t acts_bytes, float* loss, void* workspace,
                              size_t workspace_bytes, void* stream, int flags) {
    ActPlan A;
    GPT_TRY(check_train(cfg, weights, idx, targets, B, T, acts, acts_bytes, &A));
    Plan P;
    GPT_TRY(check_common(cfg, weights, B, T, workspace, workspace_bytes, &P));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Weights W;
    fill_weights(W, cfg, weights);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* ab = static_cast<uint8_t*>(acts);
    int32_t* status = status_word(ws);
    const int C = cfg->n_embd, V = cfg->vocab_size, nh = cfg->n_head, hs = C / nh, N = B * T, dt = cfg->dtype;
    const size_t es = elem_size(cfg);
    const bool bf = dt == GPT_DTYPE_BF16;
    GPT_TRY(cuda_status(cudaMemsetAsync(status, 0, sizeof(int32_t), s)));
    GPT_TRY(launch_embed(W.wte(), W.wpe(), idx, reinterpret_cast<float*>(ab + A.x_in), B, T, C, V, dt, status, s));
    for (int l = 0; l < cfg->n_layer; ++l) {
        uint8_t* L = ab + A.layer * l;
        float* x_in = reinterpret_cast<float*>(L + A.x_in);
        float* x_mid = reinterpret_cast<float*>(L + A.x_mid);
        float* x_out = l + 1 < cfg->n_layer ? reinterpret_cast<float*>(ab + A.layer * (l + 1) + A.x_in)
                                            : reinterpret_cast<float*>(ab + A.x_f);
        void* u1 = L + A.u1;
        void* qkv = L + A.qkv;
        void* y = L + A.y;
        float* lse = reinterpret_cast<float*>(L + A.lse);
        void* u2 = L + A.u2;
        void* pre = L + A.pre;
        void* hh = L + A.h;
        // ln_1 also copies x_in to x_mid, which attn c_proj then adds into (x_in stays for the backward)
        GPT_TRY(launch_layernorm(x_in, W.layer(l, W_LN1_W), W.bias(l, W_LN1_B), u1, N, C, dt, s, x_mid));
        if (bf) {
            GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(u1), C, static_cast<const bf16*>(W.layer(l, W_ATTN_W)), C,
                                     static_cast<const bf16*>(W.bias(l, W_ATTN_B)), qkv, 3LL * C, N, 3 * C, C,
                                     GPT_EPI_STORE, cfg->gelu, nullptr, status, s));
            const bf16* qb = static_cast<const bf16*>(qkv);
            AttnLayout AL{qb, qb + C, qb + 2 * C, 3LL * C * T, hs, 3LL * C, static_cast<bf16*>(y),
                          static_cast<long long>(C) * T, hs, C, lse};
            GPT_TRY(launch_attention_bf16(AL, B, nh, T, status, s));
        } else {
            GPT_TRY(launch_linear_f32(static_cast<const float*>(u1), C, static_cast<const float*>(W.layer(l, W_ATTN_W)),
                                      static_cast<const float*>(W.bias(l, W_ATTN_B)), static_cast<float*>(qkv), 3LL * C,
                                      N, 3 * C, C, GPT_EPI_STORE, cfg->gelu, s));
            const float* qf = static_cast<const float*>(qkv);
            AttnLayoutF32 AL{qf, qf + C, qf + 2 * C, 3LL * C * T, hs, 3LL * C, static_cast<float*>(y),
                             static_cast<long long>(C) * T, hs, C, lse};
            GPT_TRY(launch_attention_f32(AL, B, nh, T, hs, s));
        }
        if (bf)
            GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(y), C, static_cast<const bf16*>(W.layer(l, W_PROJ_W)), C,
                                     static_cast<const bf16*>(W.bias(l, W_PROJ_B)), x_mid, C, N, C, C, GPT_EPI_RESID,
                                     cfg->gelu, nullptr, status, s));
        else
            GPT_TRY(launch_linear_f32(static_cast<const float*>(y), C, static_cast<const float*>(W.layer(l, W_PROJ_W)),
                                      static_cast<const float*>(W.bias(l, W_PROJ_B)), x_mid, C, N, C, C, GPT_EPI_RESID,
                                      cfg->gelu, s));
        // ln_2 also copies x_mid to the next layer's x_in (x_out), which mlp c_proj adds into
        GPT_TRY(launch_layernorm(x_mid, W.layer(l, W_LN2_W), W.bias(l, W_LN2_B), u2, N, C, dt, s, x_out));
        // c_fc keeps the GELU output (for the weight gradient) and, in the bf16 path, the GELU
        // derivative at the pre-activation in `pre` (for the backward through GELU): one product
        // writing both when h directly follows pre, else a store, a GELU pass and an in-place
        // derivative pass.  The fp32 path keeps the pre-activation itself.
        const bool two_out = bf && (N % 32 == 0) &&
                             static_cast<uint8_t*>(hh) == static_cast<uint8_t*>(pre) + static_cast<size_t>(N) * 4 * C * es;
        if (two_out)
            GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(u2), C, static_cast<const bf16*>(W.layer(l, W_FC_W)), C,
                                     static_cast<const bf16*>(W.bias(l, W_FC_B)), pre, 4LL * C, N, 4 * C, C,
                                     GEMM_EPI_GELU2, cfg->gelu, nullptr, status, s));
        else if (bf)
            GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(u2), C, static_cast<const bf16*>(W.layer(l, W_FC_W)), C,
                                     static_cast<const bf16*>(W.bias(l, W_FC_B)), pre, 4LL * C, N, 4 * C, C,
                                     GPT_EPI_STORE, cfg->gelu, nullptr, status, s));
        else
            GPT_TRY(launch_linear_f32(static_cast<const float*>(u2), C, static_cast<const float*>(W.layer(l, W_FC_W)),
                                      static_cast<const float*>(W.bias(l, W_FC_B)), static_cast<float*>(pre), 4LL * C, N,
                                      4 * C, C, GPT_EPI_STORE, cfg->gelu, s));
        if (!two_out) {
            GPT_TRY(launch_gelu_forward(pre, hh, static_cast<long long>(N) * 4 * C, dt, cfg->gelu == GPT_GELU_TANH, s));
            if (bf)
                GPT_TRY(launch_gelu_deriv_inplace(pre, static_cast<long long>(N) * 4 * C, dt,
                                                  cfg->gelu == GPT_GELU_TANH, s));
        }
        if (bf)
            GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(hh), 4LL * C, static_cast<const bf16*>(W.layer(l, W_FC2_W)),
                                     4LL * C, static_cast<const bf16*>(W.bias(l, W_FC2_B)), x_out, C, N, C, 4 * C,
                                     GPT_EPI_RESID, cfg->gelu, nullptr, status, s));
        else
            GPT_TRY(launch_linear_f32(static_cast<const float*>(hh), 4LL * C, static_cast<const float*>(W.layer(l, W_FC2_W)),
                                      static_cast<const float*>(W.bias(l, W_FC2_B)), x_out, C, N, C, 4 * C, GPT_EPI_RESID,
                                      cfg->gelu, s));
    }
    void* u_f = ab + A.u_f;
    void* logits = ab + A.logits;
    double* sc = reinterpret_cast<double*>(ab + A.sum_count);
    GPT_TRY(launch_layernorm(reinterpret_cast<float*>(ab + A.x_f), W.lnf_w(), W.lnf_b(), u_f, N, C, dt, s));
    float* rl = reinterpret_cast<float*>(ws + P.rowloss);
    if (bf) {
        CeArgs ce{targets, reinterpret_cast<float2*>(ws + P.part), reinterpret_cast<float*>(ws + P.tlogit), P.n_part};
        GPT_TRY(launch_gemm_bf16(static_cast<const bf16*>(u_f), C, static_cast<const bf16*>(W.wte()), C, nullptr, logits, V,
                                 N, V, C, 3 /* EPI_CE */, cfg->gelu, &ce, status, s));
        GPT_TRY(launch_ce_rows_from_parts(ce.part, P.n_part, ce.tlogit, targets, N, V, rl, status, s,
                                          reinterpret_cast<float*>(ab + A.row_lse)));
    } else {
        GPT_TRY(launch_linear_f32(static_cast<const float*>(u_f), C, static_cast<const float*>(W.wte()), nullptr,
                                  static_cast<float*>(logits), V, N, V, C, GPT_EPI_STORE, cfg->gelu, s));
        GPT_TRY(launch_ce_rows_from_logits(static_cast<const float*>(logits), targets, N, V, rl, status, s));
    }
    GPT_TRY(launch_loss_finalize(rl, targets, N, V, loss, sc, s));
    (void)es;
    if (flags & GPT_FLAG_SYNC_CHECK) return sync_and_read_status(ws, s);
    return GPT_OK;
}

GPT_API int gpt_grad_buckets(const gpt_config_t* cfg, size_t* starts, size_t* stops, int n) {
    const int rc = validate(cfg);
    if (rc != GPT_OK) return rc;
    const int L = cfg->n_layer, count = 2 + kTensorsPerLayer * L + 2;
    if (count > kOptMaxTensors) return GPT_ERR_UNSUPPORTED;
    size_t offs[kOptMaxTensors];
    layout(cfg, offs, nullptr, count);
    const size_t es = elem_size(cfg);
    const size_t total = gpt_param_elems(cfg);
    for (int i = 0; i <= L && i < n; ++i) {
        size_t a, b;
        if (i < L) {
            const int l = L - 1 - i;  // buckets in the order the backward finishes them
            a = offs[2 + kTensorsPerLayer * l] / es;
            b = (i == 0) ? total : offs[2 + kTensorsPerLayer * (l + 1)] / es;
        } else {
            a = 0;
            b = offs[2] / es;
        }
        if (starts) starts[i] = a;
        if (stops) stops[i] = b;
    }
    return L + 1;
}

GPT_API size_t gpt_train_loss_terms_offset(const gpt_config_t* cfg, int B, int T) {
    if (validate(cfg) != GPT_OK || B < 1 || T < 1 || T > cfg->block_size) return 0;
    return plan_acts(cfg, B, T).sum_count;
}

GPT_API int gpt_backward(const gpt_config_t* cfg, const void* weights, const int64_t* idx, const int64_t* targets, int B,
                         int T, const void* acts, size_t acts_bytes, float* grads, float loss_scale, void* workspace,
                         size_t workspace_bytes, void* stream, int flags, void* const* bucket_events) {
    ActPlan A;
    GPT_TRY(check_train(cfg, weights, idx, targets, B, T, acts, acts_bytes, &A));
    if (!grads || !workspace) return GPT_ERR_NULL;
    if (!aligned(grads, 16) || !aligned(workspace, 256)) return GPT_ERR_BAD_ALIGN;
    const BwdPlan P = plan_bwd(cfg, B, T);
    if (workspace_bytes < P.total) return GPT_ERR_WS_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Weights W;
    fill_weights(W, cfg, weights);
    const uint8_t* ab = static_cast<const uint8_t*>(acts);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* status = status_word(ws);
    const int C = cfg->n_embd, V = cfg->vocab_size, nh = cfg->n_head, hs = C / nh, N = B * T, dt = cfg->dtype;
    const bool bf = dt == GPT_DTYPE_BF16;
    const size_t es = elem_size(cfg);
    // gradient slots: the packed layout in fp32 elements
    size_t offs[kOptMaxTensors];
    const int count = 2 + kTensorsPerLayer * cfg->n_layer + 2;
    if (count > kOptMaxTensors) return GPT_ERR_UNSUPPORTED;
    layout(cfg, offs, nullptr, count);
    auto G = [&](int i) { return grads + offs[i] / es; };
    auto GL = [&](int l, int which) { return G(2 + kTensorsPerLayer * l + which); };
    void* dz = ws + P.dz;
    void* dzT = ws + P.dzT;
    void* wT = ws + P.wT;
    void* gE = ws + P.gE;
    void* gT = ws + P.gT;
    void* aT = ws + P.aT;
    float* d1 = reinterpret_cast<float*>(ws + P.d1);
    float* dx = reinterpret_cast<float*>(ws + P.dx);
    void* dpre = ws + P.dpre;
    void* dqkv = ws + P.dqkv;
    void* dy = ws + P.dy;
    float* D = reinterpret_cast<float*>(ws + P.D);
    float* parts = reinterpret_cast<float*>(ws + P.parts);
    const int F32 = GPT_DTYPE_F32;
    const size_t nc = static_cast<size_t>(N) * C;

    // Linear backward: the input gradient dIn = dY W and dW (fp32) += dY^T X, for dY [N, n_out] (row
    // stride ldy), X [N, n_in] (row stride ldx) and W [n_out, n_in] in the config dtype.  dIn is
    // written as `mode` says: GEMM_BWD_STORE_F32 (fp32 [N, n_in]), GEMM_BWD_STORE_BF16, or
    // GEMM_BWD_DGELU_BF16 (bf16 (dY W) * gelu'(aux), aux the [N, n_in] pre-activation).  bf16 hands
    // the GEMM the stored dY, X and W as MN-major operands where the product needs their transposes;
    // fp32 (GEMM_BWD_STORE_F32 only) forms the transposes in scratch first (yT: room for dY^T).
    auto linear_bwd = [&](const void* dYp, long long ldy, const void* Xp, long long ldx, const void* Wp, int n_out,
                          int n_in, void* dIn, int mode, const void* aux, float* dW, void* yT,
                          float* colsum = nullptr) -> int {
        if (bf) {
            const bf16* y = static_cast<const bf16*>(dYp);
            GPT_TRY(launch_gemm_bf16_bwd(y, ldy, false, static_cast<const bf16*>(Wp), n_in, true, dIn, n_in, N, n_in,
                                         n_out, mode, static_cast<const bf16*>(aux), n_in, cfg->gelu, status, s,
                                         nullptr, colsum));
            return launch_gemm_bf16_bwd(y, ldy, true, static_cast<const bf16*>(Xp), ldx, true, dW, n_in, n_out, n_in, N,
                                        GEMM_BWD_ACC_F32, nullptr, 0, 0, status, s,
                                        reinterpret_cast<float*>(ws + P.splitk));
        }
        if (mode != GEMM_BWD_STORE_F32) return GPT_ERR_UNSUPPORTED;
        float* out = static_cast<float*>(dIn);
        GPT_TRY(cuda_status(cudaMemsetAsync(out, 0, static_cast<size_t>(N) * n_in * 4, s)));
        GPT_TRY(launch_transpose(Wp, dt, n_in, wT, dt, n_out, n_out, n_in, s));
        GPT_TRY(gemm_acc(cfg, dYp, ldy, wT, n_out, out, n_in, N, n_in, n_out, status, s));
        GPT_TRY(launch_transpose(dYp, dt, ldy, yT, dt, N, N, n_out, s));
        GPT_TRY(launch_transpose(Xp, dt, ldx, aT, dt, N, N, n_in, s));
        return gemm_acc(cfg, yT, N, aT, N, dW, n_in, n_out, n_in, N, status, s);
    };
    // The residual gradient dx stays fp32; the products read it as gx: the bf16 copy gE that each
    // LayerNorm backward writes next to dx (bf16), or dx itself (fp32).
    const void* gx = bf ? static_cast<const void*>(gE) : static_cast<const void*>(dx);
    bf16* dx16 = bf ? static_cast<bf16*>(gE) : nullptr;
    const int F32_OUT = GEMM_BWD_STORE_F32;

    GPT_TRY(cuda_status(cudaMemsetAsync(status, 0, sizeof(int32_t), s)));
    // d loss / d logits, then the tied head: du_f = dz wte, dwte += dz^T u_f
    if (!(loss_scale > 0.f) || !isfinite(loss_scale)) return GPT_ERR_BAD_SHAPE;
    // bf16: d(logits) in one pass with the row logsumexp the forward kept; fp32: reduced here
    GPT_TRY(launch_ce_backward(ab + A.logits, dt, targets, reinterpret_cast<const double*>(ab + A.sum_count), dz, N, V,
                               status, s, loss_scale, bf ? reinterpret_cast<const float*>(ab + A.row_lse) : nullptr));
    GPT_TRY(linear_bwd(dz, V, ab + A.u_f, C, W.wte(), V, C, d1, F32_OUT, nullptr, G(0), dzT));
    // The residual gradient each LayerNorm backward writes is also the bias gradient of the
    // projection that added into the stream there: the last Block's mlp c_proj at ln_f, attn c_proj
    // at ln_2, the previous Block's mlp c_proj at ln_1.  The LayerNorm backward sums it as it goes.
    const int Lm1 = cfg->n_layer - 1;
    GPT_TRY(launch_layernorm_backward(d1, reinterpret_cast<const float*>(ab + A.x_f), W.lnf_w(), dt, dx, 0, G(count - 2),
                                      cfg->bias ? G(count - 1) : nullptr, 1, parts, N, C, s, dx16,
                                      cfg->bias ? GL(Lm1, W_FC2_B) : nullptr));
    // Event i marks the end of bucket i (gpt_grad_buckets): a caller may start reducing that range
    // of grads on another stream while the rest of the backward runs.
    auto mark = [&](int i) -> int {
        if (!bucket_events || !bucket_events[i]) return GPT_OK;
        return cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(bucket_events[i]), s));
    };
    for (int l = cfg->n_layer - 1; l >= 0; --l) {
        const uint8_t* L = ab + A.layer * l;
        // mlp c_proj, then GELU: dpre = (dx W_fc2) * gelu'(pre) (bf16: one fused product reading the
        // derivative the forward stored; fp32: dh into d1, then the GELU backward from the
        // pre-activation); dW_fc2 += dx^T h (db_fc2 += sum dx came with the LayerNorm backward above)
        if (bf) {
            // the product's epilogue also leaves dpre's column sums per 32-row band (db_fc)
            GPT_TRY(linear_bwd(gx, C, L + A.h, 4LL * C, W.layer(l, W_FC2_W), C, 4 * C, dpre, GEMM_BWD_DGELU_BF16,
                               L + A.pre, GL(l, W_FC2_W), gT, cfg->bias ? parts : nullptr));
            if (cfg->bias) GPT_TRY(launch_colsum_bands(parts, (N + 31) / 32, 4 * C, GL(l, W_FC_B), 1, s));
        } else {
            GPT_TRY(linear_bwd(gx, C, L + A.h, 4LL * C, W.layer(l, W_FC2_W), C, 4 * C, d1, F32_OUT, nullptr,
                               GL(l, W_FC2_W), gT));
            GPT_TRY(launch_gelu_backward(d1, L + A.pre, dt, dpre, static_cast<long long>(nc) * 4,
                                         cfg->gelu == GPT_GELU_TANH, s));
        }
        // c_fc: du2 = dpre W_fc (into d1 [N, C]); dW_fc += dpre^T u2; db_fc += sum dpre (bf16: above)
        GPT_TRY(linear_bwd(dpre, 4LL * C, L + A.u2, C, W.layer(l, W_FC_W), 4 * C, C, d1, F32_OUT, nullptr,
                           GL(l, W_FC_W), gT));
        if (cfg->bias && !bf) GPT_TRY(launch_colsum(dpre, dt, N, 4 * C, GL(l, W_FC_B), 1, parts, s));
        GPT_TRY(launch_layernorm_backward(d1, reinterpret_cast<const float*>(L + A.x_mid), W.layer(l, W_LN2_W), dt, dx, 1,
                                          GL(l, W_LN2_W), cfg->bias ? GL(l, W_LN2_B) : nullptr, 1, parts, N, C, s,
                                          dx16, cfg->bias ? GL(l, W_PROJ_B) : nullptr));
        // attn c_proj: dy = dx W_proj (straight into the config dtype); dW_proj += dx^T y (db_proj += sum dx
        // came with ln_2's backward)
        GPT_TRY(linear_bwd(gx, C, L + A.y, C, W.layer(l, W_PROJ_W), C, C, dy, bf ? GEMM_BWD_STORE_BF16 : F32_OUT,
                           nullptr, GL(l, W_PROJ_W), gT));
        // attention backward into dqkv (the qkv layout)
        const float* lse = reinterpret_cast<const float*>(L + A.lse);
        bool attn_bias_done = false;
        const long long qsb = 3LL * C * T, ysb = static_cast<long long>(C) * T;
        if (bf) {
            const bf16* q = reinterpret_cast<const bf16*>(L + A.qkv);
            bf16* dq = static_cast<bf16*>(dqkv);
            AttnBwdLayout<bf16> AL{q, q + C, q + 2 * C, qsb, hs, 3LL * C,
                                   reinterpret_cast<const bf16*>(L + A.y), static_cast<const bf16*>(dy), ysb, hs, C,
                                   dq, dq + C, dq + 2 * C, lse};
            // the tensor-core kernels also leave dqkv's column sums per 32-row band (db_attn)
            const AttnBwdColsum cs{parts, 3LL * C, 0, C, 2 * C};
            bool cs_done = false;
            GPT_TRY(launch_attention_backward(&AL, nullptr, B, nh, T, hs, D, status, s, cfg->bias ? &cs : nullptr,
                                              &cs_done));
            if (cs_done) GPT_TRY(launch_colsum_bands(parts, B * ((T + 31) / 32), 3 * C, GL(l, W_ATTN_B), 1, s));
            attn_bias_done = cs_done;
        } else {
            const float* q = reinterpret_cast<const float*>(L + A.qkv);
            float* dq = static_cast<float*>(dqkv);
            AttnBwdLayout<float> AL{q, q + C, q + 2 * C, qsb, hs, 3LL * C,
                                    reinterpret_cast<const float*>(L + A.y), static_cast<const float*>(dy), ysb, hs, C,
                                    dq, dq + C, dq + 2 * C, lse};
            GPT_TRY(launch_attention_backward(nullptr, &AL, B, nh, T, hs, D, status, s));
        }
        // c_attn: du1 = dqkv W_attn (into d1 [N, C]); dW_attn += dqkv^T u1; db_attn += sum dqkv (unless the
        // attention backward's band sums gave it above)
        GPT_TRY(linear_bwd(dqkv, 3LL * C, L + A.u1, C, W.layer(l, W_ATTN_W), 3 * C, C, d1, F32_OUT, nullptr,
                           GL(l, W_ATTN_W), gT));
        if (cfg->bias && !attn_bias_done) GPT_TRY(launch_colsum(dqkv, dt, N, 3 * C, GL(l, W_ATTN_B), 1, parts, s));
        GPT_TRY(launch_layernorm_backward(d1, reinterpret_cast<const float*>(L + A.x_in), W.layer(l, W_LN1_W), dt, dx, 1,
                                          GL(l, W_LN1_W), cfg->bias ? GL(l, W_LN1_B) : nullptr, 1, parts, N, C, s,
                                          dx16, cfg->bias && l > 0 ? GL(l - 1, W_FC2_B) : nullptr));
        GPT_TRY(mark(cfg->n_layer - 1 - l));  // every gradient of layer l (and, for the last layer, ln_f) is final
    }
    GPT_TRY(launch_embed_backward(idx, dx, B, T, C, V, G(0), G(1), reinterpret_cast<unsigned long long*>(ws + P.sort),
                                  status, s));
    GPT_TRY(mark(cfg->n_layer));  // wte (the head's and the embedding's parts) and wpe
    if (flags & GPT_FLAG_SYNC_CHECK) return sync_and_read_status(ws, s);
    return GPT_OK;
}

