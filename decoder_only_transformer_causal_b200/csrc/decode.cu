// Incremental decoding ("nanoGPT 全局流程图", 第五阶段 generate): the forward of one new token per
// sequence against a key/value cache, and the sampling step (temperature, top-k, softmax,
// multinomial draw).
//
// A decode step reads every weight once for a handful of rows, so its matrix products are
// matrix-vector products bound by HBM bandwidth, not tensor-core work: CTAs of 8 warps stage
// the input rows in shared memory (fusing the LayerNorm that precedes ln_1 / ln_2 / ln_f
// products) and stream weight rows with 16-byte loads; the epilogue (bias, GELU, residual
// add, k/v append) is fused.  The attention of the new position against the cached keys is
// split over 64-key ranges (so a long cache is read by many CTAs at once) and merged by the
// last CTA of each head.  The position being written lives in device memory, so a recorded
// graph of a step can be replayed as the sequence grows.
//
// Element type E is the configuration's storage type (bf16 or fp32) for weights, activations
// and the cache; accumulation is fp32 throughout and the residual stream is fp32.
//
// Memory visibility.  Every kernel here is launched with programmatic stream serialisation
// and calls griddep_wait() first; the wait makes the writes of the kernel immediately before
// it visible, but data written further back (the decode position, written at the end of the
// previous step; the cache, written by earlier steps; the residual stream, last written
// several kernels earlier; the logits, written before the position update) can still be
// served stale from this SM's L1.  So every buffer that any kernel writes is read here with
// L2 loads (ld.global.cg); only the weights, which never change, use the cached path.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gpt {

namespace {

GPT_DEVINL float to_f(bf16 v) { return __bfloat162float(v); }
GPT_DEVINL float to_f(float v) { return v; }
template <typename E> GPT_DEVINL E from_f(float v);
template <> GPT_DEVINL bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }
template <> GPT_DEVINL float from_f<float>(float v) { return v; }

// L2 loads of data other kernels write (see the note at the top of the file).
GPT_DEVINL float ld_act(const bf16* p) {
    return __bfloat162float(__ushort_as_bfloat16(__ldcg(reinterpret_cast<const unsigned short*>(p))));
}
GPT_DEVINL float ld_act(const float* p) { return __ldcg(p); }

// 8 consecutive elements (16-byte aligned for bf16, 32-byte for fp32) as fp32: weights through
// the cached path, activations and the cache (load8_act) from L2.
GPT_DEVINL void unpack8(const uint4& w, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __low2float(h[i]);
        f[2 * i + 1] = __high2float(h[i]);
    }
}
GPT_DEVINL void load8_act(const bf16* p, float (&f)[8]) { unpack8(__ldcg(reinterpret_cast<const uint4*>(p)), f); }
GPT_DEVINL void load8_act(const float* p, float (&f)[8]) {
    const float4 a = __ldcg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldcg(reinterpret_cast<const float4*>(p + 4));
    f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w;
    f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}
GPT_DEVINL void load8(const bf16* p, float (&f)[8]) { unpack8(*reinterpret_cast<const uint4*>(p), f); }
GPT_DEVINL void load8(const float* p, float (&f)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w;
    f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}

GPT_DEVINL float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Asks L2 to fetch [p, p + bytes) (both multiples of 16) from HBM; no completion to wait on.
GPT_DEVINL void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// This CTA's share of an L2 prefetch of [base, base + bytes): the whole range is split over the
// grid in 16-byte-aligned pieces, so the first CTAs to start fetch all of it.
GPT_DEVINL void prefetch_l2_share(const void* base, size_t bytes) {
    const size_t per = ((bytes + gridDim.x - 1) / gridDim.x + 15) & ~static_cast<size_t>(15);
    const size_t off = per * blockIdx.x;
    if (off >= bytes) return;
    size_t n = bytes - off < per ? bytes - off : per;
    const uint8_t* p = static_cast<const uint8_t*>(base) + off;
    while (n >= 16) {
        const uint32_t chunk = n > (1u << 20) ? (1u << 20) : static_cast<uint32_t>(n & ~static_cast<size_t>(15));
        prefetch_l2(p, chunk);
        p += chunk;
        n -= chunk;
    }
}

GPT_DEVINL float gelu_erf(float v) { return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f)); }
GPT_DEVINL float gelu_tanh(float v) {
    return 0.5f * v * (1.0f + tanhf(0.79788456080286536f * (v + 0.044715f * v * v * v)));
}

// x[b, :] = wte[tok[b * ld_tok], :] + wpe[*pos, :]  (the embedding sum at one position)
template <typename E>
__global__ void embed_pos_kernel(const E* __restrict__ wte, const E* __restrict__ wpe, const int64_t* __restrict__ tok,
                                 long long ld_tok, const int* __restrict__ pos, float* __restrict__ x, int B, int C,
                                 int V, int block_size, int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= B * C) return;
    const int b = i / C, c = i % C;
    long long t = __ldcg(tok + b * ld_tok);
    if (t < 0 || t >= V) {
        set_status(status, GPT_ERR_INDEX);
        t = 0;
    }
    int p = __ldcg(pos);
    if (p < 0 || p >= block_size) {
        set_status(status, GPT_ERR_BAD_SHAPE);
        p = 0;
    }
    x[i] = to_f(wte[t * C + c]) + to_f(wpe[static_cast<long long>(p) * C + c]);
}

// ---------------------------------------------------------------- matrix-vector products
// out[r, n] = epilogue(sum_k xin[r, k] W[n, k] + bias[n]) for up to kGemvRows rows r (launches of
// more rows are split).
//
// A CTA of 8 warps stages its input rows in shared memory once (in E, as stored between
// kernels), optionally as LayerNorm of the fp32 residual stream (the ln_1 / ln_2 / ln_f that
// precedes the product, fused).  Warps then stream weight rows with 16-byte loads: KSPLIT
// warps share one column, each over a contiguous K slice (narrow outputs need the extra
// loads in flight), and each warp carries CPW columns (the vocabulary head).  Partial sums
// are reduced over lanes by a butterfly and over the KSPLIT warps in slice order.
constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvRows = 16;

template <typename E>
struct GemvArgs {
    const void* x;      // LN: fp32 residual rows [rows, K]; otherwise E rows [rows, K]; row stride ldx
    long long ldx;
    const E* ln_w;      // LN prologue weight / bias (bias may be null)
    const E* ln_b;
    const E* W;         // [N, K]
    const E* bias;      // [N] or null
    void* out;          // see DecodeEpi
    long long ldo;
    int rows, N, K, gelu_tanh;
    E* kv;              // DV_QKV: this layer's cache [rows, block_size, 2C]
    int* pos;           // DV_QKV reads it; bump_pos: CTA 0 advances it by one
    int C, block_size, bump_pos;
};

enum DecodeEpi {
    DV_GELU = 1,    // out E [rows, N] = gelu(.)
    DV_RESID = 2,   // out fp32 [rows, N] += .
    DV_F32 = 3,     // out fp32 [rows, N]
    DV_QKV = 4,     // columns [0, C) -> out E (q); [C, 3C) -> kv[row, *pos, :] (k then v)
    DV_STORE = 5,   // out E [rows, N]
};

GPT_DEVINL void store4(bf16* p, float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&lo);
    v.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = v;
}
GPT_DEVINL void store4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
GPT_DEVINL float4 load4w(const bf16* p) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
    return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
}
GPT_DEVINL float4 load4w(const float* p) { return *reinterpret_cast<const float4*>(p); }

template <typename E, int EPI, int KSPLIT, int CPW, bool LN, int ROWS>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const GemvArgs<E> a) {
    griddep_launch_dependents();
    // the weights never change: start bringing them into L2 while the previous kernel finishes
    // (when each CTA takes one column group, its share of the prefetch is exactly its rows of W)
    if (threadIdx.x == 0 && static_cast<long long>(gridDim.x) * ((kGemvWarps / KSPLIT) * CPW) >= a.N)
        prefetch_l2_share(a.W, static_cast<size_t>(a.N) * a.K * sizeof(E));
    griddep_wait();
    extern __shared__ __align__(16) uint8_t gemv_smem[];
    E* xs = reinterpret_cast<E*>(gemv_smem);  // [rows][K]
    float* xf = reinterpret_cast<float*>(gemv_smem + static_cast<size_t>(a.rows) * a.K * sizeof(E));  // LN input
    __shared__ float red[kGemvWarps][CPW][ROWS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = a.K;

    if (LN) {
        // LayerNorm of each fp32 row (population variance, eps 1e-5): the rows are copied to
        // shared memory, then one warp per row takes the mean, the squared deviations and the
        // normalised values from there
        const float* x = static_cast<const float*>(a.x);
        const int per_row = K / 4;
        for (int i = threadIdx.x; i < a.rows * per_row; i += kGemvThreads) {
            const int r = i / per_row, c = i % per_row;
            reinterpret_cast<float4*>(xf + r * K)[c] = __ldcg(reinterpret_cast<const float4*>(x + r * a.ldx) + c);
        }
        __syncthreads();
        for (int r = warp; r < a.rows; r += kGemvWarps) {
            const float* xr = xf + r * K;
            float sum = 0.f;
            for (int k = lane * 4; k < K; k += 128) {
                const float4 v = *reinterpret_cast<const float4*>(xr + k);
                sum += (v.x + v.y) + (v.z + v.w);
            }
            const float mean = warp_sum(sum) / K;
            float ss = 0.f;
            for (int k = lane * 4; k < K; k += 128) {
                const float4 v = *reinterpret_cast<const float4*>(xr + k);
                const float p = v.x - mean, q = v.y - mean, t = v.z - mean, w = v.w - mean;
                ss += (p * p + q * q) + (t * t + w * w);
            }
            const float rstd = rsqrtf(warp_sum(ss) / K + 1e-5f);
            for (int k = lane * 4; k < K; k += 128) {
                const float4 v = *reinterpret_cast<const float4*>(xr + k);
                const float4 g = load4w(a.ln_w + k);
                const float4 bb = a.ln_b ? load4w(a.ln_b + k) : make_float4(0.f, 0.f, 0.f, 0.f);
                store4(xs + r * K + k, (v.x - mean) * rstd * g.x + bb.x, (v.y - mean) * rstd * g.y + bb.y,
                       (v.z - mean) * rstd * g.z + bb.z, (v.w - mean) * rstd * g.w + bb.w);
            }
        }
    } else {
        const E* x = static_cast<const E*>(a.x);
        const int per_row = K * static_cast<int>(sizeof(E)) / 16;
        for (int i = threadIdx.x; i < a.rows * per_row; i += kGemvThreads) {
            const int r = i / per_row, c = i % per_row;
            reinterpret_cast<uint4*>(xs + r * K)[c] = __ldcg(reinterpret_cast<const uint4*>(x + r * a.ldx) + c);
        }
    }
    __syncthreads();
    if (a.bump_pos && blockIdx.x == 0 && threadIdx.x == 0) *a.pos = __ldcg(a.pos) + 1;

    constexpr int kCols = (kGemvWarps / KSPLIT) * CPW;
    const int ks = warp % KSPLIT;
    const int slice = K / KSPLIT;
    const int k_lo = ks * slice, k_hi = k_lo + slice;
    const int n_groups = (a.N + kCols - 1) / kCols;
    // column groups g = blockIdx.x, blockIdx.x + gridDim.x, ...: the staged rows serve them all
    for (int g = blockIdx.x; g < n_groups; g += gridDim.x) {
        const int n0 = g * kCols + (warp / KSPLIT) * CPW;
        float acc[CPW][ROWS];
#pragma unroll
        for (int c = 0; c < CPW; ++c)
#pragma unroll
            for (int r = 0; r < ROWS; ++r) acc[c][r] = 0.f;
        const E* wrow[CPW];
#pragma unroll
        for (int c = 0; c < CPW; ++c) wrow[c] = a.W + static_cast<long long>(min(n0 + c, a.N - 1)) * K;
#pragma unroll 4
        for (int k = k_lo + lane * 8; k < k_hi; k += 256) {
            float wf[CPW][8];
#pragma unroll
            for (int c = 0; c < CPW; ++c) load8(wrow[c] + k, wf[c]);
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                if (r < a.rows) {
                    float xf[8];
                    load8(xs + r * K + k, xf);
#pragma unroll
                    for (int c = 0; c < CPW; ++c) {
                        float sacc = acc[c][r];
#pragma unroll
                        for (int e = 0; e < 8; ++e) sacc = fmaf(wf[c][e], xf[e], sacc);
                        acc[c][r] = sacc;
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < CPW; ++c)
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                if (r < a.rows) {
                    const float v = warp_sum(acc[c][r]);
                    if (lane == 0) red[warp][c][r] = v;
                }
            }
        if (KSPLIT > 1) __syncthreads();
        else __syncwarp();
        for (int cr = lane; cr < CPW * ROWS; cr += 32) {
            const int c = cr / ROWS, r = cr % ROWS;
            const int n = n0 + c;
            if (ks == 0 && r < a.rows && n < a.N) {
                float v = 0.f;
#pragma unroll
                for (int j = 0; j < KSPLIT; ++j) v += red[warp + j][c][r];
                if (a.bias) v += to_f(a.bias[n]);
                if (EPI == DV_GELU) {
                    v = a.gelu_tanh ? gelu_tanh(v) : gelu_erf(v);
                    static_cast<E*>(a.out)[r * a.ldo + n] = from_f<E>(v);
                } else if (EPI == DV_RESID) {
                    float* o = static_cast<float*>(a.out) + r * a.ldo + n;
                    *o = __ldcg(o) + v;
                } else if (EPI == DV_F32) {
                    static_cast<float*>(a.out)[r * a.ldo + n] = v;
                } else if (EPI == DV_STORE) {
                    static_cast<E*>(a.out)[r * a.ldo + n] = from_f<E>(v);
                } else {  // DV_QKV
                    if (n < a.C) {
                        static_cast<E*>(a.out)[r * a.ldo + n] = from_f<E>(v);
                    } else {
                        const int p = __ldcg(a.pos);
                        if (p >= 0 && p < a.block_size)
                            a.kv[(static_cast<long long>(r) * a.block_size + p) * 2 * a.C + (n - a.C)] = from_f<E>(v);
                    }
                }
            }
        }
        if (KSPLIT > 1) __syncthreads();  // red is rewritten by the next group
        else __syncwarp();
    }
}

// ---------------------------------------------------------------- decode attention
// The newest position of sequence b, head h attends over cached positions 0..pos (the causal
// mask is implicit: no later key exists yet).  CTA (split, b*nh + h) takes kSplitKeys keys,
// one per thread for the scores; for p.v each warp takes half of the keys with a lane per
// pair of dimensions (coalesced rows).  With more than one split, each CTA leaves
// {m (log2 units), l, O[hs]} in part and the last CTA of the head to finish (a counter per
// head, reset by that CTA) merges them: y = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
constexpr int kSplitKeys = 64;
constexpr int kMaxHs = 128;

template <typename E> struct Pair;
template <> struct Pair<bf16> {
    static GPT_DEVINL float2 ld(const bf16* p) {
        const uint32_t v = __ldcg(reinterpret_cast<const unsigned int*>(p));
        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&v);
        return make_float2(__low2float(h), __high2float(h));
    }
    static GPT_DEVINL void st(bf16* p, float a, float b) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
    }
};
template <> struct Pair<float> {
    static GPT_DEVINL float2 ld(const float* p) { return __ldcg(reinterpret_cast<const float2*>(p)); }
    static GPT_DEVINL void st(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }
};

template <typename E>
__global__ void __launch_bounds__(kSplitKeys)
    decode_attention_kernel(const E* __restrict__ q, const E* __restrict__ kv, const int* __restrict__ pos,
                            float* __restrict__ part, int* __restrict__ counter, E* __restrict__ y, int nh, int hs,
                            int block_size, int n_split_max, float scale_log2) {
    griddep_launch_dependents();
    {
        // cached keys and values before the newest position do not change during this step:
        // prefetch this split's rows into L2 while the previous kernel finishes (a range read
        // from a position that is about to move is harmless for a prefetch)
        const int t = blockIdx.x * kSplitKeys + threadIdx.x;
        const int b = blockIdx.y / nh, h = blockIdx.y % nh, C = nh * hs;
        if (t < min(__ldcg(pos) + 1, block_size)) {
            const E* row = kv + (static_cast<long long>(b) * block_size + t) * 2 * C + h * hs;
            prefetch_l2(row, hs * sizeof(E));
            prefetch_l2(row + C, hs * sizeof(E));
        }
    }
    griddep_wait();
    __shared__ __align__(16) float qs[kMaxHs];
    __shared__ float ps[kSplitKeys];
    __shared__ float wmax[2], wsum[2];
    __shared__ float o1[kMaxHs];
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / nh, h = bh % nh;
    const int C = nh * hs;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_keys = min(__ldcg(pos) + 1, block_size);
    const int n_split = (n_keys + kSplitKeys - 1) / kSplitKeys;
    if (split >= n_split) return;
    const int k0 = split * kSplitKeys;
    for (int d = threadIdx.x; d < hs; d += kSplitKeys) qs[d] = ld_act(q + static_cast<long long>(b) * C + h * hs + d);
    __syncthreads();
    const E* base = kv + static_cast<long long>(b) * block_size * 2 * C + h * hs;
    const int t = k0 + threadIdx.x;
    float s = -INFINITY;
    if (t < n_keys) {
        const E* kr = base + static_cast<long long>(t) * 2 * C;
        float kf[kMaxHs / 8][8];  // the whole key row in flight at once
#pragma unroll
        for (int j = 0; j < kMaxHs / 8; ++j)
            if (8 * j < hs) load8_act(kr + 8 * j, kf[j]);
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxHs / 8; ++j)
            if (8 * j < hs) {
#pragma unroll
                for (int e = 0; e < 8; ++e) acc = fmaf(qs[8 * j + e], kf[j][e], acc);
            }
        s = acc * scale_log2;
    }
    float m = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[warp] = m;
    __syncthreads();
    m = fmaxf(wmax[0], wmax[1]);
    const float p = (t < n_keys) ? exp2f(s - m) : 0.f;
    ps[threadIdx.x] = p;
    const float lw = warp_sum(p);
    if (lane == 0) wsum[warp] = lw;
    __syncthreads();
    // p.v: warp w over keys [32w, 32w + 32) of the split, lane over dimension pairs
    const int n_here = min(kSplitKeys, n_keys - k0);
    const int i_lo = warp * 32, i_hi = min(i_lo + 32, n_here);
    float o[kMaxHs / 32];
#pragma unroll
    for (int j = 0; j < kMaxHs / 32; ++j) o[j] = 0.f;
    const E* vbase = base + C + static_cast<long long>(k0) * 2 * C;
#pragma unroll 16
    for (int i = i_lo; i < i_hi; ++i) {
        const float pi = ps[i];
        const E* vr = vbase + static_cast<long long>(i) * 2 * C;
#pragma unroll
        for (int j = 0; j < kMaxHs / 64; ++j) {
            const int d = 2 * lane + 64 * j;
            if (d < hs) {
                const float2 v = Pair<E>::ld(vr + d);
                o[2 * j] = fmaf(pi, v.x, o[2 * j]);
                o[2 * j + 1] = fmaf(pi, v.y, o[2 * j + 1]);
            }
        }
    }
    if (warp == 1) {
#pragma unroll
        for (int j = 0; j < kMaxHs / 64; ++j) {
            const int d = 2 * lane + 64 * j;
            if (d < hs) o1[d] = o[2 * j], o1[d + 1] = o[2 * j + 1];
        }
    }
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int j = 0; j < kMaxHs / 64; ++j) {
        const int d = 2 * lane + 64 * j;
        if (d < hs) o[2 * j] += o1[d], o[2 * j + 1] += o1[d + 1];
    }
    const float l = wsum[0] + wsum[1];
    E* yr = y + static_cast<long long>(b) * C + h * hs;
    if (n_split == 1) {
#pragma unroll
        for (int j = 0; j < kMaxHs / 64; ++j) {
            const int d = 2 * lane + 64 * j;
            if (d < hs) Pair<E>::st(yr + d, o[2 * j] / l, o[2 * j + 1] / l);
        }
        return;
    }
    float* mine = part + (static_cast<long long>(bh) * n_split_max + split) * (hs + 2);
#pragma unroll
    for (int j = 0; j < kMaxHs / 64; ++j) {
        const int d = 2 * lane + 64 * j;
        if (d < hs) mine[2 + d] = o[2 * j], mine[3 + d] = o[2 * j + 1];
    }
    if (lane == 0) mine[0] = m, mine[1] = l;
    __threadfence();
    __syncwarp();
    int ticket = 0;
    if (lane == 0) ticket = atomicAdd(counter + bh, 1);
    ticket = __shfl_sync(0xffffffffu, ticket, 0);
    if (ticket != n_split - 1) return;
    __threadfence();
    const float* pp = part + static_cast<long long>(bh) * n_split_max * (hs + 2);
    float M = -INFINITY;
#pragma unroll 8
    for (int sp = 0; sp < n_split; ++sp) M = fmaxf(M, __ldcg(pp + sp * (hs + 2)));
    float L = 0.f;
#pragma unroll 8
    for (int sp = 0; sp < n_split; ++sp) L += exp2f(__ldcg(pp + sp * (hs + 2)) - M) * __ldcg(pp + sp * (hs + 2) + 1);
#pragma unroll
    for (int j = 0; j < kMaxHs / 64; ++j) {
        const int d = 2 * lane + 64 * j;
        if (d < hs) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
            for (int sp = 0; sp < n_split; ++sp) {
                const float wgt = exp2f(__ldcg(pp + sp * (hs + 2)) - M);
                a0 = fmaf(wgt, __ldcg(pp + sp * (hs + 2) + 2 + d), a0);
                a1 = fmaf(wgt, __ldcg(pp + sp * (hs + 2) + 3 + d), a1);
            }
            Pair<E>::st(yr + d, a0 / L, a1 / L);
        }
    }
    if (lane == 0) counter[bh] = 0;
}

// k and v of positions [0, T) from the c_attn output qkv [B, T, 3C] into a layer's cache
// [B, block_size, 2C]; 16-byte units.
__global__ void kv_store_kernel(const uint8_t* __restrict__ qkv, uint8_t* __restrict__ kv, int B, int T,
                                long long row_bytes_qkv, long long c_bytes, int block_size) {
    griddep_launch_dependents();
    griddep_wait();
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long per_row = 2 * c_bytes / 16;
    if (i >= static_cast<long long>(B) * T * per_row) return;
    const long long row = i / per_row;  // b * T + t
    const long long off = (i % per_row) * 16;
    const long long b = row / T, t = row % T;
    *reinterpret_cast<uint4*>(kv + (b * block_size + t) * 2 * c_bytes + off) =
        __ldcg(reinterpret_cast<const uint4*>(qkv + row * row_bytes_qkv + c_bytes + off));
}

// dst[b, t] = src[b, t] for t < T (token buffers at row strides ld_src / ld_dst).
__global__ void copy_tokens_kernel(const int64_t* __restrict__ src, long long ld_src, int64_t* __restrict__ dst,
                                   long long ld_dst, int B, int T) {
    griddep_launch_dependents();
    griddep_wait();
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<long long>(B) * T) return;
    const long long b = i / T, t = i % T;
    dst[b * ld_dst + t] = __ldcg(src + b * ld_src + t);
}

// Sets the decode position and clears the attention merge counters (after a prefill).
__global__ void decode_reset_kernel(int* pos, int value, int* counter, int n_counter) {
    griddep_launch_dependents();
    griddep_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) *pos = value;
    if (i < n_counter) counter[i] = 0;
}

// ---------------------------------------------------------------- sampling
// Order-preserving map of a float to an unsigned key (larger float -> larger key); -0 and +0
// map to the same key, as they compare equal.
GPT_DEVINL uint32_t fkey(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSampleThreads = 1024;
constexpr int kSampleWarps = kSampleThreads / 32;
constexpr int kSampleMaxV = 52 * 1024;  // the row in shared memory: 208 KB (plus 16 KB of tables)

// Per row b: z = logits / temperature; keep z >= the top_k-th largest z (every z when
// top_k <= 0 or >= V; ties at the threshold are all kept); p = exp(z - max z) over the kept;
// choose the smallest index i with p_0 + ... + p_i > u[b] * sum(p).  The selection is made on
// the raw logits (dividing by a positive temperature keeps their order).
//
// One CTA per row stages the row in shared memory (V <= kSampleMaxV) and, in the same pass,
// counts the order-preserving 32-bit keys by their top 11 bits.  A scan from the top bin finds
// the bin holding the top_k-th largest key; its members (few, for a top-k of a spread-out
// row) are gathered and two more histogram levels over them (bits 20..10, then 9..0) give the
// k-th largest key itself.  (A bin with more than kSampleCand members is bisected over the whole
// row instead: the largest t with count(key >= t) >= top_k.)  For the draw, warp w owns the
// contiguous segment [w*seg, (w+1)*seg): the exponentials are fp32 and their sums fp64 (one
// entry's share of a flat distribution over tens of thousands of entries is not far above
// fp32 accumulation error).  Every thread adds the 32 segment sums in the same order, so
// exactly one warp's [prefix, prefix + sum) holds u * total; that warp walks its segment 32
// entries at a time with a warp scan.
constexpr int kSampleBins = 2048;
constexpr int kSampleCand = 2048;

// Block-wide sum of per-thread counts with one barrier.  Three accumulators rotate: call n adds
// into acc[n % 3] and clears acc[(n + 1) % 3], which no thread can still be reading (a thread
// reads acc[(n - 1) % 3] before it reaches call n's barrier).  acc[0] and acc[1] start at 0.
GPT_DEVINL uint32_t block_count(uint32_t c, uint32_t* acc, int& phase) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    uint32_t* cur = acc + phase % 3;
    if ((threadIdx.x & 31) == 0) atomicAdd(cur, c);
    if (threadIdx.x == 0) acc[(phase + 1) % 3] = 0;
    __syncthreads();
    ++phase;
    return *cur;
}

// Scan of hist[0, 2048) from the top bin down: the bin that holds the need-th largest entry
// (need >= 1 and at most the histogram's total), and that entry's rank inside the bin, into
// *s_bin / *s_need.  kSampleThreads threads, two bins each.
GPT_DEVINL void top_bin(const uint32_t* hist, uint32_t need, uint32_t* s_wtot, uint32_t* s_bin, uint32_t* s_need) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t h0 = hist[kSampleBins - 1 - 2 * tid], h1 = hist[kSampleBins - 2 - 2 * tid];
    uint32_t incl = h0 + h1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) s_wtot[warp] = incl;
    __syncthreads();
    uint32_t before = 0;
    for (int w = 0; w < warp; ++w) before += s_wtot[w];
    incl += before;
    const uint32_t excl = incl - h0 - h1;
    if (excl < need && incl >= need) {
        const bool first = excl + h0 >= need;
        *s_bin = first ? kSampleBins - 1 - 2 * tid : kSampleBins - 2 - 2 * tid;
        *s_need = first ? need - excl : need - excl - h0;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kSampleThreads)
    sample_kernel(const float* __restrict__ logits, long long ld_logits, int V, float temperature, int top_k,
                  const float* __restrict__ u, int64_t* __restrict__ out, long long ld_out) {
    griddep_launch_dependents();
    griddep_wait();
    extern __shared__ __align__(16) float zs[];  // the row, V floats
    __shared__ uint32_t hist[kSampleBins];
    __shared__ uint32_t cand[kSampleCand];
    __shared__ uint32_t s_acc[3], s_ncand, s_bin, s_need;
    __shared__ uint32_t s_wtot[kSampleWarps];
    __shared__ float s_wmax[kSampleWarps];
    __shared__ double s_wsum[kSampleWarps];
    const int b = blockIdx.x;
    const float* lg = logits + b * ld_logits;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool filter = top_k > 0 && top_k < V;

    for (int i = tid; i < kSampleBins; i += kSampleThreads) hist[i] = 0;
    if (tid < 2) s_acc[tid] = 0;
    if (tid == 0) s_ncand = 0;
    __syncthreads();
    float mx = -INFINITY;
    const bool vec = (V & 3) == 0 && (ld_logits & 3) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15) == 0;
    // 16-byte loads, eight in flight per thread (two rounds for V 50304)
    const int V4 = vec ? V >> 2 : 0;
    for (int i0 = tid; i0 < V4; i0 += 8 * kSampleThreads) {
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kSampleThreads;
            v[j] = i < V4 ? __ldcg(reinterpret_cast<const float4*>(lg) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kSampleThreads;
            if (i < V4) {
                reinterpret_cast<float4*>(zs)[i] = v[j];
                mx = fmaxf(mx, fmaxf(fmaxf(v[j].x, v[j].y), fmaxf(v[j].z, v[j].w)));
                if (filter) {
                    atomicAdd(&hist[fkey(v[j].x) >> 21], 1u);
                    atomicAdd(&hist[fkey(v[j].y) >> 21], 1u);
                    atomicAdd(&hist[fkey(v[j].z) >> 21], 1u);
                    atomicAdd(&hist[fkey(v[j].w) >> 21], 1u);
                }
            }
        }
    }
    // element loads otherwise, eight in flight per thread
    for (int i0 = vec ? V : tid; i0 < V; i0 += 8 * kSampleThreads) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kSampleThreads;
            v[j] = i < V ? __ldcg(lg + i) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kSampleThreads;
            if (i < V) {
                zs[i] = v[j];
                mx = fmaxf(mx, v[j]);
                if (filter) atomicAdd(&hist[fkey(v[j]) >> 21], 1u);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_wmax[warp] = mx;
    __syncthreads();
    float lmax = s_wmax[0];
    for (int w = 1; w < kSampleWarps; ++w) lmax = fmaxf(lmax, s_wmax[w]);
    const float m = lmax / temperature;  // the largest z (division is monotone)

    uint32_t thr_key = 0;  // key of the top_k-th largest logit
    if (filter) {
        top_bin(hist, static_cast<uint32_t>(top_k), s_wtot, &s_bin, &s_need);
        const uint32_t bin = s_bin, need2 = s_need;
        const uint32_t nbin = hist[bin];
        int phase = 0;
        uint32_t lo = bin << 21, hi = lo | ((1u << 21) - 1);  // invariant: count(key >= lo) >= need
        if (nbin <= kSampleCand) {
            // the bin's members, then two more histogram levels over them: bits 20..10, 9..0
            for (int i = tid; i < V; i += kSampleThreads) {
                const uint32_t key = fkey(zs[i]);
                if ((key >> 21) == bin) cand[atomicAdd(&s_ncand, 1u)] = key;
            }
            for (int i = tid; i < kSampleBins; i += kSampleThreads) hist[i] = 0;
            __syncthreads();
            for (uint32_t i = tid; i < nbin; i += kSampleThreads) atomicAdd(&hist[(cand[i] >> 10) & 2047u], 1u);
            __syncthreads();
            top_bin(hist, need2, s_wtot, &s_bin, &s_need);
            const uint32_t bin2 = s_bin, need3 = s_need;
            for (int i = tid; i < kSampleBins; i += kSampleThreads) hist[i] = 0;
            __syncthreads();
            for (uint32_t i = tid; i < nbin; i += kSampleThreads)
                if (((cand[i] >> 10) & 2047u) == bin2) atomicAdd(&hist[cand[i] & 1023u], 1u);
            __syncthreads();
            top_bin(hist, need3, s_wtot, &s_bin, &s_need);  // bins 1024.. are empty
            lo = (bin << 21) | (bin2 << 10) | s_bin;
        } else {
            for (int it = 0; it < 22 && lo < hi; ++it) {
                const uint32_t mid = lo + (hi - lo + 1) / 2;
                uint32_t c = 0;
                for (int i = tid; i < V; i += kSampleThreads) {
                    const uint32_t key = fkey(zs[i]);
                    c += (key >> 21) == bin && key >= mid;
                }
                if (block_count(c, s_acc, phase) >= need2) lo = mid;
                else hi = mid - 1;
            }
        }
        thr_key = lo;
    }

    // segment sums: lane-strided fp64 partials, then a butterfly
    const int seg = ((V + kSampleWarps * 32 - 1) / (kSampleWarps * 32)) * 32;
    const int s0 = min(V, warp * seg), s1 = min(V, s0 + seg);
    double part = 0.0;
    for (int i = s0 + lane; i < s1; i += 32) {
        const float li = zs[i];
        if (fkey(li) >= thr_key) part += static_cast<double>(expf(li / temperature - m));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) s_wsum[warp] = part;
    __syncthreads();
    double excl = 0.0, total = 0.0;
    for (int w = 0; w < kSampleWarps; ++w) {
        if (w == warp) excl = total;
        total += s_wsum[w];
    }
    const double seg_sum = s_wsum[warp];
    const double target = static_cast<double>(__ldcg(u + b)) * total;
    if (!(seg_sum > 0.0 && excl <= target && target < excl + seg_sum)) return;
    // this warp's segment holds the target: the first entry whose running sum passes it
    double cum = excl;
    long long last = -1;
    for (int i0 = s0; i0 < s1; i0 += 32) {
        const int i = i0 + lane;
        double p = 0.0;
        if (i < s1) {
            const float li = zs[i];
            if (fkey(li) >= thr_key) p = static_cast<double>(expf(li / temperature - m));
        }
        const uint32_t nz = __ballot_sync(0xffffffffu, p > 0.0);
        if (!nz) continue;  // nothing kept in these 32 entries: the running sum stays
        double c = p;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double n = __shfl_up_sync(0xffffffffu, c, o);
            if (lane >= o) c += n;
        }
        c += cum;
        const uint32_t hit = __ballot_sync(0xffffffffu, p > 0.0 && c > target);
        if (hit) {
            if (lane == __ffs(hit) - 1) out[b * ld_out] = i;
            return;
        }
        last = i0 + 31 - __clz(nz);
        cum = __shfl_sync(0xffffffffu, c, 31);
    }
    // rounding left the target past the segment's running sum: its last entry with p > 0
    if (lane == 0) out[b * ld_out] = last;
}

// The same draw with a row spread over a cluster of kSampleCtas CTAs (V >= kSampleClusterMinV): one
// CTA's instruction rate bounds the single-CTA kernel (three passes over the row by one SM).
// CTA rank r stages entries [r S, min(V, (r + 1) S)) of the row (S = ceil(V / kSampleCtas) rounded up
// to a multiple of 4) and counts their keys' top 11 bits; the counts meet in CTA 0's histogram
// (distributed shared memory), from which every CTA finds the bin of the top_k-th largest key; the
// bin's members are gathered into CTA 0, copied back by every CTA and resolved there (bits 20..10,
// 9..0), so each CTA knows the threshold key without another barrier.  (A bin of more than
// kSampleCand members is bisected: each step's count is summed across the cluster in CTA 0.)  The
// draw: each CTA sums its kept exponentials per warp segment in fp64; every CTA adds the CTAs'
// totals in rank order, so the interval [lo, hi) of warp w of CTA r has the same computed bounds in
// every CTA and the intervals tile [0, total) exactly; the one warp whose interval holds u * total
// walks its segment as in the single-CTA kernel.
constexpr int kSampleCtas = 8;
constexpr int kSampleClusterMinV = 4096;
constexpr int kCThreads = 512;
constexpr int kCWarps = kCThreads / 32;

// top_bin for kCThreads threads, four bins each.
GPT_DEVINL void top_bin_c(const uint32_t* hist, uint32_t need, uint32_t* s_wtot, uint32_t* s_bin, uint32_t* s_need) {
    constexpr int PER = kSampleBins / kCThreads;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t h[PER], sum = 0;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        h[k] = hist[kSampleBins - 1 - (PER * tid + k)];
        sum += h[k];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t nb = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nb;
    }
    if (lane == 31) s_wtot[warp] = incl;
    __syncthreads();
    uint32_t before = 0;
    for (int w = 0; w < warp; ++w) before += s_wtot[w];
    incl += before;
    uint32_t acc = incl - sum;
    if (acc < need && incl >= need) {
        bool found = false;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            if (!found && acc + h[k] >= need) {
                *s_bin = kSampleBins - 1 - (PER * tid + k);
                *s_need = need - acc;
                found = true;
            }
            acc += h[k];
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kCThreads)
    sample_cluster_kernel(const float* __restrict__ logits, long long ld_logits, int V, float temperature, int top_k,
                          const float* __restrict__ u, int64_t* __restrict__ out, long long ld_out) {
    griddep_launch_dependents();
    griddep_wait();
    extern __shared__ __align__(16) float zs[];  // this CTA's slice of the row
    __shared__ uint32_t hist[kSampleBins];       // this slice's counts; CTA 0's become the row's
    __shared__ uint32_t hist2[kSampleBins];      // the row's counts, then the finer levels
    __shared__ uint32_t cand[kSampleCand];       // the bin's members (gathered in CTA 0, copied by the rest)
    __shared__ uint32_t s_acc[3], s_ncand, s_bin, s_need;
    __shared__ uint32_t s_wtot[kCWarps];
    __shared__ float s_wmax[kCWarps];
    __shared__ double s_wsum[kCWarps];
    __shared__ uint32_t s_max;  // this slice's largest logit (float bits)
    __shared__ double s_tot;    // this slice's sum of kept exponentials
    const uint32_t rank = cluster_ctarank();
    const int b = static_cast<int>(blockIdx.x) / kSampleCtas;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float* lg = logits + b * ld_logits;
    const bool filter = top_k > 0 && top_k < V;
    const int S = ((V + kSampleCtas - 1) / kSampleCtas + 3) & ~3;
    const int c0 = min(V, static_cast<int>(rank) * S);
    const int n = min(V, c0 + S) - c0;

    for (int i = tid; i < kSampleBins; i += kCThreads) hist[i] = 0;
    if (tid < 3) s_acc[tid] = 0;
    if (tid == 0) s_ncand = 0;
    cluster_sync();  // every CTA of the cluster runs, its counters zero, before any remote access

    // 1. the slice: shared memory, its maximum, the histogram of its keys' top 11 bits
    float mx = -INFINITY;
    const bool vec = ((ld_logits | c0) & 3) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15) == 0;
    const int n4 = vec ? n >> 2 : 0;
    for (int i0 = tid; i0 < n4; i0 += 4 * kCThreads) {
        float4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * kCThreads;
            v[j] = i < n4 ? __ldcg(reinterpret_cast<const float4*>(lg + c0) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * kCThreads;
            if (i < n4) {
                reinterpret_cast<float4*>(zs)[i] = v[j];
                mx = fmaxf(mx, fmaxf(fmaxf(v[j].x, v[j].y), fmaxf(v[j].z, v[j].w)));
                if (filter) {
                    atomicAdd(&hist[fkey(v[j].x) >> 21], 1u);
                    atomicAdd(&hist[fkey(v[j].y) >> 21], 1u);
                    atomicAdd(&hist[fkey(v[j].z) >> 21], 1u);
                    atomicAdd(&hist[fkey(v[j].w) >> 21], 1u);
                }
            }
        }
    }
    for (int i = 4 * n4 + tid; i < n; i += kCThreads) {
        const float v = __ldcg(lg + c0 + i);
        zs[i] = v;
        mx = fmaxf(mx, v);
        if (filter) atomicAdd(&hist[fkey(v) >> 21], 1u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_wmax[warp] = mx;
    __syncthreads();
    if (tid == 0) {
        float m0 = s_wmax[0];
        for (int w = 1; w < kCWarps; ++w) m0 = fmaxf(m0, s_wmax[w]);
        s_max = __float_as_uint(m0);
    }
    // 2. the slice's counts into CTA 0's histogram
    if (filter && rank != 0) {
        const uint32_t h0 = map_to_rank(hist, 0);
        for (int t = tid; t < kSampleBins; t += kCThreads)
            if (hist[t]) red_cluster_add_u32(h0 + 4u * t, hist[t]);
    }
    cluster_sync();  // CTA 0 holds the row's counts; every slice maximum is written

    // 3. the row's maximum; the bin of the top_k-th largest key, found by every CTA
    float lmax = -INFINITY;
    for (int r = 0; r < kSampleCtas; ++r) lmax = fmaxf(lmax, __uint_as_float(ld_cluster_u32(map_to_rank(&s_max, r))));
    const float m = lmax / temperature;  // the largest z (division is monotone)
    uint32_t thr_key = 0;                // key of the top_k-th largest logit
    if (filter) {
        const uint32_t h0 = map_to_rank(hist, 0);
        for (int t = tid; t < kSampleBins; t += kCThreads) hist2[t] = rank == 0 ? hist[t] : ld_cluster_u32(h0 + 4u * t);
        __syncthreads();
        top_bin_c(hist2, static_cast<uint32_t>(top_k), s_wtot, &s_bin, &s_need);
        const uint32_t bin = s_bin, need2 = s_need;
        const uint32_t nbin = hist2[bin];
        uint32_t lo = bin << 21, hi = lo | ((1u << 21) - 1);  // invariant: count(key >= lo) >= need
        if (nbin <= kSampleCand) {
            // 4. the slice's members of the bin appended to CTA 0's list (one remote add per warp and pass)
            const uint32_t cnt0 = map_to_rank(&s_ncand, 0), cand0 = map_to_rank(cand, 0);
            for (int base = 0; base < n; base += kCThreads) {
                const int i = base + tid;
                const uint32_t key = i < n ? fkey(zs[i]) : 0u;
                const bool hit = i < n && (key >> 21) == bin;
                const uint32_t mask = __ballot_sync(0xffffffffu, hit);
                if (mask) {
                    uint32_t pos = 0;
                    if (lane == 0) pos = atom_cluster_add_u32(cnt0, static_cast<uint32_t>(__popc(mask)));
                    pos = __shfl_sync(0xffffffffu, pos, 0);
                    if (hit) st_cluster_u32(cand0 + 4u * (pos + __popc(mask & ((1u << lane) - 1u))), key);
                }
            }
            cluster_sync();  // CTA 0 holds the bin's nbin members
            // 5. every CTA resolves bits 20..10, then 9..0, from its own copy of the members
            if (rank != 0)
                for (uint32_t i = tid; i < nbin; i += kCThreads) cand[i] = ld_cluster_u32(cand0 + 4u * i);
            for (int i = tid; i < kSampleBins; i += kCThreads) hist2[i] = 0;
            __syncthreads();
            for (uint32_t i = tid; i < nbin; i += kCThreads) atomicAdd(&hist2[(cand[i] >> 10) & 2047u], 1u);
            __syncthreads();
            top_bin_c(hist2, need2, s_wtot, &s_bin, &s_need);
            const uint32_t bin2 = s_bin, need3 = s_need;
            for (int i = tid; i < kSampleBins; i += kCThreads) hist2[i] = 0;
            __syncthreads();
            for (uint32_t i = tid; i < nbin; i += kCThreads)
                if (((cand[i] >> 10) & 2047u) == bin2) atomicAdd(&hist2[cand[i] & 1023u], 1u);
            __syncthreads();
            top_bin_c(hist2, need3, s_wtot, &s_bin, &s_need);  // bins 1024.. are empty
            lo = (bin << 21) | (bin2 << 10) | s_bin;
        } else {
            // the bin bisected over the row; each step's count summed in CTA 0 (three rotating
            // counters: step k adds into s_acc[k % 3] and CTA 0 clears s_acc[(k + 1) % 3], which no CTA
            // can still be reading)
            const uint32_t acc0 = map_to_rank(s_acc, 0);
            for (int it = 0; it < 22 && lo < hi; ++it) {  // lo, hi agree in every CTA
                const uint32_t mid = lo + (hi - lo + 1) / 2;
                uint32_t c = 0;
                for (int i = tid; i < n; i += kCThreads) {
                    const uint32_t key = fkey(zs[i]);
                    c += (key >> 21) == bin && key >= mid;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
                if (lane == 0 && c) red_cluster_add_u32(acc0 + 4u * (it % 3), c);
                if (rank == 0 && tid == 0) s_acc[(it + 1) % 3] = 0;
                cluster_sync();
                if (ld_cluster_u32(acc0 + 4u * (it % 3)) >= need2) lo = mid;
                else hi = mid - 1;
            }
        }
        thr_key = lo;
    }

    // 6. the slice's kept exponentials summed per warp segment (fp64), then the CTAs' totals in order
    const int seg = ((n + kCWarps * 32 - 1) / (kCWarps * 32)) * 32;
    const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
    double part = 0.0;
    for (int i = s0 + lane; i < s1; i += 32) {
        const float li = zs[i];
        if (fkey(li) >= thr_key) part += static_cast<double>(expf(li / temperature - m));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) s_wsum[warp] = part;
    __syncthreads();
    double wlo = 0.0, whi = 0.0, ctot = 0.0;
    for (int w = 0; w < kCWarps; ++w) {
        if (w == warp) wlo = ctot;
        ctot += s_wsum[w];
        if (w == warp) whi = ctot;
    }
    if (tid == 0) s_tot = ctot;
    cluster_sync();  // every slice total written
    double before = 0.0, after = 0.0, total = 0.0;
    for (int r = 0; r < kSampleCtas; ++r) {
        if (r == static_cast<int>(rank)) before = total;
        total += ld_cluster_f64(map_to_rank(&s_tot, r));
        if (r == static_cast<int>(rank)) after = total;
    }
    cluster_sync();  // no CTA leaves while another may still read its shared memory
    // this warp's interval: [before + wlo, before + whi), its last warp's upper end the next slice's start
    const double target = static_cast<double>(__ldcg(u + b)) * total;
    const double lo_b = before + wlo, hi_b = warp + 1 < kCWarps ? before + whi : after;
    const double seg_sum = s_wsum[warp];
    if (!(seg_sum > 0.0 && lo_b <= target && target < hi_b)) return;
    double cum = lo_b;
    long long last = -1;
    for (int i0 = s0; i0 < s1; i0 += 32) {
        const int i = i0 + lane;
        double p = 0.0;
        if (i < s1) {
            const float li = zs[i];
            if (fkey(li) >= thr_key) p = static_cast<double>(expf(li / temperature - m));
        }
        const uint32_t nz = __ballot_sync(0xffffffffu, p > 0.0);
        if (!nz) continue;
        double c = p;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double nb = __shfl_up_sync(0xffffffffu, c, o);
            if (lane >= o) c += nb;
        }
        c += cum;
        const uint32_t hit = __ballot_sync(0xffffffffu, p > 0.0 && c > target);
        if (hit) {
            if (lane == __ffs(hit) - 1) out[b * ld_out] = c0 + i;
            return;
        }
        last = c0 + i0 + 31 - __clz(nz);
        cum = __shfl_sync(0xffffffffu, c, 31);
    }
    if (lane == 0) out[b * ld_out] = last;
}

}  // namespace

// ------------------------------------------------------------------ launchers
int launch_embed_pos(const void* wte, const void* wpe, const int64_t* tok, long long ld_tok, const int* pos, float* x,
                     int B, int C, int V, int block_size, int dtype, int32_t* status, cudaStream_t s) {
    const dim3 grid((B * C + 255) / 256), block(256);
    if (dtype == GPT_DTYPE_BF16)
        return launch_overlapped(embed_pos_kernel<bf16>, grid, block, 0, s, static_cast<const bf16*>(wte),
                                 static_cast<const bf16*>(wpe), tok, ld_tok, pos, x, B, C, V, block_size, status);
    return launch_overlapped(embed_pos_kernel<float>, grid, block, 0, s, static_cast<const float*>(wte),
                             static_cast<const float*>(wpe), tok, ld_tok, pos, x, B, C, V, block_size, status);
}

namespace {
template <typename E, int EPI, int KSPLIT, int CPW, bool LN, int ROWS>
int launch_gemv_inst(const GemvArgs<E>& a, cudaStream_t s) {
    constexpr int kCols = (kGemvWarps / KSPLIT) * CPW;
    const size_t smem = static_cast<size_t>(a.rows) * a.K * (sizeof(E) + (LN ? sizeof(float) : 0));
    auto kern = gemv_kernel<E, EPI, KSPLIT, CPW, LN, ROWS>;
    static size_t opted[kMaxDevices] = {};
    const int rc = opt_in_smem(reinterpret_cast<const void*>(kern), smem, opted);
    if (rc) return rc;
    int grid = (a.N + kCols - 1) / kCols;
    // With the LayerNorm prologue every CTA normalises all rows again: for the wide head product
    // a few CTAs per SM, each looping over column groups, share that work among more columns.
    if (LN && a.N >= 16384) grid = min(grid, 4 * num_sms());
    return launch_overlapped(kern, dim3(grid), dim3(kGemvThreads), smem, s, a);
}

// Warps per column: enough CTAs for narrow outputs, four columns a warp for the head (two with
// more than 8 rows, to keep the accumulators in registers).  ROWS: accumulator rows (8 or 16).
template <typename E, int EPI, bool LN, int ROWS>
int launch_gemv_mode(const GemvArgs<E>& a, cudaStream_t s) {
    if (a.N >= 16384) {
        if (ROWS > 8) return launch_gemv_inst<E, EPI, 1, 2, LN, ROWS>(a, s);
        return launch_gemv_inst<E, EPI, 1, 4, LN, ROWS>(a, s);
    }
    int ksplit = a.N <= 2048 ? 4 : 2;
    while (ksplit > 1 && (a.K % (8 * ksplit))) ksplit >>= 1;
    if (ksplit == 4) return launch_gemv_inst<E, EPI, 4, 1, LN, ROWS>(a, s);
    if (ksplit == 2) return launch_gemv_inst<E, EPI, 2, 1, LN, ROWS>(a, s);
    return launch_gemv_inst<E, EPI, 1, 1, LN, ROWS>(a, s);
}

template <typename E, int EPI, bool LN>
int launch_gemv_rows(const GemvArgs<E>& a, cudaStream_t s) {
    if (a.rows > 8) return launch_gemv_mode<E, EPI, LN, 16>(a, s);
    return launch_gemv_mode<E, EPI, LN, 8>(a, s);
}

template <typename E>
int gemv_typed(int epi, bool ln, const void* x, long long ldx, const E* ln_w, const E* ln_b, const E* W, const E* bias,
               void* out, long long ldo, int B, int N, int K, int gelu_tanh, E* kv, int* pos, int C, int block_size,
               int bump_pos, cudaStream_t s) {
    const size_t in_es = ln ? 4 : sizeof(E);
    const size_t out_es = (epi == DV_RESID || epi == DV_F32) ? 4 : sizeof(E);
    for (int r0 = 0; r0 < B; r0 += kGemvRows) {
        const int rows = min(kGemvRows, B - r0);
        GemvArgs<E> a{static_cast<const uint8_t*>(x) + static_cast<size_t>(r0) * ldx * in_es,
                      ldx,
                      ln_w,
                      ln_b,
                      W,
                      bias,
                      static_cast<uint8_t*>(out) + static_cast<size_t>(r0) * ldo * out_es,
                      ldo,
                      rows,
                      N,
                      K,
                      gelu_tanh,
                      kv ? kv + static_cast<long long>(r0) * block_size * 2 * C : nullptr,
                      pos,
                      C,
                      block_size,
                      (bump_pos && r0 + rows >= B) ? 1 : 0};
        int rc;
        if (ln) {
            switch (epi) {
                case DV_GELU: rc = launch_gemv_rows<E, DV_GELU, true>(a, s); break;
                case DV_F32: rc = launch_gemv_rows<E, DV_F32, true>(a, s); break;
                case DV_QKV: rc = launch_gemv_rows<E, DV_QKV, true>(a, s); break;
                case DV_STORE: rc = launch_gemv_rows<E, DV_STORE, true>(a, s); break;
                default: return GPT_ERR_UNSUPPORTED;
            }
        } else {
            switch (epi) {
                case DV_RESID: rc = launch_gemv_rows<E, DV_RESID, false>(a, s); break;
                case DV_F32: rc = launch_gemv_rows<E, DV_F32, false>(a, s); break;
                default: return GPT_ERR_UNSUPPORTED;
            }
        }
        if (rc) return rc;
    }
    return GPT_OK;
}
}  // namespace

int launch_gemv(int epi, bool ln, int dtype, const void* x, long long ldx, const void* ln_w, const void* ln_b,
                const void* W, const void* bias, void* out, long long ldo, int B, int N, int K, int gelu_tanh,
                void* kv, int* pos, int C, int block_size, int bump_pos, cudaStream_t s) {
    if (B < 1 || (K % 8) || (ln && (K % 4))) return GPT_ERR_UNSUPPORTED;
    if (dtype == GPT_DTYPE_BF16)
        return gemv_typed<bf16>(epi, ln, x, ldx, static_cast<const bf16*>(ln_w), static_cast<const bf16*>(ln_b),
                                static_cast<const bf16*>(W), static_cast<const bf16*>(bias), out, ldo, B, N, K,
                                gelu_tanh, static_cast<bf16*>(kv), pos, C, block_size, bump_pos, s);
    return gemv_typed<float>(epi, ln, x, ldx, static_cast<const float*>(ln_w), static_cast<const float*>(ln_b),
                             static_cast<const float*>(W), static_cast<const float*>(bias), out, ldo, B, N, K,
                             gelu_tanh, static_cast<float*>(kv), pos, C, block_size, bump_pos, s);
}

size_t gemv_smem_bytes(int B, int K, int dtype, bool ln) {
    const size_t es = dtype == GPT_DTYPE_BF16 ? 2 : 4;
    return static_cast<size_t>(min(B, kGemvRows)) * K * (es + (ln ? 4 : 0));
}

size_t decode_attn_part_floats(int B, int nh, int hs, int block_size) {
    const int n_split_max = (block_size + kSplitKeys - 1) / kSplitKeys;
    return static_cast<size_t>(B) * nh * n_split_max * (hs + 2);
}

int launch_decode_attention(int dtype, const void* q, const void* kv, const int* pos, float* part, int* counter,
                            void* y, int B, int nh, int hs, int block_size, cudaStream_t s) {
    if (hs > kMaxHs || (hs % 8)) return GPT_ERR_UNSUPPORTED;
    const int n_split_max = (block_size + kSplitKeys - 1) / kSplitKeys;
    const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(hs)));
    const dim3 grid(n_split_max, B * nh), block(kSplitKeys);
    if (dtype == GPT_DTYPE_BF16)
        return launch_overlapped(decode_attention_kernel<bf16>, grid, block, 0, s, static_cast<const bf16*>(q),
                                 static_cast<const bf16*>(kv), pos, part, counter, static_cast<bf16*>(y), nh, hs,
                                 block_size, n_split_max, scale_log2);
    return launch_overlapped(decode_attention_kernel<float>, grid, block, 0, s, static_cast<const float*>(q),
                             static_cast<const float*>(kv), pos, part, counter, static_cast<float*>(y), nh, hs,
                             block_size, n_split_max, scale_log2);
}

int launch_kv_store(const void* qkv, void* kv, int B, int T, int C, int elem_bytes, int block_size, cudaStream_t s) {
    const long long c_bytes = static_cast<long long>(C) * elem_bytes;
    if ((c_bytes % 16) || (reinterpret_cast<uintptr_t>(qkv) % 16) || (reinterpret_cast<uintptr_t>(kv) % 16))
        return GPT_ERR_BAD_ALIGN;
    const long long n = static_cast<long long>(B) * T * (2 * c_bytes / 16);
    return launch_overlapped(kv_store_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, s,
                             static_cast<const uint8_t*>(qkv), static_cast<uint8_t*>(kv), B, T, 3 * c_bytes, c_bytes,
                             block_size);
}

int launch_copy_tokens(const int64_t* src, long long ld_src, int64_t* dst, long long ld_dst, int B, int T,
                       cudaStream_t s) {
    const long long n = static_cast<long long>(B) * T;
    if (n == 0) return GPT_OK;
    return launch_overlapped(copy_tokens_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, s, src,
                             ld_src, dst, ld_dst, B, T);
}

int launch_decode_reset(int* pos, int value, int* counter, int n_counter, cudaStream_t s) {
    const int n = n_counter > 1 ? n_counter : 1;
    return launch_overlapped(decode_reset_kernel, dim3((n + 255) / 256), dim3(256), 0, s, pos, value, counter,
                             n_counter);
}

int sample_max_vocab() { return kSampleMaxV; }

int launch_sample(const float* logits, long long ld_logits, int B, int V, float temperature, int top_k,
                  const float* u, int64_t* out, long long ld_out, cudaStream_t s) {
    if (V > kSampleMaxV) return GPT_ERR_UNSUPPORTED;
    if (V >= kSampleClusterMinV) {
        const int S = ((V + kSampleCtas - 1) / kSampleCtas + 3) & ~3;
        // static + dynamic shared memory pass 48 KB: the dynamic part needs the opt-in
        static size_t opted_c[kMaxDevices] = {};
        const int rc = opt_in_smem(reinterpret_cast<const void*>(sample_cluster_kernel),
                                   ((kSampleMaxV + kSampleCtas - 1) / kSampleCtas + 3) / 4 * 4 * sizeof(float), opted_c);
        if (rc) return rc;
        return launch_overlapped_cluster(sample_cluster_kernel, kSampleCtas, dim3(B * kSampleCtas), dim3(kCThreads),
                                         static_cast<size_t>(S) * sizeof(float), s, logits, ld_logits, V, temperature,
                                         top_k, u, out, ld_out);
    }
    static size_t opted[kMaxDevices] = {};
    const int smem = V * static_cast<int>(sizeof(float));
    const int rc = opt_in_smem(reinterpret_cast<const void*>(sample_kernel), kSampleMaxV * sizeof(float), opted);
    if (rc) return rc;
    return launch_overlapped(sample_kernel, dim3(B), dim3(kSampleThreads), static_cast<size_t>(smem), s, logits,
                             ld_logits, V, temperature, top_k, u, out, ld_out);
}

}  // namespace gpt
