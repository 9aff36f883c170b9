// Incremental decoding ("nanoGPT 全局流程图", 第五阶段 generate): the forward of one new token per
// sequence against a key/value cache, and the sampling step (temperature, top-k, softmax,
// multinomial draw).
//
// A decode step reads every weight once for a handful of rows, so its matrix products are
// matrix-vector products bound by HBM bandwidth, not tensor-core work: one warp per output
// column streams the weight row with 16-byte loads against up to kGemvRows input rows staged
// in shared memory as fp32, and the epilogue (bias, GELU, residual add, k/v append) is fused.
// The attention of the new position against the cached keys is split over key ranges (so a
// long cache is read by many CTAs at once) and merged by a combine kernel.  The position being
// written lives in device memory, so a recorded graph of a step can be replayed as the
// sequence grows.
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

constexpr int kGemvWarps = 4;     // warps (= output columns in flight) per CTA
constexpr int kGemvRows = 8;      // input rows per launch (larger batches are split)
constexpr int kChunkK = 1024;     // K elements of each input row staged per pass
constexpr int kSplitKeys = 128;   // keys per CTA in the decode attention
constexpr int kMaxHs = 128;

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

template <typename E>
struct GemvArgs {
    const E* x;         // [rows, K] at row stride ldx
    long long ldx;
    const E* W;         // [N, K]
    const E* bias;      // [N] or null
    void* out;          // see GemvEpi
    long long ldo;
    int rows, N, K, gelu_tanh;
    E* kv;              // DV_QKV: this layer's cache [rows, block_size, 2C]
    const int* pos;
    int C, block_size;
};

enum GemvEpi {
    DV_STORE = 0,   // out E [rows, N]
    DV_GELU = 1,    // out E [rows, N] = gelu(.)
    DV_RESID = 2,   // out fp32 [rows, N] += .
    DV_F32 = 3,     // out fp32 [rows, N]
    DV_QKV = 4,     // columns [0, C) -> out E (q); [C, 3C) -> kv[row, *pos, :] (k then v)
};

// out[r, n] = epilogue(sum_k x[r, k] W[n, k] + bias[n]); one warp per column n, fixed
// summation order (lane-strided partial sums, then a butterfly).
template <typename E, int EPI>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const GemvArgs<E> a) {
    griddep_launch_dependents();
    griddep_wait();
    __shared__ __align__(16) float xs[kGemvRows * kChunkK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * kGemvWarps + warp;
    float acc[kGemvRows];
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r) acc[r] = 0.f;
    const E* wrow = a.W + static_cast<long long>(n < a.N ? n : 0) * a.K;
    for (int k0 = 0; k0 < a.K; k0 += kChunkK) {
        const int kc = min(kChunkK, a.K - k0);
        __syncthreads();
        for (int i = threadIdx.x; i < a.rows * kc; i += blockDim.x) {
            const int r = i / kc, k = i % kc;
            xs[r * kChunkK + k] = ld_act(a.x + r * a.ldx + k0 + k);
        }
        __syncthreads();
        if (n < a.N) {
#pragma unroll 2
            for (int k = lane * 8; k < kc; k += 256) {
                float wf[8];
                load8(wrow + k0 + k, wf);
#pragma unroll
                for (int r = 0; r < kGemvRows; ++r) {
                    if (r < a.rows) {
                        const float4 x0 = *reinterpret_cast<const float4*>(&xs[r * kChunkK + k]);
                        const float4 x1 = *reinterpret_cast<const float4*>(&xs[r * kChunkK + k + 4]);
                        float s = acc[r];
                        s = fmaf(wf[0], x0.x, s);
                        s = fmaf(wf[1], x0.y, s);
                        s = fmaf(wf[2], x0.z, s);
                        s = fmaf(wf[3], x0.w, s);
                        s = fmaf(wf[4], x1.x, s);
                        s = fmaf(wf[5], x1.y, s);
                        s = fmaf(wf[6], x1.z, s);
                        s = fmaf(wf[7], x1.w, s);
                        acc[r] = s;
                    }
                }
            }
        }
    }
    if (n >= a.N) return;
    const float bias = a.bias ? to_f(a.bias[n]) : 0.f;
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r) {
        if (r >= a.rows) break;
        float v = warp_sum(acc[r]) + bias;
        if (lane != 0) continue;
        if (EPI == DV_STORE) {
            static_cast<E*>(a.out)[r * a.ldo + n] = from_f<E>(v);
        } else if (EPI == DV_GELU) {
            v = a.gelu_tanh ? gelu_tanh(v) : gelu_erf(v);
            static_cast<E*>(a.out)[r * a.ldo + n] = from_f<E>(v);
        } else if (EPI == DV_RESID) {
            float* o = static_cast<float*>(a.out) + r * a.ldo + n;
            *o = __ldcg(o) + v;
        } else if (EPI == DV_F32) {
            static_cast<float*>(a.out)[r * a.ldo + n] = v;
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

// Attention of the newest position against cached keys 0..pos (the causal mask is implicit:
// no later key exists yet).  CTA (split, b*nh + h) scores keys [split*kSplitKeys, ...) with one
// key per thread and writes its partial {max m (log2 units), sum l, O[hs]} to part.
template <typename E>
__global__ void __launch_bounds__(kSplitKeys)
    decode_attn_partial(const E* __restrict__ q, const E* __restrict__ kv, const int* __restrict__ pos,
                        float* __restrict__ part, int nh, int hs, int block_size, int n_split_max, float scale_log2) {
    griddep_launch_dependents();
    griddep_wait();
    __shared__ __align__(16) float qs[kMaxHs];
    __shared__ float ps[kSplitKeys];
    __shared__ float red[kSplitKeys / 32];
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / nh, h = bh % nh;
    const int C = nh * hs;
    const int n_keys = min(__ldcg(pos) + 1, block_size);
    const int k0 = split * kSplitKeys;
    float* out = part + (static_cast<long long>(bh) * n_split_max + split) * (hs + 2);
    if (k0 >= n_keys) return;  // the combine reads only splits that hold keys
    for (int d = threadIdx.x; d < hs; d += blockDim.x) qs[d] = ld_act(q + static_cast<long long>(b) * C + h * hs + d);
    __syncthreads();
    const E* base = kv + static_cast<long long>(b) * block_size * 2 * C;
    const int t = k0 + threadIdx.x;
    float s = -INFINITY;
    if (t < n_keys) {
        const E* kr = base + static_cast<long long>(t) * 2 * C + h * hs;
        float acc = 0.f;
        for (int d = 0; d < hs; d += 8) {
            float kf[8];
            load8_act(kr + d, kf);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(qs[d + e], kf[e], acc);
        }
        s = acc * scale_log2;
    }
    float m = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < kSplitKeys / 32; ++w) m = fmaxf(m, red[w]);
    ps[threadIdx.x] = (t < n_keys) ? exp2f(s - m) : 0.f;
    __syncthreads();
    // O[d] = sum_i p_i v_i[d] over this split's keys, in key order
    const int n_here = min(kSplitKeys, n_keys - k0);
    for (int d = threadIdx.x; d < hs; d += blockDim.x) {
        const E* vc = base + static_cast<long long>(k0) * 2 * C + C + h * hs + d;
        float o = 0.f;
        for (int i = 0; i < n_here; ++i) o = fmaf(ps[i], ld_act(vc + static_cast<long long>(i) * 2 * C), o);
        out[2 + d] = o;
    }
    if (threadIdx.x == 0) {
        float l = 0.f;
        for (int i = 0; i < n_here; ++i) l += ps[i];
        out[0] = m;
        out[1] = l;
    }
}

// y = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s over the splits that hold keys.
template <typename E>
__global__ void decode_attn_combine(const float* __restrict__ part, const int* __restrict__ pos, E* __restrict__ y,
                                    int nh, int hs, int block_size, int n_split_max) {
    griddep_launch_dependents();
    griddep_wait();
    const int bh = blockIdx.x;
    const int b = bh / nh, h = bh % nh;
    const int n_keys = min(__ldcg(pos) + 1, block_size);
    const int n_split = (n_keys + kSplitKeys - 1) / kSplitKeys;
    const float* pp = part + static_cast<long long>(bh) * n_split_max * (hs + 2);
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, __ldcg(pp + s * (hs + 2)));
    float L = 0.f;
    for (int s = 0; s < n_split; ++s) L += exp2f(__ldcg(pp + s * (hs + 2)) - M) * __ldcg(pp + s * (hs + 2) + 1);
    for (int d = threadIdx.x; d < hs; d += blockDim.x) {
        float o = 0.f;
        for (int s = 0; s < n_split; ++s) o += exp2f(__ldcg(pp + s * (hs + 2)) - M) * __ldcg(pp + s * (hs + 2) + 2 + d);
        y[static_cast<long long>(b) * nh * hs + h * hs + d] = from_f<E>(o / L);
    }
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

__global__ void set_pos_kernel(int* pos, int value, int add) {
    griddep_launch_dependents();
    griddep_wait();
    *pos = add ? __ldcg(pos) + value : value;
}

// ---------------------------------------------------------------- sampling
// Order-preserving map of a float to an unsigned key (larger float -> larger key); -0 and +0
// map to the same key, as they compare equal.
GPT_DEVINL uint32_t fkey(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSampleThreads = 1024;

// Per row b: z = logits / temperature; keep z >= the top_k-th largest z (every z when
// top_k <= 0 or >= V; ties at the threshold are all kept); p = exp(z - max z) over the kept;
// choose the smallest index i with p_0 + ... + p_i > u[b] * sum(p).  The selection is made on
// the raw logits (dividing by a positive temperature keeps their order).  The exponentials
// are fp32; their sums are fp64, because with a flat distribution over tens of thousands of
// entries one entry's share (~1/V) is not far above fp32 accumulation error.  Fixed-order
// sums: thread j owns the contiguous range [j*chunk, (j+1)*chunk), and the per-thread sums
// are scanned in thread order.
__global__ void __launch_bounds__(kSampleThreads)
    sample_kernel(const float* __restrict__ logits, long long ld_logits, int V, float temperature, int top_k,
                  const float* __restrict__ u, int64_t* __restrict__ out, long long ld_out) {
    griddep_launch_dependents();
    griddep_wait();
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_prefix, s_need;
    __shared__ float s_f[kSampleThreads];
    __shared__ double s_d[kSampleThreads];
    __shared__ float s_max;
    const int b = blockIdx.x;
    const float* lg = logits + b * ld_logits;
    const int tid = threadIdx.x;
    const int chunk = (V + kSampleThreads - 1) / kSampleThreads;
    const int lo = min(V, tid * chunk), hi = min(V, lo + chunk);

    uint32_t thr_key = 0;  // key of the top_k-th largest logit (radix select, 8 bits a pass)
    if (top_k > 0 && top_k < V) {
        uint32_t prefix = 0, mask = 0, need = static_cast<uint32_t>(top_k);
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += kSampleThreads) hist[i] = 0;
            __syncthreads();
            for (int i = lo; i < hi; ++i) {
                const uint32_t key = fkey(__ldcg(lg + i));
                if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (tid == 0) {
                uint32_t cum = 0;
                int d = 255;
                for (; d > 0; --d) {
                    if (cum + hist[d] >= need) break;
                    cum += hist[d];
                }
                s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
                s_need = need - cum;
            }
            __syncthreads();
            prefix = s_prefix;
            need = s_need;
            mask |= 255u << shift;
        }
        thr_key = prefix;
    }
    float mx = -INFINITY;
    for (int i = lo; i < hi; ++i) mx = fmaxf(mx, __ldcg(lg + i) / temperature);
    s_f[tid] = mx;
    __syncthreads();
    for (int w = kSampleThreads / 2; w > 0; w >>= 1) {
        if (tid < w) s_f[tid] = fmaxf(s_f[tid], s_f[tid + w]);
        __syncthreads();
    }
    if (tid == 0) s_max = s_f[0];
    __syncthreads();
    const float m = s_max;
    double part = 0.0;
    for (int i = lo; i < hi; ++i)
        if (fkey(__ldcg(lg + i)) >= thr_key) part += static_cast<double>(expf(__ldcg(lg + i) / temperature - m));
    s_d[tid] = part;
    __syncthreads();
    if (tid != 0) return;
    double total = 0.0;
    for (int j = 0; j < kSampleThreads; ++j) total += s_d[j];
    const double target = static_cast<double>(__ldcg(u + b)) * total;
    double cum = 0.0;
    int j = 0;
    for (; j < kSampleThreads - 1; ++j) {
        if (cum + s_d[j] > target) break;
        cum += s_d[j];
    }
    long long pick = -1, last_kept = -1;
    for (int i = min(V, j * chunk), e = min(V, j * chunk + chunk); i < e; ++i) {
        if (fkey(__ldcg(lg + i)) < thr_key) continue;
        const float p = expf(__ldcg(lg + i) / temperature - m);
        if (p > 0.f) last_kept = i;
        cum += static_cast<double>(p);
        if (cum > target && p > 0.f) {
            pick = i;
            break;
        }
    }
    if (pick < 0) {
        // rounding left the target at or past the end of range j: take the last kept index
        // with nonzero probability at or before the end of that range
        for (int i = min(V, j * chunk + chunk) - 1; i >= 0 && last_kept < 0; --i)
            if (fkey(__ldcg(lg + i)) >= thr_key && expf(__ldcg(lg + i) / temperature - m) > 0.f) last_kept = i;
        pick = last_kept < 0 ? 0 : last_kept;
    }
    out[b * ld_out] = pick;
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
template <typename E>
int gemv_typed(int epi, const E* x, long long ldx, const E* W, const E* bias, void* out, long long ldo, int B, int N,
               int K, int gelu_tanh, E* kv, const int* pos, int C, int block_size, cudaStream_t s) {
    const dim3 grid((N + kGemvWarps - 1) / kGemvWarps), block(kGemvWarps * 32);
    const size_t out_es = (epi == DV_RESID || epi == DV_F32) ? 4 : sizeof(E);
    for (int r0 = 0; r0 < B; r0 += kGemvRows) {
        GemvArgs<E> a{x + r0 * ldx,
                      ldx,
                      W,
                      bias,
                      static_cast<uint8_t*>(out) + static_cast<size_t>(r0) * ldo * out_es,
                      ldo,
                      min(kGemvRows, B - r0),
                      N,
                      K,
                      gelu_tanh,
                      kv ? kv + static_cast<long long>(r0) * block_size * 2 * C : nullptr,
                      pos,
                      C,
                      block_size};
        int rc;
        switch (epi) {
            case DV_STORE: rc = launch_overlapped(gemv_kernel<E, DV_STORE>, grid, block, 0, s, a); break;
            case DV_GELU: rc = launch_overlapped(gemv_kernel<E, DV_GELU>, grid, block, 0, s, a); break;
            case DV_RESID: rc = launch_overlapped(gemv_kernel<E, DV_RESID>, grid, block, 0, s, a); break;
            case DV_F32: rc = launch_overlapped(gemv_kernel<E, DV_F32>, grid, block, 0, s, a); break;
            case DV_QKV: rc = launch_overlapped(gemv_kernel<E, DV_QKV>, grid, block, 0, s, a); break;
            default: return GPT_ERR_UNSUPPORTED;
        }
        if (rc) return rc;
    }
    return GPT_OK;
}
}  // namespace

int launch_gemv(int epi, int dtype, const void* x, long long ldx, const void* W, const void* bias, void* out,
                long long ldo, int B, int N, int K, int gelu_tanh, void* kv, const int* pos, int C, int block_size,
                cudaStream_t s) {
    if (B < 1 || (K % 8)) return GPT_ERR_UNSUPPORTED;
    if (dtype == GPT_DTYPE_BF16)
        return gemv_typed<bf16>(epi, static_cast<const bf16*>(x), ldx, static_cast<const bf16*>(W),
                                static_cast<const bf16*>(bias), out, ldo, B, N, K, gelu_tanh, static_cast<bf16*>(kv),
                                pos, C, block_size, s);
    return gemv_typed<float>(epi, static_cast<const float*>(x), ldx, static_cast<const float*>(W),
                             static_cast<const float*>(bias), out, ldo, B, N, K, gelu_tanh, static_cast<float*>(kv),
                             pos, C, block_size, s);
}

size_t decode_attn_part_floats(int B, int nh, int hs, int block_size) {
    const int n_split_max = (block_size + kSplitKeys - 1) / kSplitKeys;
    return static_cast<size_t>(B) * nh * n_split_max * (hs + 2);
}

int launch_decode_attention(int dtype, const void* q, const void* kv, const int* pos, float* part, void* y, int B,
                            int nh, int hs, int block_size, cudaStream_t s) {
    if (hs > kMaxHs || (hs % 8)) return GPT_ERR_UNSUPPORTED;
    const int n_split_max = (block_size + kSplitKeys - 1) / kSplitKeys;
    const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(hs)));
    const dim3 g1(n_split_max, B * nh), b1(kSplitKeys), g2(B * nh), b2(64);
    int rc;
    if (dtype == GPT_DTYPE_BF16) {
        rc = launch_overlapped(decode_attn_partial<bf16>, g1, b1, 0, s, static_cast<const bf16*>(q),
                               static_cast<const bf16*>(kv), pos, part, nh, hs, block_size, n_split_max, scale_log2);
        if (rc) return rc;
        return launch_overlapped(decode_attn_combine<bf16>, g2, b2, 0, s, static_cast<const float*>(part), pos,
                                 static_cast<bf16*>(y), nh, hs, block_size, n_split_max);
    }
    rc = launch_overlapped(decode_attn_partial<float>, g1, b1, 0, s, static_cast<const float*>(q),
                           static_cast<const float*>(kv), pos, part, nh, hs, block_size, n_split_max, scale_log2);
    if (rc) return rc;
    return launch_overlapped(decode_attn_combine<float>, g2, b2, 0, s, static_cast<const float*>(part), pos,
                             static_cast<float*>(y), nh, hs, block_size, n_split_max);
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

int launch_set_pos(int* pos, int value, int add, cudaStream_t s) {
    return launch_overlapped(set_pos_kernel, dim3(1), dim3(1), 0, s, pos, value, add);
}

int launch_sample(const float* logits, long long ld_logits, int B, int V, float temperature, int top_k,
                  const float* u, int64_t* out, long long ld_out, cudaStream_t s) {
    return launch_overlapped(sample_kernel, dim3(B), dim3(kSampleThreads), 0, s, logits, ld_logits, V, temperature,
                             top_k, u, out, ld_out);
}

}  // namespace gpt
