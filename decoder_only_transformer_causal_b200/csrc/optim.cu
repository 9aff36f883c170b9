// One optimizer step over the packed parameters ("nanoGPT 全局流程图", 3.6 梯度裁剪 + 参数更新 and
// 优化器配置): the global L2 norm of the gradients, clipping to max_norm, and AdamW with decoupled
// weight decay on the tensors with two or more dimensions only.
//
// Parameters, gradients and both Adam moments are fp32 arrays in the element layout of the
// packed weights (tensor i at byte offset / element size); the padding between tensors is never
// touched.  Both kernels are bound by HBM: the norm reads every gradient once (4 B per
// parameter), the update reads parameter, gradient and both moments and writes parameter, both
// moments and the configuration-dtype copy the forward reads (30 B per parameter for bf16).
//
// Work is cut into chunks of kChunk elements inside one tensor; a table of tensors (element
// offset, decay flag, first chunk) travels as a kernel parameter and a CTA finds a chunk's
// tensor by binary search.  The norm is deterministic: each CTA sums its chunks (i, i + grid,
// ...) in fp64, and the last CTA to finish adds the per-CTA sums in CTA order.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gpt {

namespace {

constexpr int kOptThreads = 256;
constexpr long long kChunk = 4096;  // elements

__device__ __forceinline__ int find_tensor(const OptTable& t, long long chunk) {
    int lo = 0, hi = t.n - 1;  // the last tensor whose first chunk is <= chunk
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (t.chunk0[mid] <= chunk) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ double block_sum(double v, double* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x == 0)
        for (int w = 0; w < kOptThreads / 32; ++w) s += red[w];  // warp order
    return s;
}

// part[blockIdx.x] = sum of g^2 over this CTA's chunks; the last CTA forms the norm, the clip
// factor min(1, max_norm / (norm + 1e-6)) (1 when max_norm <= 0) and clears the counter.
__global__ void __launch_bounds__(kOptThreads)
    grad_norm_kernel(const OptTable tab, const float* __restrict__ g, double* __restrict__ part,
                     unsigned int* __restrict__ counter, float* __restrict__ coef, float* __restrict__ norm_out,
                     float max_norm) {
    griddep_launch_dependents();
    griddep_wait();
    __shared__ double red[kOptThreads / 32];
    __shared__ bool last;
    double acc = 0.0;
    for (long long c = blockIdx.x; c < tab.chunk0[tab.n]; c += gridDim.x) {
        const int t = find_tensor(tab, c);
        const long long first = (c - tab.chunk0[t]) * kChunk;
        const long long n = min(kChunk, tab.numel[t] - first);
        const float4* src = reinterpret_cast<const float4*>(g + tab.off[t] + first);
        const long long n4 = n / 4;
        // four independent 16-byte loads in flight per thread; each float4's squares summed in
        // fp32, the running sum in fp64
        long long i = threadIdx.x;
        for (; i + 3 * kOptThreads < n4; i += 4 * kOptThreads) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = __ldcg(src + i + u * kOptThreads);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                acc += static_cast<double>((v[u].x * v[u].x + v[u].y * v[u].y) + (v[u].z * v[u].z + v[u].w * v[u].w));
        }
        for (; i < n4; i += kOptThreads) {
            const float4 v = __ldcg(src + i);
            acc += static_cast<double>((v.x * v.x + v.y * v.y) + (v.z * v.z + v.w * v.w));
        }
    }
    const double s = block_sum(acc, red);
    if (threadIdx.x == 0) {
        part[blockIdx.x] = s;
        __threadfence();
        last = atomicAdd(counter, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!last || threadIdx.x != 0) return;
    __threadfence();
    double tot = 0.0;
    for (unsigned int i = 0; i < gridDim.x; ++i) tot += __ldcg(part + i);
    const double nrm = sqrt(tot);
    double f = 1.0;
    if (max_norm > 0.f) f = fmin(1.0, static_cast<double>(max_norm) / (nrm + 1e-6));
    *coef = static_cast<float>(f);
    if (norm_out) *norm_out = static_cast<float>(nrm);
    *counter = 0;
}

template <typename E>
GPT_DEVINL void store_copy4(E* p, float a, float b, float c, float d);
template <>
GPT_DEVINL void store_copy4<bf16>(bf16* p, float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&lo);
    v.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = v;
}
template <>
GPT_DEVINL void store_copy4<float>(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}

struct AdamwArgs {
    float lr, beta1, beta2, eps, weight_decay;
    float step_size;   // lr / (1 - beta1^step)
    float bc2_sqrt;    // sqrt(1 - beta2^step)
};

GPT_DEVINL float adamw1(float& p, float g, float& m, float& v, float wd, const AdamwArgs& a) {
    p = p * (1.f - a.lr * wd);
    m = a.beta1 * m + (1.f - a.beta1) * g;
    v = a.beta2 * v + (1.f - a.beta2) * g * g;
    p = p - a.step_size * m / (sqrtf(v) / a.bc2_sqrt + a.eps);
    return p;
}

// p, m, v updated in place; copy (the packed weights the forward reads) receives p in E.
template <typename E>
__global__ void __launch_bounds__(kOptThreads)
    adamw_kernel(const OptTable tab, float* __restrict__ p, const float* __restrict__ g, float* __restrict__ m,
                 float* __restrict__ v, E* __restrict__ copy, const float* __restrict__ coef, const AdamwArgs a) {
    griddep_launch_dependents();
    griddep_wait();
    const float f = __ldcg(coef);
    for (long long c = blockIdx.x; c < tab.chunk0[tab.n]; c += gridDim.x) {
        const int t = find_tensor(tab, c);
        const long long first = tab.off[t] + (c - tab.chunk0[t]) * kChunk;
        const long long n = min(kChunk, tab.numel[t] - (c - tab.chunk0[t]) * kChunk);
        const float wd = tab.decay[t] ? a.weight_decay : 0.f;
        for (long long i = threadIdx.x * 4; i < n; i += kOptThreads * 4) {
            const long long e = first + i;
            float4 pp = __ldcg(reinterpret_cast<const float4*>(p + e));
            const float4 gg = __ldcg(reinterpret_cast<const float4*>(g + e));
            float4 mm = __ldcg(reinterpret_cast<const float4*>(m + e));
            float4 vv = __ldcg(reinterpret_cast<const float4*>(v + e));
            adamw1(pp.x, gg.x * f, mm.x, vv.x, wd, a);
            adamw1(pp.y, gg.y * f, mm.y, vv.y, wd, a);
            adamw1(pp.z, gg.z * f, mm.z, vv.z, wd, a);
            adamw1(pp.w, gg.w * f, mm.w, vv.w, wd, a);
            *reinterpret_cast<float4*>(p + e) = pp;
            *reinterpret_cast<float4*>(m + e) = mm;
            *reinterpret_cast<float4*>(v + e) = vv;
            if (copy) store_copy4<E>(copy + e, pp.x, pp.y, pp.z, pp.w);
        }
    }
}

}  // namespace

long long opt_chunk_elems() { return kChunk; }

int launch_adamw(const OptTable& tab, int dtype, float* params, const float* grads, float* m, float* v, void* copy,
                 float lr, float beta1, float beta2, float eps, float weight_decay, int step, float max_norm,
                 float* norm_out, void* ws, cudaStream_t s) {
    uint8_t* w = static_cast<uint8_t*>(ws);
    unsigned int* counter = reinterpret_cast<unsigned int*>(w);
    float* coef = reinterpret_cast<float*>(w + 4);
    double* part = reinterpret_cast<double*>(w + 256);
    const long long chunks = tab.chunk0[tab.n];
    const int grid_norm = static_cast<int>(chunks < 4LL * num_sms() ? chunks : 4LL * num_sms());
    const int grid_upd = static_cast<int>(chunks < 4LL * num_sms() ? chunks : 4LL * num_sms());
    if (grid_norm < 1) return GPT_OK;
    int rc = cuda_status(cudaMemsetAsync(counter, 0, sizeof(unsigned int), s));
    if (rc) return rc;
    rc = launch_overlapped(grad_norm_kernel, dim3(grid_norm), dim3(kOptThreads), 0, s, tab, grads, part, counter,
                           coef, norm_out, max_norm);
    if (rc) return rc;
    AdamwArgs a;
    a.lr = lr;
    a.beta1 = beta1;
    a.beta2 = beta2;
    a.eps = eps;
    a.weight_decay = weight_decay;
    a.step_size = static_cast<float>(static_cast<double>(lr) / (1.0 - pow(static_cast<double>(beta1), step)));
    a.bc2_sqrt = static_cast<float>(sqrt(1.0 - pow(static_cast<double>(beta2), step)));
    if (dtype == GPT_DTYPE_BF16)
        return launch_overlapped(adamw_kernel<bf16>, dim3(grid_upd), dim3(kOptThreads), 0, s, tab, params, grads, m,
                                 v, static_cast<bf16*>(copy), static_cast<const float*>(coef), a);
    return launch_overlapped(adamw_kernel<float>, dim3(grid_upd), dim3(kOptThreads), 0, s, tab, params, grads, m, v,
                             static_cast<float*>(copy), static_cast<const float*>(coef), a);
}

size_t adamw_workspace_bytes() { return 256 + 8 * 4096; }

int adamw_max_grid() { return 4096; }

}  // namespace gpt
