// Memory-bound row kernels: embedding gather + add, LayerNorm, and the cross-entropy
// reductions.  One warp per row where a row is reduced, 16-byte vector accesses throughout.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gpt {

namespace {

constexpr int kWarpsPerBlock = 8;

GPT_DEVINL float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
GPT_DEVINL float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

GPT_DEVINL float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
GPT_DEVINL float4 load4(const bf16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}
GPT_DEVINL void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
GPT_DEVINL void store4(bf16* p, float4 v) {
    uint2 u;
    u.x = pack_bf16x2(v.x, v.y);
    u.y = pack_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2*>(p) = u;
}

// x[b, t, :] = wte[idx[b, t], :] + wpe[t, :]   ("nanoGPT 全局流程图", §3.2 ①)
template <typename Tw>
__global__ void embed_kernel(const Tw* __restrict__ wte, const Tw* __restrict__ wpe,
                             const int64_t* __restrict__ idx, float* __restrict__ x, int T, int C,
                             int V, long long total4, int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= total4) return;
    const int c4 = C >> 2;
    const long long row = i / c4;
    const int c = static_cast<int>(i - row * c4) * 4;
    const int t = static_cast<int>(row % T);
    long long tok = idx[row];
    if (tok < 0 || tok >= V) {
        set_status(status, GPT_ERR_INDEX);
        tok = 0;
    }
    const float4 a = load4(wte + tok * C + c);
    const float4 p = load4(wpe + static_cast<long long>(t) * C + c);
    store4(x + row * C + c, make_float4(a.x + p.x, a.y + p.y, a.z + p.z, a.w + p.w));
}

// The same with a warp per row: the token id once per row, then every 4-element chunk of the
// row's wte and wpe slices loaded before any is added (VEC chunks per lane, C <= 128 VEC), so a
// warp keeps a whole row's loads in flight instead of one chunk per thread.
template <typename Tw, int VEC>
__global__ void embed_rows_kernel(const Tw* __restrict__ wte, const Tw* __restrict__ wpe,
                                  const int64_t* __restrict__ idx, float* __restrict__ x, int rows, int T, int C,
                                  int V, int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
    const int units = C >> 2;
    for (int row = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); row < rows; row += nwarps) {
        long long tok = idx[row];
        if (tok < 0 || tok >= V) {
            if (lane == 0) set_status(status, GPT_ERR_INDEX);
            tok = 0;
        }
        const Tw* er = wte + tok * C;
        const Tw* pr = wpe + static_cast<long long>(row % T) * C;
        float4 a[VEC], p[VEC];
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            const int u = lane + 32 * j;
            if (u < units) {
                a[j] = load4(er + 4 * u);
                p[j] = load4(pr + 4 * u);
            }
        }
        float* xr = x + static_cast<long long>(row) * C;
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            const int u = lane + 32 * j;
            if (u < units) store4(xr + 4 * u, make_float4(a[j].x + p[j].x, a[j].y + p[j].y, a[j].z + p[j].z, a[j].w + p[j].w));
        }
    }
}

// LayerNorm over rows of fp32 x, population variance, eps 1e-5 ("nanoGPT 全局流程图",
// §2.5 (A)).  The row stays in registers: mean, then sum of squared deviations.
constexpr int kLnMaxVec = 16;  // float4 per lane -> C <= 2048

// xcopy (optional): the input rows are also written there unchanged (the training forward keeps
// each residual stream state for the backward while the next projection adds into the copy).
template <typename To, int VEC>  // VEC = float4 per lane, ceil(C / 128): registers sized to the row
__global__ void layernorm_kernel(const float* __restrict__ x, const To* __restrict__ w,
                                 const To* __restrict__ bias, To* __restrict__ out, int rows, int C,
                                 float* __restrict__ xcopy) {
    griddep_launch_dependents();
    griddep_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kWarpsPerBlock + warp;
    if (row >= rows) return;
    const float* xr = x + static_cast<long long>(row) * C;
    const int nv = C >> 2;
    float4 v[VEC];
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
        const int j = lane + 32 * k;
        if (j < nv) {
            v[k] = load4(xr + 4 * j);
            s += (v[k].x + v[k].y) + (v[k].z + v[k].w);
        }
    }
    const float mean = warp_sum(s) / C;
    if (xcopy) {
        float* cr = xcopy + static_cast<long long>(row) * C;
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
            const int j = lane + 32 * k;
            if (j < nv) store4(cr + 4 * j, v[k]);
        }
    }
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
        const int j = lane + 32 * k;
        if (j < nv) {
            const float a = v[k].x - mean, b = v[k].y - mean, c = v[k].z - mean, d = v[k].w - mean;
            ss += (a * a + b * b) + (c * c + d * d);
        }
    }
    const float rstd = rsqrtf(warp_sum(ss) / C + 1e-5f);
    To* orow = out + static_cast<long long>(row) * C;
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
        const int j = lane + 32 * k;
        if (j < nv) {
            const float4 g = load4(w + 4 * j);
            float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
            if (bias) bb = load4(bias + 4 * j);
            float4 y;
            y.x = (v[k].x - mean) * rstd * g.x + bb.x;
            y.y = (v[k].y - mean) * rstd * g.y + bb.y;
            y.z = (v[k].z - mean) * rstd * g.z + bb.z;
            y.w = (v[k].w - mean) * rstd * g.w + bb.w;
            store4(orow + 4 * j, y);
        }
    }
}

// loss_r = logsumexp(z_r) - z_r[target]: combine the (max, sum exp(z - max)) pairs the lm_head
// epilogue left per column slice ("nanoGPT 全局流程图", §3.3).
__global__ void ce_rows_from_parts_kernel(const float2* __restrict__ part, int n_part,
                                          const float* __restrict__ tlogit,
                                          const int64_t* __restrict__ targets, int rows, int V,
                                          float* __restrict__ row_loss, int32_t* status,
                                          float* __restrict__ row_lse) {
    griddep_launch_dependents();
    griddep_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kWarpsPerBlock + warp;
    if (row >= rows) return;
    const long long t = targets[row];
    if (t == -1 || t < 0 || t >= V) {
        if (t != -1 && lane == 0) set_status(status, GPT_ERR_INDEX);
        if (lane == 0) row_loss[row] = 0.f;
        return;
    }
    const float2* pr = part + static_cast<long long>(row) * n_part;
    float m = -INFINITY;
    for (int j = lane; j < n_part; j += 32) {
        const float2 q = pr[j];
        if (q.y > 0.f) m = fmaxf(m, q.x);
    }
    m = warp_max(m);
    float s = 0.f;
    for (int j = lane; j < n_part; j += 32) {
        const float2 q = pr[j];
        if (q.y > 0.f) s += q.y * expf(q.x - m);
    }
    s = warp_sum(s);
    if (lane == 0) {
        const float l = m + logf(s);
        row_loss[row] = l - tlogit[row];
        if (row_lse) row_lse[row] = l;
    }
}

__global__ void ce_rows_from_logits_kernel(const float* __restrict__ logits,
                                           const int64_t* __restrict__ targets, int rows, int V,
                                           float* __restrict__ row_loss, int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kWarpsPerBlock + warp;
    if (row >= rows) return;
    const long long t = targets[row];
    if (t == -1 || t < 0 || t >= V) {
        if (t != -1 && lane == 0) set_status(status, GPT_ERR_INDEX);
        if (lane == 0) row_loss[row] = 0.f;
        return;
    }
    const float* z = logits + static_cast<long long>(row) * V;
    float m = -INFINITY;
    for (int j = lane; j < V; j += 32) m = fmaxf(m, z[j]);
    m = warp_max(m);
    float s = 0.f;
    for (int j = lane; j < V; j += 32) s += expf(z[j] - m);
    s = warp_sum(s);
    if (lane == 0) row_loss[row] = m + logf(s) - z[t];
}

// Mean over counted rows; one block, every thread sums a fixed stride of rows in fp64, then a
// fixed tree: the result does not depend on scheduling.
constexpr int kFinThreads = 1024;
__global__ void __launch_bounds__(kFinThreads)
    loss_finalize_kernel(const float* __restrict__ row_loss, const int64_t* __restrict__ targets,
                         int rows, int V, float* loss, double* sum_count) {
    griddep_launch_dependents();
    griddep_wait();
    __shared__ double s_sum[kFinThreads];
    __shared__ double s_cnt[kFinThreads];
    double a = 0.0, n = 0.0;
    for (int r = threadIdx.x; r < rows; r += kFinThreads) {
        const long long t = targets[r];
        if (t >= 0 && t < V) {
            a += static_cast<double>(row_loss[r]);
            n += 1.0;
        }
    }
    s_sum[threadIdx.x] = a;
    s_cnt[threadIdx.x] = n;
    __syncthreads();
    for (int w = kFinThreads / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w) {
            s_sum[threadIdx.x] += s_sum[threadIdx.x + w];
            s_cnt[threadIdx.x] += s_cnt[threadIdx.x + w];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double tot = s_sum[0], cnt = s_cnt[0];
        if (loss) *loss = cnt > 0.0 ? static_cast<float>(tot / cnt) : __int_as_float(0x7fc00000);
        if (sum_count) {
            sum_count[0] = tot;
            sum_count[1] = cnt;
        }
    }
}

}  // namespace

namespace {
template <typename Tw, int VEC = 1>
int launch_embed_rows(const Tw* wte, const Tw* wpe, const int64_t* idx, float* x, int rows, int T, int C, int V,
                      int32_t* status, cudaStream_t s) {
    if constexpr (VEC < 16) {
        if (C > 128 * VEC) return launch_embed_rows<Tw, VEC + 1>(wte, wpe, idx, x, rows, T, C, V, status, s);
    }
    const int warps = rows < 148 * 64 ? rows : 148 * 64;  // enough warps to keep every SM's loads in flight
    return launch_overlapped(embed_rows_kernel<Tw, VEC>, dim3((warps + 7) / 8), dim3(256), 0, s, wte, wpe, idx, x,
                             rows, T, C, V, status);
}
}  // namespace

int launch_embed(const void* wte, const void* wpe, const int64_t* idx, float* x, int B, int T, int C,
                 int V, int dtype, int32_t* status, cudaStream_t s) {
    const long long total4 = static_cast<long long>(B) * T * (C / 4);
    if (total4 == 0) return GPT_OK;
    if (C % 4 == 0 && C <= 2048 && static_cast<long long>(B) * T < (1LL << 31)) {
        const int rows = B * T;
        return dtype == GPT_DTYPE_BF16
                   ? launch_embed_rows(static_cast<const bf16*>(wte), static_cast<const bf16*>(wpe), idx, x, rows, T,
                                       C, V, status, s)
                   : launch_embed_rows(static_cast<const float*>(wte), static_cast<const float*>(wpe), idx, x, rows, T,
                                       C, V, status, s);
    }
    const int threads = 256;
    const unsigned blocks = static_cast<unsigned>((total4 + threads - 1) / threads);
    if (dtype == GPT_DTYPE_BF16)
        return launch_overlapped(embed_kernel<bf16>, dim3(blocks), dim3(threads), 0, s, static_cast<const bf16*>(wte),
                                 static_cast<const bf16*>(wpe), idx, x, T, C, V, total4, status);
    return launch_overlapped(embed_kernel<float>, dim3(blocks), dim3(threads), 0, s, static_cast<const float*>(wte),
                             static_cast<const float*>(wpe), idx, x, T, C, V, total4, status);
}

namespace {
template <typename To, int VEC>
int launch_ln_vec(const float* x, const void* w, const void* b, void* out, int rows, int C, float* xcopy,
                  cudaStream_t s) {
    const unsigned blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
    return launch_overlapped(layernorm_kernel<To, VEC>, dim3(blocks), dim3(32 * kWarpsPerBlock), 0, s, x,
                             static_cast<const To*>(w), static_cast<const To*>(b), static_cast<To*>(out), rows, C,
                             xcopy);
}

template <typename To, int VEC = 1>
int launch_ln(const float* x, const void* w, const void* b, void* out, int rows, int C, float* xcopy,
              cudaStream_t s) {
    if constexpr (VEC < kLnMaxVec) {
        if (C > 128 * VEC) return launch_ln<To, VEC + 1>(x, w, b, out, rows, C, xcopy, s);
    }
    return launch_ln_vec<To, VEC>(x, w, b, out, rows, C, xcopy, s);
}
}  // namespace

int launch_layernorm(const float* x, const void* w, const void* b, void* out, int rows, int C,
                     int dtype, cudaStream_t s, float* xcopy) {
    if (C > 4 * 32 * kLnMaxVec || (C & 3)) return GPT_ERR_UNSUPPORTED;
    if (rows == 0) return GPT_OK;
    if (dtype == GPT_DTYPE_BF16) return launch_ln<bf16>(x, w, b, out, rows, C, xcopy, s);
    return launch_ln<float>(x, w, b, out, rows, C, xcopy, s);
}

int launch_ce_rows_from_parts(const float2* part, int n_part, const float* tlogit,
                              const int64_t* targets, int rows, int V, float* row_loss,
                              int32_t* status, cudaStream_t s, float* row_lse) {
    if (rows == 0) return GPT_OK;
    const unsigned blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
    return launch_overlapped(ce_rows_from_parts_kernel, dim3(blocks), dim3(32 * kWarpsPerBlock), 0, s, part, n_part,
                             tlogit, targets, rows, V, row_loss, status, row_lse);
}

int launch_ce_rows_from_logits(const float* logits, const int64_t* targets, int rows, int V,
                               float* row_loss, int32_t* status, cudaStream_t s) {
    if (rows == 0) return GPT_OK;
    const unsigned blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
    return launch_overlapped(ce_rows_from_logits_kernel, dim3(blocks), dim3(32 * kWarpsPerBlock), 0, s, logits,
                             targets, rows, V, row_loss, status);
}

int launch_loss_finalize(const float* row_loss, const int64_t* targets, int rows, int V, float* loss,
                         double* sum_count, cudaStream_t s) {
    return launch_overlapped(loss_finalize_kernel, dim3(1), dim3(kFinThreads), 0, s, row_loss, targets, rows, V, loss,
                             sum_count);
}

}  // namespace gpt
