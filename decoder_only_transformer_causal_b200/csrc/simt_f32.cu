// fp32 path (GPT_DTYPE_F32) on the CUDA cores.  tcgen05 has no fp32 operand kind and tf32
// rounding (~1e-3 relative) would not hold an fp32 result to 1e-4, so the fp32 model runs
// these SIMT kernels: a tiled SGEMM with the same fused epilogues as the tensor-core GEMM,
// and a causal attention kernel with one warp per query row.  Both accumulate in a fixed
// order.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gpt {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

GPT_DEVINL float gelu32(float v, int tanh_mode) {
    if (tanh_mode)
        return 0.5f * v * (1.0f + tanhf(0.7978845608028654f * (v + 0.044715f * v * v * v)));
    return 0.5f * v * (1.0f + erff(v * 0.7071067811865476f));
}

// out[M, N] (=|+=) epi(A[M, K] W[N, K]^T + b); 256 threads, each a 4x4 block of outputs.
template <int EPI>
__global__ void __launch_bounds__(256)
    linear_f32_kernel(const float* __restrict__ A, long long lda, const float* __restrict__ W,
                      const float* __restrict__ bias, float* __restrict__ out, long long ldo, int M,
                      int N, int K, int gelu_tanh) {
    __shared__ float As[TK][TM + 4];
    __shared__ float Ws[TK][TN + 4];
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += TK) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = tid + 256 * q;
            const int r = e / TK, kk = e % TK;
            const int gm = m0 + r, gn = n0 + r, gk = k0 + kk;
            As[kk][r] = (gm < M && gk < K) ? A[static_cast<long long>(gm) * lda + gk] : 0.f;
            Ws[kk][r] = (gn < N && gk < K) ? W[static_cast<long long>(gn) * K + gk] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= N) continue;
            float v = acc[i][j] + (bias ? bias[n] : 0.f);
            float* o = out + static_cast<long long>(m) * ldo + n;
            if (EPI == GPT_EPI_GELU) v = gelu32(v, gelu_tanh);
            if (EPI == GPT_EPI_RESID) *o += v;
            else *o = v;
        }
    }
}

// Causal attention, fp32: one warp per query row i of one (b, h).  Scores for keys j <= i go
// to shared memory (each lane owns keys lane, lane+32, ...), then the row maximum, the
// exponentials and their sum, then y[d] = sum_j p_j v_j[d] / sum with lanes over d.
constexpr int kAttWarps = 4;
constexpr int kMaxHs = 128;

__global__ void __launch_bounds__(kAttWarps * 32)
    attention_f32_kernel(AttnLayoutF32 L, int B, int nh, int T, int hs, float scale) {
    extern __shared__ float sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* sq = sm + warp * (kMaxHs + T);
    float* sp = sq + kMaxHs;
    const long long gid = static_cast<long long>(blockIdx.x) * kAttWarps + warp;
    if (gid >= static_cast<long long>(B) * nh * T) return;
    const int i = static_cast<int>(gid % T);
    const int bh = static_cast<int>(gid / T);
    const int b = bh / nh, h = bh % nh;
    const float* q = L.q + b * L.sb + h * L.sh + static_cast<long long>(i) * L.st;
    const float* kb = L.k + b * L.sb + h * L.sh;
    const float* vb = L.v + b * L.sb + h * L.sh;
    for (int d = lane; d < hs; d += 32) sq[d] = q[d];
    __syncwarp();
    float mx = -INFINITY;
    for (int j = lane; j <= i; j += 32) {
        const float* kr = kb + static_cast<long long>(j) * L.st;
        float s = 0.f;
        for (int d = 0; d < hs; ++d) s = fmaf(sq[d], kr[d], s);
        s *= scale;
        sp[j] = s;
        mx = fmaxf(mx, s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int j = lane; j <= i; j += 32) {
        const float e = expf(sp[j] - mx);
        sp[j] = e;
        sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    __syncwarp();
    const float inv = 1.f / sum;
    if (L.lse && lane == 0) L.lse[static_cast<long long>(bh) * T + i] = (mx + logf(sum)) * 1.4426950408889634f;
    float* y = L.y + b * L.y_sb + h * L.y_sh + static_cast<long long>(i) * L.y_st;
    for (int d = lane; d < hs; d += 32) {
        float acc = 0.f;
        for (int j = 0; j <= i; ++j) acc = fmaf(sp[j], vb[static_cast<long long>(j) * L.st + d], acc);
        y[d] = acc * inv;
    }
}

}  // namespace

int launch_linear_f32(const float* A, long long lda, const float* W, const float* bias, float* out,
                      long long ldo, int M, int N, int K, int epilogue, int gelu, cudaStream_t s) {
    if (M == 0 || N == 0) return GPT_OK;
    dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
    switch (epilogue) {
        case GPT_EPI_STORE:
            linear_f32_kernel<GPT_EPI_STORE><<<grid, 256, 0, s>>>(A, lda, W, bias, out, ldo, M, N, K, gelu);
            break;
        case GPT_EPI_GELU:
            linear_f32_kernel<GPT_EPI_GELU><<<grid, 256, 0, s>>>(A, lda, W, bias, out, ldo, M, N, K, gelu);
            break;
        case GPT_EPI_RESID:
            linear_f32_kernel<GPT_EPI_RESID><<<grid, 256, 0, s>>>(A, lda, W, bias, out, ldo, M, N, K, gelu);
            break;
        default:
            return GPT_ERR_UNSUPPORTED;
    }
    return cuda_status(cudaGetLastError());
}

int launch_attention_f32(const AttnLayoutF32& L, int B, int nh, int T, int hs, cudaStream_t s) {
    if (hs > kMaxHs) return GPT_ERR_UNSUPPORTED;
    const long long rows = static_cast<long long>(B) * nh * T;
    if (rows == 0) return GPT_OK;
    const size_t smem = static_cast<size_t>(kAttWarps) * (kMaxHs + T) * sizeof(float);
    if (smem > 48 * 1024) {
        static size_t opted[kMaxDevices] = {};
        const int rc = opt_in_smem(reinterpret_cast<const void*>(attention_f32_kernel), smem, opted);
        if (rc) return rc;
    }
    const unsigned blocks = static_cast<unsigned>((rows + kAttWarps - 1) / kAttWarps);
    attention_f32_kernel<<<blocks, kAttWarps * 32, smem, s>>>(L, B, nh, T, hs, 1.0f / sqrtf(static_cast<float>(hs)));
    return cuda_status(cudaGetLastError());
}

}  // namespace gpt
