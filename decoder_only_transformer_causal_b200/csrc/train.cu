// Kernels the training step adds around the tensor-core GEMM ("nanoGPT 全局流程图", 3.4 反向传播):
// transposes / conversions that turn the Linear layers' backward products into the GEMM's
// A[M,K] B[N,K]^T form, the GELU applied to a stored pre-activation, and the causal attention's
// backward.
//
// Attention backward (per batch b, head h; s_ij = q_i . k_j, p_ij = 2^(s_ij * scale_log2 - lse2_i)
// with lse2 the forward's per-row log2-sum-exp, so P is recomputed, never stored):
//   D_i   = sum_d dO_i[d] O_i[d]
//   dS_ij = p_ij (dO_i . v_j - D_i)               for j <= i, 0 above the diagonal
//   dQ_i  = sum_j dS_ij k_j / sqrt(hs),  dK_j = sum_i dS_ij q_i / sqrt(hs),  dV_j = sum_i p_ij dO_i
// This first version runs on the SIMT pipes: two threads per row, each holding half of the head
// dimensions in registers, with the other side's 64-row tiles staged in shared memory and read by
// broadcast; the two halves of a dot product meet in one shuffle.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gpt {

namespace {

GPT_DEVINL float ldf(const bf16* p) {
    return __bfloat162float(__ushort_as_bfloat16(__ldcg(reinterpret_cast<const unsigned short*>(p))));
}
GPT_DEVINL float ldf(const float* p) { return __ldcg(p); }
template <typename E> GPT_DEVINL E stf(float v);
template <> GPT_DEVINL bf16 stf<bf16>(float v) { return __float2bfloat16_rn(v); }
template <> GPT_DEVINL float stf<float>(float v) { return v; }

// out[c, r] = in[r, c] for an R x Cc matrix (row strides ld_in / ld_out), converting the type;
// 32 x 32 tiles through shared memory.
template <typename Ti, typename To>
__global__ void transpose_kernel(const Ti* __restrict__ in, long long ld_in, To* __restrict__ out, long long ld_out,
                                 int R, int Cc) {
    griddep_launch_dependents();
    griddep_wait();
    __shared__ float tile[32][33];
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int k = threadIdx.y; k < 32; k += blockDim.y) {
        const int r = r0 + k, c = c0 + threadIdx.x;
        tile[k][threadIdx.x] = (r < R && c < Cc) ? ldf(in + r * ld_in + c) : 0.f;
    }
    __syncthreads();
    for (int k = threadIdx.y; k < 32; k += blockDim.y) {
        const int c = c0 + k, r = r0 + threadIdx.x;
        if (c < Cc && r < R) out[c * ld_out + r] = stf<To>(tile[threadIdx.x][k]);
    }
}

template <typename Ti, typename To>
__global__ void convert_kernel(const Ti* __restrict__ in, To* __restrict__ out, long long n) {
    griddep_launch_dependents();
    griddep_wait();
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) out[i] = stf<To>(ldf(in + i));
}

template <typename E>
__global__ void gelu_forward_kernel(const E* __restrict__ pre, E* __restrict__ h, long long n, int tanh_form) {
    griddep_launch_dependents();
    griddep_wait();
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float z = ldf(pre + i);
    const float g = tanh_form ? 0.5f * z * (1.f + tanhf(0.7978845608028654f * (z + 0.044715f * z * z * z)))
                              : 0.5f * z * (1.f + erff(z * 0.7071067811865476f));
    h[i] = stf<E>(g);
}

// ------------------------------------------------------------------ attention backward
// D[bh * T + i] = sum_d dO_i[d] O_i[d]; one warp per row.
template <typename E>
__global__ void attn_bwd_rowdot_kernel(const AttnBwdLayout<E> L, int B, int nh, int T, int hs, float* __restrict__ D) {
    griddep_launch_dependents();
    griddep_wait();
    const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= static_cast<long long>(B) * nh * T) return;
    const int i = static_cast<int>(row % T);
    const int bh = static_cast<int>(row / T), b = bh / nh, h = bh % nh;
    const E* o = L.o + b * L.o_sb + h * L.o_sh + static_cast<long long>(i) * L.o_st;
    const E* g = L.dout + b * L.o_sb + h * L.o_sh + static_cast<long long>(i) * L.o_st;
    float s = 0.f;
    for (int d = lane; d < hs; d += 32) s += ldf(o + d) * ldf(g + d);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) D[row] = s;
}

constexpr int kBwdRows = 64;  // rows per CTA and per staged tile

// dQ for 64 query rows of one (b, h): thread (row, half); key tiles of 64 in shared memory.
template <typename E, int HS>
__global__ void __launch_bounds__(2 * kBwdRows)
    attn_bwd_dq_kernel(const AttnBwdLayout<E> L, int nh, int T, float scale_log2, float inv_sqrt_hs,
                       const float* __restrict__ D) {
    griddep_launch_dependents();
    griddep_wait();
    constexpr int H2 = HS / 2;
    __shared__ float ks[kBwdRows][HS + 1], vs[kBwdRows][HS + 1];
    const int bh = blockIdx.y, b = bh / nh, h = bh % nh;
    const int half = threadIdx.x & 1;
    const int i = blockIdx.x * kBwdRows + (threadIdx.x >> 1);
    const bool live = i < T;
    const int ic = live ? i : T - 1;
    const E* q = L.q + b * L.sb + h * L.sh + static_cast<long long>(ic) * L.st + half * H2;
    const E* g = L.dout + b * L.o_sb + h * L.o_sh + static_cast<long long>(ic) * L.o_st + half * H2;
    float qr[H2], gr[H2], acc[H2];
#pragma unroll
    for (int d = 0; d < H2; ++d) qr[d] = ldf(q + d), gr[d] = ldf(g + d), acc[d] = 0.f;
    const float lse = __ldcg(L.lse + static_cast<long long>(bh) * T + ic);
    const float Di = __ldcg(D + static_cast<long long>(bh) * T + ic);
    const int last_row = min(T - 1, (blockIdx.x + 1) * kBwdRows - 1);
    for (int j0 = 0; j0 <= last_row; j0 += kBwdRows) {
        __syncthreads();
        for (int e = threadIdx.x; e < kBwdRows * HS; e += 2 * kBwdRows) {
            const int jj = e / HS, d = e % HS, j = min(j0 + jj, T - 1);
            ks[jj][d] = ldf(L.k + b * L.sb + h * L.sh + static_cast<long long>(j) * L.st + d);
            vs[jj][d] = ldf(L.v + b * L.sb + h * L.sh + static_cast<long long>(j) * L.st + d);
        }
        __syncthreads();
        const int jn = min(kBwdRows, last_row - j0 + 1);
        for (int jj = 0; jj < jn; ++jj) {
            const int j = j0 + jj;
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int d = 0; d < H2; ++d) {
                s = fmaf(qr[d], ks[jj][half * H2 + d], s);
                dp = fmaf(gr[d], vs[jj][half * H2 + d], dp);
            }
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            dp += __shfl_xor_sync(0xffffffffu, dp, 1);
            const float p = (live && j <= i) ? exp2f(s * scale_log2 - lse) : 0.f;
            const float ds = p * (dp - Di);
#pragma unroll
            for (int d = 0; d < H2; ++d) acc[d] = fmaf(ds, ks[jj][half * H2 + d], acc[d]);
        }
    }
    if (!live) return;
    E* dq = L.dq + b * L.sb + h * L.sh + static_cast<long long>(i) * L.st + half * H2;
#pragma unroll
    for (int d = 0; d < H2; ++d) dq[d] = stf<E>(acc[d] * inv_sqrt_hs);
}

// dK and dV for 64 key rows of one (b, h): thread (row, half); query tiles of 64 (with their
// lse and D) in shared memory, from the diagonal tile down.
template <typename E, int HS>
__global__ void __launch_bounds__(2 * kBwdRows)
    attn_bwd_dkdv_kernel(const AttnBwdLayout<E> L, int nh, int T, float scale_log2, float inv_sqrt_hs,
                         const float* __restrict__ D) {
    griddep_launch_dependents();
    griddep_wait();
    constexpr int H2 = HS / 2;
    __shared__ float qs[kBwdRows][HS + 1], gs[kBwdRows][HS + 1];
    __shared__ float ls[kBwdRows], dsum[kBwdRows];
    const int bh = blockIdx.y, b = bh / nh, h = bh % nh;
    const int half = threadIdx.x & 1;
    const int j = blockIdx.x * kBwdRows + (threadIdx.x >> 1);
    const bool live = j < T;
    const int jc = live ? j : T - 1;
    const E* k = L.k + b * L.sb + h * L.sh + static_cast<long long>(jc) * L.st + half * H2;
    const E* v = L.v + b * L.sb + h * L.sh + static_cast<long long>(jc) * L.st + half * H2;
    float kr[H2], vr[H2], dk[H2], dv[H2];
#pragma unroll
    for (int d = 0; d < H2; ++d) kr[d] = ldf(k + d), vr[d] = ldf(v + d), dk[d] = 0.f, dv[d] = 0.f;
    for (int i0 = blockIdx.x * kBwdRows; i0 < T; i0 += kBwdRows) {
        __syncthreads();
        for (int e = threadIdx.x; e < kBwdRows * HS; e += 2 * kBwdRows) {
            const int ii = e / HS, d = e % HS, i = min(i0 + ii, T - 1);
            qs[ii][d] = ldf(L.q + b * L.sb + h * L.sh + static_cast<long long>(i) * L.st + d);
            gs[ii][d] = ldf(L.dout + b * L.o_sb + h * L.o_sh + static_cast<long long>(i) * L.o_st + d);
        }
        for (int ii = threadIdx.x; ii < kBwdRows; ii += 2 * kBwdRows) {
            const int i = min(i0 + ii, T - 1);
            ls[ii] = __ldcg(L.lse + static_cast<long long>(bh) * T + i);
            dsum[ii] = __ldcg(D + static_cast<long long>(bh) * T + i);
        }
        __syncthreads();
        const int in = min(kBwdRows, T - i0);
        for (int ii = 0; ii < in; ++ii) {
            const int i = i0 + ii;
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int d = 0; d < H2; ++d) {
                s = fmaf(kr[d], qs[ii][half * H2 + d], s);
                dp = fmaf(vr[d], gs[ii][half * H2 + d], dp);
            }
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            dp += __shfl_xor_sync(0xffffffffu, dp, 1);
            const float p = (live && j <= i) ? exp2f(s * scale_log2 - ls[ii]) : 0.f;
            const float ds = p * (dp - dsum[ii]);
#pragma unroll
            for (int d = 0; d < H2; ++d) {
                dv[d] = fmaf(p, gs[ii][half * H2 + d], dv[d]);
                dk[d] = fmaf(ds, qs[ii][half * H2 + d], dk[d]);
            }
        }
    }
    if (!live) return;
    E* odk = L.dk + b * L.sb + h * L.sh + static_cast<long long>(j) * L.st + half * H2;
    E* odv = L.dv + b * L.sb + h * L.sh + static_cast<long long>(j) * L.st + half * H2;
#pragma unroll
    for (int d = 0; d < H2; ++d) odk[d] = stf<E>(dk[d] * inv_sqrt_hs), odv[d] = stf<E>(dv[d]);
}

template <typename E, int HS>
int attn_bwd_typed(const AttnBwdLayout<E>& L, int B, int nh, int T, float* D, cudaStream_t s) {
    const long long rows = static_cast<long long>(B) * nh * T;
    int rc = launch_overlapped(attn_bwd_rowdot_kernel<E>, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256), 0, s,
                               L, B, nh, T, HS, D);
    if (rc) return rc;
    const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(HS)));
    const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(HS)));
    const dim3 grid((T + kBwdRows - 1) / kBwdRows, B * nh), block(2 * kBwdRows);
    rc = launch_overlapped(attn_bwd_dq_kernel<E, HS>, grid, block, 0, s, L, nh, T, scale_log2, inv,
                           static_cast<const float*>(D));
    if (rc) return rc;
    return launch_overlapped(attn_bwd_dkdv_kernel<E, HS>, grid, block, 0, s, L, nh, T, scale_log2, inv,
                             static_cast<const float*>(D));
}

}  // namespace

int launch_transpose(const void* in, int in_dtype, long long ld_in, void* out, int out_dtype, long long ld_out, int R,
                     int Cc, cudaStream_t s) {
    if (R == 0 || Cc == 0) return GPT_OK;
    const dim3 grid((Cc + 31) / 32, (R + 31) / 32), block(32, 8);
    const bool ib = in_dtype == GPT_DTYPE_BF16, ob = out_dtype == GPT_DTYPE_BF16;
    if (ib && ob)
        return launch_overlapped(transpose_kernel<bf16, bf16>, grid, block, 0, s, static_cast<const bf16*>(in), ld_in,
                                 static_cast<bf16*>(out), ld_out, R, Cc);
    if (!ib && ob)
        return launch_overlapped(transpose_kernel<float, bf16>, grid, block, 0, s, static_cast<const float*>(in),
                                 ld_in, static_cast<bf16*>(out), ld_out, R, Cc);
    if (ib && !ob)
        return launch_overlapped(transpose_kernel<bf16, float>, grid, block, 0, s, static_cast<const bf16*>(in), ld_in,
                                 static_cast<float*>(out), ld_out, R, Cc);
    return launch_overlapped(transpose_kernel<float, float>, grid, block, 0, s, static_cast<const float*>(in), ld_in,
                             static_cast<float*>(out), ld_out, R, Cc);
}

int launch_convert(const void* in, int in_dtype, void* out, int out_dtype, long long n, cudaStream_t s) {
    if (n == 0) return GPT_OK;
    const dim3 grid(static_cast<unsigned>((n + 255) / 256)), block(256);
    const bool ib = in_dtype == GPT_DTYPE_BF16, ob = out_dtype == GPT_DTYPE_BF16;
    if (!ib && ob)
        return launch_overlapped(convert_kernel<float, bf16>, grid, block, 0, s, static_cast<const float*>(in),
                                 static_cast<bf16*>(out), n);
    if (ib && !ob)
        return launch_overlapped(convert_kernel<bf16, float>, grid, block, 0, s, static_cast<const bf16*>(in),
                                 static_cast<float*>(out), n);
    if (ib)
        return launch_overlapped(convert_kernel<bf16, bf16>, grid, block, 0, s, static_cast<const bf16*>(in),
                                 static_cast<bf16*>(out), n);
    return launch_overlapped(convert_kernel<float, float>, grid, block, 0, s, static_cast<const float*>(in),
                             static_cast<float*>(out), n);
}

int launch_gelu_forward(const void* pre, void* h, long long n, int dtype, int tanh_form, cudaStream_t s) {
    if (n == 0) return GPT_OK;
    const dim3 grid(static_cast<unsigned>((n + 255) / 256)), block(256);
    if (dtype == GPT_DTYPE_BF16)
        return launch_overlapped(gelu_forward_kernel<bf16>, grid, block, 0, s, static_cast<const bf16*>(pre),
                                 static_cast<bf16*>(h), n, tanh_form);
    return launch_overlapped(gelu_forward_kernel<float>, grid, block, 0, s, static_cast<const float*>(pre),
                             static_cast<float*>(h), n, tanh_form);
}

int launch_attention_backward(const AttnBwdLayout<bf16>* Lb, const AttnBwdLayout<float>* Lf, int B, int nh, int T,
                              int hs, float* D, cudaStream_t s) {
    if (B == 0 || nh == 0 || T == 0) return GPT_OK;
    if (Lb) {
        if (hs == 64) return attn_bwd_typed<bf16, 64>(*Lb, B, nh, T, D, s);
        if (hs == 32) return attn_bwd_typed<bf16, 32>(*Lb, B, nh, T, D, s);
        return GPT_ERR_UNSUPPORTED;
    }
    if (hs == 64) return attn_bwd_typed<float, 64>(*Lf, B, nh, T, D, s);
    if (hs == 32) return attn_bwd_typed<float, 32>(*Lf, B, nh, T, D, s);
    return GPT_ERR_UNSUPPORTED;
}

}  // namespace gpt
