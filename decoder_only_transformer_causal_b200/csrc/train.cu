// Kernels the training step adds around the tensor-core GEMM ("nanoGPT 全局流程图", 3.4 反向传播):
// the transpose that gives the fp32 path's backward products their A[M,K] B[N,K]^T operands (the
// bf16 path reads MN-major operands in place), the GELU and its derivative applied to a stored
// pre-activation, and the causal attention's backward.
//
// Attention backward (per batch b, head h; s_ij = q_i . k_j, p_ij = 2^(s_ij * scale_log2 - lse2_i)
// with lse2 the forward's per-row log2-sum-exp, so P is recomputed, never stored):
//   D_i   = sum_d dO_i[d] O_i[d]
//   dS_ij = p_ij (dO_i . v_j - D_i)               for j <= i, 0 above the diagonal
//   dQ_i  = sum_j dS_ij k_j / sqrt(hs),  dK_j = sum_i dS_ij q_i / sqrt(hs),  dV_j = sum_i p_ij dO_i
// bf16 with head size 64 runs on the tensor cores (attention_bwd_tc.cu); the kernels here cover fp32,
// head size 32 and operands TMA cannot address: two threads per row, each holding half of the
// head dimensions in registers, with the other side's 64-row tiles staged in shared memory and
// read by broadcast; the two halves of a dot product meet in one shuffle.
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

// Elementwise kernels: thread t takes values [8t, 8t + 8) with 16-byte accesses when `vec` (every
// buffer 16-byte aligned) and the group is whole, one value at a time otherwise.
GPT_DEVINL float gelu_value(float z, int tanh_form) {
    return tanh_form ? 0.5f * z * (1.f + tanhf(0.7978845608028654f * (z + 0.044715f * z * z * z)))
                     : 0.5f * z * (1.f + erff(z * 0.7071067811865476f));
}

template <typename E>
__global__ void gelu_forward_kernel(const E* __restrict__ pre, E* __restrict__ h, long long n, int tanh_form, int vec) {
    griddep_launch_dependents();
    griddep_wait();
    const long long i0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
    if (i0 >= n) return;
    if (vec && i0 + 8 <= n) {
        float v[8];
        ld8(pre + i0, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = gelu_value(v[e], tanh_form);
        st8(h + i0, v);
        return;
    }
    for (long long i = i0; i < n && i < i0 + 8; ++i) h[i] = stf<E>(gelu_value(ldf(pre + i), tanh_form));
}

// pre <- gelu'(pre) in place (the training forward's fallback when c_fc cannot write both outputs
// in one epilogue: the backward reads the derivative, not the pre-activation).
template <typename E>
__global__ void gelu_deriv_inplace_kernel(E* __restrict__ pre, long long n, int tanh_form, int vec) {
    griddep_launch_dependents();
    griddep_wait();
    const long long i0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
    if (i0 >= n) return;
    if (vec && i0 + 8 <= n) {
        float v[8];
        ld8(pre + i0, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = gelu_slope(v[e], tanh_form);
        st8(pre + i0, v);
        return;
    }
    for (long long i = i0; i < n && i < i0 + 8; ++i) pre[i] = stf<E>(gelu_slope(ldf(pre + i), tanh_form));
}

// ------------------------------------------------------------------ attention backward
// Per (b, h) and query row i < Tp (Tp = T rounded up to 128): D[bh * Tp + i] = sum_d dO_i[d] O_i[d]
// and L2[bh * Tp + i] = -lse2_i (the forward's, negated for the tensor-core kernels' exponent FMA);
// rows i >= T hold D = 0 and L2 = -inf (p = 0 there).
// hs / 8 threads per row, each with one 8-value slice of dO_i and O_i (16-byte loads when `vec`);
// the slices meet in shuffles within the row's lane group.
template <typename E>
__global__ void attn_bwd_rowdot_kernel(const AttnBwdLayout<E> L, int B, int nh, int T, int Tp, int hs,
                                       float* __restrict__ D, float* __restrict__ L2, int vec) {
    griddep_launch_dependents();
    griddep_wait();
    const int G = hs / 8;  // 4 or 8: divides 32, so a row's lanes sit in one warp
    const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long row = t / G;
    const int part = static_cast<int>(t % G);
    const bool valid = row < static_cast<long long>(B) * nh * Tp;
    const int i = valid ? static_cast<int>(row % Tp) : 0;
    const int bh = valid ? static_cast<int>(row / Tp) : 0, b = bh / nh, h = bh % nh;
    float s = 0.f;
    if (valid && i < T) {
        const E* o = L.o + b * L.o_sb + h * L.o_sh + static_cast<long long>(i) * L.o_st + part * 8;
        const E* g = L.dout + b * L.o_sb + h * L.o_sh + static_cast<long long>(i) * L.o_st + part * 8;
        float ov[8], gv[8];
        if (vec) {
            ld8(o, ov);
            ld8(g, gv);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) ov[e] = ldf(o + e), gv[e] = ldf(g + e);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) s = fmaf(ov[e], gv[e], s);
    }
    for (int off = G / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (valid && part == 0) {
        D[row] = i < T ? s : 0.f;
        L2[row] = i < T ? -__ldcg(L.lse + static_cast<long long>(bh) * T + i) : -INFINITY;
    }
}

constexpr int kBwdRows = 64;  // rows per CTA and per staged tile

// dQ for 64 query rows of one (b, h): thread (row, half); key tiles of 64 in shared memory.
template <typename E, int HS>
__global__ void __launch_bounds__(2 * kBwdRows)
    attn_bwd_dq_kernel(const AttnBwdLayout<E> L, int nh, int T, int Tp, float scale_log2, float inv_sqrt_hs,
                       const float* __restrict__ D) {
    griddep_launch_dependents();
    griddep_wait();
    constexpr int H2 = HS / 2;
    __shared__ __align__(16) float ks[kBwdRows][HS + 4], vs[kBwdRows][HS + 4];
    const int bh = blockIdx.y, b = bh / nh, h = bh % nh;
    const int half = threadIdx.x & 1;
    const int tile = gridDim.x - 1 - blockIdx.x;  // the last query tiles see the most keys: start them first
    const int i = tile * kBwdRows + (threadIdx.x >> 1);
    const bool live = i < T;
    const int ic = live ? i : T - 1;
    const E* q = L.q + b * L.sb + h * L.sh + static_cast<long long>(ic) * L.st + half * H2;
    const E* g = L.dout + b * L.o_sb + h * L.o_sh + static_cast<long long>(ic) * L.o_st + half * H2;
    float qr[H2], gr[H2], acc[H2];
#pragma unroll
    for (int d = 0; d < H2; ++d) qr[d] = ldf(q + d), gr[d] = ldf(g + d), acc[d] = 0.f;
    const float lse = __ldcg(L.lse + static_cast<long long>(bh) * T + ic);
    const float Di = __ldcg(D + static_cast<long long>(bh) * Tp + ic);
    const int last_row = min(T - 1, (tile + 1) * kBwdRows - 1);
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
            const float4* kr4 = reinterpret_cast<const float4*>(&ks[jj][half * H2]);
            const float4* vr4 = reinterpret_cast<const float4*>(&vs[jj][half * H2]);
            float s4[4] = {0.f, 0.f, 0.f, 0.f}, p4[4] = {0.f, 0.f, 0.f, 0.f};  // independent chains
#pragma unroll
            for (int d = 0; d < H2 / 4; ++d) {
                const float4 kk = kr4[d], vv = vr4[d];
                s4[0] = fmaf(qr[4 * d], kk.x, s4[0]);
                s4[1] = fmaf(qr[4 * d + 1], kk.y, s4[1]);
                s4[2] = fmaf(qr[4 * d + 2], kk.z, s4[2]);
                s4[3] = fmaf(qr[4 * d + 3], kk.w, s4[3]);
                p4[0] = fmaf(gr[4 * d], vv.x, p4[0]);
                p4[1] = fmaf(gr[4 * d + 1], vv.y, p4[1]);
                p4[2] = fmaf(gr[4 * d + 2], vv.z, p4[2]);
                p4[3] = fmaf(gr[4 * d + 3], vv.w, p4[3]);
            }
            float s = (s4[0] + s4[1]) + (s4[2] + s4[3]), dp = (p4[0] + p4[1]) + (p4[2] + p4[3]);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            dp += __shfl_xor_sync(0xffffffffu, dp, 1);
            const float p = (live && j <= i) ? exp2f(s * scale_log2 - lse) : 0.f;
            const float ds = p * (dp - Di);
#pragma unroll
            for (int d = 0; d < H2 / 4; ++d) {
                const float4 kk = kr4[d];
                acc[4 * d] = fmaf(ds, kk.x, acc[4 * d]);
                acc[4 * d + 1] = fmaf(ds, kk.y, acc[4 * d + 1]);
                acc[4 * d + 2] = fmaf(ds, kk.z, acc[4 * d + 2]);
                acc[4 * d + 3] = fmaf(ds, kk.w, acc[4 * d + 3]);
            }
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
    attn_bwd_dkdv_kernel(const AttnBwdLayout<E> L, int nh, int T, int Tp, float scale_log2, float inv_sqrt_hs,
                         const float* __restrict__ D) {
    griddep_launch_dependents();
    griddep_wait();
    constexpr int H2 = HS / 2;
    __shared__ __align__(16) float qs[kBwdRows][HS + 4], gs[kBwdRows][HS + 4];
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
            dsum[ii] = __ldcg(D + static_cast<long long>(bh) * Tp + i);
        }
        __syncthreads();
        const int in = min(kBwdRows, T - i0);
        for (int ii = 0; ii < in; ++ii) {
            const int i = i0 + ii;
            const float4* qr4 = reinterpret_cast<const float4*>(&qs[ii][half * H2]);
            const float4* gr4 = reinterpret_cast<const float4*>(&gs[ii][half * H2]);
            float s4[4] = {0.f, 0.f, 0.f, 0.f}, p4[4] = {0.f, 0.f, 0.f, 0.f};  // independent chains
#pragma unroll
            for (int d = 0; d < H2 / 4; ++d) {
                const float4 qq = qr4[d], gg = gr4[d];
                s4[0] = fmaf(kr[4 * d], qq.x, s4[0]);
                s4[1] = fmaf(kr[4 * d + 1], qq.y, s4[1]);
                s4[2] = fmaf(kr[4 * d + 2], qq.z, s4[2]);
                s4[3] = fmaf(kr[4 * d + 3], qq.w, s4[3]);
                p4[0] = fmaf(vr[4 * d], gg.x, p4[0]);
                p4[1] = fmaf(vr[4 * d + 1], gg.y, p4[1]);
                p4[2] = fmaf(vr[4 * d + 2], gg.z, p4[2]);
                p4[3] = fmaf(vr[4 * d + 3], gg.w, p4[3]);
            }
            float s = (s4[0] + s4[1]) + (s4[2] + s4[3]), dp = (p4[0] + p4[1]) + (p4[2] + p4[3]);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            dp += __shfl_xor_sync(0xffffffffu, dp, 1);
            const float p = (live && j <= i) ? exp2f(s * scale_log2 - ls[ii]) : 0.f;
            const float ds = p * (dp - dsum[ii]);
#pragma unroll
            for (int d = 0; d < H2 / 4; ++d) {
                const float4 qq = qr4[d], gg = gr4[d];
                dv[4 * d] = fmaf(p, gg.x, dv[4 * d]);
                dv[4 * d + 1] = fmaf(p, gg.y, dv[4 * d + 1]);
                dv[4 * d + 2] = fmaf(p, gg.z, dv[4 * d + 2]);
                dv[4 * d + 3] = fmaf(p, gg.w, dv[4 * d + 3]);
                dk[4 * d] = fmaf(ds, qq.x, dk[4 * d]);
                dk[4 * d + 1] = fmaf(ds, qq.y, dk[4 * d + 1]);
                dk[4 * d + 2] = fmaf(ds, qq.z, dk[4 * d + 2]);
                dk[4 * d + 3] = fmaf(ds, qq.w, dk[4 * d + 3]);
            }
        }
    }
    if (!live) return;
    E* odk = L.dk + b * L.sb + h * L.sh + static_cast<long long>(j) * L.st + half * H2;
    E* odv = L.dv + b * L.sb + h * L.sh + static_cast<long long>(j) * L.st + half * H2;
#pragma unroll
    for (int d = 0; d < H2; ++d) odk[d] = stf<E>(dk[d] * inv_sqrt_hs), odv[d] = stf<E>(dv[d]);
}

// D / L2: the padded [B*nh, Tp] arrays of attn_bwd_rowdot_kernel.
template <typename E, int HS>
int attn_bwd_typed(const AttnBwdLayout<E>& L, int B, int nh, int T, float* D, float* L2, int32_t* status,
                   cudaStream_t s, const AttnBwdColsum* cs, bool* cs_done) {
    const int Tp = (T + 127) / 128 * 128;
    const long long threads = static_cast<long long>(B) * nh * Tp * (HS / 8);
    const int vec = ((reinterpret_cast<uintptr_t>(L.o) | reinterpret_cast<uintptr_t>(L.dout)) & 15) == 0 &&
                    ((L.o_sb | L.o_sh | L.o_st) * static_cast<long long>(sizeof(E))) % 16 == 0;
    int rc = launch_overlapped(attn_bwd_rowdot_kernel<E>, dim3(static_cast<unsigned>((threads + 255) / 256)), dim3(256),
                               0, s, L, B, nh, T, Tp, HS, D, L2, vec);
    if (rc) return rc;
    if constexpr (sizeof(E) == 2 && HS == 64) {
        // Tensor-core kernels whenever the operands can be described by TMA maps (16-byte
        // aligned bases and strides); the SIMT kernels below otherwise.
        rc = launch_attention_backward_tc(L, B, nh, T, D, L2, status, s, cs);
        if (rc != GPT_ERR_BAD_ALIGN) {
            if (cs_done) *cs_done = cs != nullptr && rc == GPT_OK;
            return rc;
        }
    }
    const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(HS)));
    const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(HS)));
    const dim3 grid((T + kBwdRows - 1) / kBwdRows, B * nh), block(2 * kBwdRows);
    rc = launch_overlapped(attn_bwd_dq_kernel<E, HS>, grid, block, 0, s, L, nh, T, Tp, scale_log2, inv,
                           static_cast<const float*>(D));
    if (rc) return rc;
    return launch_overlapped(attn_bwd_dkdv_kernel<E, HS>, grid, block, 0, s, L, nh, T, Tp, scale_log2, inv,
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

namespace {
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
dim3 grid8(long long n) { return dim3(static_cast<unsigned>((n + 8LL * 256 - 1) / (8LL * 256))); }
}  // namespace

int launch_gelu_forward(const void* pre, void* h, long long n, int dtype, int tanh_form, cudaStream_t s) {
    if (n == 0) return GPT_OK;
    const dim3 grid = grid8(n), block(256);
    const int vec = al16(pre) && al16(h);
    if (dtype == GPT_DTYPE_BF16)
        return launch_overlapped(gelu_forward_kernel<bf16>, grid, block, 0, s, static_cast<const bf16*>(pre),
                                 static_cast<bf16*>(h), n, tanh_form, vec);
    return launch_overlapped(gelu_forward_kernel<float>, grid, block, 0, s, static_cast<const float*>(pre),
                             static_cast<float*>(h), n, tanh_form, vec);
}

int launch_gelu_deriv_inplace(void* pre, long long n, int dtype, int tanh_form, cudaStream_t s) {
    if (n == 0) return GPT_OK;
    const dim3 grid = grid8(n), block(256);
    const int vec = al16(pre);
    if (dtype == GPT_DTYPE_BF16)
        return launch_overlapped(gelu_deriv_inplace_kernel<bf16>, grid, block, 0, s, static_cast<bf16*>(pre), n,
                                 tanh_form, vec);
    return launch_overlapped(gelu_deriv_inplace_kernel<float>, grid, block, 0, s, static_cast<float*>(pre), n,
                             tanh_form, vec);
}

int launch_attention_backward(const AttnBwdLayout<bf16>* Lb, const AttnBwdLayout<float>* Lf, int B, int nh, int T,
                              int hs, float* scratch, int32_t* status, cudaStream_t s, const AttnBwdColsum* cs,
                              bool* cs_done) {
    if (cs_done) *cs_done = false;
    if (B == 0 || nh == 0 || T == 0) return GPT_OK;
    float* D = scratch;
    float* L2 = scratch + static_cast<long long>(B) * nh * ((T + 127) / 128 * 128);
    if (Lb) {
        if (hs == 64) return attn_bwd_typed<bf16, 64>(*Lb, B, nh, T, D, L2, status, s, cs, cs_done);
        if (hs == 32) return attn_bwd_typed<bf16, 32>(*Lb, B, nh, T, D, L2, status, s, cs, cs_done);
        return GPT_ERR_UNSUPPORTED;
    }
    if (hs == 64) return attn_bwd_typed<float, 64>(*Lf, B, nh, T, D, L2, status, s, cs, cs_done);
    if (hs == 32) return attn_bwd_typed<float, 32>(*Lf, B, nh, T, D, L2, status, s, cs, cs_done);
    return GPT_ERR_UNSUPPORTED;
}

}  // namespace gpt
