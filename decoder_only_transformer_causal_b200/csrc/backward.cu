// Backward kernels of the pieces of the forward that are not matrix products ("nanoGPT 全局流程图",
// 3.4 反向传播: loss.backward() applies the chain rule from the loss back to every parameter):
// the cross-entropy's gradient with respect to the logits, LayerNorm's backward, GELU's
// derivative, column sums for bias (and LayerNorm weight) gradients, and the embedding's
// backward.  Every reduction runs in a fixed order, so results are deterministic.
//
// All are HBM-bound row or column sweeps: the logits gradient reads the logits twice (an online
// max/sum pass, then the write pass) and writes one gradient per logit; LayerNorm's backward
// reads dy and x once and writes dx; the column sums read their input once.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gpt {

namespace {

constexpr int kBwdWarps = 8;

// Every load is an L2 load (ld.global.cg): these kernels run under programmatic dependent launch
// and read data written several kernels earlier (the logits, the saved activations), which only
// the immediately preceding kernel's writes are guaranteed visible past griddepcontrol.wait.
GPT_DEVINL float ld1(const bf16* p) {
    return __bfloat162float(__ushort_as_bfloat16(__ldcg(reinterpret_cast<const unsigned short*>(p))));
}
GPT_DEVINL float ld1(const float* p) { return __ldcg(p); }
template <typename E> GPT_DEVINL E st1(float v);
template <> GPT_DEVINL bf16 st1<bf16>(float v) { return __float2bfloat16_rn(v); }
template <> GPT_DEVINL float st1<float>(float v) { return v; }

// 16-byte L2 loads / stores of 8 bf16 or 4 fp32 values.
GPT_DEVINL void ld_vec(const bf16* p, float (&f)[8]) {
    const uint4 w = __ldcg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) f[2 * i] = __low2float(h[i]), f[2 * i + 1] = __high2float(h[i]);
}
GPT_DEVINL void ld_vec(const float* p, float (&f)[4]) {
    const float4 w = __ldcg(reinterpret_cast<const float4*>(p));
    f[0] = w.x, f[1] = w.y, f[2] = w.z, f[3] = w.w;
}
GPT_DEVINL void st_vec(bf16* p, const float (&f)[8]) {
    uint4 w;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = w;
}
GPT_DEVINL void st_vec(float* p, const float (&f)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
}

GPT_DEVINL float wsum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// dlogits[r, v] = scale (exp(z_rv - lse_r) - [v == t_r]) / n for rows whose target is not -1,
// and 0 for the rest; n = the number of counted rows, read from sum_count[1] (the forward's {sum
// of row losses, counted rows}, or its sum over data-parallel ranks).  One warp per row: an online (max, sum) pass over the row, then the
// write pass.
template <typename E>
__global__ void __launch_bounds__(kBwdWarps * 32)
    ce_backward_kernel(const E* __restrict__ z, const int64_t* __restrict__ targets, const double* __restrict__ sum_count,
                       E* __restrict__ dz, int rows, int V, float scale, int32_t* status,
                       const float* __restrict__ row_lse) {
    griddep_launch_dependents();
    griddep_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * kBwdWarps + warp;
    if (r >= rows) return;
    const E* zr = z + static_cast<long long>(r) * V;
    E* dr = dz + static_cast<long long>(r) * V;
    const long long t = __ldcg(targets + r);
    const double n = __ldcg(sum_count + 1);
    if (t == -1 || n <= 0.0) {
        for (int v = lane; v < V; v += 32) dr[v] = st1<E>(0.f);
        return;
    }
    if (t < 0 || t >= V) {
        if (lane == 0) set_status(status, GPT_ERR_INDEX);
        for (int v = lane; v < V; v += 32) dr[v] = st1<E>(0.f);
        return;
    }
    constexpr int VW = 16 / sizeof(E);  // elements per 16-byte access
    const bool vec = (V % VW) == 0;     // rows are then 16-byte aligned
    float lse;
    if (row_lse) {
        lse = __ldcg(row_lse + r);  // the forward's logsumexp of the row: one pass below
    } else {
        float m = -INFINITY, s = 0.f;
        if (vec) {
            for (int v = lane * VW; v < V; v += 32 * VW) {
                float f[VW];
                ld_vec(zr + v, f);
                float mx = f[0];
#pragma unroll
                for (int e = 1; e < VW; ++e) mx = fmaxf(mx, f[e]);
                const float mn = fmaxf(m, mx);
                float add = 0.f;
#pragma unroll
                for (int e = 0; e < VW; ++e) add += __expf(f[e] - mn);
                s = (m == -INFINITY ? 0.f : s * __expf(m - mn)) + add;
                m = mn;
            }
        } else {
            for (int v = lane; v < V; v += 32) {
                const float x = ld1(zr + v);
                if (x > m) {
                    s = s * __expf(m - x) + 1.f;
                    m = x;
                } else {
                    s += __expf(x - m);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
            const float mm = fmaxf(m, m2);
            s = (m == -INFINITY ? 0.f : s * __expf(m - mm)) + (m2 == -INFINITY ? 0.f : s2 * __expf(m2 - mm));
            m = mm;
        }
        lse = m + __logf(s);
    }
    const float inv_n = static_cast<float>(static_cast<double>(scale) / n);
    if (vec) {
        for (int v = lane * VW; v < V; v += 32 * VW) {
            float f[VW];
            ld_vec(zr + v, f);
#pragma unroll
            for (int e = 0; e < VW; ++e) f[e] = (__expf(f[e] - lse) - (v + e == t ? 1.f : 0.f)) * inv_n;
            st_vec(dr + v, f);
        }
    } else {
        for (int v = lane; v < V; v += 32) {
            const float p = __expf(ld1(zr + v) - lse);
            dr[v] = st1<E>((p - (v == t ? 1.f : 0.f)) * inv_n);
        }
    }
}

// LayerNorm backward, one warp per row: y = xhat w + b, xhat = (x - mean) * rstd;
// dx (+)= rstd (dxhat - mean(dxhat) - xhat mean(dxhat xhat)), dxhat = dy w.  Each CTA also
// leaves its rows' sums of dy * xhat and dy per column in part[blockIdx.x] (the weight and bias
// gradients after the column reduction) and, with nsum 3, the column sums of dx as written: the
// residual stream's gradient, which is also the bias gradient of the projection whose output
// was added to the stream here (attn c_proj before ln_2, the previous Block's mlp c_proj before
// ln_1 or ln_f).
template <typename Tw>
__global__ void __launch_bounds__(kBwdWarps * 32)
    layernorm_backward_kernel(const float* __restrict__ dy, const float* __restrict__ x, const Tw* __restrict__ w,
                              float* __restrict__ dx, int accumulate, float* __restrict__ part, int rows, int C,
                              bf16* __restrict__ dx16, int nsum) {
    griddep_launch_dependents();
    griddep_wait();
    extern __shared__ float sm[];  // [kBwdWarps][nsum][C] per-warp column sums
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* my = sm + static_cast<size_t>(warp) * nsum * C;
    for (int c = lane; c < nsum * C; c += 32) my[c] = 0.f;
    __syncwarp();
    const int r = blockIdx.x * kBwdWarps + warp;
    if (r < rows) {
        const float* xr = x + static_cast<long long>(r) * C;
        const float* dyr = dy + static_cast<long long>(r) * C;
        float s = 0.f;
        for (int c = lane; c < C; c += 32) s += __ldcg(xr + c);
        const float mean = wsum(s) / C;
        float ss = 0.f;
        for (int c = lane; c < C; c += 32) {
            const float d = __ldcg(xr + c) - mean;
            ss += d * d;
        }
        const float rstd = rsqrtf(wsum(ss) / C + 1e-5f);
        float a = 0.f, bsum = 0.f;  // sum of dxhat, sum of dxhat * xhat
        for (int c = lane; c < C; c += 32) {
            const float xh = (__ldcg(xr + c) - mean) * rstd;
            const float g = __ldcg(dyr + c);
            const float dxh = g * ld1(w + c);
            a += dxh;
            bsum += dxh * xh;
            my[c] += g * xh;
            my[C + c] += g;
        }
        const float ma = wsum(a) / C, mb = wsum(bsum) / C;
        float* dxr = dx + static_cast<long long>(r) * C;
        for (int c = lane; c < C; c += 32) {
            const float xh = (__ldcg(xr + c) - mean) * rstd;
            const float v = rstd * (__ldcg(dyr + c) * ld1(w + c) - ma - xh * mb);
            const float o = accumulate ? __ldcg(dxr + c) + v : v;
            dxr[c] = o;
            if (dx16) dx16[static_cast<long long>(r) * C + c] = __float2bfloat16_rn(o);
            if (nsum == 3) my[2 * C + c] += o;
        }
    }
    __syncthreads();
    // this CTA's column sums, warps added in order
    for (int c = threadIdx.x; c < nsum * C; c += kBwdWarps * 32) {
        float v = 0.f;
        for (int wp = 0; wp < kBwdWarps; ++wp) v += sm[static_cast<size_t>(wp) * nsum * C + c];
        part[static_cast<long long>(blockIdx.x) * nsum * C + c] = v;
    }
}

// The same with each row held in registers (VEC float4 of x and of dy per lane, C <= 128 VEC):
// x and dy are read once; each warp takes ln_rows_per_warp(rows) consecutive rows.  Up to C = 768 (VEC 6)
// the next row's x, dy (and the dx it adds to) are loaded while the current one is reduced and
// the lanes' dw / db column sums stay in registers; wider rows (whose registers would spill) load
// row by row and add into per-warp sums in shared memory.  The warps' sums meet in warp order, so
// a CTA leaves one partial per kBwdWarps * ln_rows_per_warp(rows) rows.
constexpr int kLnRowsPerWarp = 4;  // rows per warp in the register kernel, at least

// Rows per warp of the register kernel: enough that the grid is one wave of CTAs (one per SM), so
// no SM idles in a partial last wave and every warp's one-row lookahead runs over many rows.
int ln_rows_per_warp(int rows) {
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int per = (rows + sms * kBwdWarps - 1) / (sms * kBwdWarps);
    return per > kLnRowsPerWarp ? per : kLnRowsPerWarp;
}

template <int VEC>
struct LnRow {
    float4 x[VEC], g[VEC], old[VEC];
};

template <int VEC>
GPT_DEVINL void ln_row_load(LnRow<VEC>& R, const float* x, const float* dy, const float* dx, int accumulate, int lane,
                            int C) {
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
        const int c = (lane + 32 * j) * 4;
        if (c < C) {
            R.x[j] = __ldcg(reinterpret_cast<const float4*>(x + c));
            R.g[j] = __ldcg(reinterpret_cast<const float4*>(dy + c));
            R.old[j] = accumulate ? __ldcg(reinterpret_cast<const float4*>(dx + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

template <typename Tw, int VEC>
__global__ void __launch_bounds__(kBwdWarps * 32)
    layernorm_backward_reg_kernel(const float* __restrict__ dy, const float* __restrict__ x, const Tw* __restrict__ w,
                                  float* __restrict__ dx, int accumulate, float* __restrict__ part, int rows, int C,
                                  bf16* __restrict__ dx16, int rows_per_warp, int nsum) {
    griddep_launch_dependents();
    griddep_wait();
    extern __shared__ float sm[];  // [kBwdWarps][nsum][C] per-warp column sums
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float4 wv[VEC], dwa[VEC], dba[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
        const int c = (lane + 32 * j) * 4;
        wv[j] = c < C ? make_float4(ld1(w + c), ld1(w + c + 1), ld1(w + c + 2), ld1(w + c + 3))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
        dwa[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        dba[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    constexpr bool kPipe = VEC <= 6;
    float* my = sm + static_cast<size_t>(warp) * nsum * C;
    // dw / db sums: registers (kPipe) or shared memory; the dx sums (nsum 3) always shared memory
    for (int c = kPipe ? 2 * C + lane : lane; c < nsum * C; c += 32) my[c] = 0.f;
    __syncwarp();
    const int r0 = (blockIdx.x * kBwdWarps + warp) * rows_per_warp;
    const int r1 = min(rows, r0 + rows_per_warp);
    LnRow<VEC> cur, nxt;
    if (kPipe && r0 < r1) {
        const long long o = static_cast<long long>(r0) * C;
        ln_row_load(cur, x + o, dy + o, dx + o, accumulate, lane, C);
    }
    for (int r = r0; r < r1; ++r) {
        if constexpr (kPipe) {
            if (r + 1 < r1) {
                const long long o = static_cast<long long>(r + 1) * C;
                ln_row_load(nxt, x + o, dy + o, dx + o, accumulate, lane, C);
            }
        } else {
            const long long o = static_cast<long long>(r) * C;
            ln_row_load(cur, x + o, dy + o, dx + o, accumulate, lane, C);
        }
        float4* xv = cur.x;
        const float4* gv = cur.g;
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < VEC; ++j)
            if ((lane + 32 * j) * 4 < C) s += (xv[j].x + xv[j].y) + (xv[j].z + xv[j].w);
        const float mean = wsum(s) / C;
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            if ((lane + 32 * j) * 4 < C) {
                xv[j].x -= mean, xv[j].y -= mean, xv[j].z -= mean, xv[j].w -= mean;
                ss += (xv[j].x * xv[j].x + xv[j].y * xv[j].y) + (xv[j].z * xv[j].z + xv[j].w * xv[j].w);
            }
        }
        const float rstd = rsqrtf(wsum(ss) / C + 1e-5f);
        float a = 0.f, bsum = 0.f;  // sums of dxhat and dxhat * xhat
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            if ((lane + 32 * j) * 4 < C) {
                xv[j].x *= rstd, xv[j].y *= rstd, xv[j].z *= rstd, xv[j].w *= rstd;  // xhat
                a += (gv[j].x * wv[j].x + gv[j].y * wv[j].y) + (gv[j].z * wv[j].z + gv[j].w * wv[j].w);
                bsum += (gv[j].x * wv[j].x * xv[j].x + gv[j].y * wv[j].y * xv[j].y) +
                        (gv[j].z * wv[j].z * xv[j].z + gv[j].w * wv[j].w * xv[j].w);
                if constexpr (kPipe) {
                    dwa[j].x += gv[j].x * xv[j].x, dwa[j].y += gv[j].y * xv[j].y;
                    dwa[j].z += gv[j].z * xv[j].z, dwa[j].w += gv[j].w * xv[j].w;
                    dba[j].x += gv[j].x, dba[j].y += gv[j].y, dba[j].z += gv[j].z, dba[j].w += gv[j].w;
                } else {
                    const int c = (lane + 32 * j) * 4;
                    my[c] += gv[j].x * xv[j].x, my[c + 1] += gv[j].y * xv[j].y;
                    my[c + 2] += gv[j].z * xv[j].z, my[c + 3] += gv[j].w * xv[j].w;
                    my[C + c] += gv[j].x, my[C + c + 1] += gv[j].y, my[C + c + 2] += gv[j].z, my[C + c + 3] += gv[j].w;
                }
            }
        }
        const float ma = wsum(a) / C, mb = wsum(bsum) / C;
        float* dxr = dx + static_cast<long long>(r) * C;
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            const int c = (lane + 32 * j) * 4;
            if (c < C) {
                const float4 o = make_float4(cur.old[j].x + rstd * (gv[j].x * wv[j].x - ma - xv[j].x * mb),
                                             cur.old[j].y + rstd * (gv[j].y * wv[j].y - ma - xv[j].y * mb),
                                             cur.old[j].z + rstd * (gv[j].z * wv[j].z - ma - xv[j].z * mb),
                                             cur.old[j].w + rstd * (gv[j].w * wv[j].w - ma - xv[j].w * mb));
                *reinterpret_cast<float4*>(dxr + c) = o;
                if (dx16)
                    *reinterpret_cast<uint2*>(dx16 + static_cast<long long>(r) * C + c) =
                        make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w));
                if (nsum == 3) {
                    float4* ds = reinterpret_cast<float4*>(my + 2 * C + c);
                    const float4 t = *ds;
                    *ds = make_float4(t.x + o.x, t.y + o.y, t.z + o.z, t.w + o.w);
                }
            }
        }
        if constexpr (kPipe) cur = nxt;
    }
    if constexpr (kPipe) {
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            const int c = (lane + 32 * j) * 4;
            if (c < C) {
                *reinterpret_cast<float4*>(my + c) = dwa[j];
                *reinterpret_cast<float4*>(my + C + c) = dba[j];
            }
        }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < nsum * C; c += kBwdWarps * 32) {
        float v = 0.f;
        for (int wp = 0; wp < kBwdWarps; ++wp) v += sm[static_cast<size_t>(wp) * nsum * C + c];
        part[static_cast<long long>(blockIdx.x) * nsum * C + c] = v;
    }
}

// The second stage of a column reduction with up to three destinations: column c of the
// [n_part, n_out * C] partials goes to out_{c / C}[c % C] (+)= the sum over parts in order; a
// null out is skipped.  Block (32, 32): slice y adds parts y, y + 32, ... (eight loads in flight),
// then the 32 slice sums are added in order.
__global__ void __launch_bounds__(1024)
    colsum_parts3_kernel(const float* __restrict__ part, int n_part, int C, int n_out, float* out0, float* out1,
                         float* out2, int accumulate) {
    griddep_launch_dependents();
    griddep_wait();
    __shared__ float red[32][33];
    const int c = blockIdx.x * 32 + threadIdx.x;
    const long long ld = static_cast<long long>(n_out) * C;
    float v = 0.f;
    if (c < ld) {
#pragma unroll 8
        for (int i = threadIdx.y; i < n_part; i += 32) v += __ldcg(part + i * ld + c);
    }
    red[threadIdx.y][threadIdx.x] = v;
    __syncthreads();
    if (threadIdx.y == 0 && c < ld) {
        float t = red[0][threadIdx.x];
#pragma unroll
        for (int k = 1; k < 32; ++k) t += red[k][threadIdx.x];
        const int which = c / C, cc = c - which * C;
        float* out = which == 0 ? out0 : which == 1 ? out1 : out2;
        if (out) out[cc] = accumulate ? __ldcg(out + cc) + t : t;
    }
}

// out[c] (+)= sum over i < n_part of part[i * ld + c], in order of i (the second stage of a
// column reduction).
__global__ void __launch_bounds__(256)
    colsum_parts_kernel(const float* __restrict__ part, long long ld, int n_part, int C, float* __restrict__ out,
                        int accumulate) {
    griddep_launch_dependents();
    griddep_wait();
    // block (32, 8): column blockIdx.x * 32 + x; slice y sums parts y, y + 8, ... in order, then the
    // eight slice sums are added in order (a fixed summation order for any launch).
    __shared__ float red[8][33];
    const int c = blockIdx.x * 32 + threadIdx.x;
    float v = 0.f;
    if (c < C) {
#pragma unroll 4
        for (int i = threadIdx.y; i < n_part; i += 8) v += __ldcg(part + i * ld + c);
    }
    red[threadIdx.y][threadIdx.x] = v;
    __syncthreads();
    if (threadIdx.y == 0 && c < C) {
        float t = red[0][threadIdx.x];
#pragma unroll
        for (int k = 1; k < 8; ++k) t += red[k][threadIdx.x];
        out[c] = accumulate ? __ldcg(out + c) + t : t;
    }
}

// part[blockIdx.y][c] = sum of y[r, c] over this CTA's row block; first stage of the bias gradient
// (column sums of the output gradient).  Thread t takes columns [4t, 4t + 4) with one 16-byte
// (fp32) or 8-byte (bf16) load per row when `vec`, eight rows at a time into eight running sums
// (loads in flight), which are added in a fixed order at the end.
constexpr int kColRows = 64;
GPT_DEVINL float4 ld4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }
GPT_DEVINL float4 ld4(const bf16* p) {
    const uint2 w = __ldcg(reinterpret_cast<const uint2*>(p));
    return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u), __uint_as_float(w.y << 16),
                       __uint_as_float(w.y & 0xffff0000u));
}
template <typename E>
__global__ void colsum_rows_kernel(const E* __restrict__ y, int rows, int C, float* __restrict__ part, int vec) {
    griddep_launch_dependents();
    griddep_wait();
    const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (c0 >= C) return;
    const int r0 = blockIdx.y * kColRows, r1 = min(rows, r0 + kColRows);
    float* out = part + static_cast<long long>(blockIdx.y) * C;
    if (vec && c0 + 4 <= C) {
        float4 acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        int r = r0;
        for (; r + 8 <= r1; r += 8) {
            float4 v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = ld4(y + static_cast<long long>(r + k) * C + c0);
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k].x += v[k].x, acc[k].y += v[k].y, acc[k].z += v[k].z, acc[k].w += v[k].w;
        }
        for (; r < r1; ++r) {
            const float4 v = ld4(y + static_cast<long long>(r) * C + c0);
            acc[0].x += v.x, acc[0].y += v.y, acc[0].z += v.z, acc[0].w += v.w;
        }
#pragma unroll
        for (int k = 1; k < 8; ++k)
            acc[0].x += acc[k].x, acc[0].y += acc[k].y, acc[0].z += acc[k].z, acc[0].w += acc[k].w;
        *reinterpret_cast<float4*>(out + c0) = acc[0];
        return;
    }
    for (int c = c0; c < C && c < c0 + 4; ++c) {
        float v = 0.f;
        for (int r = r0; r < r1; ++r) v += ld1(y + static_cast<long long>(r) * C + c);
        out[c] = v;
    }
}

// dpre = dh * gelu'(pre): erf form Phi(z) + z phi(z); tanh form 0.5 (1 + tanh a) +
// 0.5 z (1 - tanh^2 a) sqrt(2/pi) (1 + 3 * 0.044715 z^2), a = sqrt(2/pi) (z + 0.044715 z^3).
template <typename E>
__global__ void gelu_backward_kernel(const float* __restrict__ dh, const E* __restrict__ pre, E* __restrict__ dpre,
                                     long long n, int tanh_form, int vec) {
    griddep_launch_dependents();
    griddep_wait();
    // thread t: values [8t, 8t + 8), 16-byte accesses when `vec` and the group is whole
    const long long i0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
    if (i0 >= n) return;
    if (vec && i0 + 8 <= n) {
        float z[8], g[8];
        ld8(pre + i0, z);
        ld8(dh + i0, g);
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] *= gelu_slope(z[e], tanh_form);
        st8(dpre + i0, g);
        return;
    }
    for (long long i = i0; i < n && i < i0 + 8; ++i) dpre[i] = st1<E>(__ldcg(dh + i) * gelu_slope(ld1(pre + i), tanh_form));
}

// ------------------------------------------------------------------ embedding backward
// dwte[v] += sum of dx[r] over rows r with idx[r] = v, in row order; dwpe[t] += sum over the
// batch of dx[b, t].  The rows are ordered by (token, row) in one CTA's shared memory (N <=
// kEmbSortMax rows), then each run of equal tokens is summed by one warp in row order.  The order
// comes from a stable radix sort of 32-bit keys token << 14 | row on the token bits, 8 at a time
// from the least significant (rows start in order and every pass keeps equal digits in order),
// when the tokens fit 18 bits; else from a bitonic sort of 64-bit keys.
constexpr int kEmbSortMax = 16384;
constexpr int kEmbSortThreads = 1024;
constexpr int kEmbRowBits = 14;  // rows < kEmbSortMax
constexpr int kEmbRadixMaxV = (1 << (32 - kEmbRowBits)) - 1;  // tokens 0..V (V: a bad index) in 18 bits

__global__ void __launch_bounds__(kEmbSortThreads)
    embed_radix_sort_kernel(const int64_t* __restrict__ idx, int N, int V, unsigned long long* __restrict__ sorted,
                            int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();
    extern __shared__ uint32_t sbuf[];  // two buffers of N keys
    __shared__ uint32_t whist[32][257];  // per warp: digit counts, then running offsets
    __shared__ uint32_t s_dbase[256];
    uint32_t* ka = sbuf;
    uint32_t* kb = sbuf + N;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < N; i += kEmbSortThreads) {
        long long t = __ldcg(idx + i);
        if (t < 0 || t >= V) {
            set_status(status, GPT_ERR_INDEX);
            t = V;  // sorts after every valid token; skipped by the run kernel
        }
        ka[i] = (static_cast<uint32_t>(t) << kEmbRowBits) | static_cast<uint32_t>(i);
    }
    const int nb = 32 - __clz(V);  // bits of the largest key token, V
    const int E = (N + 31) / 32;   // each warp's contiguous chunk
    const int w0 = min(N, warp * E), w1 = min(N, w0 + E);
    for (int shift = kEmbRowBits; shift < kEmbRowBits + nb; shift += 8) {
        for (int d = lane; d < 256; d += 32) whist[warp][d] = 0;
        __syncthreads();  // the keys (first pass: their construction) and the zeroed counts
        for (int i = w0 + lane; i < w1; i += 32) atomicAdd(&whist[warp][(ka[i] >> shift) & 255u], 1u);
        __syncthreads();
        // digit d's slots: after every smaller digit, then warp by warp
        uint32_t tot = 0;
        if (threadIdx.x < 256) {
            const int d = threadIdx.x;
            for (int w = 0; w < 32; ++w) {
                const uint32_t c = whist[w][d];
                whist[w][d] = tot;
                tot += c;
            }
            s_dbase[d] = tot;
        }
        __syncthreads();
        if (warp == 0) {  // exclusive scan of the 256 digit totals, eight digits a lane
            uint32_t v[8], sum = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                v[k] = s_dbase[8 * lane + k];
                sum += v[k];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            uint32_t run = incl - sum;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                s_dbase[8 * lane + k] = run;
                run += v[k];
            }
        }
        __syncthreads();
        // stable scatter: each warp walks its chunk in order, lanes with equal digits in lane order
        for (int base = w0; base < w1; base += 32) {
            const int i = base + lane;
            const bool ok = i < w1;
            const uint32_t k = ok ? ka[i] : 0u;
            const uint32_t d = ok ? (k >> shift) & 255u : 256u + static_cast<uint32_t>(lane);
            const uint32_t peers = __match_any_sync(0xffffffffu, d);
            const uint32_t rank = __popc(peers & ((1u << lane) - 1u));
            if (ok) kb[s_dbase[d] + whist[warp][d] + rank] = k;
            __syncwarp();
            if (ok && rank == 0) whist[warp][d] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
        uint32_t* t = ka;
        ka = kb;
        kb = t;
    }
    for (int i = threadIdx.x; i < N; i += kEmbSortThreads) {
        const uint32_t k = ka[i];
        sorted[i] = (static_cast<unsigned long long>(k >> kEmbRowBits) << 32) | (k & ((1u << kEmbRowBits) - 1u));
    }
}

__global__ void __launch_bounds__(kEmbSortThreads)
    embed_sort_kernel(const int64_t* __restrict__ idx, int N, int V, unsigned long long* __restrict__ sorted,
                      int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();
    extern __shared__ unsigned long long keys[];  // next power of two >= N
    int n2 = 1;
    while (n2 < N) n2 <<= 1;
    for (int i = threadIdx.x; i < n2; i += kEmbSortThreads) {
        unsigned long long k = ~0ull;
        if (i < N) {
            long long t = __ldcg(idx + i);
            if (t < 0 || t >= V) {
                set_status(status, GPT_ERR_INDEX);
                t = V;  // sorts after every valid token; skipped below
            }
            k = (static_cast<unsigned long long>(t) << 32) | static_cast<unsigned>(i);
        }
        keys[i] = k;
    }
    __syncthreads();
    for (int size = 2; size <= n2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < n2; i += kEmbSortThreads) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool up = (i & size) == 0;
                    const unsigned long long a = keys[i], b = keys[j];
                    if ((a > b) == up) {
                        keys[i] = b;
                        keys[j] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = threadIdx.x; i < N; i += kEmbSortThreads) sorted[i] = keys[i];
}

// One warp per sorted position that starts a run of equal tokens: adds the run's dx rows (in
// row order) into dwte[token].
__global__ void embed_runs_kernel(const unsigned long long* __restrict__ sorted, int N, int V,
                                  const float* __restrict__ dx, int C, float* __restrict__ dwte) {
    griddep_launch_dependents();
    griddep_wait();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= N) return;
    const unsigned long long k = __ldcg(sorted + warp);
    const unsigned tok = static_cast<unsigned>(k >> 32);
    if (tok >= static_cast<unsigned>(V)) return;
    if (warp > 0 && static_cast<unsigned>(__ldcg(sorted + warp - 1) >> 32) == tok) return;  // not a run start
    int end = warp + 1;
    while (end < N && static_cast<unsigned>(__ldcg(sorted + end) >> 32) == tok) ++end;
    float* out = dwte + static_cast<long long>(tok) * C;
    // lane l owns columns c0 + l + 32 j, j < 8: a row's eight loads are issued together
    for (int c0 = 0; c0 < C; c0 += 256) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = 0.f;
        for (int s = warp; s < end; ++s) {
            const unsigned r = static_cast<unsigned>(__ldcg(sorted + s) & 0xffffffffull);
            const float* xr = dx + static_cast<long long>(r) * C + c0 + lane;
            float t[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) t[j] = c0 + lane + 32 * j < C ? __ldcg(xr + 32 * j) : 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] += t[j];
        }
        float o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = c0 + lane + 32 * j < C ? __ldcg(out + c0 + lane + 32 * j) : 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (c0 + lane + 32 * j < C) out[c0 + lane + 32 * j] = o[j] + v[j];
    }
}

__global__ void embed_wpe_kernel(const float* __restrict__ dx, int B, int T, int C, float* __restrict__ dwpe) {
    griddep_launch_dependents();
    griddep_wait();
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<long long>(T) * C) return;
    float v = 0.f;
    for (int b = 0; b < B; ++b) v += __ldcg(dx + static_cast<long long>(b) * T * C + i);
    dwpe[i] = __ldcg(dwpe + i) + v;
}

}  // namespace

int launch_ce_backward(const void* logits, int dtype, const int64_t* targets, const double* sum_count, void* dlogits,
                       int rows, int V, int32_t* status, cudaStream_t s, float scale, const float* row_lse) {
    const dim3 grid((rows + kBwdWarps - 1) / kBwdWarps), block(kBwdWarps * 32);
    if (dtype == GPT_DTYPE_BF16)
        return launch_overlapped(ce_backward_kernel<bf16>, grid, block, 0, s, static_cast<const bf16*>(logits),
                                 targets, sum_count, static_cast<bf16*>(dlogits), rows, V, scale, status, row_lse);
    return launch_overlapped(ce_backward_kernel<float>, grid, block, 0, s, static_cast<const float*>(logits), targets,
                             sum_count, static_cast<float*>(dlogits), rows, V, scale, status, row_lse);
}

int layernorm_backward_parts(int rows, int C) {  // partials of 2C (3C with dsum) floats each
    const int per = (C <= 2048 && C % 4 == 0) ? kBwdWarps * ln_rows_per_warp(rows) : kBwdWarps;
    return (rows + per - 1) / per;
}

namespace {
template <typename Tw, int VEC = 1>
int launch_ln_bwd_reg(const float* dy, const float* x, const void* w, float* dx, bf16* dx16, int accumulate, float* part, int rows,
                      int C, int nsum, size_t smem, cudaStream_t s) {
    if constexpr (VEC < 16) {
        if (C > 128 * VEC)
            return launch_ln_bwd_reg<Tw, VEC + 1>(dy, x, w, dx, dx16, accumulate, part, rows, C, nsum, smem, s);
    }
    static size_t opted[kMaxDevices] = {};
    const int rc = opt_in_smem(reinterpret_cast<const void*>(layernorm_backward_reg_kernel<Tw, VEC>), smem, opted);
    if (rc) return rc;
    return launch_overlapped(layernorm_backward_reg_kernel<Tw, VEC>, dim3(layernorm_backward_parts(rows, C)),
                             dim3(kBwdWarps * 32), smem, s, dy, x, static_cast<const Tw*>(w), dx, accumulate, part,
                             rows, C, dx16, ln_rows_per_warp(rows), nsum);
}
}  // namespace

int launch_layernorm_backward(const float* dy, const float* x, const void* w, int dtype, float* dx, int accumulate,
                              float* dw, float* db, int accumulate_wb, float* part, int rows, int C, cudaStream_t s,
                              bf16* dx16, float* dsum) {
    const int n_part = layernorm_backward_parts(rows, C);
    const int nsum = dsum ? 3 : 2;
    const size_t smem = static_cast<size_t>(kBwdWarps) * nsum * C * sizeof(float);
    int rc;
    if (C <= 2048 && C % 4 == 0) {
        rc = dtype == GPT_DTYPE_BF16
                 ? launch_ln_bwd_reg<bf16>(dy, x, w, dx, dx16, accumulate, part, rows, C, nsum, smem, s)
                 : launch_ln_bwd_reg<float>(dy, x, w, dx, dx16, accumulate, part, rows, C, nsum, smem, s);
    } else if (dtype == GPT_DTYPE_BF16) {
        static size_t opted[kMaxDevices] = {};
        rc = opt_in_smem(reinterpret_cast<const void*>(layernorm_backward_kernel<bf16>), smem, opted);
        if (!rc)
            rc = launch_overlapped(layernorm_backward_kernel<bf16>, dim3(n_part), dim3(kBwdWarps * 32), smem, s, dy,
                                   x, static_cast<const bf16*>(w), dx, accumulate, part, rows, C, dx16, nsum);
    } else {
        static size_t opted[kMaxDevices] = {};
        rc = opt_in_smem(reinterpret_cast<const void*>(layernorm_backward_kernel<float>), smem, opted);
        if (!rc)
            rc = launch_overlapped(layernorm_backward_kernel<float>, dim3(n_part), dim3(kBwdWarps * 32), smem, s, dy,
                                   x, static_cast<const float*>(w), dx, accumulate, part, rows, C, dx16, nsum);
    }
    if (rc) return rc;
    // dsum always accumulates (bias gradients add into the caller's gradient buffer)
    if (dsum && !accumulate_wb) return GPT_ERR_UNSUPPORTED;
    return launch_overlapped(colsum_parts3_kernel, dim3((nsum * C + 31) / 32), dim3(32, 32), 0, s,
                             static_cast<const float*>(part), n_part, C, nsum, dw, db, dsum, accumulate_wb);
}

int launch_colsum_bands(const float* part, int n_part, int C, float* out, int accumulate, cudaStream_t s) {
    if (n_part < 1 || C < 1) return GPT_OK;
    return launch_overlapped(colsum_parts3_kernel, dim3((C + 31) / 32), dim3(32, 32), 0, s, part, n_part, C, 1, out,
                             static_cast<float*>(nullptr), static_cast<float*>(nullptr), accumulate);
}

int colsum_parts(int rows) { return (rows + kColRows - 1) / kColRows; }

int launch_colsum(const void* y, int dtype, int rows, int C, float* out, int accumulate, float* part,
                  cudaStream_t s) {
    const int n_part = colsum_parts(rows);
    const dim3 g1((C + 4 * 256 - 1) / (4 * 256), n_part), b(256);
    // 16-byte rows of 4 values: C % 4 == 0 and aligned base and partial buffer
    const int vec = (C % 4 == 0) && ((reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(part)) & 15) == 0;
    int rc = dtype == GPT_DTYPE_BF16
                 ? launch_overlapped(colsum_rows_kernel<bf16>, g1, b, 0, s, static_cast<const bf16*>(y), rows, C, part,
                                     vec)
                 : launch_overlapped(colsum_rows_kernel<float>, g1, b, 0, s, static_cast<const float*>(y), rows, C,
                                     part, vec);
    if (rc) return rc;
    return launch_overlapped(colsum_parts_kernel, dim3((C + 31) / 32), dim3(32, 8), 0, s,
                             static_cast<const float*>(part), static_cast<long long>(C), n_part, C, out, accumulate);
}

int launch_gelu_backward(const float* dh, const void* pre, int dtype, void* dpre, long long n, int tanh_form,
                         cudaStream_t s) {
    if (n == 0) return GPT_OK;
    const dim3 g(static_cast<unsigned>((n + 8LL * 256 - 1) / (8LL * 256))), b(256);
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    const int vec = al(dh) && al(pre) && al(dpre);
    if (dtype == GPT_DTYPE_BF16)
        return launch_overlapped(gelu_backward_kernel<bf16>, g, b, 0, s, dh, static_cast<const bf16*>(pre),
                                 static_cast<bf16*>(dpre), n, tanh_form, vec);
    return launch_overlapped(gelu_backward_kernel<float>, g, b, 0, s, dh, static_cast<const float*>(pre),
                             static_cast<float*>(dpre), n, tanh_form, vec);
}

int embed_backward_max_rows() { return kEmbSortMax; }

int launch_embed_backward(const int64_t* idx, const float* dx, int B, int T, int C, int V, float* dwte, float* dwpe,
                          unsigned long long* sorted, int32_t* status, cudaStream_t s) {
    const int N = B * T;
    if (N > kEmbSortMax) return GPT_ERR_UNSUPPORTED;
    int rc;
    if (V <= kEmbRadixMaxV) {
        const size_t smem = static_cast<size_t>(2) * N * sizeof(uint32_t);
        static size_t opted_r[kMaxDevices] = {};
        rc = opt_in_smem(reinterpret_cast<const void*>(embed_radix_sort_kernel), smem, opted_r);
        if (rc) return rc;
        rc = launch_overlapped(embed_radix_sort_kernel, dim3(1), dim3(kEmbSortThreads), smem, s, idx, N, V, sorted,
                               status);
    } else {
        int n2 = 1;
        while (n2 < N) n2 <<= 1;
        const size_t smem = static_cast<size_t>(n2) * sizeof(unsigned long long);
        static size_t opted[kMaxDevices] = {};
        rc = opt_in_smem(reinterpret_cast<const void*>(embed_sort_kernel), smem, opted);
        if (rc) return rc;
        rc = launch_overlapped(embed_sort_kernel, dim3(1), dim3(kEmbSortThreads), smem, s, idx, N, V, sorted, status);
    }
    if (rc) return rc;
    rc = launch_overlapped(embed_runs_kernel, dim3((N * 32 + 255) / 256), dim3(256), 0, s,
                           static_cast<const unsigned long long*>(sorted), N, V, dx, C, dwte);
    if (rc) return rc;
    const long long n = static_cast<long long>(T) * C;
    return launch_overlapped(embed_wpe_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, s, dx, B,
                             T, C, dwpe);
}

}  // namespace gpt
