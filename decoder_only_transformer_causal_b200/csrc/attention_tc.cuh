// Causal flash-style self-attention for sm_100a, head size 64, bf16 in / bf16 out.
//
// Computes, for every (batch b, head h, query row i) ("nanoGPT 全局流程图", §2.5 (B) 步骤3-6):
//   y_i = sum_{j <= i} p_ij v_j,  p_ij = exp(s_ij - max_j s) / sum_j exp(s_ij - max_j s),
//   s_ij = q_i . k_j / sqrt(64)
// without materialising the T x T matrix: keys are visited in 128-wide tiles with an online
// (running-maximum) softmax, and tiles entirely above the diagonal are never touched.
//
// One CTA owns one 128-row query tile of one (b, h) and runs four roles:
//   warp 0      TMA: Q once, then K_j / V_j tiles (128 x 64, 128-byte swizzle) into a
//               two-deep ring;
//   warp 1      one thread issues tcgen05.mma: S = Q K_j^T (M=128, N=128, K=64) into TMEM, and
//               O += P V_j (M=128, N=64, K=128) with P read from TMEM and V as an MN-major
//               shared-memory operand;
//   warps 2-5   softmax, one query row per thread: load the S row from TMEM, mask the
//               diagonal tile, update the running maximum / sum, write P (bf16) to TMEM,
//               rescale O in TMEM when the maximum moved by more than 2^8, and finally
//               write y = O / l.  3-input maxima cut the issue count; the exponents' arguments
//               and the row sums are packed f32x2 FMAs and adds (one instruction per two
//               scores); on the diagonal tile the 32-column chunks right of a warp's last row are
//               fully masked and skip the exponential, one branch per chunk.  The exponential
//               (MUFU ex2, 16 per clock per SM) bounds this kernel at head size 64.
// TMEM columns: S [0,128), P [128,192) (bf16 pairs), O [192,256).  256 columns and 80 KB of
// shared memory let two CTAs share an SM, so one CTA's softmax overlaps the other's MMAs.
//
// q, k and v are addressed through 4-D TMA maps {hs, head, t, b} with arbitrary strides, which
// covers both the standalone [B, nh, T, hs] layout and the fused c_attn output
// [B, T, 3, nh, hs] (heads of q, k, v read in place: no transpose copy).
#pragma once

#include "common.cuh"

namespace gpt {
namespace attn {

constexpr int HS = 64;
constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int THREADS = 192;
constexpr int TILE_BYTES = BQ * HS * 2;  // 16 KB for Q, K or V
constexpr int SMEM_BYTES = 5 * TILE_BYTES + 256 + 1024;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_S = 0, COL_P = 128, COL_O = 192;
// The running maximum is only moved (forcing an O rescale) when it grows by more than this
// many powers of two; P values then stay below 2^8, harmless in fp32 and bf16.
constexpr float kRescaleThreshold = 8.0f;


GPT_DEVINL float max3(float a, float b, float c) { float d; asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c)); return d; }

struct Params {
    int B, nh, T;
    int head_inner;          // 1: TMA coordinates {0, h, t, b}; 0: {0, t, h, b}
    bf16* y;                 // output base
    long long y_sb, y_sh, y_st;  // element strides of y for b, h, t (hs is contiguous)
    float scale_log2;        // log2(e) / sqrt(hs)
    int32_t* status;
    float* lse;              // optional [B, nh, T]: m + log2(l) per row (log2 units of the scaled score)
};

__global__ void __launch_bounds__(THREADS, 2)
    attention_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = smem + TILE_BYTES;       // 2 stages
    uint8_t* sV = smem + 3 * TILE_BYTES;   // 2 stages
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 5 * TILE_BYTES);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;   // [2]
    uint64_t* k_empty = bars + 3;  // [2]
    uint64_t* v_full = bars + 5;   // [2]
    uint64_t* v_empty = bars + 7;  // [2]
    uint64_t* s_full = bars + 9;   // S_j in TMEM
    uint64_t* s_free = bars + 10;  // softmax has read S_j
    uint64_t* p_full = bars + 11;  // P_j (and rescaled O) written
    uint64_t* o_done = bars + 12;  // O += P_j V_j finished
    uint64_t* drain = bars + 13;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Longest query tiles first: blocks are dispatched roughly in index order.
    const int BH = p.B * p.nh;
    const int n_qt = (p.T + BQ - 1) / BQ;
    const int qt = n_qt - 1 - static_cast<int>(blockIdx.x) / BH;
    const int bh = static_cast<int>(blockIdx.x) % BH;
    const int b = bh / p.nh;
    const int h = bh % p.nh;
    const int q0 = qt * BQ;
    const int n_kv = qt + 1;  // key tiles 0..qt; the last one is the diagonal tile

    if (threadIdx.x == 0) {
        for (int i = 0; i < 14; ++i) mbar_init(&bars[i], (i == 10 || i == 11) ? 128u : 1u);
        *abort_flag = 0;
        fence_barrier_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The set-up above overlapped the previous kernel; its outputs are read from here on.
    griddep_launch_dependents();
    griddep_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            // Coordinates of row t of head h in the 4-D maps.
            const int c1h = p.head_inner ? h : 0, c2h = p.head_inner ? 0 : h;
            auto c1 = [&](int t) { return p.head_inner ? c1h : t; };
            auto c2 = [&](int t) { return p.head_inner ? t : c2h; };
            mbar_arrive_expect_tx(q_full, TILE_BYTES);
            tma_load_4d(sQ, &tmQ, q_full, 0, c1(q0), c2(q0), b);
            int issued_k = 0, issued_v = 0;
            for (int j = 0; j < n_kv; ++j) {
                const int st = j & 1;
                const uint32_t ph = (j >> 1) & 1;
                if (!mbar_wait(&k_empty[st], ph ^ 1u, abort_flag)) break;
                mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
                tma_load_4d(sK + st * TILE_BYTES, &tmK, &k_full[st], 0, c1(j * BKV), c2(j * BKV), b);
                ++issued_k;
                if (!mbar_wait(&v_empty[st], ph ^ 1u, abort_flag)) break;
                mbar_arrive_expect_tx(&v_full[st], TILE_BYTES);
                tma_load_4d(sV + st * TILE_BYTES, &tmV, &v_full[st], 0, c1(j * BKV), c2(j * BKV), b);
                ++issued_v;
            }
            // No bulk copy may still target shared memory when the CTA exits.
            mbar_drain(q_full, 0);
            for (int i = 1; i <= 2; ++i) {
                if (issued_k - i >= 0) mbar_drain(&k_full[(issued_k - i) & 1], ((issued_k - i) >> 1) & 1);
                if (issued_v - i >= 0) mbar_drain(&v_full[(issued_v - i) & 1], ((issued_v - i) >> 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = make_idesc_bf16(BQ, BKV, false);
            constexpr uint32_t idesc_o = make_idesc_bf16(BQ, HS, true);
            const uint32_t tS = tmem + COL_S, tP = tmem + COL_P, tO = tmem + COL_O;
            // Testing aid: nothing arrives on `drain` before the commit below, so this wait can only
            // give up, which sends the whole CTA down its time-out path.
            if (g_force_timeout) mbar_wait(drain, 0, abort_flag);
            bool ok = !g_force_timeout && mbar_wait(q_full, 0, abort_flag);
            tc_fence_after();
            const uint32_t q_addr = smem_addr(sQ);
            for (int j = 0; ok && j <= n_kv; ++j) {
                if (j < n_kv) {
                    // S_j = Q K_j^T once the softmax has taken S_{j-1} out of TMEM.
                    const int st = j & 1;
                    const uint32_t ph = (j >> 1) & 1;
                    if (!mbar_wait(&k_full[st], ph, abort_flag)) break;
                    if (j > 0 && !mbar_wait(s_free, (j - 1) & 1, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t k_addr = smem_addr(sK + st * TILE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < HS / 16; ++kk)
                        umma_ss(tS, make_sdesc_sw128(q_addr + kk * 32), make_sdesc_sw128(k_addr + kk * 32),
                                idesc_s, kk > 0 ? 1u : 0u);
                    umma_commit(&k_empty[st]);
                    umma_commit(s_full);
                }
                if (j > 0) {
                    // O += P_{j-1} V_{j-1} once the softmax has written P_{j-1}.
                    const int jj = j - 1;
                    const int st = jj & 1;
                    const uint32_t ph = (jj >> 1) & 1;
                    if (!mbar_wait(p_full, jj & 1, abort_flag)) break;
                    if (!mbar_wait(&v_full[st], ph, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t v_addr = smem_addr(sV + st * TILE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BKV / 16; ++kk)
                        umma_ts(tO, tP + kk * 8, make_sdesc_sw128(v_addr + kk * 2048), idesc_o,
                                (jj > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&v_empty[st]);
                    umma_commit(o_done);
                }
            }
            umma_commit(drain);
            mbar_drain(drain, 0);
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // row within the query tile
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + COL_S + lane_off;
        const uint32_t tP = tmem + COL_P + lane_off;
        const uint32_t tO = tmem + COL_O + lane_off;
        float m_used = -INFINITY;  // running maximum (log2 units) the P values are taken against
        float l = 0.f;             // running sum of P
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            const bool got = mbar_wait(s_full, j & 1, abort_flag);
            __syncwarp();  // tcgen05.ld / st below are warp-collective
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // S row -> registers (raw scores; the 1/sqrt(hs) * log2(e) scale is folded into the
            // exponent below).  Independent partial maxima / sums keep the dependency chains short.
            float s[BKV];
#pragma unroll
            for (int c = 0; c < BKV; c += 64) {
                uint32_t u[64];
                tmem_ld64(tS + c, u);
#pragma unroll
                for (int e = 0; e < 64; ++e) s[c + e] = __uint_as_float(u[e]);
            }
            tc_fence_before();
            mbar_arrive(s_free);
            if (j == n_kv - 1) {
                // Diagonal tile: key column c is visible to row r iff c <= r.
#pragma unroll
                for (int c = 0; c < BKV; ++c)
                    if (c > r) s[c] = -INFINITY;
            }
            float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
            for (int cc = 4; cc < BKV; cc += 8) {
                m4[0] = max3(m4[0], s[cc], s[cc + 1]);
                m4[1] = max3(m4[1], s[cc + 2], s[cc + 3]);
                if (cc + 4 < BKV) {
                    m4[2] = max3(m4[2], s[cc + 4], s[cc + 5]);
                    m4[3] = max3(m4[3], s[cc + 6], s[cc + 7]);
                }
            }
            const float mx = max3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * p.scale_log2;
            float alpha = 1.f;
            if (mx > m_used + kRescaleThreshold || m_used == -INFINITY) {
                alpha = exp2_approx(m_used - mx);
                m_used = mx;
            }
            const bool diag = (j == n_kv - 1);
            const float SCs = p.scale_log2, NMs = -m_used;
            uint64_t acc4[4] = {0, 0, 0, 0};
            uint32_t pk0[32], pk1[32];
            // Off the diagonal every column is live (a loop with no per-column test).  On the
            // diagonal tile, 32-column chunks to the right of this warp's last row are masked for
            // every lane: P is 0 there and no exponential is evaluated.
            const int live_cols = diag ? (quarter + 1) * 32 : BKV;  // warp-uniform
            if (!diag) {
                const uint64_t SC2 = f2_pack(SCs, SCs), NM2 = f2_pack(NMs, NMs);
#pragma unroll
                for (int c = 0; c < BKV; c += 2) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), SC2, NM2), x0, x1);
                    const float p0 = exp2_approx(x0), p1 = exp2_approx(x1);
                    acc4[(c >> 1) & 3] = f2_add(acc4[(c >> 1) & 3], f2_pack(p0, p1));
                    if (c < 64) pk0[c / 2] = pack_bf16x2(p0, p1);
                    else pk1[(c - 64) / 2] = pack_bf16x2(p0, p1);
                }
            } else {
                const uint64_t SC = f2_pack(p.scale_log2, p.scale_log2), NM = f2_pack(-m_used, -m_used);
#pragma unroll
                for (int ch = 0; ch < BKV / 32; ++ch) {
                    if (ch * 32 < live_cols) {  // warp-uniform: one branch per 32-column chunk
#pragma unroll
                        for (int c = ch * 32; c < ch * 32 + 32; c += 2) {
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), SC, NM), x0, x1);
                            const float p0 = exp2_approx(x0), p1 = exp2_approx(x1);
                            acc4[(c >> 1) & 3] = f2_add(acc4[(c >> 1) & 3], f2_pack(p0, p1));
                            if (c < 64) pk0[c / 2] = pack_bf16x2(p0, p1);
                            else pk1[(c - 64) / 2] = pack_bf16x2(p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int c = ch * 32; c < ch * 32 + 32; c += 2) {
                            if (c < 64) pk0[c / 2] = 0u;
                            else pk1[(c - 64) / 2] = 0u;
                        }
                    }
                }
            }
            float a0, a1, b0, b1, c0, c1, d0, d1;
            f2_unpack(acc4[0], a0, a1); f2_unpack(acc4[1], b0, b1); f2_unpack(acc4[2], c0, c1); f2_unpack(acc4[3], d0, d1);
            const float rs = ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
            l = l * alpha + rs;
            // P_j may overwrite P_{j-1} and O may be rescaled only after O += P_{j-1} V_{j-1}.
            if (j > 0) {
                const bool done = mbar_wait(o_done, (j - 1) & 1, abort_flag);
                __syncwarp();
                if (!__all_sync(0xffffffffu, done)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            tmem_st32(tP, pk0);
            tmem_st32(tP + 32, pk1);
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                for (int c = 0; c < HS; c += 32) {
                    uint32_t u[32];
                    tmem_ld32(tO + c, u);
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
                    tmem_st32(tO + c, u);
                }
            }
            tc_fence_before();
            mbar_arrive(p_full);
        }
        bool last = ok && mbar_wait(o_done, (n_kv - 1) & 1, abort_flag);
        __syncwarp();
        if (__all_sync(0xffffffffu, last)) {
            tc_fence_after();
            const int t = q0 + r;
            const float inv_l = 1.f / l;
            if (p.lse && t < p.T) p.lse[(static_cast<long long>(b) * p.nh + h) * p.T + t] = m_used + __log2f(l);
            uint32_t out[32];
#pragma unroll
            for (int c = 0; c < HS; c += 32) {
                uint32_t u[32];
                tmem_ld32(tO + c, u);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    out[c / 2 + e] = pack_bf16x2(__uint_as_float(u[2 * e]) * inv_l,
                                                 __uint_as_float(u[2 * e + 1]) * inv_l);
            }
            if (t < p.T) {
                uint4* dst = reinterpret_cast<uint4*>(p.y + b * p.y_sb + h * p.y_sh + static_cast<long long>(t) * p.y_st);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    dst[q] = make_uint4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if (threadIdx.x == 0 && *abort_flag) set_status(p.status, GPT_ERR_TIMEOUT);
}

}  // namespace attn
}  // namespace gpt
