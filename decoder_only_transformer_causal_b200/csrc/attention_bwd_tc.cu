// Tensor-core backward of the causal attention for sm_100a, head size 64, bf16 ("nanoGPT 全局流程图",
// 3.4 反向传播 through §2.5 (B)'s softmax(Q K^T / sqrt(d)) V).
//
// With s_ij = q_i . k_j, p_ij = 2^(s_ij * scale_log2 - lse2_i) (lse2: the forward's per-row
// log2-sum-exp, so P is recomputed, never stored) and D_i = dO_i . O_i:
//   dP_ij = dO_i . v_j,   dS_ij = p_ij (dP_ij - D_i)   (p_ij = dS_ij = 0 for j > i)
//   dV_j = sum_i p_ij dO_i,   dK_j = sum_i dS_ij q_i / sqrt(hs),   dQ_i = sum_j dS_ij k_j / sqrt(hs)
// Two kernels, each owning 128 "outer" rows of one (b, h) and sweeping 64-row "inner" tiles, so
// every result is summed inside one CTA in a fixed order (no atomics: bit-reproducible):
//   dK/dV kernel  outer = 128 keys, inner = the query tiles from the diagonal to T.
//                 S^T = K Q_n^T and dP^T = V dO_n^T (M=128, N=64, K=64) into TMEM; the four
//                 row warps turn key row j into P^T and dS^T (bf16) in shared memory, written in
//                 the K-major 128-byte-swizzled layout a TMA load would produce; then
//                 dV += P^T dO_n and dK += dS^T Q_n (M=128, N=64, K=64), dO_n and Q_n read as
//                 MN-major operands.
//   dQ kernel     outer = 128 queries, inner = the key tiles up to the diagonal.  S = Q K_n^T and
//                 dP = dO V_n^T into TMEM; dS (bf16) goes back to TMEM and dQ += dS K_n takes it
//                 as the A operand, K_n as an MN-major operand.
// -lse2 and D come from [B*nh, Tp] arrays (Tp = T rounded up to 128) whose padding holds
// -lse2 = -inf and D = 0, so queries past T get p = 0 with no test; the dK/dV kernel copies the
// 64 entries of each query tile next to its Q / dO tiles with one bulk copy each.  The row warps
// form P and dS with packed f32x2 arithmetic.  The inner tiles stream through a ring: two stages in
// the dK/dV kernel (its P^T and dS^T operands take the rest of the shared memory two CTAs per SM
// allow), four in the dQ kernel (three tiles in flight ahead of the one being used).
// Roles (192 threads, two CTAs per SM): warp 0 TMA producer, warp 1 MMA issuer (one thread),
// warps 2-5 one outer row per thread.  TMEM (256 columns): dK/dV kernel S^T [0,64), dP^T
// [64,128), dV [128,192), dK [192,256); dQ kernel S [0,64), dP [64,128), dQ [128,192),
// dS [192,224).  Every wait is bounded; a timeout records GPT_ERR_TIMEOUT and the CTA drains its
// copies and MMAs, frees TMEM and returns.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gpt {
namespace attn_bwd {

constexpr int HS = 64;
constexpr int BM = 128;  // outer rows per CTA
constexpr int BN = 64;   // inner tile rows
constexpr int THREADS = 192;
constexpr int OUTER_BYTES = BM * HS * 2;  // 16 KB
constexpr int INNER_BYTES = BN * HS * 2;  // 8 KB
constexpr int ROWS_BYTES = BM * BN * 2;   // 16 KB: a bf16 [128 x 64] operand written by the row warps
constexpr int VEC_BYTES = BN * 4;         // 64 fp32
constexpr uint32_t TMEM_COLS = 256;
constexpr int kNumBars = 11;
constexpr int QNST = 4;  // dQ kernel: stages of the key / value tiles (prefetch three tiles ahead)
constexpr int kQBars = 7 + 2 * QNST;

// dK/dV kernel: K, V | Q[2], dO[2] | P^T, dS^T | lse2[2], D[2] | barriers
constexpr int KV_OFF_Q = 2 * OUTER_BYTES;
constexpr int KV_OFF_G = KV_OFF_Q + 2 * INNER_BYTES;
constexpr int KV_OFF_P = KV_OFF_G + 2 * INNER_BYTES;
constexpr int KV_OFF_DS = KV_OFF_P + ROWS_BYTES;
constexpr int KV_OFF_VEC = KV_OFF_DS + ROWS_BYTES;
constexpr int KV_OFF_BAR = KV_OFF_VEC + 4 * VEC_BYTES;
constexpr int KV_SMEM = KV_OFF_BAR + 256 + 1024;
// dQ kernel: Q, dO | K[QNST], V[QNST] | barriers
constexpr int Q_OFF_K = 2 * OUTER_BYTES;
constexpr int Q_OFF_V = Q_OFF_K + QNST * INNER_BYTES;
constexpr int Q_OFF_BAR = Q_OFF_V + QNST * INNER_BYTES;
constexpr int Q_SMEM = Q_OFF_BAR + 256 + 1024;

struct Params {
    int B, nh, T, Tp;
    int qk_head_inner, o_head_inner;  // TMA coordinate order of the q/k/v maps and of the dO map
    bf16 *dq, *dk, *dv;
    long long sb, sh, st;             // element strides of dq / dk / dv (hs contiguous)
    const float* lse2;                // [B*nh, Tp]: -lse2 per query, padding -inf
    const float* D;                   // [B*nh, Tp], padding 0
    float scale_log2, inv_sqrt_hs;
    int32_t* status;
    // Optional: column sums of dq / dk / dv per 32-row band of each sequence (the first stage of the
    // bias gradient of the layer that produced q, k, v): row b * bands + t / 32 of colsum
    // [B * bands, cs_ld]; head h's columns of q, k, v start at cs_q, cs_k, cs_v + h * HS.
    float* colsum;
    long long cs_ld;
    int cs_q, cs_k, cs_v, bands;
};

// Rows [t, t + box) of head h, batch b in a 4-D map {hs, head, t, b} or {hs, t, head, b}.
GPT_DEVINL void load_rows(void* dst, const CUtensorMap* m, uint64_t* bar, int head_inner, int h, int t, int b) {
    tma_load_4d(dst, m, bar, 0, head_inner ? h : t, head_inner ? t : h, b);
}

// Row r of a bf16 [128 x 64] tile in the K-major 128-byte-swizzled layout (rows of 128 bytes,
// 16-byte chunk c of row r stored at chunk c ^ (r mod 8)); w holds the row's 64 values as pairs.
GPT_DEVINL void store_swizzled_row(uint8_t* tile, int r, const uint32_t (&w)[32]) {
    uint8_t* row = tile + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) =
            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}

GPT_DEVINL void store_row_bf16(bf16* dst, const uint32_t (&w)[32]) {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 8; ++q) d[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

// 64 accumulator columns of this thread's TMEM lane -> 32 bf16 pairs, times `scale`.
GPT_DEVINL void tmem_row_bf16(uint32_t taddr, float scale, uint32_t (&w)[32]) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        uint32_t u[32];
        tmem_ld32(taddr + half * 32, u);
#pragma unroll
        for (int e = 0; e < 16; ++e)
            w[half * 16 + e] = pack_bf16x2(__uint_as_float(u[2 * e]) * scale, __uint_as_float(u[2 * e + 1]) * scale);
    }
}

// As tmem_row_bf16, and with cs (warp-uniform) the column sums of the warp's 32 rows of the scaled
// fp32 values (rows with !valid add zero) into cs[0, 64): lane l writes columns l and 32 + l.
GPT_DEVINL void tmem_row_bf16_colsum(uint32_t taddr, float scale, uint32_t (&w)[32], bool valid, float* cs) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        uint32_t u[32];
        tmem_ld32(taddr + half * 32, u);
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(u[e]) * scale;
#pragma unroll
        for (int e = 0; e < 16; ++e) w[half * 16 + e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
        if (cs) {
            if (!valid) {
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = 0.f;
            }
            cs[half * 32 + lane] = warp_colsum32(v);
        }
    }
}

// The band row of this warp's 32 rows [t0, t0 + 32) of sequence b in p.colsum, or null (no sums
// asked for, or a band entirely past T).
GPT_DEVINL float* colsum_band(const Params& p, int b, int t0) {
    if (!p.colsum || t0 >= p.T) return nullptr;
    return p.colsum + (static_cast<long long>(b) * p.bands + t0 / 32) * p.cs_ld;
}

// One 32-column half of a key row of the dK/dV kernel: P^T and dS^T for queries c0 + e, with packed
// f32x2 arithmetic (one exponent FMA, one subtraction and one product per pair).  nl: the negated
// lse2 per query; MASK: the tile touches the diagonal and columns c < cmin (queries before the key)
// are zero.
template <bool MASK>
GPT_DEVINL void kv_half(const uint32_t (&su)[32], const uint32_t (&du)[32], const float* nl, const float* dv,
                        float sc, int c0, int cmin, uint32_t* pw, uint32_t* dw) {
    const uint64_t* nl2 = reinterpret_cast<const uint64_t*>(nl + c0);
    const uint64_t* d2 = reinterpret_cast<const uint64_t*>(dv + c0);
    const uint64_t SC = f2_pack(sc, sc);
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
        float p0, p1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(su[k]), __uint_as_float(su[k + 1])), SC, nl2[k / 2]), p0, p1);
        p0 = exp2_approx(p0);
        p1 = exp2_approx(p1);
        if (MASK && c0 + k < cmin) p0 = 0.f;
        if (MASK && c0 + k + 1 < cmin) p1 = 0.f;
        const uint64_t pp = f2_pack(p0, p1);
        float s0, s1;
        f2_unpack(f2_mul(pp, f2_sub(f2_pack(__uint_as_float(du[k]), __uint_as_float(du[k + 1])), d2[k / 2])), s0, s1);
        pw[k / 2] = pack_bf16x2(p0, p1);
        dw[k / 2] = pack_bf16x2(s0, s1);
    }
}

// One 32-column half of a query row of the dQ kernel: dS for keys c0 + e (packed f32x2).  nlse: the
// row's negated lse2; MASK: columns c > cmax (keys after the query) are zero.
template <bool MASK>
GPT_DEVINL void q_half(const uint32_t (&su)[32], const uint32_t (&du)[32], float sc, float nlse, float Di, int c0,
                       int cmax, uint32_t* dw) {
    const uint64_t SC = f2_pack(sc, sc), NL = f2_pack(nlse, nlse), DD = f2_pack(Di, Di);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float p0, p1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(su[e]), __uint_as_float(su[e + 1])), SC, NL), p0, p1);
        p0 = exp2_approx(p0);
        p1 = exp2_approx(p1);
        if (MASK && c0 + e > cmax) p0 = 0.f;
        if (MASK && c0 + e + 1 > cmax) p1 = 0.f;
        float s0, s1;
        f2_unpack(f2_mul(f2_pack(p0, p1), f2_sub(f2_pack(__uint_as_float(du[e]), __uint_as_float(du[e + 1])), DD)),
                  s0, s1);
        dw[e / 2] = pack_bf16x2(s0, s1);
    }
}

// ------------------------------------------------------------------ dK / dV
__global__ void __launch_bounds__(THREADS, 2)
    attn_bwd_dkdv_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
                     const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sK = smem;
    uint8_t* sV = smem + OUTER_BYTES;
    uint8_t* sQ = smem + KV_OFF_Q;  // 2 stages
    uint8_t* sG = smem + KV_OFF_G;  // 2 stages
    uint8_t* sP = smem + KV_OFF_P;
    uint8_t* sDS = smem + KV_OFF_DS;
    float* vlse = reinterpret_cast<float*>(smem + KV_OFF_VEC);  // [2][64]
    float* vD = vlse + 2 * BN;                                  // [2][64]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + KV_OFF_BAR);
    uint64_t* a_full = bars + 0;
    uint64_t* b_full = bars + 1;   // [2]
    uint64_t* b_empty = bars + 3;  // [2]
    uint64_t* s_full = bars + 5;   // S^T, dP^T in TMEM
    uint64_t* s_free = bars + 6;   // row warps have read them (128 arrivals)
    uint64_t* p_full = bars + 7;   // P^T, dS^T in shared memory (128 arrivals)
    uint64_t* ps_free = bars + 8;  // dV / dK MMAs have read P^T, dS^T
    uint64_t* acc_done = bars + 9;
    uint64_t* drain = bars + 10;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int BH = p.B * p.nh;
    const int kt = static_cast<int>(blockIdx.x) / BH;  // key tile 0 (the most query tiles) first
    const int bh = static_cast<int>(blockIdx.x) % BH;
    const int b = bh / p.nh, h = bh % p.nh;
    const int k0 = kt * BM;
    const int nq = (p.T - k0 + BN - 1) / BN;  // query tiles k0 + n * 64, n < nq

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], (i == 6 || i == 7) ? 128u : 1u);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmG);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_launch_dependents();
    griddep_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const float* lrow = p.lse2 + static_cast<long long>(bh) * p.Tp;
            const float* drow = p.D + static_cast<long long>(bh) * p.Tp;
            mbar_arrive_expect_tx(a_full, 2 * OUTER_BYTES);
            load_rows(sK, &tmK, a_full, p.qk_head_inner, h, k0, b);
            load_rows(sV, &tmV, a_full, p.qk_head_inner, h, k0, b);
            int issued = 0;
            for (int n = 0; n < nq; ++n) {
                const int st = n & 1;
                if (!mbar_wait(&b_empty[st], ((n >> 1) & 1) ^ 1u, abort_flag)) break;
                const int i0 = k0 + n * BN;
                mbar_arrive_expect_tx(&b_full[st], 2 * INNER_BYTES + 2 * VEC_BYTES);
                load_rows(sQ + st * INNER_BYTES, &tmQ, &b_full[st], p.qk_head_inner, h, i0, b);
                load_rows(sG + st * INNER_BYTES, &tmG, &b_full[st], p.o_head_inner, h, i0, b);
                bulk_load_1d(vlse + st * BN, lrow + i0, VEC_BYTES, &b_full[st]);
                bulk_load_1d(vD + st * BN, drow + i0, VEC_BYTES, &b_full[st]);
                ++issued;
            }
            // No copy may still target shared memory when the CTA exits.
            mbar_drain(a_full, 0);
            for (int i = 1; i <= 2; ++i)
                if (issued - i >= 0) mbar_drain(&b_full[(issued - i) & 1], ((issued - i) >> 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = make_idesc_bf16(BM, BN, false);
            constexpr uint32_t idesc_acc = make_idesc_bf16(BM, HS, true);
            const uint32_t tS = tmem, tdP = tmem + 64, tdV = tmem + 128, tdK = tmem + 192;
            const uint32_t k_addr = smem_addr(sK), v_addr = smem_addr(sV);
            const uint32_t p_addr = smem_addr(sP), ds_addr = smem_addr(sDS);
            bool ok = mbar_wait(a_full, 0, abort_flag);
            tc_fence_after();
            for (int n = 0; ok && n <= nq; ++n) {
                if (n < nq) {
                    // S^T_n = K Q_n^T and dP^T_n = V dO_n^T once the row warps have read tile n-1.
                    const int st = n & 1;
                    if (!mbar_wait(&b_full[st], (n >> 1) & 1, abort_flag)) break;
                    if (n > 0 && !mbar_wait(s_free, (n - 1) & 1, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t q_addr = smem_addr(sQ + st * INNER_BYTES);
                    const uint32_t g_addr = smem_addr(sG + st * INNER_BYTES);
#pragma unroll
                    for (int kk = 0; kk < HS / 16; ++kk)
                        umma_ss(tS, make_sdesc_sw128(k_addr + kk * 32), make_sdesc_sw128(q_addr + kk * 32), idesc_s,
                                kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < HS / 16; ++kk)
                        umma_ss(tdP, make_sdesc_sw128(v_addr + kk * 32), make_sdesc_sw128(g_addr + kk * 32), idesc_s,
                                kk > 0 ? 1u : 0u);
                    umma_commit(s_full);
                }
                if (n > 0) {
                    // dV += P^T_m dO_m, dK += dS^T_m Q_m for the previous tile m.
                    const int m = n - 1, st = m & 1;
                    if (!mbar_wait(p_full, m & 1, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t q_addr = smem_addr(sQ + st * INNER_BYTES);
                    const uint32_t g_addr = smem_addr(sG + st * INNER_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        umma_ss(tdV, make_sdesc_sw128(p_addr + kk * 32), make_sdesc_sw128(g_addr + kk * 2048),
                                idesc_acc, (m > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        umma_ss(tdK, make_sdesc_sw128(ds_addr + kk * 32), make_sdesc_sw128(q_addr + kk * 2048),
                                idesc_acc, (m > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&b_empty[st]);
                    umma_commit(ps_free);
                }
            }
            umma_commit(acc_done);
            umma_commit(drain);
            mbar_drain(drain, 0);
        }
    } else {
        // ------------------------------------------------------------ row warps: key row r
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off, tdP = tmem + 64 + lane_off;
        const float sc = p.scale_log2;
        bool ok = true;
        for (int n = 0; n < nq; ++n) {
            const int st = n & 1;
            const bool got = mbar_wait(&b_full[st], (n >> 1) & 1, abort_flag) && mbar_wait(s_full, n & 1, abort_flag);
            __syncwarp();  // tcgen05.ld below is warp-collective
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float* lv = vlse + st * BN;  // negated lse2 of the tile's queries
            const float* dv = vD + st * BN;
            const int cmin = r - n * BN;  // key k0 + r sees query k0 + n*64 + c iff c >= cmin
            uint32_t pw[32], dw[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t su[32], du[32];
                tmem_ld32(tS + half * 32, su);
                tmem_ld32(tdP + half * 32, du);
                if (half == 1) {
                    tc_fence_before();
                    mbar_arrive(s_free);
                }
                if (n < 2)  // warp-uniform: only the two tiles at the diagonal hold masked entries
                    kv_half<true>(su, du, lv, dv, sc, half * 32, cmin, pw + half * 16, dw + half * 16);
                else
                    kv_half<false>(su, du, lv, dv, sc, half * 32, cmin, pw + half * 16, dw + half * 16);
            }
            if (n > 0) {
                const bool fr = mbar_wait(ps_free, (n - 1) & 1, abort_flag);
                __syncwarp();
                if (!__all_sync(0xffffffffu, fr)) {
                    ok = false;
                    break;
                }
            }
            store_swizzled_row(sP, r, pw);
            store_swizzled_row(sDS, r, dw);
            fence_proxy_async_shared();  // generic-proxy writes -> visible to the tensor core
            mbar_arrive(p_full);
        }
        bool last = ok && mbar_wait(acc_done, 0, abort_flag);
        last = last && !*abort_flag;
        __syncwarp();
        if (__all_sync(0xffffffffu, last)) {
            tc_fence_after();
            uint32_t w[32];
            const int j = k0 + r;
            const long long off = b * p.sb + h * p.sh + static_cast<long long>(j) * p.st;
            float* cs = colsum_band(p, b, k0 + quarter * 32);
            tmem_row_bf16_colsum(tmem + 128 + lane_off, 1.f, w, j < p.T, cs ? cs + p.cs_v + h * HS : nullptr);
            if (j < p.T) store_row_bf16(p.dv + off, w);
            tmem_row_bf16_colsum(tmem + 192 + lane_off, p.inv_sqrt_hs, w, j < p.T, cs ? cs + p.cs_k + h * HS : nullptr);
            if (j < p.T) store_row_bf16(p.dk + off, w);
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

// ------------------------------------------------------------------ dQ
__global__ void __launch_bounds__(THREADS, 2)
    attn_bwd_dq_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem;
    uint8_t* sG = smem + OUTER_BYTES;
    uint8_t* sK = smem + Q_OFF_K;  // 2 stages
    uint8_t* sV = smem + Q_OFF_V;  // 2 stages
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Q_OFF_BAR);
    uint64_t* a_full = bars + 0;
    uint64_t* b_full = bars + 1;
    uint64_t* b_empty = bars + 1 + QNST;
    uint64_t* s_full = bars + 1 + 2 * QNST;
    uint64_t* s_free = s_full + 1;
    uint64_t* p_full = s_full + 2;
    uint64_t* ds_free = s_full + 3;
    uint64_t* acc_done = s_full + 4;
    uint64_t* drain = s_full + 5;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kQBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int BH = p.B * p.nh;
    const int n_qt = (p.T + BM - 1) / BM;
    const int qt = n_qt - 1 - static_cast<int>(blockIdx.x) / BH;  // longest query tiles first
    const int bh = static_cast<int>(blockIdx.x) % BH;
    const int b = bh / p.nh, h = bh % p.nh;
    const int q0 = qt * BM;
    const int nk = (min(q0 + BM, p.T) + BN - 1) / BN;  // key tiles n * 64, n < nk

    if (threadIdx.x == 0) {
        for (int i = 0; i < kQBars; ++i) mbar_init(&bars[i], (i == 2 + 2 * QNST || i == 3 + 2 * QNST) ? 128u : 1u);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmG);
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
    griddep_launch_dependents();
    griddep_wait();

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(a_full, 2 * OUTER_BYTES);
            load_rows(sQ, &tmQ, a_full, p.qk_head_inner, h, q0, b);
            load_rows(sG, &tmG, a_full, p.o_head_inner, h, q0, b);
            int issued = 0;
            for (int n = 0; n < nk; ++n) {
                const int st = n % QNST;
                if (!mbar_wait(&b_empty[st], ((n / QNST) & 1) ^ 1u, abort_flag)) break;
                mbar_arrive_expect_tx(&b_full[st], 2 * INNER_BYTES);
                load_rows(sK + st * INNER_BYTES, &tmK, &b_full[st], p.qk_head_inner, h, n * BN, b);
                load_rows(sV + st * INNER_BYTES, &tmV, &b_full[st], p.qk_head_inner, h, n * BN, b);
                ++issued;
            }
            mbar_drain(a_full, 0);
            for (int i = 1; i <= QNST; ++i)
                if (issued - i >= 0) mbar_drain(&b_full[(issued - i) % QNST], ((issued - i) / QNST) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = make_idesc_bf16(BM, BN, false);
            constexpr uint32_t idesc_acc = make_idesc_bf16(BM, HS, true);
            const uint32_t tS = tmem, tdP = tmem + 64, tdQ = tmem + 128, tdS = tmem + 192;
            const uint32_t q_addr = smem_addr(sQ), g_addr = smem_addr(sG);
            bool ok = mbar_wait(a_full, 0, abort_flag);
            tc_fence_after();
            for (int n = 0; ok && n <= nk; ++n) {
                if (n < nk) {
                    const int st = n % QNST;
                    if (!mbar_wait(&b_full[st], (n / QNST) & 1, abort_flag)) break;
                    if (n > 0 && !mbar_wait(s_free, (n - 1) & 1, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t k_addr = smem_addr(sK + st * INNER_BYTES);
                    const uint32_t v_addr = smem_addr(sV + st * INNER_BYTES);
#pragma unroll
                    for (int kk = 0; kk < HS / 16; ++kk)
                        umma_ss(tS, make_sdesc_sw128(q_addr + kk * 32), make_sdesc_sw128(k_addr + kk * 32), idesc_s,
                                kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < HS / 16; ++kk)
                        umma_ss(tdP, make_sdesc_sw128(g_addr + kk * 32), make_sdesc_sw128(v_addr + kk * 32), idesc_s,
                                kk > 0 ? 1u : 0u);
                    umma_commit(s_full);
                }
                if (n > 0) {
                    // dQ += dS_m K_m
                    const int m = n - 1, st = m % QNST;
                    if (!mbar_wait(p_full, m & 1, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t k_addr = smem_addr(sK + st * INNER_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        umma_ts(tdQ, tdS + kk * 8, make_sdesc_sw128(k_addr + kk * 2048), idesc_acc,
                                (m > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&b_empty[st]);
                    umma_commit(ds_free);
                }
            }
            umma_commit(acc_done);
            umma_commit(drain);
            mbar_drain(drain, 0);
        }
    } else {
        // ------------------------------------------------------------ row warps: query row r
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int i = q0 + r;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off, tdP = tmem + 64 + lane_off, tdS = tmem + 192 + lane_off;
        const float sc = p.scale_log2;
        const long long vi = static_cast<long long>(bh) * p.Tp + i;  // i < Tp: Tp is a multiple of 128
        const float nlse = __ldcg(p.lse2 + vi);  // stored negated
        const float Di = __ldcg(p.D + vi);
        bool ok = true;
        for (int n = 0; n < nk; ++n) {
            const bool got = mbar_wait(s_full, n & 1, abort_flag);
            __syncwarp();
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int cmax = i - n * BN;  // query i sees key n*64 + c iff c <= cmax
            const bool diag = n * BN + BN - 1 > q0;  // warp-uniform
            uint32_t dw[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t su[32], du[32];
                tmem_ld32(tS + half * 32, su);
                tmem_ld32(tdP + half * 32, du);
                if (half == 1) {
                    tc_fence_before();
                    mbar_arrive(s_free);
                }
                if (diag)
                    q_half<true>(su, du, sc, nlse, Di, half * 32, cmax, dw + half * 16);
                else
                    q_half<false>(su, du, sc, nlse, Di, half * 32, cmax, dw + half * 16);
            }
            if (n > 0) {
                const bool fr = mbar_wait(ds_free, (n - 1) & 1, abort_flag);
                __syncwarp();
                if (!__all_sync(0xffffffffu, fr)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            tmem_st32(tdS, dw);
            tc_fence_before();
            mbar_arrive(p_full);
        }
        bool last = ok && mbar_wait(acc_done, 0, abort_flag);
        last = last && !*abort_flag;
        __syncwarp();
        if (__all_sync(0xffffffffu, last)) {
            tc_fence_after();
            uint32_t w[32];
            float* cs = colsum_band(p, b, q0 + quarter * 32);
            tmem_row_bf16_colsum(tmem + 128 + lane_off, p.inv_sqrt_hs, w, i < p.T, cs ? cs + p.cs_q + h * HS : nullptr);
            if (i < p.T) store_row_bf16(p.dq + b * p.sb + h * p.sh + static_cast<long long>(i) * p.st, w);
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

// 4-D map over rows of 64 bf16 (one head's row) with a box of `rows` rows; the coordinate order
// keeps the strides non-decreasing: {hs, head, t, b} when heads are interleaved inside a position,
// {hs, t, head, b} when each head is a contiguous [T, hs] block.
int make_rows_map(CUtensorMap* m, const void* base, int B, int nh, int T, long long sb, long long sh, long long st,
                  int rows, int* head_inner) {
    const bool hi = sh <= st;
    uint64_t dims[4], strides[3];
    dims[0] = HS;
    dims[1] = hi ? nh : T;
    dims[2] = hi ? T : nh;
    dims[3] = B;
    strides[0] = static_cast<uint64_t>(hi ? sh : st) * 2;
    strides[1] = static_cast<uint64_t>(hi ? st : sh) * 2;
    strides[2] = static_cast<uint64_t>(sb) * 2;
    const uint32_t box_hi[4] = {HS, 1, static_cast<uint32_t>(rows), 1};
    const uint32_t box_ti[4] = {HS, static_cast<uint32_t>(rows), 1, 1};
    *head_inner = hi ? 1 : 0;
    return make_tmap_bf16_4d(m, base, dims, strides, hi ? box_hi : box_ti);
}

}  // namespace attn_bwd

size_t attn_bwd_scratch_bytes(long long B, long long nh, long long T) {
    const long long Tp = (T + attn_bwd::BM - 1) / attn_bwd::BM * attn_bwd::BM;
    return static_cast<size_t>(2 * B * nh * Tp) * sizeof(float);
}

int launch_attention_backward_tc(const AttnBwdLayout<bf16>& L, int B, int nh, int T, const float* D,
                                 const float* lse2, int32_t* status, cudaStream_t s, const AttnBwdColsum* cs) {
    using namespace attn_bwd;
    // Results are stored as 16-byte rows: 16-byte aligned bases and strides that are multiples of 8.
    auto aligned = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    if (!aligned(L.dq) || !aligned(L.dk) || !aligned(L.dv) || ((L.sb | L.sh | L.st) & 7)) return GPT_ERR_BAD_ALIGN;
    CUtensorMap k128, v128, q64, g64, q128, g128, k64, v64;
    int qk_hi = 0, o_hi = 0;
    int rc = make_rows_map(&k128, L.k, B, nh, T, L.sb, L.sh, L.st, BM, &qk_hi);
    if (!rc) rc = make_rows_map(&v128, L.v, B, nh, T, L.sb, L.sh, L.st, BM, &qk_hi);
    if (!rc) rc = make_rows_map(&q64, L.q, B, nh, T, L.sb, L.sh, L.st, BN, &qk_hi);
    if (!rc) rc = make_rows_map(&g64, L.dout, B, nh, T, L.o_sb, L.o_sh, L.o_st, BN, &o_hi);
    if (!rc) rc = make_rows_map(&q128, L.q, B, nh, T, L.sb, L.sh, L.st, BM, &qk_hi);
    if (!rc) rc = make_rows_map(&g128, L.dout, B, nh, T, L.o_sb, L.o_sh, L.o_st, BM, &o_hi);
    if (!rc) rc = make_rows_map(&k64, L.k, B, nh, T, L.sb, L.sh, L.st, BN, &qk_hi);
    if (!rc) rc = make_rows_map(&v64, L.v, B, nh, T, L.sb, L.sh, L.st, BN, &qk_hi);
    if (rc) return rc;
    Params p{};
    p.B = B;
    p.nh = nh;
    p.T = T;
    p.Tp = (T + BM - 1) / BM * BM;
    p.qk_head_inner = qk_hi;
    p.o_head_inner = o_hi;
    p.dq = L.dq;
    p.dk = L.dk;
    p.dv = L.dv;
    p.sb = L.sb;
    p.sh = L.sh;
    p.st = L.st;
    p.lse2 = lse2;
    p.D = D;
    p.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(HS)));
    p.inv_sqrt_hs = static_cast<float>(1.0 / sqrt(static_cast<double>(HS)));
    p.status = status;
    if (cs) {
        p.colsum = cs->part;
        p.cs_ld = cs->ld;
        p.cs_q = cs->col_q;
        p.cs_k = cs->col_k;
        p.cs_v = cs->col_v;
        p.bands = (T + 31) / 32;
    }
    static size_t opted_q[kMaxDevices] = {}, opted_kv[kMaxDevices] = {};
    rc = opt_in_smem(reinterpret_cast<const void*>(attn_bwd_dq_tc), Q_SMEM, opted_q);
    if (!rc) rc = opt_in_smem(reinterpret_cast<const void*>(attn_bwd_dkdv_tc), KV_SMEM, opted_kv);
    if (rc) return rc;
    const long long blocks = static_cast<long long>((T + BM - 1) / BM) * B * nh;
    if (blocks > 0x7fffffffLL) return GPT_ERR_UNSUPPORTED;
    rc = launch_overlapped(attn_bwd_dq_tc, dim3(static_cast<unsigned>(blocks)), dim3(THREADS), Q_SMEM, s, q128, g128,
                           k64, v64, p);
    if (rc) return rc;
    return launch_overlapped(attn_bwd_dkdv_tc, dim3(static_cast<unsigned>(blocks)), dim3(THREADS), KV_SMEM, s, k128,
                             v128, q64, g64, p);
}

// Pipeline-wait limit of this file's kernels on the current device (0: the default).
GPT_DEFINE_WAIT_LIMIT_SETTER(set_wait_limit_attention_bwd)

}  // namespace gpt
