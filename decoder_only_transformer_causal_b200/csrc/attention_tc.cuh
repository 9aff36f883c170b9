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
//   warps 2-5   softmax, one query row per thread: load the S row from TMEM (both halves in
//               flight together, one wait; P's two halves likewise stored with one wait), mask the
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


// The 128 S columns of this warp's TMEM lanes: two 32x32b.x64 loads in flight together, one wait
// (the empty asm statements after it tie every register's later use to the wait).
GPT_DEVINL void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]),
          "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
          "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
          "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),
          "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]),
          "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]),
          "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]),
          "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]),
          "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]),
          "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]),
          "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]),
          "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]),
          "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]),
          "=r"(r[127])
        : "r"(taddr + 64u));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 128; ++i) asm volatile("" : "+r"(r[i]));
}

// P (64 columns of bf16 pairs) into this warp's TMEM lanes: two stores, one wait.
GPT_DEVINL void tmem_st64_pair(uint32_t taddr, const uint32_t (&a)[32], const uint32_t (&b)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        :: "r"(taddr), "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]),
           "r"(a[8]), "r"(a[9]), "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]), "r"(a[15]),
           "r"(a[16]), "r"(a[17]), "r"(a[18]), "r"(a[19]), "r"(a[20]), "r"(a[21]), "r"(a[22]), "r"(a[23]),
           "r"(a[24]), "r"(a[25]), "r"(a[26]), "r"(a[27]), "r"(a[28]), "r"(a[29]), "r"(a[30]), "r"(a[31])
        : "memory");
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        :: "r"(taddr + 32u), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(b[4]), "r"(b[5]), "r"(b[6]),
           "r"(b[7]), "r"(b[8]), "r"(b[9]), "r"(b[10]), "r"(b[11]), "r"(b[12]), "r"(b[13]), "r"(b[14]),
           "r"(b[15]), "r"(b[16]), "r"(b[17]), "r"(b[18]), "r"(b[19]), "r"(b[20]), "r"(b[21]), "r"(b[22]),
           "r"(b[23]), "r"(b[24]), "r"(b[25]), "r"(b[26]), "r"(b[27]), "r"(b[28]), "r"(b[29]), "r"(b[30]),
           "r"(b[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

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
            {
                uint32_t u[BKV];
                tmem_ld128(tS, u);
#pragma unroll
                for (int e = 0; e < BKV; ++e) s[e] = __uint_as_float(u[e]);
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
            tmem_st64_pair(tP, pk0, pk1);
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
