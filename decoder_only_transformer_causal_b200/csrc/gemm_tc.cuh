// Tensor-core GEMM for sm_100a: Y[M, N] = epilogue(A[M, K] * W[N, K]^T), bf16 operands,
// fp32 accumulation in tensor memory.
//
// Used for every nn.Linear of the forward pass ("nanoGPT 全局流程图", §2.5: c_attn, attn
// c_proj, c_fc, mlp c_proj) and for the tied lm_head (§3.2 ④), each with its epilogue fused:
//   EPI_STORE  out_bf16 = acc + b                 (c_attn)
//   EPI_GELU   out_bf16 = gelu(acc + b)           (c_fc; "nanoGPT架构逐步详解", 4. MLP)
//   EPI_RESID  x_fp32  += acc + b                 (both c_proj: the residual add of Block)
//   EPI_CE     logits_bf16 = acc, plus per (row, column slice) the running maximum and the sum
//              of exp(z - max) and, in the slice holding the row's target, z[target] in fp32:
//              the pieces of F.cross_entropy's logsumexp (§3.3), reduced by ce_rows.
//
// Design: one persistent CTA per SM walks the output tiles (128 x BN).  Tiles are visited so
// that the larger operand is streamed from HBM once: n-fastest when A is the larger (the CTAs
// sharing an A row-block run together), m-fastest when W is (the head: the CTAs of a wave share
// W columns).  Warp 0 streams 128x64 A and BNx64 W tiles with TMA (128-byte swizzle) through a
// kStages-deep shared-memory ring; one thread of warp 1 issues tcgen05.mma (M=128, N=BN, K=16)
// into one of two TMEM accumulators; 8 epilogue warps drain the other accumulator while the
// next tile's MMAs run.  Each epilogue warp owns 32 rows (its TMEM lane quarter) and half of the
// tile's columns; it turns 32 columns at a time into a 32 x 64-byte tile in a private shared-
// memory buffer (64-byte swizzle: conflict-free from one-row-per-thread writes) and one lane hands
// that tile to TMA: a tile store for the bf16 outputs, a tile reduce-add for the residual stream
// (x += acc + b happens at the destination; x never travels to the SM).  TMA clips the ragged
// edges.  The tile's bias is staged in shared memory before the accumulator wait.  Every wait is
// bounded (common.cuh).
#pragma once

#include "common.cuh"

namespace gpt {
namespace gemm {

constexpr int BM = 128;
constexpr int BK = 64;  // one 128-byte swizzle row of bf16
constexpr int kStages = 4;
constexpr int NEPI = 8;  // epilogue warps: two per TMEM lane quarter, each half of BN

// EPI_F32: out_fp32 = acc, plain store (a backward product, or the partial products of a split-K
//          launch).
// EPI_DGELU: out_bf16 = acc * aux, aux the bf16 GELU derivative [M, ld_aux] that the training
//          forward stored (the MLP's backward through GELU, fused into the product that yields
//          d loss / d gelu output).  Each epilogue warp's 32 x 128 slice of aux is copied by TMA into
//          shared memory when the warp starts the tile, so it arrives while the products run.
// EPI_GELU2: gelu'(acc + b) at rows [0, M) of out and gelu(acc + b) at rows [M, 2M) (the training
//          forward keeps the GELU output for the weight gradient and its derivative for the
//          backward through GELU; M % 32 == 0).
enum Epi { EPI_STORE = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_CE = 3, EPI_F32 = 4, EPI_DGELU = 5, EPI_GELU2 = 6 };

struct Params {
    int M, N, K;
    int n_fastest;     // tile order: 1 = n fastest (A-heavy), 0 = m fastest (W-heavy)
    const bf16* bias;  // [N] or nullptr
    void* out;         // bf16 [M, ldo] (STORE / GELU / CE logits) or fp32 [M, ldo] (RESID)
    long long ldo;
    const int64_t* targets;  // EPI_CE: [M]
    float2* part;            // EPI_CE: [M, n_part] of (max, sum exp(z - max))
    float* tlogit;           // EPI_CE: [M], z[target] in fp32
    int n_part;
    int32_t* status;
    // Split-K (EPI_F32 only): the K blocks are cut into k_splits ranges of kb_per_split blocks;
    // split s stores its partial product at rows [s * M, s * M + M) of out (M % 32 == 0).
    int k_splits;
    int kb_per_split;
    const bf16* aux;  // EPI_DGELU: [M, ld_aux]
    long long ld_aux;
    // EPI_DGELU (optional): the output's column sums per 32-row band, [ceil(M / 32), ld_colsum]
    // (the first stage of the bias gradient of the layer whose input gradient this is)
    float* colsum;
    long long ld_colsum;
};

// PAIR: a cluster of two CTAs computes one 256 x BN tile with the 2-SM MMA; each CTA stages its
// own 128 rows of A and half of B's BN rows, so a stage is 32 KB and six fit.  AUX (EPI_DGELU):
// each epilogue warp also stages its 32 x 128 slice of the tile's GELU derivatives (two 64-column
// TMA boxes, 128-byte swizzle, 8 KB), which costs two stages of the ring.
template <int BN, int PAIR = 0, int AUX = 0>
struct Cfg {
    static_assert(BN == 256, "BN");
    static constexpr int STAGES = PAIR ? (AUX ? 4 : 6) : (AUX ? 2 : kStages);
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;         // rows of B this CTA stages
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = B_ROWS * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int AUX_OFF = STAGES * STAGE_BYTES;      // AUX: [NEPI][2 boxes][32 rows][64]
    static constexpr int AUX_WARP_BYTES = 32 * (BN / (NEPI / 4)) * 2;
    static constexpr int BIAS_OFF = AUX_OFF + (AUX ? NEPI * AUX_WARP_BYTES : 0);  // a bias slice per epilogue warp
    static constexpr int STG_OFF = BIAS_OFF + NEPI * (BN / (NEPI / 4)) * 4;
    static constexpr int STG_BYTES = 32 * 64;                 // 32 rows x 64 bytes per warp
    static constexpr int BAR_OFF = STG_OFF + NEPI * STG_BYTES;
    static constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;  // barriers + alignment slack
    static constexpr int TMEM_COLS = 2 * BN;                  // two accumulators
    static constexpr int THREADS = 64 + NEPI * 32;
    static constexpr int COLS_PER_WARP = BN / (NEPI / 4);     // 128
    static constexpr int PARTS_PER_TILE = NEPI / 4;
};

// GELU for the epilogue, cheap enough to hide under the next tile's MMAs.
//  erf form:  x * Phi(x) with the normal CDF Phi in a logistic form, Phi(x) ~ 1 / (1 + exp(-2 x
//             (a + b x^2 + c x^4))) (the shape of the logistic approximations of Phi in the
//             literature, e.g. Bowling, Khasawneh, Kaewkuekool and Cho, J. Industrial Engineering
//             and Management 2(1), 2009), with a, b, c fitted here by minimising the largest
//             |x Phi~(x) - x Phi(x)| over [-10, 10].  The quintic's bracket a + b x^2 + c x^4 turns
//             positive past |x| = 11.1 (c < 0), so x^2 is clamped at 110 inside it: the bracket
//             stays at its value there (-1.77 / -2 log2 e) and the exponent keeps growing with |x|.
//             Largest error over [-60, 60]: 2.6e-5 absolute (0.12% relative where |gelu| > 0.01,
//             under a third of the bf16 step of the output); of the derivative 4.4e-4.  One
//             exponential and one reciprocal per element; the polynomial on packed f32x2 pairs
//             where a loop has them.
//  tanh form: 0.5 x (1 + tanh(u)) = x / (1 + exp(-2u)), u = sqrt(2/pi) (x + 0.044715 x^3).
GPT_DEVINL float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kGeluA = 0.7975078821182251f, kGeluB = 0.03700564429163933f, kGeluC = -0.0003515167918521911f;
constexpr float kGeluNeg2Log2e = -2.0f * 1.4426950408889634f;
constexpr float kGeluX2Max = 110.0f;  // x^2 clamp inside the bracket
// the exponent e(x) = -2 log2(e) x (a + b x^2 + c x^4), and its derivative
constexpr float kGeluK1 = kGeluNeg2Log2e * kGeluA, kGeluK3 = kGeluNeg2Log2e * kGeluB, kGeluK5 = kGeluNeg2Log2e * kGeluC;

// gelu(x) and gelu'(x) together.  Erf form: g = x r, r = 1 / (1 + E), E = 2^e(x), so
// g' = r - x r^2 E ln2 e'(x) = r - r (1 - r) x ln2 e'(x), e'(x) = K1 + 3 K3 x^2 + 5 K5 x^4.
template <int TANH>
GPT_DEVINL void gelu_pair_f(float x, float& g, float& dg) {
    constexpr float kLog2e = 1.4426950408889634f;
    if (TANH) {
        const float c = 0.7978845608028654f;
        const float u = c * x * fmaf(0.044715f * x, x, 1.0f);
        const float r = rcp_approx(1.0f + exp2_approx(2.0f * u * kLog2e));  // (1 - tanh u) / 2
        const float th = 1.0f - 2.0f * r;
        g = x * (1.0f - r);
        dg = 0.5f * (1.0f + th) + 0.5f * x * (1.0f - th * th) * c * fmaf(3.0f * 0.044715f * x, x, 1.0f);
        return;
    }
    const float xx = x * x, x2 = fminf(xx, kGeluX2Max);
    const float bracket = fmaf(x2, fmaf(x2, kGeluK5, kGeluK3), kGeluK1);
    const float e = bracket * x;
    // e'(x): the quintic's inside the clamp, the constant bracket outside
    const float de = xx < kGeluX2Max ? fmaf(x2, fmaf(x2, 5.0f * kGeluK5, 3.0f * kGeluK3), kGeluK1) : bracket;
    const float r = rcp_approx(1.0f + exp2_approx(e));
    g = x * r;
    dg = fmaf(-fmaf(-r, r, r), x * de * 0.6931471805599453f, r);
}

template <int TANH>
GPT_DEVINL float gelu_f(float x) {
    constexpr float kLog2e = 1.4426950408889634f;
    if (TANH) {
        const float u2 = -2.0f * 0.7978845608028654f * x * fmaf(0.044715f * x, x, 1.0f);
        return x * rcp_approx(1.0f + exp2_approx(u2 * kLog2e));
    }
    const float x2 = fminf(x * x, kGeluX2Max);
    return x * rcp_approx(1.0f + exp2_approx(fmaf(x2, fmaf(x2, kGeluK5, kGeluK3), kGeluK1) * x));
}

// The erf form on 32 values, the polynomial on packed pairs.
GPT_DEVINL void gelu32_erf(float (&v)[32]) {
    const uint64_t K1 = f2_pack(kGeluK1, kGeluK1), K3 = f2_pack(kGeluK3, kGeluK3), K5 = f2_pack(kGeluK5, kGeluK5);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
        const uint64_t xv = f2_pack(v[j], v[j + 1]);
        const uint64_t x2 = f2_pack(fminf(v[j] * v[j], kGeluX2Max), fminf(v[j + 1] * v[j + 1], kGeluX2Max));
        float e0, e1;
        f2_unpack(f2_mul(f2_fma(x2, f2_fma(x2, K5, K3), K1), xv), e0, e1);
        v[j] *= rcp_approx(1.0f + exp2_approx(e0));
        v[j + 1] *= rcp_approx(1.0f + exp2_approx(e1));
    }
}

// A_MN / B_MN: the operand is stored MN-major, i.e. as the [K, M] (or [K, N]) row-major matrix
// whose transpose the product needs (the backward's dY^T X and dY W).  Its tile is then loaded
// as 64-column TMA boxes (64 K rows x 128 bytes each, 8 KB apart) and described to the MMA with
// the MN-major layout; no transposed copy is made.
//
// PAIR: launched in clusters of two.  Rank 0 (the leader) owns the barriers the pair shares: each
// CTA's TMA loads count on the leader's `full`, the leader's one MMA thread issues the 2-SM MMAs
// (M = 256) and its commits arrive on `empty` and `tfull` in both CTAs, and both CTAs' epilogue
// threads arrive on the leader's `tempty`.  Each CTA's epilogue drains its own 128 rows.
// tmX: EPI_DGELU's map of the GELU derivatives ([M, N] bf16, 64 x 32 boxes, 128-byte swizzle);
// unused otherwise.
template <int BN, int EPI, int GELU_TANH, int A_MN = 0, int B_MN = 0, int PAIR = 0>
__global__ void __launch_bounds__(Cfg<BN>::THREADS, 1)  // 10 warps: <= 168 registers per thread
    gemm_bf16_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
                 const Params p) {
    using L = Cfg<BN, PAIR, EPI == EPI_DGELU>;
    constexpr int kStages = L::STAGES;
    constexpr int TM = PAIR ? 2 * BM : BM;  // output rows per tile
    constexpr int COLS = L::COLS_PER_WARP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    float* sbias = reinterpret_cast<float*>(smem + L::BIAS_OFF);  // [NEPI][COLS]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* peer_done = drain + 1;            // PAIR, leader: the peer's producer has finished
    uint64_t* aux_full = peer_done + 1;         // EPI_DGELU: [NEPI] a warp's derivative slice landed
    volatile unsigned long long* peer_issued =  // PAIR, leader: the peer's count of issued stage loads
        reinterpret_cast<volatile unsigned long long*>(aux_full + NEPI);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aux_full + NEPI + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0: leader
    const int unit0 = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
    const int n_units = PAIR ? static_cast<int>(num_clusters_x()) : static_cast<int>(gridDim.x);
    const int num_m = (p.M + TM - 1) / TM;
    const int num_n = (p.N + BN - 1) / BN;
    const int num_mn = num_m * num_n;
    const int num_tiles = num_mn * p.k_splits;
    const int num_kb = (p.K + BK - 1) / BK;
    // K-block range of a tile: splits are the slowest tile index, so a wave works on one K range.
    auto tile_kb = [&](int tile, int& kb0, int& kb1) {
        const int ks = tile / num_mn;
        kb0 = ks * p.kb_per_split;
        kb1 = min(num_kb, kb0 + p.kb_per_split);
    };
    auto tile_mn = [&](int tile, int& m_blk, int& n_blk) {
        tile %= num_mn;
        if (p.n_fastest) {
            n_blk = tile % num_n;
            m_blk = tile / num_n;
        } else {
            m_blk = tile % num_m;
            n_blk = tile / num_m;
        }
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], (PAIR ? 2 : 1) * NEPI * 32);
        }
        mbar_init(drain, 1);
        mbar_init(peer_done, 1);
        for (int w = 0; w < NEPI; ++w) mbar_init(&aux_full[w], 1);
        *peer_issued = 0ull;
        *abort_flag = 0;
        fence_barrier_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmC);
        if (EPI == EPI_DGELU) tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, L::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();  // the leader's barriers are initialised before the peer's loads count on them
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // The set-up above overlapped the previous kernel; its outputs are read from here on.
    griddep_launch_dependents();
    griddep_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t ph = 0;
            long long issued = 0;
            bool ok = true;
            const uint32_t full_leader = PAIR ? map_to_rank(full, 0) : 0u;  // cluster address of full[0]
            auto load = [&](void* dst, const CUtensorMap* map, int x, int y) {
                if (PAIR)
                    tma_load_2d_pair(dst, map, full_leader + 8u * static_cast<uint32_t>(stage), x, y);
                else
                    tma_load_2d(dst, map, &full[stage], x, y);
            };
            for (int tile = unit0; tile < num_tiles && ok; tile += n_units) {
                int m_blk, n_blk;
                tile_mn(tile, m_blk, n_blk);
                const int m0 = m_blk * TM + static_cast<int>(rank) * BM;           // this CTA's A rows
                const int n0 = n_blk * BN + static_cast<int>(rank) * L::B_ROWS;    // this CTA's B rows
                int kb0, kb1;
                tile_kb(tile, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&empty[stage], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + stage * L::STAGE_BYTES;
                    // the leader expects both CTAs' bytes
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], (PAIR ? 2 : 1) * L::STAGE_BYTES);
                    if (A_MN) {
#pragma unroll
                        for (int j = 0; j < BM / 64; ++j) load(st + j * 8192, &tmA, m0 + 64 * j, kb * BK);
                    } else {
                        load(st, &tmA, kb * BK, m0);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int j = 0; j < L::B_ROWS / 64; ++j)
                            load(st + L::A_BYTES + j * 8192, &tmB, n0 + 64 * j, kb * BK);
                    } else {
                        load(st + L::A_BYTES, &tmB, kb * BK, n0);
                    }
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        ph ^= 1u;
                    }
                }
            }
            // Make sure no bulk copy is still writing shared memory when the CTA exits: wait
            // for the latest load issued into each stage (already complete on the normal path).
            // The leader's `full` phases count the peer's bytes too, so the leader drains for both
            // CTAs.  After a time-out the two producers may have issued different numbers of
            // stage loads: the peer reports its count, and the leader balances the byte count of
            // every phase only one of them issued (the peer's bytes expected on a phase the leader
            // never armed; a peer half that will never come completed by hand), so that every
            // issued copy is waited for before the pair's final cluster barrier.
            long long total = issued;
            if (PAIR && rank != 0) {
                st_cluster_u64(map_to_rank(const_cast<unsigned long long*>(peer_issued), 0),
                               static_cast<unsigned long long>(issued));
                mbar_arrive_remote(map_to_rank(peer_done, 0));
            }
            if (PAIR && rank == 0) {
                const long long peer = mbar_wait_cluster_bounded(peer_done, 0)
                                           ? static_cast<long long>(*peer_issued) : issued;
                const long long lo = peer < issued ? peer : issued, hi = peer < issued ? issued : peer;
                for (long long idx = lo; idx < hi; ++idx) {
                    uint64_t* b = &full[idx % kStages];
                    if (idx >= kStages) mbar_drain(b, static_cast<uint32_t>(((idx - kStages) / kStages) & 1));
                    if (peer > issued)
                        mbar_arrive_expect_tx(b, L::STAGE_BYTES);  // only the peer's half arrives
                    else
                        mbar_complete_tx(b, L::STAGE_BYTES);       // the peer's half never comes
                }
                total = hi;
            }
            const long long n_check = rank != 0 ? 0 : (total < kStages ? total : kStages);
            for (long long i = 1; i <= n_check; ++i) {
                const long long idx = total - i;
                mbar_drain(&full[idx % kStages], static_cast<uint32_t>((idx / kStages) & 1));
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = make_idesc_bf16(TM, BN, B_MN != 0, A_MN != 0);
            int stage = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            bool ok = true;
            // Testing aid: nothing arrives on `drain` before the commit below, so this wait can only
            // give up, which sends the CTA (for a pair: the leader; the peer's own waits then give
            // up too) down its time-out path.
            if (g_force_timeout) {
                mbar_wait(drain, 0, abort_flag);
                ok = false;
            }
            for (int tile = unit0; tile < num_tiles && ok; tile += n_units) {
                if (!(PAIR ? mbar_wait_cluster(&tempty[acc], acc_ph ^ 1u, abort_flag)
                           : mbar_wait(&tempty[acc], acc_ph ^ 1u, abort_flag)))
                    break;
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
                int kb0, kb1;
                tile_kb(tile, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&full[stage], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_addr(smem + stage * L::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + L::A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        // K step of 16: 32 bytes along a K-major row, 16 rows (2048 bytes) of an
                        // MN-major tile.
                        const uint64_t da = A_MN ? make_sdesc_sw128_mn(a_addr + k * 2048, 8192)
                                                 : make_sdesc_sw128(a_addr + k * 32);
                        const uint64_t db = B_MN ? make_sdesc_sw128_mn(b_addr + k * 2048, 8192)
                                                 : make_sdesc_sw128(b_addr + k * 32);
                        if (PAIR)
                            umma_ss_pair(d, da, db, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
                        else
                            umma_ss(d, da, db, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
                    }
                    if (PAIR)
                        umma_commit_pair(&empty[stage], 0x3);
                    else
                        umma_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                if (PAIR)
                    umma_commit_pair(&tfull[acc], 0x3);
                else
                    umma_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_ph ^= 1u;
            }
            // All MMAs issued by this thread must be finished before TMEM is released.
            if (PAIR)
                umma_commit_pair(drain, 0x1);
            else
                umma_commit(drain);
            mbar_drain(drain, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue warps
        const int ew = warp - 2;
        const int quarter = warp & 3;        // TMEM lanes this warp may access
        const int half = ew >> 2;            // which BN/2 columns of the tile
        int acc = 0;
        uint32_t acc_ph = 0;
        uint32_t aux_ph = 0;
        bool aux_pending = false;  // EPI_DGELU: a derivative load of this warp not yet waited for
        uint8_t* abuf = smem + L::AUX_OFF + ew * L::AUX_WARP_BYTES;  // EPI_DGELU: this warp's slice
        for (int tile = unit0; tile < num_tiles; tile += n_units) {
            int m_blk, n_blk;
            tile_mn(tile, m_blk, n_blk);
            const int m0 = m_blk * TM + static_cast<int>(rank) * BM, n0 = n_blk * BN;  // this CTA's rows
            const int row = m0 + quarter * 32 + lane;
            const bool row_ok = row < p.M;
            const int nw0 = n0 + half * COLS;  // first column of this warp's slice
            float* sb = sbias + ew * COLS;  // this warp's private bias slice
            uint8_t* stg = smem + L::STG_OFF + ew * L::STG_BYTES;  // this warp's staging tile

            // EPI_DGELU: this warp's 32 x 128 slice of the GELU derivatives is copied into shared
            // memory while the tile's products run (rows past M and columns past N read as zero).
            if (EPI == EPI_DGELU) {
                __syncwarp();  // every lane's reads of the previous tile's slice are done
                if (lane == 0) {
                    fence_proxy_async_shared();
                    mbar_arrive_expect_tx(&aux_full[ew], static_cast<uint32_t>(L::AUX_WARP_BYTES));
                    tma_load_2d(abuf, &tmX, &aux_full[ew], nw0, m0 + quarter * 32);
                    tma_load_2d(abuf + L::AUX_WARP_BYTES / 2, &tmX, &aux_full[ew], nw0 + 64, m0 + quarter * 32);
                }
                aux_pending = true;
            }

            // Before the accumulator is ready: this warp's bias slice into shared memory.
            if (EPI != EPI_CE) {
                __syncwarp();  // the previous tile's reads of sb are done
                for (int c = lane; c < COLS; c += 32) {
                    const int n = nw0 + c;
                    sb[c] = (p.bias && n < p.N) ? __bfloat162float(p.bias[n]) : 0.f;
                }
                __syncwarp();
            }
            long long tgt = -1;
            if (EPI == EPI_CE && row_ok) tgt = p.targets[row];

            const bool got = mbar_wait(&tfull[acc], acc_ph, abort_flag);
            __syncwarp();  // tcgen05.ld below is warp-collective
            if (!__all_sync(0xffffffffu, got)) break;
            if (EPI == EPI_DGELU) {
                const bool ag = mbar_wait(&aux_full[ew], aux_ph, abort_flag);
                __syncwarp();
                if (!__all_sync(0xffffffffu, ag)) break;
                aux_ph ^= 1u;
                aux_pending = false;
            }
            tc_fence_after();
            const uint32_t tbase = tmem_base + static_cast<uint32_t>(acc * BN + half * COLS) +
                                   (static_cast<uint32_t>(quarter * 32) << 16);
            const int row0 = m0 + quarter * 32;      // first row of this warp's band
            const bool band_ok = row0 < p.M;         // warp-uniform
            // Row `lane` of the staging tile; its four 16-byte chunks are swizzled by bits 1-2 of
            // the row (the 64-byte TMA swizzle).
            uint4* srow = reinterpret_cast<uint4*>(stg + lane * 64);
            const int swz = (lane >> 1) & 3;

            float run_max = -INFINITY, run_sum = 0.f;
            constexpr float kLog2e = 1.4426950408889634f;

            if (EPI == EPI_RESID || EPI == EPI_F32) {
                const int out_row0 = row0 + (EPI == EPI_F32 ? (tile / num_mn) * p.M : 0);
#pragma unroll 1
                for (int c = 0; c < COLS; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(tbase + c, r);
#pragma unroll
                    for (int sub = 0; sub < 2; ++sub) {
                        const int n = nw0 + c + 16 * sub;
                        if (n >= p.N || !band_ok) continue;  // warp-uniform
                        float v[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[16 * sub + j]) + sb[c + 16 * sub + j];
                        if (lane == 0) bulk_wait_read_all();  // the buffer's previous tile was read
                        __syncwarp();
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            srow[q ^ swz] = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                                       __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
                        fence_proxy_async_shared();
                        __syncwarp();
                        if (lane == 0) {
                            if (EPI == EPI_RESID)
                                tma_reduce_add_2d(&tmC, stg, n, out_row0);
                            else
                                tma_store_2d(&tmC, stg, n, out_row0);
                            bulk_commit();
                        }
                    }
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < COLS; c += 64) {
                    uint32_t r[64];
                    tmem_ld64(tbase + c, r);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int cc = c + 32 * h;
                        const int n = nw0 + cc;
                        if (n >= p.N) continue;  // warp-uniform
                        const bool full_chunk = (n + 32 <= p.N);
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[32 * h + j]);
                        if (EPI == EPI_STORE || EPI == EPI_GELU || EPI == EPI_GELU2) {
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float4 b4 = *reinterpret_cast<const float4*>(sb + cc + 4 * q);
                                v[4 * q + 0] += b4.x;
                                v[4 * q + 1] += b4.y;
                                v[4 * q + 2] += b4.z;
                                v[4 * q + 3] += b4.w;
                            }
                        }
                        if (EPI == EPI_GELU && !GELU_TANH) {
                            gelu32_erf(v);
                        } else if (EPI == EPI_GELU) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = gelu_f<GELU_TANH>(v[j]);
                        }
                        if (EPI == EPI_DGELU) {
                            // this row's 32 derivatives of the chunk from the staged slice: row `lane`
                            // of box cc / 64, 16-byte chunks (cc % 64) / 8 .. + 3, swizzled by row % 8
                            const uint8_t* rp = abuf + (cc >> 6) * (L::AUX_WARP_BYTES / 2) + lane * 128;
                            const int c16 = (cc & 63) >> 3;
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const uint4 w = *reinterpret_cast<const uint4*>(rp + (((c16 + q) ^ (lane & 7)) << 4));
                                const uint32_t u4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    v[8 * q + 2 * e] *= __uint_as_float(u4[e] << 16);
                                    v[8 * q + 2 * e + 1] *= __uint_as_float(u4[e] & 0xffff0000u);
                                }
                            }
                        }
                        if (EPI == EPI_CE) {
                            float cmax = -INFINITY;
                            if (full_chunk) {
                                float m4[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
                                for (int j = 4; j < 32; ++j) m4[j & 3] = fmaxf(m4[j & 3], v[j]);
                                cmax = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                            } else {
                                for (int j = 0; j < 32; ++j)
                                    if (n + j < p.N) cmax = fmaxf(cmax, v[j]);
                            }
                            const float new_max = fmaxf(run_max, cmax);
                            const float off = new_max * kLog2e;
                            float s4[4] = {0.f, 0.f, 0.f, 0.f};
                            if (full_chunk) {
#pragma unroll
                                for (int j = 0; j < 32; ++j) s4[j & 3] += exp2_approx(fmaf(v[j], kLog2e, -off));
                            } else {
                                for (int j = 0; j < 32; ++j)
                                    if (n + j < p.N) s4[0] += exp2_approx(fmaf(v[j], kLog2e, -off));
                            }
                            run_sum = run_sum * exp2_approx((run_max - new_max) * kLog2e) +
                                      ((s4[0] + s4[1]) + (s4[2] + s4[3]));
                            run_max = new_max;
                            const long long rel = tgt - n;
                            if (rel >= 0 && rel < 32) {
                                float zt = 0.f;
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    if (j == rel) zt = v[j];
                                if (row_ok) p.tlogit[row] = zt;
                            }
                        }
                        if (!band_ok) continue;  // warp-uniform: no row of this band exists
                        float vg[EPI == EPI_GELU2 ? 32 : 1];  // EPI_GELU2: the GELU outputs of pass 1
                        if (EPI == EPI_GELU2) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                float g, dg;
                                gelu_pair_f<GELU_TANH>(v[j], g, dg);
                                v[j] = dg;
                                vg[j] = g;
                            }
                        }
                        for (int pass = 0; pass < (EPI == EPI_GELU2 ? 2 : 1); ++pass) {
                            if (EPI == EPI_GELU2 && pass == 1) {
#pragma unroll
                                for (int j = 0; j < 32; ++j) v[j] = vg[j];
                            }
                            if (lane == 0) bulk_wait_read_all();  // the buffer's previous tile was read
                            __syncwarp();
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                srow[q ^ swz] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]),
                                                           pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                                           pack_bf16x2(v[8 * q + 4], v[8 * q + 5]),
                                                           pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
                            fence_proxy_async_shared();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_2d(&tmC, stg, n, row0 + pass * p.M);
                                bulk_commit();
                            }
                        }
                        if (EPI == EPI_DGELU && p.colsum) {
                            // this band's column sums of the 32 columns (rows past M add zero)
                            if (!row_ok) {
#pragma unroll
                                for (int j = 0; j < 32; ++j) v[j] = 0.f;
                            }
                            const float cs = warp_colsum32(v);
                            if (n + lane < p.N) p.colsum[static_cast<long long>(row0 >> 5) * p.ld_colsum + n + lane] = cs;
                        }
                    }
                }
            }
            if (EPI == EPI_CE && row_ok) {
                p.part[static_cast<size_t>(row) * p.n_part + n_blk * L::PARTS_PER_TILE + half] =
                    make_float2(run_max, run_sum);
            }
            tc_fence_before();
            if (PAIR && rank != 0)
                mbar_arrive_remote(map_to_rank(&tempty[acc], 0));
            else
                mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_ph ^= 1u;
        }
        if (lane == 0) bulk_wait_all();  // this warp's stores and reduce-adds have completed
        // a derivative load issued for a tile this warp did not finish (time-out) lands before exit
        if (EPI == EPI_DGELU && aux_pending && lane == 0) mbar_drain(&aux_full[ew], aux_ph);
        __syncwarp();
    }

    __syncthreads();
    // A pair releases its tensor memory together, once neither CTA's MMAs, loads or arrivals can
    // still reach the other.
    if (PAIR) cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if (PAIR)
            tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
        else
            tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
    if (threadIdx.x == 0 && *abort_flag) set_status(p.status, GPT_ERR_TIMEOUT);
}

}  // namespace gemm
}  // namespace gpt
