// Host launcher of the tensor-core GEMM (kernel in gemm_tc.cuh).
#include "gemm_tc.cuh"
#include "internal.h"

namespace gpt {

namespace {

constexpr int kBN = 256;

// Co-resident clusters of two for a kernel (cached per device; 0 if the query fails).
int max_pairs(const void* kern, int threads, size_t smem, int* cache) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    if (cache[dev] > 0) return cache[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * num_sms());
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cache[dev] = n;
    return n;
}

// PAIR: 256-row tiles on CTA pairs (the 2-SM MMA); the B map's box must then be 128 rows
// (K-major B) — see b_box_rows().
// tx: EPI_DGELU's derivative map (any map otherwise; it is not read).
template <int EPI, int GELU_TANH, int A_MN = 0, int B_MN = 0, int PAIR = 0>
int launch_one(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const gemm::Params& p,
               cudaStream_t s, const CUtensorMap* tx = nullptr) {
    using L = gemm::Cfg<kBN, PAIR, EPI == gemm::EPI_DGELU>;
    const CUtensorMap& txr = tx ? *tx : tc;
    auto kern = gemm::gemm_bf16_tc<kBN, EPI, GELU_TANH, A_MN, B_MN, PAIR>;
    static size_t opted[kMaxDevices] = {};
    const int rc = opt_in_smem(reinterpret_cast<const void*>(kern), L::SMEM_BYTES, opted);
    if (rc) return rc;
    const int tm = PAIR ? 2 * gemm::BM : gemm::BM;
    const int tiles = ((p.M + tm - 1) / tm) * ((p.N + kBN - 1) / kBN) * p.k_splits;
    if (PAIR) {
        static int cache[kMaxDevices] = {};
        int units = max_pairs(reinterpret_cast<const void*>(kern), L::THREADS, L::SMEM_BYTES, cache);
        if (units <= 0) units = num_sms() / 2;
        units = tiles < units ? tiles : units;
        return launch_overlapped_pairs(kern, dim3(2 * units), dim3(L::THREADS), L::SMEM_BYTES, s, ta, tb, tc, txr, p);
    }
    const int grid = tiles < num_sms() ? tiles : num_sms();
    return launch_overlapped(kern, dim3(grid), dim3(L::THREADS), L::SMEM_BYTES, s, ta, tb, tc, txr, p);
}

// 2-SM pairs pay off once there are two 128-row blocks to pair.
bool use_pairs(int M) { return M >= 2 * gemm::BM; }

// out[m, n] += sum over s = 0..S-1, in order, of part[s * M + m][n]: the partial products of a
// split-K launch (part rows of N fp32; N, ldo multiples of 4 and 16-byte aligned buffers).
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int S, int M, int N, float* __restrict__ out,
                                     long long ldo) {
    griddep_launch_dependents();
    griddep_wait();
    const long long n4 = N / 4;
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<long long>(M) * n4) return;
    const long long m = i / n4, c = (i % n4) * 4;
    float4 t = __ldcg(reinterpret_cast<const float4*>(part + m * N + c));
    for (int s = 1; s < S; ++s) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(part + (static_cast<long long>(s) * M + m) * N + c));
        t.x += v.x, t.y += v.y, t.z += v.z, t.w += v.w;
    }
    float4* o = reinterpret_cast<float4*>(out + m * ldo + c);
    float4 d = __ldcg(o);
    d.x += t.x, d.y += t.y, d.z += t.z, d.w += t.w;
    *o = d;
}

// Split count for an accumulating product with MN-major A: the S that minimises the modelled
// time  P * ceil(tiles * S / 148) / S  +  2 * S * M * N * 4 / B  — the product's time P at full
// occupancy of a 148-SM part, stretched by the wave quantisation of tiles * S CTAs, plus writing
// and re-reading the S partial products at HBM bandwidth B — with every K range non-empty.
// 1 = no split (also when M % 32 != 0 or N % 4 != 0).
constexpr int kSplitSms = 148;
void split_plan(int M, int N, int K, int* splits, int* kb_per) {
    const long long tiles = static_cast<long long>((M + gemm::BM - 1) / gemm::BM) * ((N + kBN - 1) / kBN);
    const int num_kb = (K + gemm::BK - 1) / gemm::BK;
    *splits = 1;
    *kb_per = num_kb;
    if ((M % 32) || (N % 4) || tiles >= kSplitSms || num_kb < 2) return;
    const double prod = 2.0 * M * N * K / 1.0e15;  // seconds at ~1 PFLOP/s
    const double part = 2.0 * 4.0 * M * N / 5.0e12;  // seconds per split of partial traffic
    double best = 1e30;
    int best_s = 1;
    const int s_max = num_kb < 32 ? num_kb : 32;
    for (int S = 1; S <= s_max; ++S) {
        const int per = (num_kb + S - 1) / S;
        const int Se = (num_kb + per - 1) / per;  // non-empty ranges
        if (Se != S) continue;
        const double waves = static_cast<double>((tiles * S + kSplitSms - 1) / kSplitSms);
        const double t = prod * waves * kSplitSms / (static_cast<double>(S) * tiles) + (S > 1 ? part * S : 0.0);
        if (t < best * 0.999) {
            best = t;
            best_s = S;
        }
    }
    *splits = best_s;
    *kb_per = (num_kb + best_s - 1) / best_s;
}

}  // namespace

size_t gemm_acc_split_bytes(int M, int N, int K) {
    int S, per;
    split_plan(M, N, K, &S, &per);
    return S > 1 ? static_cast<size_t>(S) * M * N * 4 : 0;
}

int gemm_ce_parts(int N) { return ((N + kBN - 1) / kBN) * gemm::Cfg<kBN>::PARTS_PER_TILE; }

int launch_gemm_bf16(const bf16* A, long long lda, const bf16* W, long long ldw, const bf16* bias,
                     void* out, long long ldo, int M, int N, int K, int epilogue, int gelu,
                     const CeArgs* ce, int32_t* status, cudaStream_t s) {
    if (M == 0 || N == 0) return GPT_OK;
    CUtensorMap ta, tb;
    int rc = make_tmap_bf16_2d(&ta, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                               static_cast<uint64_t>(lda) * 2, gemm::BK, gemm::BM);
    if (rc) return rc;
    const bool pair = use_pairs(M);
    rc = make_tmap_bf16_2d(&tb, W, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                           static_cast<uint64_t>(ldw) * 2, gemm::BK, pair ? kBN / 2 : kBN);
    if (rc) return rc;
    // Output map for the epilogue's TMA stores: 32-row boxes of 64 bytes (32 bf16 or 16 fp32);
    // 2M rows for EPI_GELU2 (pre-activation, then GELU output).
    CUtensorMap tc;
    const bool out_f32 = epilogue == GPT_EPI_RESID;
    if (epilogue == gemm::EPI_GELU2 && (M % 32)) return GPT_ERR_UNSUPPORTED;
    const uint64_t out_rows = static_cast<uint64_t>(M) * (epilogue == gemm::EPI_GELU2 ? 2 : 1);
    rc = make_tmap_2d_sw64(&tc, out, out_f32, static_cast<uint64_t>(N), out_rows,
                           static_cast<uint64_t>(ldo) * (out_f32 ? 4 : 2), out_f32 ? 16 : 32, 32);
    if (rc) return rc;
    gemm::Params p{};
    p.M = M;
    p.N = N;
    p.K = K;
    p.bias = bias;
    p.out = out;
    p.ldo = ldo;
    // Visit tiles so that the larger operand streams from memory once (see gemm_tc.cuh).
    p.n_fastest = static_cast<long long>(M) >= static_cast<long long>(N) ? 1 : 0;
    p.status = status;
    p.k_splits = 1;
    p.kb_per_split = (K + gemm::BK - 1) / gemm::BK;
    if (epilogue == gemm::EPI_CE) {
        if (!ce) return GPT_ERR_NULL;
        p.targets = ce->targets;
        p.part = ce->part;
        p.tlogit = ce->tlogit;
        p.n_part = ce->n_part;
    }
    switch (epilogue) {
        case GPT_EPI_STORE:
            return pair ? launch_one<gemm::EPI_STORE, 0, 0, 0, 1>(ta, tb, tc, p, s)
                        : launch_one<gemm::EPI_STORE, 0>(ta, tb, tc, p, s);
        case GPT_EPI_GELU:
            if (gelu == GPT_GELU_TANH)
                return pair ? launch_one<gemm::EPI_GELU, 1, 0, 0, 1>(ta, tb, tc, p, s)
                            : launch_one<gemm::EPI_GELU, 1>(ta, tb, tc, p, s);
            return pair ? launch_one<gemm::EPI_GELU, 0, 0, 0, 1>(ta, tb, tc, p, s)
                        : launch_one<gemm::EPI_GELU, 0>(ta, tb, tc, p, s);
        case GPT_EPI_RESID:
            return pair ? launch_one<gemm::EPI_RESID, 0, 0, 0, 1>(ta, tb, tc, p, s)
                        : launch_one<gemm::EPI_RESID, 0>(ta, tb, tc, p, s);
        case gemm::EPI_CE:
            return pair ? launch_one<gemm::EPI_CE, 0, 0, 0, 1>(ta, tb, tc, p, s)
                        : launch_one<gemm::EPI_CE, 0>(ta, tb, tc, p, s);
        case gemm::EPI_GELU2:
            if (gelu == GPT_GELU_TANH)
                return pair ? launch_one<gemm::EPI_GELU2, 1, 0, 0, 1>(ta, tb, tc, p, s)
                            : launch_one<gemm::EPI_GELU2, 1>(ta, tb, tc, p, s);
            return pair ? launch_one<gemm::EPI_GELU2, 0, 0, 0, 1>(ta, tb, tc, p, s)
                        : launch_one<gemm::EPI_GELU2, 0>(ta, tb, tc, p, s);
        default: return GPT_ERR_UNSUPPORTED;
    }
}

int launch_gemm_bf16_bwd(const bf16* A, long long lda, bool a_mn, const bf16* W, long long ldw, bool b_mn, void* out,
                         long long ldo, int M, int N, int K, int mode, const bf16* aux, long long ld_aux, int gelu,
                         int32_t* status, cudaStream_t s, float* split_ws, float* colsum) {
    if (M == 0 || N == 0) return GPT_OK;
    if (!b_mn || (a_mn && mode != GEMM_BWD_ACC_F32)) return GPT_ERR_UNSUPPORTED;
    CUtensorMap ta, tb, tc;
    int rc = a_mn ? make_tmap_bf16_2d(&ta, A, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                                      static_cast<uint64_t>(lda) * 2, 64, gemm::BK)
                  : make_tmap_bf16_2d(&ta, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                                      static_cast<uint64_t>(lda) * 2, gemm::BK, gemm::BM);
    if (rc) return rc;
    rc = make_tmap_bf16_2d(&tb, W, static_cast<uint64_t>(N), static_cast<uint64_t>(K), static_cast<uint64_t>(ldw) * 2,
                           64, gemm::BK);
    if (rc) return rc;
    gemm::Params p{};
    p.M = M;
    p.N = N;
    p.K = K;
    p.n_fastest = static_cast<long long>(M) >= static_cast<long long>(N) ? 1 : 0;
    p.status = status;
    p.k_splits = 1;
    p.kb_per_split = (K + gemm::BK - 1) / gemm::BK;
    p.out = out;
    p.ldo = ldo;
    const bool f32 = mode == GEMM_BWD_ACC_F32 || mode == GEMM_BWD_STORE_F32;
    if (mode == GEMM_BWD_ACC_F32 && a_mn && split_ws) {
        int S, per;
        split_plan(M, N, K, &S, &per);
        if (S > 1) {
            // Deterministic split-K: each K range stores its partial product into its own slice of
            // split_ws, then one pass adds the slices to out in order.
            if (((reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(split_ws)) & 15) || (ldo % 4))
                return GPT_ERR_BAD_ALIGN;
            rc = make_tmap_2d_sw64(&tc, split_ws, true, static_cast<uint64_t>(N), static_cast<uint64_t>(S) * M,
                                   static_cast<uint64_t>(N) * 4, 16, 32);
            if (rc) return rc;
            p.out = split_ws;
            p.ldo = N;
            p.k_splits = S;
            p.kb_per_split = per;
            rc = launch_one<gemm::EPI_F32, 0, 1, 1>(ta, tb, tc, p, s);
            if (rc) return rc;
            const long long n4 = static_cast<long long>(M) * (N / 4);
            return launch_overlapped(splitk_reduce_kernel, dim3(static_cast<unsigned>((n4 + 255) / 256)), dim3(256), 0,
                                     s, static_cast<const float*>(split_ws), S, M, N, static_cast<float*>(out), ldo);
        }
    }
    rc = make_tmap_2d_sw64(&tc, out, f32, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                           static_cast<uint64_t>(ldo) * (f32 ? 4 : 2), f32 ? 16 : 32, 32);
    if (rc) return rc;
    // The input-gradient products (K-major A, M = token rows) run on CTA pairs; MN-major B boxes are
    // 64 columns wide either way.
    const bool pair = !a_mn && use_pairs(M);
    CUtensorMap tx;
    if (mode == GEMM_BWD_DGELU_BF16) {
        if (!aux) return GPT_ERR_NULL;
        if ((reinterpret_cast<uintptr_t>(aux) & 15) || (ld_aux % 8)) return GPT_ERR_BAD_ALIGN;
        // the epilogue warps' 64-column x 32-row boxes of the derivatives
        rc = make_tmap_bf16_2d(&tx, aux, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                               static_cast<uint64_t>(ld_aux) * 2, 64, 32);
        if (rc) return rc;
        p.aux = aux;
        p.ld_aux = ld_aux;
        p.colsum = colsum;
        p.ld_colsum = N;
    }
    switch (mode) {
        case GEMM_BWD_ACC_F32:
            if (a_mn) return launch_one<gemm::EPI_RESID, 0, 1, 1>(ta, tb, tc, p, s);
            return pair ? launch_one<gemm::EPI_RESID, 0, 0, 1, 1>(ta, tb, tc, p, s)
                        : launch_one<gemm::EPI_RESID, 0, 0, 1>(ta, tb, tc, p, s);
        case GEMM_BWD_STORE_F32:
            return pair ? launch_one<gemm::EPI_F32, 0, 0, 1, 1>(ta, tb, tc, p, s)
                        : launch_one<gemm::EPI_F32, 0, 0, 1>(ta, tb, tc, p, s);
        case GEMM_BWD_STORE_BF16:
            return pair ? launch_one<gemm::EPI_STORE, 0, 0, 1, 1>(ta, tb, tc, p, s)
                        : launch_one<gemm::EPI_STORE, 0, 0, 1>(ta, tb, tc, p, s);
        case GEMM_BWD_DGELU_BF16:
            if (gelu == GPT_GELU_TANH)
                return pair ? launch_one<gemm::EPI_DGELU, 1, 0, 1, 1>(ta, tb, tc, p, s, &tx)
                            : launch_one<gemm::EPI_DGELU, 1, 0, 1>(ta, tb, tc, p, s, &tx);
            return pair ? launch_one<gemm::EPI_DGELU, 0, 0, 1, 1>(ta, tb, tc, p, s, &tx)
                        : launch_one<gemm::EPI_DGELU, 0, 0, 1>(ta, tb, tc, p, s, &tx);
        default: return GPT_ERR_UNSUPPORTED;
    }
}

int launch_gemm_bf16_acc(const bf16* A, long long lda, bool a_mn, const bf16* W, long long ldw, bool b_mn, float* out,
                         long long ldo, int M, int N, int K, int32_t* status, cudaStream_t s, float* split_ws) {
    if (!a_mn && !b_mn)
        return launch_gemm_bf16(A, lda, W, ldw, nullptr, out, ldo, M, N, K, GPT_EPI_RESID, 0, nullptr, status, s);
    return launch_gemm_bf16_bwd(A, lda, a_mn, W, ldw, b_mn, out, ldo, M, N, K, GEMM_BWD_ACC_F32, nullptr, 0, 0, status,
                                s, split_ws);
}

// Pipeline-wait limit of this file's kernels on the current device (0: the default).
GPT_DEFINE_WAIT_LIMIT_SETTER(set_wait_limit_gemm)

}  // namespace gpt
