// Host launcher of the tensor-core GEMM (kernel in gemm_tc.cuh).
#include "gemm_tc.cuh"
#include "internal.h"

namespace gpt {

namespace {

constexpr int kBN = 256;

template <int EPI, int GELU_TANH, int A_MN = 0, int B_MN = 0>
int launch_one(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const gemm::Params& p,
               cudaStream_t s) {
    using L = gemm::Cfg<kBN>;
    auto kern = gemm::gemm_bf16_tc<kBN, EPI, GELU_TANH, A_MN, B_MN>;
    static size_t opted[kMaxDevices] = {};
    const int rc = opt_in_smem(reinterpret_cast<const void*>(kern), L::SMEM_BYTES, opted);
    if (rc) return rc;
    const int tiles = ((p.M + gemm::BM - 1) / gemm::BM) * ((p.N + kBN - 1) / kBN);
    const int grid = tiles < num_sms() ? tiles : num_sms();
    return launch_overlapped(kern, dim3(grid), dim3(L::THREADS), L::SMEM_BYTES, s, ta, tb, tc, p);
}

}  // namespace

int gemm_ce_parts(int N) { return ((N + kBN - 1) / kBN) * gemm::Cfg<kBN>::PARTS_PER_TILE; }

int launch_gemm_bf16(const bf16* A, long long lda, const bf16* W, long long ldw, const bf16* bias,
                     void* out, long long ldo, int M, int N, int K, int epilogue, int gelu,
                     const CeArgs* ce, int32_t* status, cudaStream_t s) {
    if (M == 0 || N == 0) return GPT_OK;
    CUtensorMap ta, tb;
    int rc = make_tmap_bf16_2d(&ta, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                               static_cast<uint64_t>(lda) * 2, gemm::BK, gemm::BM);
    if (rc) return rc;
    rc = make_tmap_bf16_2d(&tb, W, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                           static_cast<uint64_t>(ldw) * 2, gemm::BK, kBN);
    if (rc) return rc;
    // Output map for the epilogue's TMA stores: 32-row boxes of 64 bytes (32 bf16 or 16 fp32).
    CUtensorMap tc;
    const bool out_f32 = epilogue == GPT_EPI_RESID;
    rc = make_tmap_2d_sw64(&tc, out, out_f32, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
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
    switch (epilogue) {
        case GPT_EPI_STORE: return launch_one<gemm::EPI_STORE, 0>(ta, tb, tc, p, s);
        case GPT_EPI_GELU:
            return gelu == GPT_GELU_TANH ? launch_one<gemm::EPI_GELU, 1>(ta, tb, tc, p, s)
                                         : launch_one<gemm::EPI_GELU, 0>(ta, tb, tc, p, s);
        case GPT_EPI_RESID: return launch_one<gemm::EPI_RESID, 0>(ta, tb, tc, p, s);
        case gemm::EPI_CE:
            if (!ce) return GPT_ERR_NULL;
            p.targets = ce->targets;
            p.part = ce->part;
            p.tlogit = ce->tlogit;
            p.n_part = ce->n_part;
            return launch_one<gemm::EPI_CE, 0>(ta, tb, tc, p, s);
        default: return GPT_ERR_UNSUPPORTED;
    }
}

int launch_gemm_bf16_acc(const bf16* A, long long lda, bool a_mn, const bf16* W, long long ldw, bool b_mn, float* out,
                         long long ldo, int M, int N, int K, int32_t* status, cudaStream_t s) {
    if (M == 0 || N == 0) return GPT_OK;
    if (a_mn == false && b_mn == false)
        return launch_gemm_bf16(A, lda, W, ldw, nullptr, out, ldo, M, N, K, GPT_EPI_RESID, 0, nullptr, status, s);
    if (!b_mn) return GPT_ERR_UNSUPPORTED;  // MN-major A is only paired with MN-major B
    CUtensorMap ta, tb, tc;
    int rc = a_mn ? make_tmap_bf16_2d(&ta, A, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                                      static_cast<uint64_t>(lda) * 2, 64, gemm::BK)
                  : make_tmap_bf16_2d(&ta, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                                      static_cast<uint64_t>(lda) * 2, gemm::BK, gemm::BM);
    if (rc) return rc;
    rc = make_tmap_bf16_2d(&tb, W, static_cast<uint64_t>(N), static_cast<uint64_t>(K), static_cast<uint64_t>(ldw) * 2,
                           64, gemm::BK);
    if (rc) return rc;
    rc = make_tmap_2d_sw64(&tc, out, true, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                           static_cast<uint64_t>(ldo) * 4, 16, 32);
    if (rc) return rc;
    gemm::Params p{};
    p.M = M;
    p.N = N;
    p.K = K;
    p.out = out;
    p.ldo = ldo;
    p.n_fastest = static_cast<long long>(M) >= static_cast<long long>(N) ? 1 : 0;
    p.status = status;
    return a_mn ? launch_one<gemm::EPI_RESID, 0, 1, 1>(ta, tb, tc, p, s)
                : launch_one<gemm::EPI_RESID, 0, 0, 1>(ta, tb, tc, p, s);
}

}  // namespace gpt
