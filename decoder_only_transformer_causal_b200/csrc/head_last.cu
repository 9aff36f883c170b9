// The head of the inference branch for sm_100a: logits[b, :] = LayerNorm(x_b; ln_f) wte^T for the
// last position of each sequence ("nanoGPT 全局流程图", §3.2 ④: without targets only x[:, [-1], :]
// goes through ln_f and lm_head).
//
// The product reads all of wte (V x C bf16, 77 MB for GPT-2 124M, 161 MB for XL) once and does
// only 2 B C V FLOP, so it is bound by HBM.  wte is the streamed operand: 128-row tiles of it
// (the vocabulary entries) are the MMA's A operand, fed by TMA through a deep shared-memory ring,
// and the at most 16 normalised rows u (bf16, the precision of every other product input) are the
// B operand, resident in shared memory for the whole launch: D[128 x 16] = wte_tile u^T, one
// tcgen05.mma (M=128, N=16, K=16) per 16 columns of C.  The tensor core's share is small; the
// kernel's job is to keep enough of wte in flight.
//
// One persistent CTA per SM walks the 128-row tiles of wte.  Warp 0: TMA producer; warp 1: MMA
// issuer (two 16-column accumulators in tensor memory, so one tile's epilogue overlaps the next
// tile's products); warps 2-5: epilogue, one vocabulary entry per thread, writing its B logits.
// All six warps first compute the LayerNorm of the B rows (population variance, eps 1e-5) and
// write u into shared memory in the 128-byte-swizzled K-major layout the MMA reads.
#include "common.cuh"
#include "internal.h"

namespace gpt {
namespace {

constexpr int kHeadRows = 16;                 // N of the product: rows u per launch
constexpr int kTileV = 128;                   // vocabulary entries per tile (M)
constexpr int kBK = 64;                       // one 128-byte swizzle row of bf16
constexpr int kStages = 8;
constexpr int kTileBytes = kTileV * kBK * 2;  // 16 KB of wte per stage
constexpr int kUBlockBytes = kHeadRows * kBK * 2;  // 2 KB of u per 64 columns of C
constexpr int kMaxC = 2048;
constexpr int kThreads = 192;
constexpr int kOffU = kStages * kTileBytes;
constexpr int kOffBar = kOffU + (kMaxC / kBK) * kUBlockBytes;
// full[kStages] empty[kStages] tfull[2] tempty[2] drain
constexpr int kNumBars = 2 * kStages + 5;
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;

struct HeadArgs {
    const float* x;      // row b at x + b * ldx (fp32 residual stream)
    long long ldx;
    const bf16* lnw;     // [C]
    const bf16* lnb;     // [C] or null
    bf16* out;           // row b at out + b * ldo
    long long ldo;
    int rows, C, V;
    int32_t* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    head_last_kernel(const __grid_constant__ CUtensorMap tmW, const HeadArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* su = smem + kOffU;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = a.C;
    const int num_kb = (C + kBK - 1) / kBK;
    const int num_tiles = (a.V + kTileV - 1) / kTileV;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 32);
        tmem_relinquish();
    }
    griddep_launch_dependents();
    griddep_wait();

    // The producer's sequence of loads: this CTA's tiles in turn, each as num_kb 128 x 64 boxes.
    const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;
    const long long n_loads = static_cast<long long>(my_tiles) * num_kb;
    long long issued = 0;
    auto issue = [&](long long i) {  // load i into stage i % kStages (its previous use is free)
        const int st = static_cast<int>(i % kStages);
        const int tile = static_cast<int>(blockIdx.x) + static_cast<int>(i / num_kb) * static_cast<int>(gridDim.x);
        mbar_arrive_expect_tx(&full[st], kTileBytes);
        tma_load_2d(smem + st * kTileBytes, &tmW, &full[st], static_cast<int>(i % num_kb) * kBK, tile * kTileV);
    };
    // The first loads need no free slot: issue them before the prologue below.
    if (threadIdx.x == 0)
        for (; issued < n_loads && issued < kStages; ++issued) issue(issued);

    // ---- LayerNorm of the rows into u (rows >= a.rows and columns >= C are zero).  Element
    // (r, k) of k-block kb sits at byte kb * 2048 + (r / 8) * 1024 + (r % 8) * 128 + 16 * (chunk ^
    // (r % 8)) + 2 * (k % 8), chunk = (k % 64) / 8: the layout a 128-byte-swizzled TMA box of 16 rows
    // x 64 columns would have.
    for (int r = warp; r < kHeadRows; r += kThreads / 32) {
        float mean = 0.f, rstd = 0.f;
        const float* xr = a.x + static_cast<long long>(r) * a.ldx;
        if (r < a.rows) {
            float s = 0.f;
            for (int k = lane * 4; k < C; k += 128) {
                const float4 v = __ldcg(reinterpret_cast<const float4*>(xr + k));
                s += (v.x + v.y) + (v.z + v.w);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            mean = s / C;
            float ss = 0.f;
            for (int k = lane * 4; k < C; k += 128) {
                const float4 v = __ldcg(reinterpret_cast<const float4*>(xr + k));
                const float d0 = v.x - mean, d1 = v.y - mean, d2 = v.z - mean, d3 = v.w - mean;
                ss += (d0 * d0 + d1 * d1) + (d2 * d2 + d3 * d3);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            rstd = rsqrtf(ss / C + 1e-5f);
        }
        // 8 columns (one 16-byte chunk) per lane and step
        for (int k = lane * 8; k < num_kb * kBK; k += 256) {
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            if (r < a.rows && k < C) {
                float v[8];
                const float4 v0 = __ldcg(reinterpret_cast<const float4*>(xr + k));
                const float4 v1 = __ldcg(reinterpret_cast<const float4*>(xr + k) + 1);
                v[0] = v0.x, v[1] = v0.y, v[2] = v0.z, v[3] = v0.w, v[4] = v1.x, v[5] = v1.y, v[6] = v1.z, v[7] = v1.w;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float g = __bfloat162float(a.lnw[k + e]);
                    const float bb = a.lnb ? __bfloat162float(a.lnb[k + e]) : 0.f;
                    v[e] = (v[e] - mean) * rstd * g + bb;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) w[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
            }
            const int kb = k / kBK, chunk = (k % kBK) / 8;
            uint8_t* dst = su + kb * kUBlockBytes + (r / 8) * 1024 + (r % 8) * 128 + 16 * (chunk ^ (r % 8));
            *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    fence_proxy_async_shared();  // u, written by these threads, is read by the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (; issued < n_loads; ++issued) {
                // slot issued % kStages is free once the products of load issued - kStages are done
                const uint32_t ph = static_cast<uint32_t>(((issued - kStages) / kStages) & 1);
                if (!mbar_wait(&empty[issued % kStages], ph, abort_flag)) break;
                issue(issued);
            }
            const long long n_check = issued < kStages ? issued : kStages;
            for (long long i = 1; i <= n_check; ++i) {
                const long long idx = issued - i;
                mbar_drain(&full[idx % kStages], static_cast<uint32_t>((idx / kStages) & 1));
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc_bf16(kTileV, kHeadRows, false);
            const uint32_t u_addr = smem_addr(su);
            int stage = 0, acc = 0;
            uint32_t ph = 0, acc_ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                if (!mbar_wait(&tempty[acc], acc_ph ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(acc * kHeadRows);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&full[stage], ph, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t w_addr = smem_addr(smem + stage * kTileBytes);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_ss(d, make_sdesc_sw128(w_addr + k * 32), make_sdesc_sw128(u_addr + kb * kUBlockBytes + k * 32),
                                idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    umma_commit(&empty[stage]);
                    if (++stage == kStages) { stage = 0; ph ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_ph ^= 1u;
            }
            umma_commit(drain);
            mbar_drain(drain, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue: one entry per thread
        const int quarter = warp & 3;
        int acc = 0;
        uint32_t acc_ph = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const bool got = mbar_wait(&tfull[acc], acc_ph, abort_flag);
            __syncwarp();
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            uint32_t r[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
                "tcgen05.wait::ld.sync.aligned;"
                : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                  "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                : "r"(tmem + static_cast<uint32_t>(acc * kHeadRows) + (static_cast<uint32_t>(quarter * 32) << 16))
                : "memory");
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            const int v = tile * kTileV + quarter * 32 + lane;
            if (v < a.V) {
#pragma unroll
                for (int b = 0; b < kHeadRows; ++b)
                    if (b < a.rows) a.out[b * a.ldo + v] = __float2bfloat16_rn(__uint_as_float(r[b]));
            }
            acc ^= 1;
            if (acc == 0) acc_ph ^= 1u;
        }
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 32);
    }
    if (threadIdx.x == 0 && *abort_flag) set_status(a.status, GPT_ERR_TIMEOUT);
}

}  // namespace

bool head_last_tc_supported(int C) { return C % 8 == 0 && C <= kMaxC; }

int launch_head_last_bf16(const float* x, long long ldx, const bf16* lnw, const bf16* lnb, const bf16* wte, int B,
                          int C, int V, bf16* out, long long ldo, int32_t* status, cudaStream_t s) {
    if (!head_last_tc_supported(C)) return GPT_ERR_UNSUPPORTED;
    CUtensorMap tm;
    int rc = make_tmap_bf16_2d(&tm, wte, static_cast<uint64_t>(C), static_cast<uint64_t>(V),
                               static_cast<uint64_t>(C) * 2, kBK, kTileV);
    if (rc) return rc;
    static size_t opted[kMaxDevices] = {};
    rc = opt_in_smem(reinterpret_cast<const void*>(head_last_kernel), kSmemBytes, opted);
    if (rc) return rc;
    const int tiles = (V + kTileV - 1) / kTileV;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    for (int r0 = 0; r0 < B; r0 += kHeadRows) {
        HeadArgs a{x + static_cast<long long>(r0) * ldx, ldx, lnw, lnb, out + static_cast<long long>(r0) * ldo, ldo,
                   B - r0 < kHeadRows ? B - r0 : kHeadRows, C, V, status};
        rc = launch_overlapped(head_last_kernel, dim3(grid), dim3(kThreads), kSmemBytes, s, tm, a);
        if (rc) return rc;
    }
    return GPT_OK;
}

// Pipeline-wait limit of this file's kernel on the current device (0: the default).
GPT_DEFINE_WAIT_LIMIT_SETTER(set_wait_limit_head)

}  // namespace gpt
