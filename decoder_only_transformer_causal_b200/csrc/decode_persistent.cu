// One decode step of the bf16 model as a single persistent kernel ("nanoGPT 全局流程图", 第五阶段
// generate: the newest position of each sequence through every Block against the cached keys and
// values of the earlier ones, then ln_f and the tied head).
//
// The step is a chain of matrix-vector products whose weights (1-5 MB each for GPT-2 124M) are far
// below HBM's bandwidth-delay product, so as separate launches each is bound by latency.  Here one
// cooperative launch (one CTA per SM, all resident) walks the whole chain:
//   per layer { LN1 + c_attn (q out, k/v appended to the cache) | attention over the cache |
//   attn c_proj + residual | LN2 + c_fc + GELU | mlp c_proj + residual }; ln_f + head
// with a grid barrier between dependent phases (5 per layer; layer 0's first phase embeds the tokens
// itself).  Every wait is bounded: on expiry the CTA records GPT_ERR_TIMEOUT, lets its copies in
// flight land and returns (the others give up at their next barrier).
//
// What bounds it.  Each phase is a short dependent chain (one L2 round trip for its input rows, a
// few hundred instructions, the barrier), so the step is bound by latency and by instruction fetch:
// the four product phases therefore run from one copy of the code (a loop over the phase), loops
// stay rolled where unrolling buys nothing, and no helper is called out of line (no stack traffic
// through an L1 that the shared-memory carve-out leaves small).
//
// Weights stay off the critical path.  A product's output columns are split over the CTAs in tiles
// of 8 weight rows (each CTA owns one contiguous range); the CTA's rows of a phase (and their bias,
// and the LayerNorm weights that precede c_attn and c_fc) are copied into shared memory by bulk
// copies (cp.async.bulk, one per row, rows padded by 16 bytes so that fragment loads are free of
// bank conflicts).  A slot is refilled as soon as its product is done, between the CTA's arrival at
// the barrier and its wait, one copy per thread: with S = 4 slots the next layer's
// weights are in flight while this one runs; smaller shared-memory budgets (larger B or C) use S = 2
// or 1.  The products are tensor-core mma.sync m16n8k16 (bf16 in, fp32 accumulate): up to 16 staged
// rows are the A operand, 8 weight rows the B operand, K split over the CTA's warps when it owns
// fewer tiles than warps.  The head streams wte through per-warp buffers of one tile each; its rows
// are sent to L2 while the last layer runs, and the next step's first weights at the end.
//
// Attention: with at least two CTAs per (sequence, head) unit, cpu CTAs share a unit (each an equal
// share of the keys, split again over its 8 warps; c_proj's staging merges their partials);
// otherwise (larger batches) each unit's keys are split over single warps
// anywhere in the grid, merged by the unit's last warp.  A warp copies up to
// 32 key and value rows with cp.async, lane t scores key t, and lane l accumulates output
// dimensions 2l, 2l + 1 (online softmax across chunks).  The cache rows are prefetched into L2 a
// phase ahead.  Data written during the step (residual, q, the cache, y, h) is read through L2
// (ld.cg), never through the per-SM L1.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gpt {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRows = 16;     // sequences per launch (the mma's M)
constexpr int kTile = 8;         // weight rows per tile (the mma's N)
constexpr int kPad = 8;          // bf16 elements of padding per staged row
constexpr int kChunk = 32;       // keys per attention chunk: a lane per key
constexpr int kMaxCtaSplit = 4;  // CTAs sharing one (sequence, head): 4 measured best at B 1 (of 1, 4, 6, 8, 12)
constexpr int kMaxHs = 64;       // head size (every GPT-2 size has 64)
constexpr int kMaxC = 1024;      // a LayerNorm row lives in registers: C / 128 float4 per lane
constexpr int kResidCols = 32;   // residual columns one CTA may own
constexpr int kMaxHeadBufs = 2;  // head buffers per warp
constexpr int kSmemLimit = 232448;

// attention staging per warp: kChunk key rows (padded), kChunk value rows, the query
constexpr int kKld = kMaxHs + 8;
constexpr int kAttnWarpBytes = kChunk * kKld * 2 + kChunk * kMaxHs * 2 + kMaxHs * 2;
constexpr int kAttnStageBytes = kWarps * kAttnWarpBytes;

// dynamic shared memory: [barriers][reduce / attention partials][residual addend][staged rows][weights];
// while attention runs, the staged-row region holds its staging instead
constexpr int kBarBytes = 256;                                  // 4 slot + 16 head barriers, abort flag
constexpr int kRedBytes = 4352;                                 // >= max(8 x 16 x 8, 8 x (2 + kMaxHs)) floats
constexpr int kXsBytes = kMaxRows * kResidCols * 4;
constexpr int kFixedBytes = kBarBytes + kRedBytes + kXsBytes;   // staged rows start here

struct StepArgs {
    const bf16* wte;
    const bf16* wpe;
    const uint8_t* layer0;       // layer 0's tensors; layer l at layer0 + l * layer_bytes
    long long layer_bytes;
    long long off[12];           // byte offsets of the 12 tensors inside a layer (packed order)
    int has_bias;
    const bf16* lnf_w;
    const bf16* lnf_b;
    const int64_t* tok;
    long long ld_tok;
    bf16* kv;                    // cache; layer l at kv + l * kv_layer, [B, block_size, 2C]
    long long kv_layer;          // elements
    float* logits;
    long long ldl;
    int* pos;
    float* x;                    // [B, C] fp32 residual
    bf16* q;                     // [B, C]
    bf16* y;                     // [B, C]
    bf16* h;                     // [B, 4C]
    float* part;                 // per (sequence, head): n_split_max attention partials of hs + 2 floats
    int* counter;                // per (sequence, head): partials written, zero between steps
    int n_split_max;
    unsigned* bar;               // grid barrier counter, zero at launch
    int32_t* status;
    int B, C, nh, hs, V, L, block_size, gelu_tanh;
    float scale_log2;
    int S;                       // weight slots (4, 2 or 1)
    int slot_off[4];             // byte offsets of the slots in dynamic shared memory
    int head_nb;                 // head buffers per warp
    int head_off;                // byte offset of the head buffers
};

enum { T_LN1W = 0, T_LN1B, T_ATTNW, T_ATTNB, T_PROJW, T_PROJB, T_LN2W, T_LN2B, T_FCW, T_FCB, T_FC2W, T_FC2B };
enum { P_QKV = 0, P_PROJ = 1, P_FC = 2, P_FC2 = 3 };

GPT_DEVINL const bf16* tensor(const StepArgs& a, int l, int which) {
    return reinterpret_cast<const bf16*>(a.layer0 + a.layer_bytes * l + a.off[which]);
}

// Shape of weight phase x of a layer: W [N, K] and its bias (nullptr without biases).
GPT_DEVINL void phase_shape(const StepArgs& a, int x, int l, int& N, int& K, const bf16*& W, const bf16*& bias) {
    const int C = a.C;
    const int w = x == P_QKV ? T_ATTNW : x == P_PROJ ? T_PROJW : x == P_FC ? T_FCW : T_FC2W;
    N = x == P_QKV ? 3 * C : x == P_FC ? 4 * C : C;
    K = x == P_FC2 ? 4 * C : C;
    W = tensor(a, l, w);
    bias = a.has_bias ? tensor(a, l, w + 1) : nullptr;
}

// This CTA's tiles [t0, t1) of a product with N columns.
GPT_DEVINL void cta_tiles(int N, int& t0, int& t1) {
    const int tiles = N / kTile;
    t0 = static_cast<int>(static_cast<long long>(blockIdx.x) * tiles / gridDim.x);
    t1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * tiles / gridDim.x);
}

GPT_DEVINL float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
GPT_DEVINL float bf(bf16 v) { return __bfloat162float(v); }
GPT_DEVINL void unpack8(const uint4& w, float (&f)[8]) {
    const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __low2float(hh[i]);
        f[2 * i + 1] = __high2float(hh[i]);
    }
}
GPT_DEVINL void unpack4(const uint2& w, float (&f)[4]) {
    const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&w);
    f[0] = __low2float(hh[0]), f[1] = __high2float(hh[0]);
    f[2] = __low2float(hh[1]), f[3] = __high2float(hh[1]);
}
GPT_DEVINL float gelu_erf(float v) { return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f)); }
GPT_DEVINL float gelu_tanh(float v) { return 0.5f * v * (1.0f + tanhf(0.79788456080286536f * (v + 0.044715f * v * v * v))); }

GPT_DEVINL void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct Ctx {
    const StepArgs& a;
    uint8_t* smem;
    uint64_t* slot_bar;    // [4]
    uint64_t* head_bar;    // [kWarps * kMaxHeadBufs]
    volatile int* abort;
    unsigned target;       // arrivals the next barrier waits for
    int issued;            // weight phases issued so far (phase j = 4 layer + x)
    int consumed;          // weight phases that have landed and been waited for
};

GPT_DEVINL int slot_of(const StepArgs& a, int j) { return a.S == 4 ? (j & 3) : j % a.S; }

// Bytes at the start of a slot that hold the LayerNorm weight (and bias) applied before the product
// of phase x: ln_1 before c_attn, ln_2 before c_fc; none before the two c_proj.
GPT_DEVINL int ln_bytes(const StepArgs& a, int x) {
    return (x == P_QKV || x == P_FC) ? a.C * 2 * (a.has_bias ? 2 : 1) : 0;
}

GPT_DEVINL void cp_async16(void* dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
// Waits for every cp.async this thread has issued.
GPT_DEVINL void cp_async_wait_all() { asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory"); }

// Bulk copies of this CTA's rows (and bias, and the LayerNorm weights) of weight phase j into its
// slot, one copy per thread (thread i: row i), so that their issue runs in parallel.
GPT_DEVINL void issue_phase(Ctx& c, int j) {
    const StepArgs& a = c.a;
    if (j >= 4 * a.L) return;
    int N, K, t0, t1;
    const bf16 *W, *bias;
    phase_shape(a, j & 3, j >> 2, N, K, W, bias);
    cta_tiles(N, t0, t1);
    const int nrows = (t1 - t0) * kTile;
    const int si = slot_of(a, j), x = j & 3, lnb = ln_bytes(a, x);
    const int n_ln = lnb ? (a.has_bias ? 2 : 1) : 0;
    const int n_copies = n_ln + nrows + (bias && nrows ? 1 : 0);
    const int i = threadIdx.x;
    uint8_t* dst = c.smem + a.slot_off[si];
    const uint32_t row_bytes = static_cast<uint32_t>(K) * 2, ld_bytes = static_cast<uint32_t>(K + kPad) * 2;
    if (i == 0) mbar_arrive_expect_tx(c.slot_bar + si, lnb + nrows * row_bytes + (bias ? nrows * 2 : 0));
    if (i >= n_copies) return;
    fence_proxy_async_shared();  // this CTA's earlier reads of the slot (ordered by a CTA barrier)
    if (i < n_ln) {
        bulk_load_1d(dst + i * a.C * 2, tensor(a, j >> 2, (x == P_QKV ? T_LN1W : T_LN2W) + i), a.C * 2, c.slot_bar + si);
    } else if (i < n_ln + nrows) {
        const int r = i - n_ln;
        bulk_load_1d(dst + lnb + static_cast<size_t>(r) * ld_bytes, W + static_cast<long long>(t0 * kTile + r) * K,
                     row_bytes, c.slot_bar + si);
    } else {
        bulk_load_1d(dst + lnb + static_cast<size_t>(nrows) * ld_bytes, bias + t0 * kTile, nrows * 2, c.slot_bar + si);
    }
}

// Waits until weight phase j has landed; the result is the same for every thread of the CTA.
GPT_DEVINL bool wait_phase(Ctx& c, int j) {
    if (mbar_wait(c.slot_bar + slot_of(c.a, j), (j / c.a.S) & 1, c.abort)) c.consumed = j + 1;
    __syncthreads();
    return *c.abort == 0;
}

// On the way out: lets every weight copy this CTA has in flight land before it exits.
GPT_DEVINL void drain_slots(Ctx& c) {
    for (int j = c.consumed; j < c.issued; ++j) mbar_drain(c.slot_bar + slot_of(c.a, j), (j / c.a.S) & 1);
}

// After weight phase j's product (and a CTA barrier): its slot takes phase j + S.
GPT_DEVINL void refill(Ctx& c, int j) {
    if (j + c.a.S < 4 * c.a.L) {
        issue_phase(c, j + c.a.S);
        c.issued = j + c.a.S + 1;
    }
}

// The LayerNorm weights (at the start) and the weight rows of phase j's slot.
GPT_DEVINL const bf16* slot_ln(const Ctx& c, int j) {
    return reinterpret_cast<const bf16*>(c.smem + c.a.slot_off[slot_of(c.a, j)]);
}
GPT_DEVINL const bf16* slot_ptr(const Ctx& c, int j) {
    return reinterpret_cast<const bf16*>(c.smem + c.a.slot_off[slot_of(c.a, j)] + ln_bytes(c.a, j & 3));
}

// Warp-wide: the bulk copies of the 8 wte rows of head tile `tile` into buffer bi of this warp.
GPT_DEVINL void issue_head_tile(const StepArgs& a, int tile, uint8_t* buf, uint64_t* bar) {
    const int lane = threadIdx.x & 31, ldh = a.C + kPad;
    fence_proxy_async_shared();
    if (lane == 0) mbar_arrive_expect_tx(bar, kTile * a.C * 2);
    __syncwarp();
    if (lane < kTile)
        bulk_load_1d(buf + static_cast<size_t>(lane) * ldh * 2, a.wte + static_cast<long long>(tile * kTile + lane) * a.C,
                     a.C * 2, bar);
}

// Grid barrier, split so that work which the other CTAs do not wait for (the next weights' copies,
// the next cache prefetch) runs between this CTA's arrival and its wait.  Arrival: every thread of
// the CTA is done with the phase, then one release of the count.
GPT_DEVINL void grid_arrive(Ctx& c) {
    __syncthreads();
    c.target += gridDim.x;
    if (threadIdx.x == 0)  // release: this CTA's writes of the phase (ordered by the barrier above) first
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(c.a.bar) : "memory");
}

// The wait, bounded.  Returns false (every thread) once any wait has given up.
GPT_DEVINL bool grid_wait(Ctx& c) {
    if (threadIdx.x == 0) {
        const uint64_t t0 = globaltimer_ns();
        const uint64_t limit = g_wait_limit_ns;
        // the testing aid: a forced time-out waits for one arrival more than there will be
        const unsigned target = c.target + (g_force_timeout ? 1u : 0u);
        for (uint32_t it = 1;; ++it) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c.a.bar) : "memory");
            if (v >= target) break;
            if ((it & 15u) == 0u && globaltimer_ns() - t0 > limit) {  // the clock read every 16 polls
                *c.abort = 1;
                set_status(c.a.status, GPT_ERR_TIMEOUT);
                break;
            }
        }
    }
    __syncthreads();  // the acquiring load above, before every thread's reads of the next phase
    return *c.abort == 0;
}

GPT_DEVINL bool grid_sync(Ctx& c) {
    grid_arrive(c);
    return grid_wait(c);
}

// LayerNorm of the B input rows into bf16 rows of shared memory (row stride ldu): the fp32
// residual rows, or (embed, layer 0) wte[tok_b] + wpe[p], which CTA 0 also stores as the residual.
// A warp per row, the row held in registers (one read), lane l owning elements 4l + 128 i.  w, b:
// the LayerNorm weight and bias (b may be nullptr), in shared or global memory.
GPT_DEVINL void stage_ln(const StepArgs& a, const bf16* w, const bf16* b, bool embed, int p, bf16* us, int ldu) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = a.C, nv = C / 128;
#pragma unroll 1
    for (int r = warp; r < a.B; r += kWarps) {
        float4 xv[kMaxC / 128];
        uint2 wv[kMaxC / 128], bv[kMaxC / 128];
#pragma unroll
        for (int i = 0; i < kMaxC / 128; ++i)
            if (i < nv) {
                wv[i] = *reinterpret_cast<const uint2*>(w + lane * 4 + 128 * i);
                bv[i] = b ? *reinterpret_cast<const uint2*>(b + lane * 4 + 128 * i) : make_uint2(0u, 0u);
            }
        if (embed) {
            long long t = __ldcg(a.tok + r * a.ld_tok);
            if (t < 0 || t >= a.V) {
                if (blockIdx.x == 0 && lane == 0) set_status(a.status, GPT_ERR_INDEX);
                t = 0;
            }
            const bf16* er = a.wte + t * C;
            const bf16* pr = a.wpe + static_cast<long long>(p < 0 ? 0 : p) * C;
#pragma unroll
            for (int i = 0; i < kMaxC / 128; ++i)
                if (i < nv) {
                    float e4[4], p4[4];
                    unpack4(__ldg(reinterpret_cast<const uint2*>(er + lane * 4 + 128 * i)), e4);
                    unpack4(__ldg(reinterpret_cast<const uint2*>(pr + lane * 4 + 128 * i)), p4);
                    xv[i] = make_float4(e4[0] + p4[0], e4[1] + p4[1], e4[2] + p4[2], e4[3] + p4[3]);
                    if (blockIdx.x == 0)
                        *reinterpret_cast<float4*>(a.x + static_cast<long long>(r) * C + lane * 4 + 128 * i) = xv[i];
                }
        } else {
            const float* xr = a.x + static_cast<long long>(r) * C;
#pragma unroll
            for (int i = 0; i < kMaxC / 128; ++i)
                if (i < nv) xv[i] = __ldcg(reinterpret_cast<const float4*>(xr + lane * 4 + 128 * i));
        }
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxC / 128; ++i)
            if (i < nv) s += (xv[i].x + xv[i].y) + (xv[i].z + xv[i].w);
        const float mean = warp_sum(s) / C;
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxC / 128; ++i)
            if (i < nv) {
                const float d0 = xv[i].x - mean, d1 = xv[i].y - mean, d2 = xv[i].z - mean, d3 = xv[i].w - mean;
                ss += (d0 * d0 + d1 * d1) + (d2 * d2 + d3 * d3);
            }
        const float rstd = rsqrtf(warp_sum(ss) / C + 1e-5f);
#pragma unroll
        for (int i = 0; i < kMaxC / 128; ++i)
            if (i < nv) {
                float w4[4], b4[4];
                unpack4(wv[i], w4);
                unpack4(bv[i], b4);
                const __nv_bfloat162 lo = __floats2bfloat162_rn((xv[i].x - mean) * rstd * w4[0] + b4[0],
                                                                (xv[i].y - mean) * rstd * w4[1] + b4[1]);
                const __nv_bfloat162 hi = __floats2bfloat162_rn((xv[i].z - mean) * rstd * w4[2] + b4[2],
                                                                (xv[i].w - mean) * rstd * w4[3] + b4[3]);
                uint2 pk;
                pk.x = *reinterpret_cast<const uint32_t*>(&lo);
                pk.y = *reinterpret_cast<const uint32_t*>(&hi);
                *reinterpret_cast<uint2*>(us + r * ldu + lane * 4 + 128 * i) = pk;
            }
    }
}

// Copies B bf16 rows [B][K] written by an earlier phase into shared memory (row stride ldu).
GPT_DEVINL void stage_rows(const bf16* src, int B, int K, bf16* us, int ldu) {
    const int per = K / 8;
    for (int i = threadIdx.x; i < B * per; i += kThreads) {
        const int r = i / per, k = (i % per) * 8;
        *reinterpret_cast<uint4*>(us + r * ldu + k) = __ldcg(reinterpret_cast<const uint4*>(src) + i);
    }
}

// The residual entries x[b, n0 + j] (j < ncols) of this CTA's columns, for the epilogue x += v.
GPT_DEVINL void stage_resid(const StepArgs& a, int n0, int ncols, float* xs) {
    for (int i = threadIdx.x; i < a.B * ncols; i += kThreads) {
        const int b = i / ncols, j = i % ncols;
        xs[b * kResidCols + j] = __ldcg(a.x + static_cast<long long>(b) * a.C + n0 + j);
    }
}

enum { OUT_QKV = 0, OUT_RESID = 1, OUT_GELU = 2 };

GPT_DEVINL void store_out(const StepArgs& a, int OUT, int r, int n, int n0, float v, int layer, int p, const float* xs) {
    const int C = a.C;
    if (OUT == OUT_QKV) {
        if (n < C) {
            a.q[r * C + n] = __float2bfloat16_rn(v);
        } else if (p >= 0) {
            bf16* kvl = a.kv + a.kv_layer * layer;
            kvl[(static_cast<long long>(r) * a.block_size + p) * 2 * C + (n - C)] = __float2bfloat16_rn(v);
        }
    } else if (OUT == OUT_RESID) {
        a.x[static_cast<long long>(r) * C + n] = xs[r * kResidCols + (n - n0)] + v;
    } else {
        a.h[static_cast<long long>(r) * 4 * C + n] = __float2bfloat16_rn(a.gelu_tanh ? gelu_tanh(v) : gelu_erf(v));
    }
}

// acc = the m16n8 fragment (rows g and g + 8 = sequences, columns 2q, 2q + 1 = weight rows) of the
// staged rows us (stride ldu) against 8 weight rows wt (stride ldw) over k in [k0, k1), steps of 16
// alternating between two accumulators.  Rows 8..15 of us are read only when two (B > 8).
GPT_DEVINL void tile_dot(const bf16* us, int ldu, const bf16* wt, int ldw, int k0, int k1, bool two, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const uint32_t* a0p = reinterpret_cast<const uint32_t*>(us + g * ldu) + q;
    const uint32_t* a1p = reinterpret_cast<const uint32_t*>(us + (g + 8) * ldu) + q;
    const uint32_t* bp = reinterpret_cast<const uint32_t*>(wt + g * ldw) + q;
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
    for (int k = k0; k < k1; k += 32) {
        const int w0 = k >> 1;
        mma_16816(c0, a0p[w0], two ? a1p[w0] : 0u, a0p[w0 + 4], two ? a1p[w0 + 4] : 0u, bp[w0], bp[w0 + 4]);
        if (k + 16 < k1) {
            const int w1 = w0 + 8;
            mma_16816(c1, a0p[w1], two ? a1p[w1] : 0u, a0p[w1 + 4], two ? a1p[w1 + 4] : 0u, bp[w1], bp[w1 + 4]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = c0[i] + c1[i];
}

// out[:, n] (+ bias) for this CTA's tiles [t0, t1) of W, held in shared memory at wsm (rows of
// stride K + kPad, then the bias), against the staged rows.  K % 16 == 0.
GPT_DEVINL void product(const StepArgs& a, int out, const bf16* us, int ldu, const bf16* wsm, int K, int t0, int t1, int layer,
                        int p, float* red, const float* xs) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int B = a.B, nt = t1 - t0, ldw = K + kPad;
    if (nt <= 0) return;
    const bool two = B > 8;
    const int n0 = t0 * kTile;
    const bf16* bias = a.has_bias ? wsm + static_cast<size_t>(nt) * kTile * ldw : nullptr;
    if (nt >= kWarps) {
        // a warp per tile, the whole of K
        for (int tl = warp; tl < nt; tl += kWarps) {
            float acc[4];
            tile_dot(us, ldu, wsm + static_cast<size_t>(tl) * kTile * ldw, ldw, 0, K, two, acc);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = g + 8 * (i >> 1), nl = tl * kTile + 2 * q + (i & 1);
                if (r < B) store_out(a, out, r, n0 + nl, n0, acc[i] + (bias ? bf(bias[nl]) : 0.f), layer, p, xs);
            }
        }
        return;
    }
    // fewer tiles than warps: each tile's K split into `slices` pieces, summed through shared memory
    const int steps = K / 16;
    const int slices = min(kWarps / nt, steps);
    if (warp < nt * slices) {
        const int tl = warp % nt, sl = warp / nt;
        float acc[4];
        tile_dot(us, ldu, wsm + static_cast<size_t>(tl) * kTile * ldw, ldw, (sl * steps / slices) * 16,
                 ((sl + 1) * steps / slices) * 16, two, acc);
#pragma unroll
        for (int i = 0; i < 4; ++i) red[(warp * kMaxRows + g + 8 * (i >> 1)) * kTile + 2 * q + (i & 1)] = acc[i];
    }
    __syncthreads();
    for (int t = threadIdx.x; t < nt * kTile * B; t += kThreads) {
        const int nl = t % (nt * kTile), r = t / (nt * kTile);
        const int tl = nl / kTile, cl = nl % kTile;
        float v = bias ? bf(bias[nl]) : 0.f;
        for (int sl = 0; sl < slices; ++sl) v += red[((sl * nt + tl) * kMaxRows + r) * kTile + cl];
        store_out(a, out, r, n0 + nl, n0, v, layer, p, xs);
    }
}

// Attention work split.  With at least two CTAs per (sequence, head) unit, cpu CTAs share a unit
// (CTA b: unit b / cpu, an equal share b % cpu of the keys, split again over its 8 warps) and the
// last of them to finish merges their partials through global memory.  Otherwise a unit gets wpu =
// 8, 4, 2 or 1 warps of one CTA, which take 64-key chunks in turn.
GPT_DEVINL int attention_cpu(const StepArgs& a) {
    const int cpu = static_cast<int>(gridDim.x) / (a.B * a.nh);
    return cpu >= 2 ? min(min(cpu, a.n_split_max), kMaxCtaSplit) : 1;
}
GPT_DEVINL int attention_wpu(const StepArgs& a) {
    if (attention_cpu(a) > 1) return kWarps;
    const int per = gridDim.x * kWarps / (a.B * a.nh);
    return per >= 8 ? 8 : per >= 4 ? 4 : per >= 2 ? 2 : 1;
}

// Warp-level split (used when attention_cpu is 1): every (sequence, head) unit is cut into `parts`
// equal key ranges (parts <= 16, each at least one 32-key chunk, as many as the grid's warps
// allow), and global warp
// g takes items g, g + W, ... (item = unit * parts + part).  Each warp leaves its partial (m, l, O)
// in global memory; the last warp of a unit to finish (a per-unit ticket) merges them.
GPT_DEVINL int attention_parts(const StepArgs& a, int n_keys) {
    const int per = static_cast<int>(gridDim.x) * kWarps / (a.B * a.nh);
    const int by_keys = (n_keys + kChunk - 1) / kChunk;
    return max(1, min(min(per, by_keys), min(a.n_split_max, 16)));
}

// L2 prefetch of [p, p + bytes) by the calling warp, in pieces of at most 32 KB spread over its
// lanes.  p and bytes are multiples of 16.
GPT_DEVINL void prefetch_span(const void* p, size_t bytes) {
    constexpr size_t kPiece = 32768;
    const int lane = threadIdx.x & 31;
    for (size_t o = static_cast<size_t>(lane) * kPiece; o < bytes; o += 32 * kPiece) {
        const uint32_t n = static_cast<uint32_t>(bytes - o < kPiece ? bytes - o : kPiece);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(static_cast<const uint8_t*>(p) + o), "r"(n)
                     : "memory");
    }
}

// L2 prefetch (warp-wide) of this CTA's rows, bias and LayerNorm weights of weight phase j, the
// data issue_phase copies for it.
GPT_DEVINL void prefetch_phase(const StepArgs& a, int j) {
    int N, K, t0, t1;
    const bf16 *W, *bias;
    phase_shape(a, j & 3, j >> 2, N, K, W, bias);
    cta_tiles(N, t0, t1);
    prefetch_span(W + static_cast<long long>(t0) * kTile * K, static_cast<size_t>(t1 - t0) * kTile * K * 2);
    if (bias && t1 > t0 && (threadIdx.x & 31) == 0)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(bias + t0 * kTile), "r"((t1 - t0) * kTile * 2)
                     : "memory");
    if (ln_bytes(a, j & 3) && (threadIdx.x & 31) == 1)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(tensor(a, j >> 2, (j & 3) == P_QKV ? T_LN1W : T_LN2W)),
                     "r"(a.C * 2)
                     : "memory");
}

// L2 prefetch of layer `layer`'s cached key and value rows [0, p) of every (sequence, head), spread
// over every thread of the grid: one prefetch per row slice of hs * 2 <= 128 bytes (two when the
// slice straddles a 128-byte line).
GPT_DEVINL void prefetch_kv(const StepArgs& a, int layer, int p) {
    if (p <= 0) return;
    const int n_keys = min(p, a.block_size);
    const int total = a.B * a.nh * n_keys * 2;  // < 2^31: B <= 16, block_size and nh small
    const bf16* kvl = a.kv + a.kv_layer * layer;
    for (int i = blockIdx.x * kThreads + threadIdx.x; i < total; i += gridDim.x * kThreads) {
        const int sel = i & 1, r = i >> 1;
        const int key = r % n_keys, bh = r / n_keys;
        const uint8_t* pt = reinterpret_cast<const uint8_t*>(
            kvl + (static_cast<long long>(bh / a.nh) * a.block_size + key) * 2 * a.C + sel * a.C + (bh % a.nh) * a.hs);
        asm volatile("prefetch.global.L2 [%0];" ::"l"(pt));
        if ((reinterpret_cast<uintptr_t>(pt) & 127) + a.hs * 2 > 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(pt + a.hs * 2 - 1));
    }
}

// Attention when there are at least as many (sequence, head) units as CTAs (larger batches): the
// units' key ranges are split over single warps (attention_parts).  A warp
// copies up to 32 key and value rows of its range (lane t: key k0 + t) and the query into its
// staging area with cp.async, lane t scores key t, the warp takes the chunk's max and sum, and lane
// l accumulates output dimensions 2l, 2l + 1 (online softmax across chunks).
GPT_DEVINL void attention_warps(const StepArgs& a, int layer, int p, uint8_t* stage) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = a.C, hs = a.hs, nh = a.nh, nv16 = hs / 8;
    const int n_keys = min(p + 1, a.block_size);
    const int parts = attention_parts(a, n_keys), units = a.B * nh, items = units * parts;
    const bf16* kvl = a.kv + a.kv_layer * layer;
    bf16* ks = reinterpret_cast<bf16*>(stage + warp * kAttnWarpBytes);
    bf16* vs = ks + kChunk * kKld;
    bf16* qs = vs + kChunk * kMaxHs;
    const int d = 2 * lane;  // this lane's output dimensions d, d + 1 (hs <= 64)
    for (int it = blockIdx.x * kWarps + warp; it < items; it += gridDim.x * kWarps) {
        const int u = it / parts, sh = it % parts;
        const int b = u / nh, h = u % nh;
        const int kb = sh * n_keys / parts, ke = (sh + 1) * n_keys / parts;
        const bf16* base = kvl + static_cast<long long>(b) * a.block_size * 2 * C + h * hs;
        if (lane < nv16) cp_async16(qs + 8 * lane, a.q + static_cast<long long>(b) * C + h * hs + 8 * lane, 16);
        float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll 1
        for (int k0 = kb; k0 < ke; k0 += kChunk) {
            const int nk = min(kChunk, ke - k0);
            const bool in = lane < nk;
            const bf16* kr = base + static_cast<long long>(k0 + (in ? lane : 0)) * 2 * C;
#pragma unroll 1
            for (int i = 0; i < nv16; ++i) {
                cp_async16(ks + lane * kKld + 8 * i, kr + 8 * i, in ? 16 : 0);
                cp_async16(vs + lane * kMaxHs + 8 * i, kr + C + 8 * i, in ? 16 : 0);
            }
            cp_async_wait_all();
            __syncwarp();
            float sc = 0.f;
#pragma unroll 1
            for (int i = 0; i < nv16; ++i) {
                float kf[8], qf[8];
                unpack8(*reinterpret_cast<const uint4*>(ks + lane * kKld + 8 * i), kf);
                unpack8(*reinterpret_cast<const uint4*>(qs + 8 * i), qf);
#pragma unroll
                for (int e = 0; e < 8; ++e) sc = fmaf(qf[e], kf[e], sc);
            }
            sc = in ? sc * a.scale_log2 : -INFINITY;
            float mc = sc;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
            const float mn = fmaxf(m, mc);    // finite: every chunk has a key (nk >= 1)
            const float corr = exp2f(m - mn);  // 0 on the warp's first chunk (m = -inf)
            const float pl = in ? exp2f(sc - mn) : 0.f;
            l = l * corr + warp_sum(pl);
            o0 *= corr;
            o1 *= corr;
            m = mn;
            // lanes with 2 lane >= hs accumulate what lies past the copied dimensions and store nothing
#pragma unroll 2
            for (int t = 0; t < nk; ++t) {
                const float pt = __shfl_sync(0xffffffffu, pl, t);
                const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(vs + t * kMaxHs + 2 * lane);
                o0 = fmaf(pt, __low2float(v2), o0);
                o1 = fmaf(pt, __high2float(v2), o1);
            }
            __syncwarp();  // the next chunk's copies overwrite the staging area
        }
        cp_async_wait_all();  // the query copy of a range without keys
        __syncwarp();
        bf16* yr = a.y + static_cast<long long>(b) * C + h * hs;
        if (parts == 1) {
            if (d < hs) *reinterpret_cast<__nv_bfloat162*>(yr + d) = __floats2bfloat162_rn(o0 / l, o1 / l);
            continue;
        }
        // this warp's partial; the unit's last warp merges them:
        // y = sum_i 2^(m_i - M) O_i / sum_i 2^(m_i - M) l_i
        float* gp = a.part + (static_cast<long long>(u) * a.n_split_max + sh) * (hs + 2);
        if (d < hs) __stcg(gp + 2 + d, o0), __stcg(gp + 3 + d, o1);
        if (lane == 0) __stcg(gp, m), __stcg(gp + 1, l);
        __threadfence();
        __syncwarp();
        int ticket = 0;
        if (lane == 0) ticket = atomicAdd(a.counter + u, 1);
        ticket = __shfl_sync(0xffffffffu, ticket, 0);
        if (ticket != parts - 1) continue;
        __threadfence();
        const float* g0 = a.part + static_cast<long long>(u) * a.n_split_max * (hs + 2);
        const float mine = lane < parts ? __ldcg(g0 + lane * (hs + 2)) : -INFINITY;  // parts <= 16
        float M = mine;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f, z0 = 0.f, z1 = 0.f;
#pragma unroll 4
        for (int i = 0; i < parts; ++i) {
            const float mi = __shfl_sync(0xffffffffu, mine, i);
            const float* gi = g0 + i * (hs + 2);
            const float wgt = mi == -INFINITY ? 0.f : exp2f(mi - M);  // a range without keys: 0
            L = fmaf(wgt, __ldcg(gi + 1), L);
            if (d < hs) z0 = fmaf(wgt, __ldcg(gi + 2 + d), z0), z1 = fmaf(wgt, __ldcg(gi + 3 + d), z1);
        }
        if (d < hs) *reinterpret_cast<__nv_bfloat162*>(yr + d) = __floats2bfloat162_rn(z0 / L, z1 / L);
        if (lane == 0) a.counter[u] = 0;
    }
}

// Attention of the newest position over the cache [0, p] for every (sequence, head).  Per chunk of
// up to 32 keys a warp copies the key and value rows (lane t: key k0 + t) and the query into its
// staging area with cp.async, lane t scores key t, the warp takes the chunk's max and sum, and lane
// l accumulates output dimensions 2l, 2l + 1 over the chunk's keys (online softmax across chunks).
// The loops stay rolled: the code is short and is fetched once per layer.
GPT_DEVINL void attention(const StepArgs& a, int layer, int p, float* part, uint8_t* stage) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = a.C, hs = a.hs, nh = a.nh, nv16 = hs / 8;
    const int n_keys = min(p + 1, a.block_size);
    const int cpu = attention_cpu(a), wpu = attention_wpu(a), upc = kWarps / wpu, units = a.B * nh;
    const int wi = warp % wpu;
    const bf16* kvl = a.kv + a.kv_layer * layer;
    float* mine = part + warp * (2 + kMaxHs);
    bf16* ks = reinterpret_cast<bf16*>(stage + warp * kAttnWarpBytes);
    bf16* vs = ks + kChunk * kKld;
    bf16* qs = vs + kChunk * kMaxHs;
    // this warp's keys: [kfirst, kend) in chunks of kChunk, kstride apart
    int kfirst = wi * kChunk, kend = n_keys, kstride = wpu * kChunk;
    if (cpu > 1) {
        const int sh = blockIdx.x % cpu, kb = sh * n_keys / cpu, nkp = (sh + 1) * n_keys / cpu - kb;
        kfirst = kb + warp * nkp / kWarps;
        kend = kb + (warp + 1) * nkp / kWarps;
        kstride = kChunk;
    }
    const int u_first = cpu > 1 ? static_cast<int>(blockIdx.x) / cpu * upc : blockIdx.x * upc;
    const int u_step = cpu > 1 ? units * upc : gridDim.x * upc;  // one round when cpu > 1
    for (int u0 = u_first; u0 < units; u0 += u_step) {
        const int u = u0 + warp / wpu;
        if (u < units) {
            const int b = u / nh, h = u % nh;
            const bf16* base = kvl + static_cast<long long>(b) * a.block_size * 2 * C + h * hs;
            if (lane < nv16) cp_async16(qs + 8 * lane, a.q + static_cast<long long>(b) * C + h * hs + 8 * lane, 16);
            float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll 1
            for (int k0 = kfirst; k0 < kend; k0 += kstride) {
                const int nk = min(kChunk, kend - k0);
                const bool in = lane < nk;
                const bf16* kr = base + static_cast<long long>(k0 + (in ? lane : 0)) * 2 * C;
#pragma unroll 1
                for (int i = 0; i < nv16; ++i) {
                    cp_async16(ks + lane * kKld + 8 * i, kr + 8 * i, in ? 16 : 0);
                    cp_async16(vs + lane * kMaxHs + 8 * i, kr + C + 8 * i, in ? 16 : 0);
                }
                cp_async_wait_all();
                __syncwarp();
                float sc = 0.f;
#pragma unroll 1
                for (int i = 0; i < nv16; ++i) {
                    float kf[8], qf[8];
                    unpack8(*reinterpret_cast<const uint4*>(ks + lane * kKld + 8 * i), kf);
                    unpack8(*reinterpret_cast<const uint4*>(qs + 8 * i), qf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) sc = fmaf(qf[e], kf[e], sc);
                }
                sc = in ? sc * a.scale_log2 : -INFINITY;
                float mc = sc;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
                const float mn = fmaxf(m, mc);    // finite: every chunk has a key (nk >= 1)
                const float corr = exp2f(m - mn);  // 0 on the warp's first chunk (m = -inf)
                const float pl = in ? exp2f(sc - mn) : 0.f;
                l = l * corr + warp_sum(pl);
                o0 *= corr;
                o1 *= corr;
                m = mn;
                // lanes with 2 lane >= hs accumulate what lies past the copied dimensions and store nothing
#pragma unroll 2
                for (int t = 0; t < nk; ++t) {
                    const float pt = __shfl_sync(0xffffffffu, pl, t);
                    const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(vs + t * kMaxHs + 2 * lane);
                    o0 = fmaf(pt, __low2float(v2), o0);
                    o1 = fmaf(pt, __high2float(v2), o1);
                }
                __syncwarp();  // the next chunk's copies overwrite the staging area
            }
            cp_async_wait_all();  // the query copy of a warp that had no keys
            if (2 * lane < hs) mine[2 + 2 * lane] = o0, mine[3 + 2 * lane] = o1;
            if (lane == 0) mine[0] = m, mine[1] = l;
        }
        __syncthreads();
        // the unit's first warp merges its warps: y = sum_i 2^(m_i - M) O_i / sum_i 2^(m_i - M) l_i;
        // with cpu > 1 the merged (M, L, O) is this CTA's partial, which c_proj's staging merges
        if (u < units && wi == 0) {
            const float* pw = part + warp * (2 + kMaxHs);
            float M = -INFINITY;
            for (int i = 0; i < wpu; ++i) M = fmaxf(M, pw[i * (2 + kMaxHs)]);
            float Ls = 0.f, y0 = 0.f, y1 = 0.f;
            const int d = 2 * lane;  // this lane's two dimensions (hs <= 64)
            for (int i = 0; i < wpu; ++i) {
                const float* pi = pw + i * (2 + kMaxHs);
                const float wgt = pi[0] == -INFINITY ? 0.f : exp2f(pi[0] - M);  // a warp without keys: 0
                Ls = fmaf(wgt, pi[1], Ls);
                if (d < hs) y0 = fmaf(wgt, pi[2 + d], y0), y1 = fmaf(wgt, pi[3 + d], y1);
            }
            bf16* yr = a.y + static_cast<long long>(u / nh) * C + (u % nh) * hs;
            if (cpu == 1) {
                if (d < hs) *reinterpret_cast<__nv_bfloat162*>(yr + d) = __floats2bfloat162_rn(y0 / Ls, y1 / Ls);
            } else {
                // this CTA's partial to global memory, for c_proj's staging (the barrier orders it)
                float* gp = a.part + (static_cast<long long>(u) * a.n_split_max + blockIdx.x % cpu) * (hs + 2);
                if (d < hs) __stcg(gp + 2 + d, y0), __stcg(gp + 3 + d, y1);
                if (lane == 0) __stcg(gp, M), __stcg(gp + 1, Ls);
            }
        }
        __syncthreads();
    }
}

// c_proj's input rows when attention split its (sequence, head) units over cpu > 1 CTAs: y[b, h hs
// + d] = sum_i 2^(m_i - M) O_i[d] / sum_i 2^(m_i - M) l_i over the unit's cpu partials (M the
// largest m_i), rounded to bf16 into the staged rows (stride ldu).
GPT_DEVINL void stage_y_merge(const StepArgs& a, bf16* us, int ldu) {
    const int hs = a.hs, cpu = attention_cpu(a), lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // a warp per (sequence, head) unit: lane l merges dimensions 2l, 2l + 1 over the cpu partials
    for (int u = warp; u < a.B * a.nh; u += kWarps) {
        const float* g0 = a.part + static_cast<long long>(u) * a.n_split_max * (hs + 2);
        const int d = 2 * lane;
        // every load of the unit's (at most kMaxCtaSplit) partials goes out at once
        float mi[kMaxCtaSplit], li[kMaxCtaSplit];
        float2 oi[kMaxCtaSplit];
#pragma unroll
        for (int i = 0; i < kMaxCtaSplit; ++i) {
            const bool in = i < cpu;
            mi[i] = in ? __ldcg(g0 + i * (hs + 2)) : -INFINITY;
            li[i] = in ? __ldcg(g0 + i * (hs + 2) + 1) : 0.f;
            oi[i] = (in && d < hs) ? __ldcg(reinterpret_cast<const float2*>(g0 + i * (hs + 2) + 2 + d)) : make_float2(0.f, 0.f);
        }
        float M = mi[0];
#pragma unroll
        for (int i = 1; i < kMaxCtaSplit; ++i) M = fmaxf(M, mi[i]);
        float L = 0.f, z0 = 0.f, z1 = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxCtaSplit; ++i) {
            const float wgt = mi[i] == -INFINITY ? 0.f : exp2f(mi[i] - M);
            L = fmaf(wgt, li[i], L);
            z0 = fmaf(wgt, oi[i].x, z0);
            z1 = fmaf(wgt, oi[i].y, z1);
        }
        if (d < hs)
            *reinterpret_cast<__nv_bfloat162*>(us + (u / a.nh) * ldu + (u % a.nh) * hs + d) =
                __floats2bfloat162_rn(z0 / L, z1 / L);
    }
}

__global__ void __launch_bounds__(kThreads, 1) decode_step_kernel(const __grid_constant__ StepArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + (4 + kWarps * kMaxHeadBufs) * 8);
    float* red = reinterpret_cast<float*>(smem + kBarBytes);
    float* xs = reinterpret_cast<float*>(smem + kBarBytes + kRedBytes);
    bf16* us = reinterpret_cast<bf16*>(smem + kFixedBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 4 + kWarps * kMaxHeadBufs; ++i) mbar_init(bars + i, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    Ctx c{a, smem, bars, bars + 4, abort_flag, 0u, 0, 0};
    const int B = a.B, C = a.C, L = a.L, J = 4 * L;
    const int p_raw = __ldcg(a.pos);
    const int p = (p_raw >= 0 && p_raw < a.block_size) ? p_raw : -1;
    if (p < 0 && blockIdx.x == 0 && threadIdx.x == 0) set_status(a.status, GPT_ERR_BAD_SHAPE);

    // the first S weight phases; after phase j's product its slot takes phase j + S
    for (int j = 0; j < a.S && j < J; ++j) issue_phase(c, j);
    c.issued = min(a.S, J);
    bool ok = true;
    int t0, t1;
    // Every layer: phase x = 0 (c_attn, then attention), 1 (attn c_proj), 2 (c_fc), 3 (mlp c_proj).
    // The four product phases share one copy of the code (a loop over x), which keeps the step's
    // instruction footprint small enough to stay in the SM's instruction caches across layers.
    prefetch_kv(a, 0, p);
#pragma unroll 1
    for (int j = 0; j < J; ++j) {
        const int l = j >> 2, x = j & 3;
        const int N = x == P_QKV ? 3 * C : x == P_FC ? 4 * C : C;
        const int K = x == P_FC2 ? 4 * C : C;
        cta_tiles(N, t0, t1);
        if (x == P_PROJ || x == P_FC2) {
            // x += c_proj(y) or c_proj(h): the input rows, and the residual entries the epilogue adds to
            if (x == P_PROJ && attention_cpu(a) > 1)
                stage_y_merge(a, us, K + kPad);
            else
                stage_rows(x == P_PROJ ? a.y : a.h, B, K, us, K + kPad);
            stage_resid(a, t0 * kTile, (t1 - t0) * kTile, xs);
            if (!(ok = wait_phase(c, j))) break;
        } else {
            // q, k, v = c_attn(ln_1(x)) (layer 0 embeds: x = wte[tok] + wpe[p]); h = gelu(c_fc(ln_2(x)))
            if (!(ok = wait_phase(c, j))) break;
            stage_ln(a, slot_ln(c, j), a.has_bias ? slot_ln(c, j) + C : nullptr, x == P_QKV && l == 0, p, us, K + kPad);
            __syncthreads();
        }
        product(a, x == P_QKV ? OUT_QKV : x == P_FC ? OUT_GELU : OUT_RESID, us, K + kPad, slot_ptr(c, j), K, t0, t1, l,
                p, red, xs);
        if (j + 1 == J) {
            __syncthreads();  // the last product's reads, before the head's copies below
            break;
        }
        // each phase's slot is refilled between the CTA's arrival at the barrier and its wait
        grid_arrive(c);
        refill(c, j);
        if (x == P_FC2) prefetch_kv(a, l + 1, p);
        if (l == L - 1 && x == P_QKV && threadIdx.x >= 32 && threadIdx.x < 64) {
            // warp 1: the head's wte rows of this CTA go to L2 while the last layer runs
            int h0, h1;
            cta_tiles(a.V, h0, h1);
            prefetch_span(a.wte + static_cast<long long>(h0) * kTile * C, static_cast<size_t>(h1 - h0) * kTile * C * 2);
        }
        if (!(ok = grid_wait(c))) break;
        if (x == P_QKV) {
            if (p >= 0) {
                if (attention_cpu(a) > 1)
                    attention(a, l, p, red, smem + kFixedBytes);
                else
                    attention_warps(a, l, p, smem + kFixedBytes);
            }
            if (!(ok = grid_sync(c))) break;
        }
    }
    if (!ok) {
        drain_slots(c);
        return;
    }
    // logits = ln_f(x) wte^T (fp32): warp w streams tiles T0 + w + 8 i of this CTA's range through
    // its head_nb buffers (one tile of 8 wte rows each)
    cta_tiles(a.V, t0, t1);
    const int ldh = C + kPad;
    const size_t tile_bytes = static_cast<size_t>(kTile) * ldh * 2;
    const int nb = a.head_nb;
    uint64_t* hb = c.head_bar + warp * kMaxHeadBufs;
    uint8_t* hbuf = smem + a.head_off + static_cast<size_t>(warp) * nb * tile_bytes;
    const int n_mine = t1 - t0 > warp ? (t1 - t0 - warp + kWarps - 1) / kWarps : 0;
    for (int i = 0; i < nb && i < n_mine; ++i)
        issue_head_tile(a, t0 + warp + kWarps * i, hbuf + (i % nb) * tile_bytes, hb + i % nb);
    int landed = 0;
    ok = grid_sync(c);
    if (ok) {
        stage_ln(a, a.lnf_w, a.lnf_b, false, p, us, ldh);
        __syncthreads();
        const int g = lane >> 2, q = lane & 3;
        for (int i = 0; i < n_mine; ++i) {
            const int bi = i % nb;
            if (!mbar_wait(hb + bi, (i / nb) & 1, abort_flag)) {
                ok = false;
                break;
            }
            landed = i + 1;
            float acc[4];
            tile_dot(us, ldh, reinterpret_cast<const bf16*>(hbuf + bi * tile_bytes), ldh, 0, C, B > 8, acc);
            __syncwarp();
            if (i + nb < n_mine)
                issue_head_tile(a, t0 + warp + kWarps * (i + nb), hbuf + bi * tile_bytes, hb + bi);
            const int n = (t0 + warp + kWarps * i) * kTile + 2 * q;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = g + 8 * (e >> 1);
                if (r < B) a.logits[static_cast<long long>(r) * a.ldl + n + (e & 1)] = acc[e];
            }
        }
    }
    if (!ok) {
        set_status(a.status, GPT_ERR_TIMEOUT);
        // the head copies of this warp still in flight
        const int issued = min(n_mine, landed + nb);
        for (int i = landed; i < issued; ++i) mbar_drain(hb + i % nb, (i / nb) & 1);
        return;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.pos = p_raw + 1;
    // the next step starts with layer 0's first S weight phases: each warp w < S sends its part to L2
    if (warp < a.S && warp < J) prefetch_phase(a, warp);
}

struct SmemPlan {
    int S;
    int slot_off[4];
    int head_nb, head_off;
    size_t bytes;
};

// Shared-memory plan: staged rows (8 or 16 of width 4C + kPad), then four exact weight slots if
// they fit, else two or one slot of the largest phase; the head's buffers follow its staged rows.
bool plan_smem(int B, int C, bool bias, int grid, SmemPlan& sp) {
    const int rows = B <= 8 ? 8 : 16;
    size_t us_bytes = static_cast<size_t>(rows) * (4 * C + kPad) * 2;
    if (us_bytes < static_cast<size_t>(kAttnStageBytes)) us_bytes = kAttnStageBytes;
    size_t bytes[4], mx = 0, sum = 0;
    for (int x = 0; x < 4; ++x) {
        const int N = x == P_QKV ? 3 * C : x == P_FC ? 4 * C : C;
        const int K = x == P_FC2 ? 4 * C : C;
        const size_t maxt = (static_cast<size_t>(N / kTile) + grid - 1) / grid;
        const size_t lnb = (x == P_QKV || x == P_FC) ? static_cast<size_t>(C) * 2 * (bias ? 2 : 1) : 0;
        bytes[x] = lnb + maxt * kTile * (K + kPad) * 2 + (bias ? maxt * kTile * 2 : 0);
        mx = bytes[x] > mx ? bytes[x] : mx;
        sum += bytes[x];
    }
    const size_t base = kFixedBytes + us_bytes;
    for (int x = 0; x < 4; ++x) sp.slot_off[x] = 0;
    if (base + sum <= kSmemLimit) {
        sp.S = 4;
        size_t o = base;
        for (int x = 0; x < 4; ++x) sp.slot_off[x] = static_cast<int>(o), o += bytes[x];
        sp.bytes = o;
    } else if (base + 2 * mx <= kSmemLimit) {
        sp.S = 2;
        sp.slot_off[0] = static_cast<int>(base), sp.slot_off[1] = static_cast<int>(base + mx);
        sp.bytes = base + 2 * mx;
    } else if (base + mx <= kSmemLimit) {
        sp.S = 1;
        sp.slot_off[0] = static_cast<int>(base);
        sp.bytes = base + mx;
    } else {
        return false;
    }
    const size_t head_base = kFixedBytes + static_cast<size_t>(rows) * (C + kPad) * 2;
    const size_t tile_bytes = static_cast<size_t>(kTile) * (C + kPad) * 2;
    size_t nb = (kSmemLimit - head_base) / (kWarps * tile_bytes);
    if (nb < 1) return false;
    if (nb > kMaxHeadBufs) nb = kMaxHeadBufs;
    sp.head_nb = static_cast<int>(nb);
    sp.head_off = static_cast<int>(head_base);
    const size_t head_end = head_base + nb * kWarps * tile_bytes;
    if (head_end > sp.bytes) sp.bytes = head_end;
    return true;
}

}  // namespace

bool decode_persistent_supported(int dtype, int B, int C, int hs, int V, int has_bias) {
    if (dtype != GPT_DTYPE_BF16 || B < 1 || B > kMaxRows || C % 128 != 0 || C > kMaxC || hs % 8 != 0 ||
        hs > kMaxHs || V % kTile != 0)
        return false;
    const int grid = num_sms();
    SmemPlan sp;
    // residual columns per CTA fit the addend buffer; a phase's copies (rows + LayerNorm + bias) fit one per thread
    return grid > 0 && (C / kTile + grid - 1) / grid * kTile <= kResidCols &&
           (4 * C / kTile + grid - 1) / grid * kTile + 3 <= kThreads && plan_smem(B, C, has_bias != 0, grid, sp);
}

int launch_decode_persistent(const void* wte, const void* wpe, const void* layer0, long long layer_bytes,
                             const long long (&off)[12], int has_bias, const void* lnf_w, const void* lnf_b,
                             const int64_t* tok, long long ld_tok, void* kv, long long kv_layer_elems, float* logits,
                             long long ldl, int* pos, float* x, void* q, void* y, void* h, float* part,
                             int* counter, int n_split_max, unsigned* bar, int32_t* status, int B, int C, int nh,
                             int V, int L, int block_size, int gelu_tanh, cudaStream_t s) {
    const int hs = C / nh;
    if (!decode_persistent_supported(GPT_DTYPE_BF16, B, C, hs, V, has_bias)) return GPT_ERR_UNSUPPORTED;
    const int grid = num_sms();
    SmemPlan sp;
    if (!plan_smem(B, C, has_bias != 0, grid, sp)) return GPT_ERR_UNSUPPORTED;
    StepArgs a{};
    a.wte = static_cast<const bf16*>(wte);
    a.wpe = static_cast<const bf16*>(wpe);
    a.layer0 = static_cast<const uint8_t*>(layer0);
    a.layer_bytes = layer_bytes;
    for (int i = 0; i < 12; ++i) a.off[i] = off[i];
    a.has_bias = has_bias;
    a.lnf_w = static_cast<const bf16*>(lnf_w);
    a.lnf_b = static_cast<const bf16*>(lnf_b);
    a.tok = tok;
    a.ld_tok = ld_tok;
    a.kv = static_cast<bf16*>(kv);
    a.kv_layer = kv_layer_elems;
    a.logits = logits;
    a.ldl = ldl;
    a.pos = pos;
    a.x = x;
    a.q = static_cast<bf16*>(q);
    a.y = static_cast<bf16*>(y);
    a.h = static_cast<bf16*>(h);
    a.part = part;
    a.counter = counter;
    a.n_split_max = n_split_max;
    a.bar = bar;
    a.status = status;
    a.B = B, a.C = C, a.nh = nh, a.hs = hs, a.V = V, a.L = L, a.block_size = block_size;
    a.gelu_tanh = gelu_tanh;
    a.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(hs)));
    a.S = sp.S;
    for (int i = 0; i < 4; ++i) a.slot_off[i] = sp.slot_off[i];
    a.head_nb = sp.head_nb;
    a.head_off = sp.head_off;
    static size_t opted[kMaxDevices] = {};
    int rc = opt_in_smem(reinterpret_cast<const void*>(decode_step_kernel), kSmemLimit, opted);
    if (rc) return rc;
    int per_sm = 0;
    rc = cuda_status(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_step_kernel, kThreads, sp.bytes));
    if (rc) return rc;
    if (per_sm < 1) return GPT_ERR_UNSUPPORTED;
    rc = cuda_status(cudaMemsetAsync(bar, 0, sizeof(unsigned), s));
    if (rc) return rc;
    void* params[] = {&a};
    return cuda_status(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(decode_step_kernel), dim3(grid),
                                                   dim3(kThreads), params, sp.bytes, s));
}

// Pipeline-wait limit of this file's kernel on the current device (0: the default).
GPT_DEFINE_WAIT_LIMIT_SETTER(set_wait_limit_decode)

}  // namespace gpt
