// Device helpers shared by the sm_100a kernels: mbarriers with bounded waits, TMA tile
// loads, tcgen05 (TMEM allocation, MMA, commit, loads/stores) and shared-memory matrix
// descriptors.  Inline PTX only; no CUTLASS.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gpt.h"

#define GPT_DEVINL __device__ __forceinline__

namespace gpt {

typedef __nv_bfloat16 bf16;

// A pipeline wait gives up after this long; the kernel then records GPT_ERR_TIMEOUT,
// drains what it has in flight and returns instead of hanging.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

// The limit the pipeline waits (mbar_wait, mbar_wait_cluster) apply on this device: kWaitLimitNs
// unless gpt_set_wait_limit_ns lowered it (to exercise the time-out path).  Internal linkage: each
// translation unit with pipeline waits holds its own copy and defines a setter for it with
// GPT_DEFINE_WAIT_LIMIT_SETTER.  The drains on the way out (mbar_drain) always keep kWaitLimitNs,
// so no kernel leaves a copy or a product in flight because of a lowered limit.
static __device__ uint64_t g_wait_limit_ns = kWaitLimitNs;
// Testing aid (same linkage): when nonzero, the MMA-issuing thread of the attention kernel and of
// the product kernel first waits for an event that never happens, so that the time-out path runs
// on purpose: nothing has arrived on the kernel's drain barrier before its final commit.
static __device__ int g_force_timeout = 0;
#define GPT_DEFINE_WAIT_LIMIT_SETTER(name)                                                       \
    int name(unsigned long long ns, int force) {                                                 \
        const uint64_t v = ns ? static_cast<uint64_t>(ns) : kWaitLimitNs;                       \
        const int f = force ? 1 : 0;                                                             \
        if (cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return GPT_ERR_CUDA; \
        return cudaMemcpyToSymbol(g_force_timeout, &f, sizeof(f)) == cudaSuccess ? GPT_OK : GPT_ERR_CUDA; \
    }

GPT_DEVINL uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

GPT_DEVINL uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier
GPT_DEVINL void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

GPT_DEVINL void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

GPT_DEVINL void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

GPT_DEVINL void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

GPT_DEVINL bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits until the phase with the given parity has completed.  Returns false (and raises
// the CTA's abort flag) when the time limit passes, or when another thread already raised
// it.  Every wait in every kernel of this library goes through here.
GPT_DEVINL bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    const uint32_t a = smem_addr(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = g_wait_limit_ns;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(a, parity)) return true;
        if ((it & 63u) == 0u) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// As mbar_wait, acquiring at cluster scope (the phase's arrivals include other CTAs' threads).
GPT_DEVINL bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    const uint32_t a = smem_addr(bar);
    auto try_wait = [&]() {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(a), "r"(parity)
            : "memory");
        return ok != 0;
    };
    if (try_wait()) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = g_wait_limit_ns;
    for (uint32_t it = 1;; ++it) {
        if (try_wait()) return true;
        if ((it & 63u) == 0u) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Waits for a phase with only a time bound and no abort check: used on the way out, to
// let copies or MMAs already in flight finish before shared or tensor memory is released.
GPT_DEVINL void mbar_drain(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_addr(bar);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(a, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) return;
    }
}

// ------------------------------------------------------------------ CTA pairs (clusters of two)
GPT_DEVINL uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
GPT_DEVINL uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
GPT_DEVINL uint32_t num_clusters_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// Every thread of both CTAs of the cluster (warp-aligned).
GPT_DEVINL void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Cluster address of the same shared-memory object in CTA `rank` of this cluster.
GPT_DEVINL uint32_t map_to_rank(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}
// Arrive on a barrier of another CTA of the cluster.
GPT_DEVINL void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Loads, stores and adds on another CTA's shared memory (cluster addresses from map_to_rank).
GPT_DEVINL uint32_t ld_cluster_u32(uint32_t cluster_addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}
GPT_DEVINL double ld_cluster_f64(uint32_t cluster_addr) {
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(cluster_addr) : "memory");
    return v;
}
GPT_DEVINL void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
GPT_DEVINL void red_cluster_add_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
GPT_DEVINL uint32_t atom_cluster_add_u32(uint32_t cluster_addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(cluster_addr), "r"(v) : "memory");
    return old;
}
// Stores a 64-bit value into another CTA's shared memory (cluster address).
GPT_DEVINL void st_cluster_u64(uint32_t cluster_addr, unsigned long long v) {
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(cluster_addr), "l"(v) : "memory");
}
// Counts `bytes` as arrived on the barrier's current phase without a copy (cancels an expected
// transfer that will never be issued).
GPT_DEVINL void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}
// A wait with only a time bound (no abort flag), acquiring at cluster scope; false on time-out.
GPT_DEVINL bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_addr(bar);
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(a), "r"(parity)
            : "memory");
        if (ok) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// ------------------------------------------------------------------ TMA
GPT_DEVINL void tma_prefetch_desc(const void* desc) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(desc)) : "memory");
}

GPT_DEVINL void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
        : "memory");
}

GPT_DEVINL void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3)
        : "memory");
}

// Contiguous global -> shared copy of `bytes` (a multiple of 16; both addresses 16-byte aligned),
// counted on `bar` like a tensor load.
GPT_DEVINL void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// 2-D tensor load by either CTA of a pair for a 2-SM MMA: data into this CTA's shared memory, the
// bytes counted on the barrier at cluster address `bar` (the leader CTA's).  Each CTA's copy
// lands in that CTA's own shared memory only.
GPT_DEVINL void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// Shared -> global tile store and tile reduce-add (fp32 add at the destination), tracked by the
// issuing thread's bulk-async group.  The tile must have been written to shared memory by
// threads that then executed fence_proxy_async_shared() and synchronised with the issuer.
GPT_DEVINL void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_addr(src)), "r"(x), "r"(y)
                 : "memory");
}
GPT_DEVINL void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_addr(src)), "r"(x), "r"(y)
        : "memory");
}
GPT_DEVINL void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Until the shared-memory source of every committed bulk store of this thread has been read.
GPT_DEVINL void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Until every committed bulk store of this thread has completed.
GPT_DEVINL void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
GPT_DEVINL void fence_proxy_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ------------------------------------------------------------------ tcgen05
// Allocation is warp-wide: the whole warp executes these.
GPT_DEVINL void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
GPT_DEVINL void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
GPT_DEVINL void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// The same for a CTA pair: one warp with the same warp index in each CTA executes these; the
// columns are allocated in both CTAs' tensor memory at the same address.
GPT_DEVINL void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
GPT_DEVINL void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
GPT_DEVINL void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

GPT_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
GPT_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate).
GPT_DEVINL void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Same with the A operand read from tensor memory.
GPT_DEVINL void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 2-SM MMA issued by the leader CTA of a pair: A rows [0, 128) from this CTA's shared memory and
// [128, 256) from the peer's (same offsets), B's N columns split the same way, D in both CTAs'
// tensor memory (each its 128 rows).
GPT_DEVINL void umma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives on `bar` in each CTA of the pair named by `mask` (bit r = rank r) once the pair's MMAs
// issued so far have completed.
GPT_DEVINL void umma_commit_pair(uint64_t* bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_addr(bar)),
        "h"(mask)
        : "memory");
}

// Arrives once on `bar` when every tcgen05.mma issued so far by this thread has completed.
GPT_DEVINL void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> fp32, M x N, A K-major unless a_mn_major,
// B K-major unless b_mn_major.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, bool b_mn_major, bool a_mn_major = false) {
    return (1u << 4)                         // D format fp32
           | (1u << 7)                       // A format bf16
           | (1u << 10)                      // B format bf16
           | ((a_mn_major ? 1u : 0u) << 15)  // A major-ness
           | ((b_mn_major ? 1u : 0u) << 16)  // B major-ness
           | ((uint32_t)(N >> 3) << 17)      // N / 8
           | ((uint32_t)(M >> 4) << 24);     // M / 16
}

// Shared-memory matrix descriptor for a tile written by TMA with 128-byte swizzling:
// rows of 128 bytes, 8-row groups 1024 bytes apart.  Used for K-major operands (rows =
// M or N, 64 bf16 of K per row) and for MN-major operands (rows = K, 64 bf16 of MN per row).
GPT_DEVINL uint64_t make_sdesc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4)  // start address
           | ((uint64_t)1 << 16)                // leading byte offset (16 B; unused here)
           | ((uint64_t)(1024 >> 4) << 32)      // stride byte offset: 8 rows x 128 B
           | ((uint64_t)1 << 46)                // descriptor version for sm_100
           | ((uint64_t)2 << 61);               // 128-byte swizzle
}

// MN-major operand wider than one 64-element swizzle atom: rows of 128 bytes along K (8-row groups
// 1024 bytes apart), and the next 64 elements of M or N `mn_stride` bytes further on (the leading
// byte offset of the canonical MN-major 128-byte-swizzle layout).
GPT_DEVINL uint64_t make_sdesc_sw128_mn(uint32_t saddr, uint32_t mn_stride) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4)
           | ((uint64_t)((mn_stride >> 4) & 0x3FFFu) << 16)
           | ((uint64_t)(1024 >> 4) << 32)
           | ((uint64_t)1 << 46)
           | ((uint64_t)2 << 61);
}

// 32 lanes x 32 bit, 32 consecutive columns per thread: thread i of the warp receives
// columns [col, col+32) of lane (warp's lane quarter)*32 + i.  Load and wait in one
// statement so no use of the registers can be scheduled before the data arrives.
GPT_DEVINL void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 64 consecutive columns in one load (same lane rule as tmem_ld32).
GPT_DEVINL void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}

// Barrier over a subset of warps (id 1..15, `threads` a multiple of 32).
GPT_DEVINL void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Stores 32 consecutive 32-bit columns of this thread's lane; waits for completion.
GPT_DEVINL void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// 16 columns of this thread's lane; waits for completion.
GPT_DEVINL void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Packed pairs of fp32 (one 64-bit register pair) and the f32x2 arithmetic of sm_100.
GPT_DEVINL uint64_t f2_pack(float lo, float hi) { uint64_t r; asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi)); return r; }
GPT_DEVINL void f2_unpack(uint64_t v, float& lo, float& hi) { asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v)); }
GPT_DEVINL uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) { uint64_t d; asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c)); return d; }
GPT_DEVINL uint64_t f2_add(uint64_t a, uint64_t b) { uint64_t d; asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b)); return d; }
GPT_DEVINL uint64_t f2_sub(uint64_t a, uint64_t b) { uint64_t d; asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b)); return d; }
GPT_DEVINL uint64_t f2_mul(uint64_t a, uint64_t b) { uint64_t d; asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b)); return d; }

GPT_DEVINL float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

GPT_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Column sums of a warp's 32 x 32 block (lane = row, v[c] = column c): lane l returns the sum of
// v[l] over the 32 lanes.  A transposing butterfly: at distance k each lane keeps the half of its
// live columns on its own side of bit k and adds its partner's copy of that half (31 exchanges
// and adds per lane, in an order fixed by the lane index).  v is consumed.
GPT_DEVINL float warp_colsum32(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
        const bool up = (lane & k) != 0;
#pragma unroll
        for (int j = 0; j < k; ++j) {
            const float send = up ? v[j] : v[j + k];
            const float keep = up ? v[j + k] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, k);
        }
    }
    return v[0];
}

// Programmatic dependent launch.  A kernel launched with programmatic stream serialisation may
// start before its predecessor in the stream has finished: it must call griddep_wait() before
// it reads or writes memory the predecessor touches (the wait returns once the predecessor has
// completed and its writes are visible).  griddep_launch_dependents() lets the successor start
// as soon as every CTA of this grid has started or finished.
GPT_DEVINL void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
GPT_DEVINL void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Eight consecutive values through one 16-byte L2 load (bf16) or two (fp32), and the matching
// plain stores; p must be 16-byte aligned.  The loads bypass L1 (data written by earlier kernels of
// an overlapped launch chain may be stale there).
GPT_DEVINL void ld8(const bf16* p, float (&f)[8]) {
    const uint4 w = __ldcg(reinterpret_cast<const uint4*>(p));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) f[2 * i] = __uint_as_float(u[i] << 16), f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
}
GPT_DEVINL void ld8(const float* p, float (&f)[8]) {
    const float4 a = __ldcg(reinterpret_cast<const float4*>(p)), b = __ldcg(reinterpret_cast<const float4*>(p) + 1);
    f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}
GPT_DEVINL void st8(bf16* p, const float (&f)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                              pack_bf16x2(f[6], f[7]));
}
GPT_DEVINL void st8(float* p, const float (&f)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// d gelu(z) / dz (CUDA's erff / tanhf): erf form Phi(z) + z phi(z); tanh form 0.5 (1 + tanh a) +
// 0.5 z (1 - tanh^2 a) sqrt(2/pi) (1 + 3 * 0.044715 z^2), a = sqrt(2/pi) (z + 0.044715 z^3).
GPT_DEVINL float gelu_slope(float z, int tanh_form) {
    if (tanh_form) {
        const float c = 0.7978845608028654f;
        const float th = tanhf(c * (z + 0.044715f * z * z * z));
        return 0.5f * (1.f + th) + 0.5f * z * (1.f - th * th) * c * (1.f + 3.f * 0.044715f * z * z);
    }
    return 0.5f * (1.f + erff(z * 0.7071067811865476f)) + z * 0.3989422804014327f * __expf(-0.5f * z * z);
}

// Records a device-side status (first writer wins).
GPT_DEVINL void set_status(int32_t* status, int32_t code) {
    if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

}  // namespace gpt
