// sm_100a building blocks: mbarriers, TMA, tensor memory (TMEM) and tcgen05.mma.
//
// Conventions used by the kernels of this library:
//  * MMA operands in shared memory are tf32 (fp32 bit patterns rounded to tf32) in the
//    K-major, 128-byte-swizzled canonical layout: the tile is split into K-blocks of 32
//    elements (128 B per row); inside a K-block, row r lives at (r/8)*1024 + (r%8)*128 and
//    its 16-byte chunk c is stored at chunk position c ^ (r%8). Tiles are 1024-byte aligned.
//  * Accumulators (fp32) and TMEM-sourced A operands use lane = row, column = element.
//  * Every wait is bounded in wall time; a wait that gives up reports false.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wkv7 {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarriers -------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits until the phase with the given parity has completed, at most timeout_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    return true;
}

// Non-blocking test of the phase with the given parity (no suspension).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait by a single thread that spins on the non-blocking test: it sees the phase
// complete as soon as it does (a suspended try_wait can wake late), at the cost of one
// polling thread's issue slots.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t *bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((i & 255u) == 0 && globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// ---- proxies and tcgen05 ordering ------------------------------------------------------------
// Generic-proxy shared-memory writes -> visible to the async proxy (tensor core, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---- TMEM allocation (one warp) ---------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---- TMEM <-> registers: 32 lanes x 32 consecutive columns (one value per column) -------------
// The load includes its wait so the outputs are valid when the statement completes.
#define WKV7_R8(i) "=f"(v[i]), "=f"(v[i + 1]), "=f"(v[i + 2]), "=f"(v[i + 3]), "=f"(v[i + 4]), "=f"(v[i + 5]), \
                   "=f"(v[i + 6]), "=f"(v[i + 7])
#define WKV7_W8(i) "f"(v[i]), "f"(v[i + 1]), "f"(v[i + 2]), "f"(v[i + 3]), "f"(v[i + 4]), "f"(v[i + 5]), \
                   "f"(v[i + 6]), "f"(v[i + 7])
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : WKV7_R8(0), WKV7_R8(8), WKV7_R8(16), WKV7_R8(24)
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        WKV7_W8(0), WKV7_W8(8), WKV7_W8(16), WKV7_W8(24)
        : "memory");
}
// 32 lanes x 8 consecutive columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : WKV7_R8(0)
        : "r"(taddr)
        : "memory");
}
// Same without the wait: several loads in flight, then one tmem_ld_wait(...) naming every
// destination array before any use (the operands keep the compiler from moving uses above it).
__device__ __forceinline__ void tmem_ld8_nowait(uint32_t taddr, float (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : WKV7_R8(0)
                 : "r"(taddr)
                 : "memory");
}
#define WKV7_RW8(a) "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3]), "+f"(a[4]), "+f"(a[5]), "+f"(a[6]), "+f"(a[7])
__device__ __forceinline__ void tmem_ld_wait(float (&a)[8], float (&b)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : WKV7_RW8(a), WKV7_RW8(b) : : "memory");
}
__device__ __forceinline__ void tmem_ld_wait(float (&a)[8], float (&b)[8], float (&c)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : WKV7_RW8(a), WKV7_RW8(b), WKV7_RW8(c) : : "memory");
}
__device__ __forceinline__ void tmem_ld_wait(float (&a)[8], float (&b)[8], float (&c)[8], float (&d)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : WKV7_RW8(a), WKV7_RW8(b), WKV7_RW8(c), WKV7_RW8(d) : : "memory");
}
#undef WKV7_RW8
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), WKV7_W8(0)
                 : "memory");
}
#undef WKV7_R8
#undef WKV7_W8
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// TMEM address of (lane, column) relative to an allocation base.
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// ---- tf32 rounding -----------------------------------------------------------------------------
// Round a finite fp32 value to the nearest tf32 value (10 explicit mantissa bits), ties away
// from zero: add half of the 13 dropped bits' range to the sign-magnitude pattern, then clear
// them (a carry into the exponent is the correct round-up). The tensor core then reads the
// operand exactly. Two integer instructions; the conversion instruction is several times
// slower on this part.
__device__ __forceinline__ float to_tf32(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

// ---- shared-memory operand layout (K-major, 128-byte swizzle, tf32) -------------------------------
// Byte offset of element (row, k) in a tile of `rows` rows and 64 K-elements.
__device__ __forceinline__ uint32_t sw128_off(int row, int k, int rows) {
    const int kb = k >> 5, kk = k & 31;
    return uint32_t(kb * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 + ((((kk >> 2) ^ (row & 7))) << 4) +
                    ((kk & 3) << 2));
}
// Byte offset of the 16-byte group holding elements (row, k..k+3), k a multiple of 4.
__device__ __forceinline__ uint32_t sw128_off4(int row, int k, int rows) { return sw128_off(row, k, rows); }

// Shared-memory matrix descriptor: K-major, SWIZZLE_128B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= uint64_t((smem_addr & 0x3FFFFu) >> 4);   // start address (16-byte units)
    d |= uint64_t(1) << 16;                       // leading byte offset (unused for this layout)
    d |= uint64_t(1024 >> 4) << 32;               // stride byte offset: next 8-row group
    d |= uint64_t(1) << 46;                       // descriptor version (sm_100)
    d |= uint64_t(2) << 61;                       // swizzle mode: 128-byte
    return d;
}
// Descriptor of the 8-wide K-step `ks` (0..7) of a K-major tile with `rows` rows at smem_addr.
__device__ __forceinline__ uint64_t desc_kstep(uint32_t smem_addr, int ks, int rows) {
    return desc_sw128(smem_addr + uint32_t((ks >> 2) * rows * 128 + (ks & 3) * 32));
}

// Offset to add to a desc_sw128 descriptor for K-step `ks` (start address field, 16-byte units).
__device__ __forceinline__ uint64_t kstep_off(int ks, int rows) {
    return uint64_t(((ks >> 2) * rows * 128 + (ks & 3) * 32) >> 4);
}

// ---- MN-major operand layout (128-byte swizzle, tf32) ----------------------------------------------
// A K x MN operand stored MN-major: for each K index (a row here) 32 consecutive MN elements
// fill one 128-byte line; 8 consecutive K rows form a 1024-byte swizzle atom (16-byte chunk c of
// row r at chunk position c ^ (r % 8)). Atoms of successive K groups are MN_SBO bytes apart and
// blocks of 32 MN elements are `kdim/8 * 1024` bytes apart. A thread owning one K row writes its
// MN elements with 16-byte stores.
constexpr uint32_t MN_SBO = 1024;
__device__ __forceinline__ uint32_t mn_off(int k, int n, int kdim) {
    return uint32_t((n >> 5) * (kdim >> 3) * 1024 + (k >> 3) * 1024 + (k & 7) * 128 +
                    ((((n & 31) >> 2) ^ (k & 7)) << 4) + ((n & 3) << 2));
}
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t smem_addr, int kdim) {
    uint64_t d = 0;
    d |= uint64_t((smem_addr & 0x3FFFFu) >> 4);                 // start address
    d |= uint64_t(((kdim >> 3) * 1024) >> 4) << 16;             // leading byte offset: next 32 MN elements
    d |= uint64_t(MN_SBO >> 4) << 32;                           // stride byte offset: next 8 K rows
    d |= uint64_t(1) << 46;
    d |= uint64_t(2) << 61;
    return d;
}
// Offset (16-byte units) of K-step `ks` (8 K rows) in an MN-major tile.
__device__ __forceinline__ uint64_t mn_kstep_off(int ks) { return uint64_t(ks * MN_SBO >> 4); }

// Instruction descriptor of kind::tf32 with fp32 accumulation, K-major A and B.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
// Same with B stored MN-major.
__host__ __device__ constexpr uint32_t idesc_tf32_bmn(int M, int N) { return idesc_tf32(M, N) | (1u << 16); }
// Same with the A operand negated (D = D - A B when accumulating).
__host__ __device__ constexpr uint32_t idesc_neg_a(uint32_t idesc) { return idesc | (1u << 13); }

// ---- tcgen05.mma (issued by a single thread) -----------------------------------------------------
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Instruction descriptor of kind::f16 with bf16 A and B (K-major) and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Plain arrival (release, CTA scope) of the calling thread.
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Arrive on `bar` once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// ---- TMA (no multicast) ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_4d(void *dst, const void *tmap, uint64_t *bar, int c0, int c1, int c2,
                                            int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
        "%6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Global -> shared copy of `bytes` contiguous bytes (both addresses 16-byte aligned, bytes a
// multiple of 16), completing on an mbarrier.
__device__ __forceinline__ void bulk_load_1d(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// Fetches a tensor map (a __grid_constant__ kernel parameter) ahead of its first use.
__device__ __forceinline__ void prefetch_tensormap(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, uint64_t *bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// Shared -> global tile store through a tensor map (bulk-group completion). The source must stay
// untouched until tma_store_wait_read() in the issuing thread has returned.
__device__ __forceinline__ void tma_store_4d(const void *tmap, const void *src, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(tmap),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void tma_store_2d(const void *tmap, const void *src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(tmap),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1)
                 : "memory");
}
// Waits until at most one committed bulk group still reads its shared-memory source.
__device__ __forceinline__ void tma_store_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The sources of this thread's committed stores have been read (shared memory reusable).
__device__ __forceinline__ void tma_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// This thread's committed stores are complete.
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---- thread-block clusters and distributed shared memory ------------------------------------------
// A kernel launched without a cluster attribute runs as clusters of one CTA: rank 0 of 1.
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Address, in the shared::cluster window, of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster(uint32_t cluster_addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}
// Generic-proxy writes to (any CTA's) shared memory -> visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_cluster() {
    asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}
// Arrive (release, cluster scope) on an mbarrier in another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for a phase completed by arrivals from other CTAs (acquire at cluster scope).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_acq_cluster(bar, parity))
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    return true;
}

}  // namespace tc
}  // namespace wkv7
