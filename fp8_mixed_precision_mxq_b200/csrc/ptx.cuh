// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers with bounded waits,
// TMA / bulk copies, and the tcgen05 family (TMEM allocation, block-scaled MMA,
// shared->tensor-memory copies of scale factors, tensor-memory loads).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mxq {

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// One try_wait: true once the phase with the given parity has completed.  The thread may
// be suspended until then, for at most kMbarSuspendNs (the instruction's suspend-time hint);
// with the hint the GEMM runs 2.0-2.6 % faster than with the hardware's default limit
// (paired A/B, W4A4 and W4A8, output identical), and it bounds each try for the time-outs.
constexpr uint32_t kMbarSuspendNs = 100000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kMbarSuspendNs)
        : "memory");
    return done != 0;
}

// Wait until the phase with the given parity has completed, giving up after
// limit_ns nanoseconds.  Returns false on time-out; never spins forever.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// ---------------------------------------------------------------------------
// TMA and bulk copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled TMA load of box (c0, c1) into this CTA's shared memory, completing on the
// mbarrier at shared::cluster address bar (this CTA's own, or with kPair == 2 the
// pair leader's), with an L2 cache policy.
template <int kPair>
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, int32_t c0, int32_t c1,
                                            uint32_t bar, uint64_t policy)
{
    if constexpr (kPair == 2)
        asm volatile(
            "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
            ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
            : "memory");
    else
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
            ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
            : "memory");
}

// L2 eviction policies for the cache-hinted copies.
__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------------------
// clusters
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// shared::cluster address of the variable at local address p in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(p), "r"(rank));
    return r;
}

// Arrive on an mbarrier given by its shared::cluster address (possibly another CTA's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

// 2-D tiled TMA store from shared memory (bulk-group completion), with an L2 policy.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int32_t c0, int32_t c1,
                                             uint64_t policy)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::
                     "l"(reinterpret_cast<uint64_t>(m)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait()
{
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy (TMA store).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Named barrier `id` (1 ... 15) over `threads` threads of the CTA (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation tensor cores
// ---------------------------------------------------------------------------
// TMEM allocation (whole warp).  With kPair == 2 one warp of each CTA of the pair
// executes it, and the allocation serves MMAs that span both CTAs.
template <int kPair>
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols)
{
    if constexpr (kPair == 2)
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(dst_smem)),
                     "r"(ncols)
                     : "memory");
    else
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(dst_smem)),
                     "r"(ncols)
                     : "memory");
}

template <int kPair>
__device__ __forceinline__ void tmem_relinquish()
{
    if constexpr (kPair == 2)
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    else
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

template <int kPair>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    if constexpr (kPair == 2)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
    else
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive (once) on bar when every tcgen05 operation this thread issued so far is done.
// With kPair == 2 the arrive goes to the barrier at the same offset in both CTAs.
template <int kPair>
__device__ __forceinline__ void tc_commit(uint64_t* bar)
{
    if constexpr (kPair == 2)
        asm volatile(
            "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::
                "r"(smem_u32(bar))
            : "memory");
    else
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(bar))
                     : "memory");
}

// Commit that arrives only on this CTA's barrier (also for a pair leader).
template <int kPair>
__device__ __forceinline__ void tc_commit_local(uint64_t* bar)
{
    if constexpr (kPair == 2)
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(bar))
                     : "memory");
    else
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(bar))
                     : "memory");
}

// Copy one 512-byte scale-factor atom (32 rows x 16 bytes in shared memory) into
// 4 TMEM columns of lanes 0-31, replicated into all four 32-lane sub-partitions.
// With kPair == 2 (issued by the pair leader) each CTA copies from its own shared
// memory at the same offset into its own TMEM.
template <int kPair>
__device__ __forceinline__ void tc_copy_sf_atom(uint32_t taddr, uint64_t sdesc)
{
    if constexpr (kPair == 2)
        asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
    else
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A[smem] . B[smem]^T with per-32-element E8M0 block scales in TMEM.
// kind::mxf4: both operands packed E2M1, K = 64 per instruction.  With kPair == 2
// (M = 256) each CTA holds 128 rows of A and 128 rows of B at the same offsets.
template <int kPair>
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    if constexpr (kPair == 2)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
}

// Same, with the two shared-memory descriptors given as (low word, common high word).
template <int kPair, bool kF8F6F4>
__device__ __forceinline__ void mma_block_scaled(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t d_hi,
                                                 uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                 uint32_t accumulate)
{
#define MXQ_MMA_ASM(GROUP, KIND)                                                                             \
    asm volatile("{\n\t.reg .pred p;\n\t.reg .b64 ad, bd;\n\t"                                             \
                 "mov.b64 ad, {%1, %3};\n\tmov.b64 bd, {%2, %3};\n\t"                                         \
                 "setp.ne.b32 p, %5, 0;\n\t"                                                                   \
                 "tcgen05.mma.cta_group::" GROUP ".kind::" KIND " [%0], ad, bd, %4, [%6], [%7], p;\n\t}" ::"r"(  \
                     d_tmem),                                                                                  \
                 "r"(a_lo), "r"(b_lo), "r"(d_hi), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)    \
                 : "memory")
    if constexpr (kPair == 2 && kF8F6F4) MXQ_MMA_ASM("2", "mxf8f6f4.block_scale");
    else if constexpr (kPair == 2) MXQ_MMA_ASM("2", "mxf4.block_scale.block32");
    else if constexpr (kF8F6F4) MXQ_MMA_ASM("1", "mxf8f6f4.block_scale");
    else MXQ_MMA_ASM("1", "mxf4.block_scale.block32");
#undef MXQ_MMA_ASM
}

// kind::f16 with bf16 A and B (both K-major, the same type as this kind requires), fp32
// accumulation, K = 16: a 16-bit operand pair added into the same TMEM accumulator the
// block-scaled MMAs use.  Descriptors as for mma_block_scaled.
template <int kPair>
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t d_hi, uint32_t idesc,
                                         uint32_t accumulate)
{
#define MXQ_MMA16_ASM(GROUP)                                                                     \
    asm volatile("{\n\t.reg .pred p;\n\t.reg .b64 ad, bd;\n\t"                                 \
                 "mov.b64 ad, {%1, %3};\n\tmov.b64 bd, {%2, %3};\n\t"                             \
                 "setp.ne.b32 p, %5, 0;\n\t"                                                       \
                 "tcgen05.mma.cta_group::" GROUP ".kind::f16 [%0], ad, bd, %4, p;\n\t}" ::"r"(d_tmem), \
                 "r"(a_lo), "r"(b_lo), "r"(d_hi), "r"(idesc), "r"(accumulate)                          \
                 : "memory")
    if constexpr (kPair == 2) MXQ_MMA16_ASM("2");
    else MXQ_MMA16_ASM("1");
#undef MXQ_MMA16_ASM
}

// kind::mxf8f6f4: 8-bit A (E4M3), B in the byte-padded 4-bit layout (E2M1), K = 32.
template <int kPair>
__device__ __forceinline__ void mma_mxf8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    if constexpr (kPair == 2)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
}

// Each thread of a warp reads 32 consecutive 32-bit TMEM columns of its own lane.
__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// After tmem_ld_wait(): ties the 32 destination registers of a finished tcgen05.ld to
// the wait, so the compiler cannot schedule a use of them above it (the registers of
// an asynchronous load hold garbage until the wait).
__device__ __forceinline__ void tmem_regs_ready(uint32_t (&r)[32])
{
#pragma unroll
    for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}

// Each thread of a warp writes 4 consecutive 32-bit TMEM columns of its own lane.
__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, uint4 v)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t saddr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(saddr));
    return v;
}

// Shared-memory matrix descriptor (sm_100 form, version 1) for a K-major tile whose
// rows are 128 bytes wide, stored with the 128-byte swizzle: 8-row groups are
// 1024 bytes apart.  The tile base must be 1024-byte aligned; stepping along K
// inside the swizzle span is done by adding the byte offset to the start address.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);   // start address
    d |= static_cast<uint64_t>(1u) << 16;                  // leading byte offset (unused here)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;          // stride byte offset: 8 rows x 128 B
    d |= static_cast<uint64_t>(1u) << 46;                  // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2u) << 61;                  // layout: 128-byte swizzle
    return d;
}

// Upper 32 bits of the K-major 128-byte-swizzle descriptor (stride, version, layout);
// the lower word is the start address (>> 4) and the unused leading byte offset.
constexpr uint32_t kSdescSw128Hi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t sdesc_sw128_lo(uint32_t saddr) { return ((saddr >> 4) & 0x3FFFu) | (1u << 16); }

// Descriptor of a scale-factor atom: 32 rows x 16 bytes, no swizzle, 8-row core
// matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sf_atom(uint32_t saddr)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(128u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    return d;
}

// Instruction descriptor of a block-scaled MMA with E8M0 scales, both operands
// K-major, fp32 accumulation.  a_fmt / b_fmt are the element-type codes of the
// instruction kind; sfa_id / sfb_id pick the byte of the 32-bit TMEM scale word.
__host__ __device__ __forceinline__ uint32_t idesc_block_scaled(uint32_t a_fmt, uint32_t b_fmt, uint32_t M,
                                                                 uint32_t N, uint32_t sfa_id, uint32_t sfb_id)
{
    uint32_t d = 0;
    d |= (sfb_id & 3u) << 4;
    d |= (a_fmt & 7u) << 7;
    d |= (b_fmt & 7u) << 10;
    d |= ((N >> 3) & 63u) << 17;
    d |= 1u << 23;  // scale type: UE8M0
    d |= ((M >> 4) & 31u) << 24;
    d |= (sfa_id & 3u) << 29;
    return d;
}

// Instruction descriptor of kind::f16 with bf16 A and B (K-major) and an fp32 accumulator.
__host__ __device__ __forceinline__ uint32_t idesc_bf16(uint32_t M, uint32_t N)
{
    uint32_t d = 0;
    d |= 1u << 4;   // D format: F32
    d |= 1u << 7;   // A format: BF16
    d |= 1u << 10;  // B format: BF16
    d |= ((N >> 3) & 63u) << 17;
    d |= ((M >> 4) & 31u) << 24;
    return d;
}

}  // namespace mxq
