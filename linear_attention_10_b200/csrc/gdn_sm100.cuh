// gdn_sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the kernels use:
// mbarriers with bounded waits, tcgen05 TMEM allocation / MMA / commit / load, async-proxy fences,
// and the shared-memory matrix descriptors of the 128-byte-swizzled K-major operand layout.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace gdn {
namespace sm100 {

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------------------------------------
// mbarrier
// ------------------------------------------------------------------------------------------------
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

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
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

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity to complete.  Gives up (returns false) when `abort` is
// set by another thread or after about `limit_ns` nanoseconds; never spins forever.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns = 2000000000ull)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if ((it & 63u) == 63u && globaltimer_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Adds `bytes` to the transaction count of the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// ------------------------------------------------------------------------------------------------
// Bulk copies into this CTA's shared memory (the tensor-memory-access engine; no multicast).
// ------------------------------------------------------------------------------------------------
// 2-D tiled load described by a tensor map (a __grid_constant__ kernel parameter); completes `bar`
// by the tile's byte count.  x must be a multiple of 16 bytes / element size.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// Contiguous copy; src, dst 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Contiguous copy from this CTA's shared memory to global memory, in the issuing thread's bulk
// group; src, dst 16-byte aligned, bytes a multiple of 16.  The shared-memory writes it copies must
// have been made visible to the async proxy (fence_async_smem() by the writers, then a barrier).
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until the issuing thread's committed bulk stores have read their shared-memory source.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Waits until the issuing thread's committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ------------------------------------------------------------------------------------------------
// fences and named barriers
// ------------------------------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched as a dependent of the previous kernel in its
// stream may become resident before that kernel ends; grid_dep_wait() returns once the previous
// kernel has completed and its memory writes are visible (at once when there is no such
// dependency).  grid_dep_launch() lets the next kernel, if it is launched as a dependent, be
// scheduled now; it does not relax that kernel's own wait.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// generic-proxy shared-memory writes -> visible to the async proxy (tensor-core operand reads)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void named_bar(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also returns, to every participating thread, whether any of them passed
// pred = true.  A group that leaves a loop on a flag another group may set at any moment takes the
// decision from this value, so that all of its threads leave together.
__device__ __forceinline__ bool named_bar_any(int id, int nthreads, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// ------------------------------------------------------------------------------------------------
// Tensor memory
// ------------------------------------------------------------------------------------------------
// Executed by one full warp.  The allocated base address is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::tf32, issued by one thread.
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 with bf16 operands and fp32 accumulation.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The mbarrier receives one arrival once every tcgen05 operation issued so far by this thread has
// completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 bits, 16 or 32 consecutive columns: thread i of the warp receives lane
// (warp's lane quarter base + i), columns [col, col + N).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16])
{
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32])
{
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
          "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
          "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&r)[8])
{
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
                 : "r"(taddr));
}
// 16 lanes x 32 bits, 16 consecutive columns, twice: thread i < 16 receives lane (quarter base + i),
// columns [col, col + 16); thread i >= 16 lane (quarter base + i - 16), columns [col + 16, col + 32).
__device__ __forceinline__ void tmem_ld16x2(uint32_t taddr, float (&r)[16])
{
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 16;"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&r)[N])
{
    static_assert(N == 8 || N == 16 || N == 32, "tmem_ld: 8, 16 or 32 columns");
    if constexpr (N == 8) tmem_ld8(taddr, r);
    else if constexpr (N == 16) tmem_ld16(taddr, r);
    else tmem_ld32(taddr, r);
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------------------------------------
// Operand layout: K-major, 128-byte swizzle, 32-bit elements.
//
// A tile of R rows (R % 8 == 0) by KC 32-bit elements is stored as KC/32 panels of R x 128 bytes.
// Inside a panel, 8-row groups are 1024 bytes apart; row r of a group occupies 128 bytes whose
// 16-byte chunks are permuted by XOR with (r % 8).  Panels must start on 1024-byte boundaries.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t sw128_off(int r, int k, int R)
{
    return (uint32_t)((k >> 5) * (R * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                      ((((k & 31) >> 2) ^ (r & 7)) << 4) + ((k & 3) << 2));
}

// Descriptor of the 8-element (32-byte) K-slice `ks` of such a tile at shared address `base`.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t base, int ks, int R)
{
    const uint32_t addr = base + (uint32_t)((ks >> 2) * (R * 128) + (ks & 3) * 32);
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)1u << 16;                          // leading byte offset (unused when swizzled)
    d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset: 8-row groups
    d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                          // 128-byte swizzle
    return d;
}

// Offset, in the descriptor's 16-byte start-address units, of K-slice `ks` relative to slice 0 of
// a tile of R rows: adding it to the slice-0 descriptor gives the slice-ks descriptor (the start
// address field cannot overflow for tiles inside the 227 KB of shared memory).
__host__ __device__ constexpr uint64_t sw128_ks_off(int ks, int R)
{
    return (uint64_t)((ks >> 2) * (R * 8) + (ks & 3) * 2);
}

// Same layout with 16-bit elements: 64 elements per 128-byte row.
__device__ __forceinline__ uint32_t sw128_off_h(int r, int k, int R)
{
    return (uint32_t)((k >> 6) * (R * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                      ((((k & 63) >> 3) ^ (r & 7)) << 4) + ((k & 7) << 1));
}

// Descriptor of a tile read M/N-major (the M index runs along the 128-byte rows): 8-row groups of
// the K index are `sbo` bytes apart, 64-element blocks of the M index `lbo` bytes apart.
__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B, fp32 accumulator; each operand K-major or
// M/N-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_m_major = false, bool b_n_major = false)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_m_major ? 1u : 0u) << 15) | ((b_n_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// 16-bit K-major tile with the 64-byte swizzle (rows of 32 elements): 8-row groups of 512 bytes;
// the 16-byte chunks of row r are permuted by XOR with ((r / 2) % 4).
__device__ __forceinline__ uint32_t sw64_off_h(int r, int k)
{
    return (uint32_t)((r >> 3) * 512 + (r & 7) * 64 + ((((k >> 3) ^ ((r >> 1) & 3))) << 4) + ((k & 7) << 1));
}
__device__ __forceinline__ uint64_t sw64_desc(uint32_t addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(512u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)4u << 61;                          // 64-byte swizzle
    return d;
}

// Byte offset of element (n, k) of a 16-bit tile stored N-major with the 128-byte swizzle: N runs
// along 128-byte rows (64 elements), one row per K index, 8 K-rows per 1024-byte group; 64-wide
// N-blocks are `lbo` bytes apart.
__device__ __forceinline__ uint32_t sw128_off_nmaj(int n, int k, uint32_t lbo)
{
    return (uint32_t)((n >> 6) * lbo + (k >> 3) * 1024 + (k & 7) * 128 + (((((n & 63) >> 3) ^ (k & 7))) << 4) +
                      ((n & 7) << 1));
}

// Three-way bf16 split of two values at once, packed in pairs (first value in the low half), for
// N-major tiles where the two values are adjacent along N.  Each part is the top 16 bits of what
// the previous parts left (truncation), and every remainder is exact in fp32: x = b1 + b2 + b3 + r
// with |r| < 2^-23 |x|, so the three parts carry fp32 precision.  Only integer byte permutes,
// masks and fp32 subtractions are used -- no format conversions, which issue at a quarter of the
// fp32 rate and would make the split the slowest step of an epilogue.
__device__ __forceinline__ void bf16x2_split3(float x, float y, uint32_t& p1, uint32_t& p2, uint32_t& p3)
{
    const uint32_t xb = __float_as_uint(x), yb = __float_as_uint(y);
    p1 = __byte_perm(xb, yb, 0x7632);
    const float rx = x - __uint_as_float(xb & 0xFFFF0000u), ry = y - __uint_as_float(yb & 0xFFFF0000u);
    const uint32_t rxb = __float_as_uint(rx), ryb = __float_as_uint(ry);
    p2 = __byte_perm(rxb, ryb, 0x7632);
    const float sx = rx - __uint_as_float(rxb & 0xFFFF0000u), sy = ry - __uint_as_float(ryb & 0xFFFF0000u);
    p3 = __byte_perm(__float_as_uint(sx), __float_as_uint(sy), 0x7632);
}

// Instruction descriptor: kind::tf32, fp32 accumulator, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N)
{
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// TF32 split x = hi + lo: hi keeps the sign, exponent and the 10 leading mantissa bits of x (the
// bits a TF32 operand carries), lo = x - hi is exact in fp32 and the tensor core reads its leading
// 11 significant bits.  hi*hi + hi*lo + lo*hi then recovers an fp32-accurate product; the dropped
// lo*lo term and the unread tail of lo are both below 2^-21 relative.
__device__ __forceinline__ void tf32_split(float x, float& hi, float& lo)
{
    hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
    lo = x - hi;
}

// Three-way bf16 split x = b1 + b2 + b3 (bit patterns returned in the low 16 bits): each part keeps
// the leading 8 significant bits of what the previous parts left, so b1 + b2 + b3 carries 24
// significant bits -- fp32 precision.  With an operand that is exactly bf16, the three products
// on bf16 tensor cores give an fp32-accurate product.
__device__ __forceinline__ void bf16_split3(float x, uint32_t& b1, uint32_t& b2, uint32_t& b3)
{
    const uint32_t u1 = __float_as_uint(x) & 0xFFFF0000u;
    const float r1 = x - __uint_as_float(u1);
    const uint32_t u2 = __float_as_uint(r1) & 0xFFFF0000u;
    const float r2 = r1 - __uint_as_float(u2);
    b1 = u1 >> 16;
    b2 = u2 >> 16;
    b3 = __float_as_uint(r2) >> 16;
}

}  // namespace sm100
}  // namespace gdn
