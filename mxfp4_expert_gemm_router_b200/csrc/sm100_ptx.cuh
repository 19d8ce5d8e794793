// sm100_ptx.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// layer's kernels use: mbarriers, dependent-launch control, bulk / tensor TMA
// copies, tcgen05 tensor-memory allocation, scale-factor copies, block-scaled
// MMAs, loads and commits, and the E2M1 conversions.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

namespace moe {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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
// As mbar_try_wait, but the thread may sleep up to `hint_ns` for the phase to
// complete instead of returning at once.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// ------------------------------------------------------------------ dependent launches
// The next kernel in the stream may launch (it blocks in pdl_wait until this
// grid has finished and its memory operations are visible).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// Wait until the preceding kernel in the stream has completed and its writes
// are visible; a no-op for a kernel launched without programmatic serialization.
// Pointers to what the preceding kernels write must not be `const __restrict__`
// in a kernel that waits here: the compiler may then load through them before
// the wait (the asm's memory clobber does not cover restrict-qualified data),
// which, with the kernel launched early, reads values not yet written.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Device-side status word shared with the host: a set of bits.
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BOUNDS = 2 };

// Index checks of the debug build (MOE_DEBUG_CHECKS): a failed check records
// DEV_BOUNDS in the status word and the caller skips the access; it never
// traps.  In the release build every check is `true` and compiles away.
#ifdef MOE_DEBUG_CHECKS
__device__ __forceinline__ bool moe_in_bounds(bool ok, int* status) {
    if (!ok) atomicOr(status, DEV_BOUNDS);
    return ok;
}
#define MOE_IN_BOUNDS(cond, status) ::moe::moe_in_bounds((cond), (status))
#else
#define MOE_IN_BOUNDS(cond, status) true
#endif

// Bounded wait on an mbarrier phase.  Returns false (and raises the CTA's abort
// flag and the global status word) when `limit_ns` passes, or when another role
// of the CTA has already aborted.  No wait in the expert kernels is unbounded.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int* abort_flag, int* status,
                                                  uint64_t limit_ns) {
    // One quick check, then suspend in hardware until the phase completes (or
    // the hint expires): polling here takes issue slots from the warps that
    // share this warp's scheduler (measured: every expert GEMM got slower).
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 50000u)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicOr(status, DEV_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag (used to drain copies in flight).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > limit_ns) return false;
    return true;
}

// Bounded wait until *p (a counter other CTAs raise with atomics) reaches
// `target` (compared as a signed difference, so the counter may wrap).  Load
// with acquire semantics at GPU scope: what the raising CTA wrote before its
// release is visible afterwards.  Returns false on the abort flag or after
// `limit_ns` (then it raises the abort flag and the status word).
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// The polling interval backs off from 32 ns to 512 ns: many CTAs polling one
// line of L2 at a high rate slow down the slice that holds it, and with it
// every stream that passes through that slice.
__device__ __forceinline__ bool spin_until_reached(const uint32_t* p, uint32_t target, volatile int* abort_flag,
                                                   int* status, uint64_t limit_ns) {
    if (static_cast<int>(ld_acquire_u32(p) - target) >= 0) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t pause = 32;
#pragma unroll 1
    while (true) {
        __nanosleep(pause);
        if (pause < 512) pause <<= 1;
        if (static_cast<int>(ld_acquire_u32(p) - target) >= 0) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicOr(status, DEV_TIMEOUT);
            return false;
        }
    }
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy reads (tcgen05.mma / tcgen05.cp operands).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Order global-memory accesses of the generic proxy (what this thread has
// acquired: data other CTAs wrote with ordinary stores) before this thread's
// later async-proxy accesses (bulk copies reading that data).
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Named barrier over `count` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier that also returns the AND of `v` over the participating
// threads: every participant takes the same decision (e.g. to leave a loop
// after a bounded wait ran out in one of them).
__device__ __forceinline__ bool named_barrier_and(uint32_t id, uint32_t count, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(v ? 1u : 0u), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// ------------------------------------------------------------------ TMA
// 1-D bulk copy global -> shared; both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// Warp-collective forms of the copy-side instructions (one elected lane issues).
__device__ __forceinline__ void mbar_arrive_expect_tx_warp(uint32_t bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar), "r"(bytes)
        : "memory");
}
__device__ __forceinline__ void bulk_g2s_warp(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// 3-D tiled tensor copy global -> shared (no multicast); c0 is the innermost
// coordinate and must be a multiple of 16 bytes' worth of elements.
__device__ __forceinline__ void tma_load_3d_warp(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                                 uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n\t}" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_dst), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_commit_warp(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
        : "memory");
}
// D[tmem] (+)= (A . diag) * (B . diag)^T with kind::mxf4 block scaling: A and B
// packed E2M1 in shared memory (descriptors), one E8M0 scale per 32 elements of
// K for every row of A and B, read from tensor memory at `sfa` / `sfb`; the
// instruction consumes K = 64 (two scale bytes per row, chosen by the sf ids in
// the instruction descriptor).  Warp-collective: elect.sync picks the issuer.
__device__ __forceinline__ void mma_mxf4_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
}
// As mma_mxf4_warp with kind::mxf8f6f4 (32-element block scaling): here A is
// E2M1 in the 16-byte-padded shared-memory form (16 codes in the low 8 bytes
// of every 16), B is E4M3; the instruction consumes K = 32, one scale byte per
// row chosen by the sf ids (0..3).
__device__ __forceinline__ void mma_mxf8f6f4_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                  uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
}
// Copy one 512-byte scale-factor atom (32 rows x 16 B) from shared memory to 4
// tensor-memory columns of lanes 0..31, replicated to the four lane quarters.
// Warp-collective; ordered with the tcgen05.mma instructions the same thread issues.
__device__ __forceinline__ void tc_cp_sf_warp(uint32_t taddr, uint64_t sdesc) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
        "l"(sdesc)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Load 8 consecutive 32-bit columns of this thread's TMEM lane (warp-collective).
// (x8: the epilogue reads accumulators in groups of 8 token columns.)
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(taddr)
        : "memory");
}

// Shared-memory matrix descriptor, no swizzle, K-major: core matrices of 8 rows
// x 16 B stored as 128 contiguous bytes; `sbo` = bytes between 8-row groups,
// `lbo` = bytes between K-adjacent core matrices; descriptor version 1.
__host__ __device__ constexpr uint64_t desc_noswz(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (static_cast<uint64_t>(1) << 46);
}
// Shared-memory matrix descriptor, K-major with the 128-byte swizzle: rows of
// 128 B, 8-row groups of 1024 B (the group must start 1024-byte aligned), the
// 16-byte chunks of row r stored at chunk position (c ^ r % 8).  A K step
// inside the 128-byte row advances the start address.
__host__ __device__ constexpr uint64_t desc_sw128(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}
// Instruction descriptor, kind::mxf8f6f4 block-scaled: A E2M1 (format 5), B
// E4M3 (format 0), E8M0 scales, f32 accumulator, both K-major.
__host__ __device__ constexpr uint32_t idesc_mxf8f6f4_e2m1_e4m3(int M, int N) {
    return (5u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
// Instruction descriptor, kind::mxf4 block-scaled: E2M1 A and B (format 1),
// E8M0 scales (bit 23), f32 accumulator, both K-major.  The scale-factor ids
// (bits 4-5 for B, 29-30 for A) are or-ed in per instruction.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N) {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_sf_ids(uint32_t sf_id) { return (sf_id << 29) | (sf_id << 4); }

// Two floats -> one byte of two E2M1 codes (lo in the low nibble), rounded to
// nearest with ties to the even code, saturating at +-6.
__device__ __forceinline__ uint32_t e2m1x2_from_f32(float lo, float hi) {
    uint32_t d;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(d)
        : "f"(hi), "f"(lo));
    return d;
}
// One byte of two E2M1 codes -> f16x2 (low nibble in the low half), exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t d;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
        : "=r"(d)
        : "r"(byte));
    return d;
}

// Two floats -> two E4M3 codes (lo in the low byte), rounded to nearest even,
// saturating at +-448 (the largest finite E4M3 value).
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}
// Two E4M3 codes (low 16 bits) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t pair) {
    uint32_t d;
    const uint16_t h = static_cast<uint16_t>(pair);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(h));
    return d;
}

}  // namespace moe
