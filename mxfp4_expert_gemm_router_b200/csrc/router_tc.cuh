// router_tc.cuh -- the router's scores on the tensor cores, for bf16 activations.
//
// Method (page "GPT-OSS-20B : Architecture MoE & Résumé du Model Card", §3.1 Le
// Routeur): scores = W_router . h (+ bias), top-k, softmax over the k selected.
// The scores are a dense [T x d] . [d x E] product, so each CTA runs it as
// tcgen05.mma kind::f16 (bf16 operands, fp32 accumulation in tensor memory):
// M = 128 tokens (A = x, K-major), N = 32 experts per plane (B = the router
// weight, K-major), K chunks of 64 staged by TMA with the 128-byte swizzle.
//
// Precision: bf16 x bf16 products are exact in fp32.  Each 64-wide K chunk is
// summed in fp32 by the tensor core (into one of two accumulator buffers) and
// read out at once into fp64 per-thread totals, as the CUDA-core router sums
// fp32 within a chunk and fp64 across chunks.  With the pre-norm the weight is
// gamma * W_router rounded once to fp32 (as the CUDA-core router stages it)
// and held as three bf16 planes hi + mid + lo whose sum is that fp32 value
// exactly; the planes are stacked as N = 96 rows of one MMA and the three
// columns of each expert are added in the readout, so the products are the
// same exact values.  Without the pre-norm one plane (W_router itself).
//
// Grid: token tiles x K splits x expert tiles of 32, linearised with the
// expert tile fastest so the CTAs that share an x tile run together (L2
// reuse).  Warp roles (256 threads): warps 0..3 read tensor memory (lanes
// 32 w .. : one token each) and, with the pre-norm, sum x^2 of their token from
// the staged x chunk; warp 4 issues the TMA copies; warp 5 owns tensor memory
// and issues the MMAs; then all threads run router_tail (top-k, softmax,
// ranks, schedule).  Every wait is bounded (timeout -> status bit, abort).
#pragma once
#include <cstdint>
#include <cuda.h>

#include "routing.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int RTC_THREADS = 256;
constexpr int RTC_STAGES = 4;
constexpr uint32_t RTC_XBYTES = 128u * 128u;   // x chunk: 128 tokens x 64 bf16
__host__ __device__ constexpr uint32_t rtc_wbytes(int P) { return 32u * 128u * static_cast<uint32_t>(P); }
__host__ __device__ constexpr uint32_t rtc_stage_bytes(int P) { return RTC_XBYTES + rtc_wbytes(P); }
__host__ __device__ constexpr size_t rtc_smem_bytes(int P) {
    return 1024 + static_cast<size_t>(RTC_STAGES) * rtc_stage_bytes(P) + 8 * (2 * RTC_STAGES + 5) + 64;
}

// Instruction descriptor, kind::f16: bf16 A and B (format 1), f32 accumulator
// (format 1 at bit 4), both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tma_load_2d_warp(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n\t}" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// 32 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// gamma * W_router, rounded to fp32, as three bf16 planes hi, mid, lo ([3][E][d])
// with hi + mid + lo equal to the fp32 value: each plane is the round-to-
// nearest bf16 of what the planes before it leave, and 3 x 8 significant bits
// cover fp32's 24.
__global__ void router_planes_kernel(const __nv_bfloat16* __restrict__ wr, const float* __restrict__ gamma,
                                     __nv_bfloat16* __restrict__ planes, int E, int d) {
    const long n = static_cast<long>(E) * d;
    for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long>(gridDim.x) * blockDim.x) {
        const float v = __bfloat162float(wr[i]) * gamma[i % d];
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
        planes[i] = hi;
        planes[n + i] = mid;
        planes[2 * n + i] = lo;
    }
}


// tmap_x: x [T][d] bf16, box {64, 128}, 128-byte swizzle (rows past T read as
// zeros).  tmap_w: the weight planes [P][E][d] bf16, box {64, 32, P}, landing
// as P x 32 rows of 128 B (experts past E read as zeros).
__global__ void __launch_bounds__(RTC_THREADS, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                 const RouterArgs a, int Z, int P, int* status, uint64_t timeout_ns) {
    extern __shared__ uint8_t smem_raw[];
    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x;
    const int z = b % Z, split = (b / Z) % a.S, tile = b / (Z * a.S);
    const int ntiles = static_cast<int>(gridDim.x) / (Z * a.S);
    const int t0 = tile * ROUTER_TOKENS;
    const int ntok = min(ROUTER_TOKENS, a.T - t0);
    const int e0 = ROUTER_ETILE * z;
    const int KCH = (a.d + ROUTER_KCHUNK - 1) / ROUTER_KCHUNK;
    const int kc0 = split * KCH / a.S, kc1 = (split + 1) * KCH / a.S;
    const int nch = kc1 - kc0;
    const bool norm = a.gamma != nullptr;
    const uint32_t SB = rtc_stage_bytes(P);
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t bar0 = base + RTC_STAGES * SB;
    auto st_addr = [&](int s) { return base + static_cast<uint32_t>(s) * SB; };
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (RTC_STAGES + s); };
    auto accf_bar = [&](int u) { return bar0 + 8u * (2 * RTC_STAGES + u); };
    auto acce_bar = [&](int u) { return bar0 + 8u * (2 * RTC_STAGES + 2 + u); };
    const uint32_t drain_bar = bar0 + 8u * (2 * RTC_STAGES + 4);
    uint8_t* ctl = smem_raw + (drain_bar + 8u - raw);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 16);

    if (tid == 0) {
        for (int s = 0; s < RTC_STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), norm ? 5 : 1);   // the MMA commit (+ the 4 readers of x)
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(accf_bar(u), 1);
            mbar_init(acce_bar(u), 4);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(tmem_slot), 256);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_w);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        int pend[RTC_STAGES];
        for (int s = 0; s < RTC_STAGES; ++s) pend[s] = -1;
        for (int i = 0; i < nch; ++i) {
            const int s = i % RTC_STAGES;
            const uint32_t ph = static_cast<uint32_t>(i / RTC_STAGES) & 1u;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, status, timeout_ns)))
                break;
            const int kk = (kc0 + i) * ROUTER_KCHUNK;
            mbar_arrive_expect_tx_warp(full_bar(s), RTC_XBYTES + rtc_wbytes(P));
            tma_load_2d_warp(st_addr(s), &tmap_x, kk, t0, full_bar(s));
            tma_load_3d_warp(st_addr(s) + RTC_XBYTES, &tmap_w, kk, e0, 0, full_bar(s));
            pend[s] = static_cast<int>(ph);
        }
        // copies still in flight land before the shared memory is reused
        if (lane == 0)
            for (int s = 0; s < RTC_STAGES; ++s)
                if (pend[s] >= 0) mbar_wait_drain(full_bar(s), static_cast<uint32_t>(pend[s]), 200000000ull);
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = idesc_bf16(128, 32 * P);
        for (int i = 0; i < nch; ++i) {
            const int s = i % RTC_STAGES, u = i & 1;
            const uint32_t ph = static_cast<uint32_t>(i / RTC_STAGES) & 1u;
            const uint32_t uph = static_cast<uint32_t>(i >> 1) & 1u;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(acce_bar(u), uph ^ 1u, abort_flag, status, timeout_ns)))
                break;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), ph, abort_flag, status, timeout_ns)))
                break;
            tc_fence_after();
            const uint32_t xs = st_addr(s), ws = xs + RTC_XBYTES;
#pragma unroll
            for (int kq = 0; kq < ROUTER_KCHUNK / 16; ++kq)
                mma_bf16_warp(tmem + 128u * u, desc_sw128(xs + 32 * kq), desc_sw128(ws + 32 * kq), idesc,
                              kq > 0 ? 1u : 0u);
            tc_commit_warp(empty_bar(s));
            tc_commit_warp(accf_bar(u));
        }
        tc_commit_warp(drain_bar);
        if (lane == 0) mbar_wait_drain(drain_bar, 0, 200000000ull);
        __syncwarp();
    } else if (warp < 4) {
        // ------------------------------------------------------------ readers
        const int tl = 32 * warp + lane;
        double tot[ROUTER_ETILE];
#pragma unroll
        for (int j = 0; j < ROUTER_ETILE; ++j) tot[j] = 0.0;
        double ss = 0.0;
        for (int i = 0; i < nch; ++i) {
            const int s = i % RTC_STAGES, u = i & 1;
            const uint32_t ph = static_cast<uint32_t>(i / RTC_STAGES) & 1u;
            const uint32_t uph = static_cast<uint32_t>(i >> 1) & 1u;
            if (norm) {
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), ph, abort_flag, status, timeout_ns)))
                    break;
                // this token's 64 values: 128 B at row tl (its 16-byte pieces
                // permuted by the swizzle, which the sum does not see)
                const uint4* row = reinterpret_cast<const uint4*>(smem_raw + (st_addr(s) - raw) + 128u * tl);
                float sq = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 q = row[c];
                    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float lo = __uint_as_float(w4[h] << 16), hi = __uint_as_float(w4[h] & 0xFFFF0000u);
                        sq = fmaf(lo, lo, sq);
                        sq = fmaf(hi, hi, sq);
                    }
                }
                ss += static_cast<double>(sq);
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(s));
            }
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(accf_bar(u), uph, abort_flag, status, timeout_ns))) break;
            tc_fence_after();
            for (int pl = 0; pl < P; ++pl) {
                uint32_t r[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 128u * u + 32u * pl, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < ROUTER_ETILE; ++j) tot[j] += static_cast<double>(__uint_as_float(r[j]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce_bar(u));
        }
        if (tl < ntok) {
            double* dst = a.part + (static_cast<size_t>(split) * a.T + t0 + tl) * a.E;
#pragma unroll
            for (int j = 0; j < ROUTER_ETILE; ++j)
                if (e0 + j < a.E) dst[e0 + j] = tot[j];
            if (norm && z == 0) a.part_ss[static_cast<size_t>(split) * a.T + t0 + tl] = ss;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
    // the stages are free again: the tail's scores reuse them
    router_tail(a, tile, ntiles, a.S * Z, reinterpret_cast<float*>(smem_raw + (base - raw)),
                     static_cast<size_t>(RTC_STAGES) * SB);
}

}  // namespace moe
