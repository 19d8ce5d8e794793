// expert_gemm.cuh -- grouped expert GEMMs on tcgen05 tensor cores.
//
// Method (page "GPT-OSS-20B : Architecture MoE & Résumé du Model Card", §3.2 Les
// Experts): each expert is (Swish(x . W_gate) (.) (x . W_up)) . W_down with
// Swish(z) = z sigma(z); §2.1: the k expert outputs of a token are summed with
// the router weights.
//
// Orientation: the MMA computes D[feature, token] = W[feature, :] . X[token, :]^T
// with M = 128 weight rows (output features) and N = BN grouped token rows, so
// the weight tile is the A operand.  A lives in tensor memory: decoder warps
// read the MXFP4 tile that a bulk copy brought into shared memory, turn each
// byte into two f16 values in registers, scale them by the block's power of two
// relative to the row scale, and store them to TMEM with tcgen05.st.  B, the
// grouped f16 activations, arrives by 2-D TMA with 128-byte swizzle.  fp32
// accumulators stay in TMEM; the epilogue warps read them back with tcgen05.ld.
//
//   MODE 0 (gate/up): stages of K = 128 holding gate and up (17408 weight
//     bytes); two accumulators (gate, up) for the same 128 features; epilogue:
//     H[row, f] = Swish(g * 2^sg) * (u * 2^su), stored as f16; with a K split,
//     fp32 partials are added into GU instead.
//   MODE 1 (down): stages of K = 128 (8704 weight bytes); one accumulator;
//     epilogue: y[token, f] += w_row * (d * 2^sd), red.add into the fp32 output
//     accumulator (the weighted scatter-combine).
// Each decoder thread decodes two 32-blocks per round: MODE 0 two blocks of
// one stage, MODE 1 one block of each of two stages.
//
// Persistent kernel: one CTA per SM, units (expert, token tile, feature tile,
// K split) taken round-robin from a device-built list.  Warp roles:
//   warp 0       TMA producer (one thread)
//   warp 1       TMEM allocator and MMA issuer (one thread)
//   warps 2..17  decoders, then epilogue.  Warp w serves TMEM lanes
//                32*(w%4) .. +31 and role (w-2)/4 in 0..3: MODE 0 matrix
//                role>>1, block role&1 of the stage; MODE 1 block role.
// Every mbarrier wait is bounded; on a timeout the CTA raises an abort flag,
// all roles leave their loops, in-flight copies and MMAs are drained, TMEM is
// freed and the status word reports the timeout.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "quantize.cuh"
#include "routing.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int GEMM_DEC_WARPS = 16;
constexpr int GEMM_THREADS = (2 + GEMM_DEC_WARPS) * 32;
constexpr int GEMM_MAX_STAGES = 16;
constexpr int GEMM_MAX_A_SLOTS = 7;
constexpr int GEMM_TMEM_COLS = 512;
constexpr int GEMM_KSTAGE = 128;                              // K per pipeline stage, both modes
constexpr int GEMM_MIN_SMEM = 120 * 1024;  // keeps one CTA (and one TMEM owner) per SM

struct GemmParams {
    const uint8_t* wpack;     // tiled MXFP4 weights (quantize.cuh layout)
    const uint8_t* rowscale;  // MODE 0: [E][2][N] (gate, up); MODE 1: [E][N]
    const int4* units;        // {expert, first grouped row, valid rows, feature tile | split << 16}
    const int32_t* sched;
    TiledMatrix M;            // geometry of the (first) matrix streamed
    int N;                    // output features
    int K;                    // contraction length
    int BN;                   // token rows per tile (MMA N), multiple of 16
    int stages;
    int a_slots;              // TMEM A slots (gemm_a_cols(MODE) columns each); accumulators follow them
    uint32_t idesc;
    __half* H;                // MODE 0 output [rows][N]
    float* GU;                // MODE 0 split partials [rows][2N]
    float* yacc;              // MODE 1 output accumulator [T][N]
    const int32_t* row_token; // MODE 1
    const float* row_weight;  // MODE 1
    int* status;
    uint64_t timeout_ns;
    uint32_t skip_first_copy; // test hook: producer skips its first copy
};

// Weight bytes per stage (128 rows x 4 blocks x 17 B per matrix), TMEM columns
// per A slot (K = 128 of f16 per matrix = 64 columns), B bytes per stage (two
// 64-wide K sub-tiles of BN rows x 128 B).
__host__ __device__ constexpr int gemm_w_stage(int mode) { return mode == 0 ? 2 * 128 * 4 * 17 : 128 * 4 * 17; }
__host__ __device__ constexpr int gemm_a_cols(int mode) { return mode == 0 ? 128 : 64; }
__host__ __device__ inline size_t gemm_b_stage_bytes(int mode, int BN) {
    (void)mode;
    return static_cast<size_t>(BN) * 128 * 2;
}
__host__ inline size_t gemm_stage_bytes(int mode, int BN) { return gemm_w_stage(mode) + gemm_b_stage_bytes(mode, BN); }
// A slots that fit in TMEM beside the accumulators (2*BN columns for gate/up, BN for down).
__host__ inline int gemm_a_slots(int mode, int BN) {
    const int d_cols = mode == 0 ? 2 * BN : BN;
    int n = (GEMM_TMEM_COLS - d_cols) / gemm_a_cols(mode);
    return n > GEMM_MAX_A_SLOTS ? GEMM_MAX_A_SLOTS : n;
}
__host__ inline size_t gemm_smem_bytes(int mode, int BN, int stages) {
    size_t b = 1024 + stages * gemm_stage_bytes(mode, BN) + (2 * stages + 2 * GEMM_MAX_A_SLOTS + 3) * 8 + 64;
    return b < static_cast<size_t>(GEMM_MIN_SMEM) ? static_cast<size_t>(GEMM_MIN_SMEM) : b;
}

template <int MODE>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
expert_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int KSTAGE = GEMM_KSTAGE;
    constexpr int W_STAGE = gemm_w_stage(MODE);
    constexpr int A_COLS = gemm_a_cols(MODE);

    const int S = p.stages;
    const uint32_t b_bytes = static_cast<uint32_t>(gemm_b_stage_bytes(MODE, p.BN));
    const uint32_t b_sub = static_cast<uint32_t>(p.BN) * 128u;   // one 64-K sub-tile of B
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t b_sm = base;                                   // S x B tiles (1024-aligned)
    const uint32_t w_sm = b_sm + S * b_bytes;                     // S x weight chunks
    const uint32_t bar0 = w_sm + S * W_STAGE;                     // barriers (8-byte aligned)
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    const int NA = p.a_slots;
    const uint32_t d_col0 = static_cast<uint32_t>(NA * A_COLS);        // first accumulator column
    auto afull_bar = [&](int a) { return bar0 + 8u * (2 * S + a); };
    auto aempty_bar = [&](int a) { return bar0 + 8u * (2 * S + GEMM_MAX_A_SLOTS + a); };
    const uint32_t accf_bar = bar0 + 8u * (2 * S + 2 * GEMM_MAX_A_SLOTS);
    const uint32_t acce_bar = accf_bar + 8u;
    const uint32_t drain_bar = acce_bar + 8u;
    uint8_t* ctl = smem_raw + (drain_bar + 8u - raw);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 16);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), GEMM_DEC_WARPS + 1);  // decoder warps + 1 MMA commit
        }
        for (int a = 0; a < NA; ++a) {
            mbar_init(afull_bar(a), GEMM_DEC_WARPS);
            mbar_init(aempty_bar(a), 1);
        }
        mbar_init(accf_bar, 1);
        mbar_init(acce_bar, GEMM_DEC_WARPS);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), GEMM_TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&tmap_b);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int num_units = p.sched[MODE == 0 ? SCHED_UNITS_GU : SCHED_UNITS_DN];
    const int nsplit = p.sched[MODE == 0 ? SCHED_SPLIT_GU : SCHED_SPLIT_DN];
    const int KC = p.M.chunks();
    const size_t expert_bytes = p.M.expert_bytes();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // Warp-uniform loop; one elected lane issues each copy.
        int s = 0;
        uint32_t ph = 0;
        int pend_ph[GEMM_MAX_STAGES];
        for (int i = 0; i < GEMM_MAX_STAGES; ++i) pend_ph[i] = -1;
        bool skip = p.skip_first_copy != 0;
        bool ok = true;
        for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
            const int4 U = p.units[u];
            const int ft = U.w & 0xFFFF, sp = U.w >> 16;
            const int c0 = sp * KC / nsplit, c1 = (sp + 1) * KC / nsplit;
            const int rf = min(128, p.N - ft * 128);
            const uint8_t* we = p.wpack + static_cast<size_t>(U.x) * expert_bytes;
            for (int c = c0; c < c1; ++c) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, p.status, p.timeout_ns));
                if (!ok) break;
                if (skip) {
                    skip = false;  // test hook: this stage is never filled
                } else {
                    const uint32_t wb = static_cast<uint32_t>(p.M.chunk_bytes(c, rf));
                    const int k0 = c * KSTAGE;
                    const bool second = k0 + 64 < p.K;
                    mbar_arrive_expect_tx_warp(full_bar(s), wb + (second ? 2u : 1u) * b_sub);
                    bulk_g2s_warp(w_sm + s * W_STAGE, we + p.M.chunk_offset(ft, c, rf), wb, full_bar(s));
                    tma_load_2d_warp(b_sm + s * b_bytes, &tmap_b, k0, U.y, full_bar(s));
                    if (second) tma_load_2d_warp(b_sm + s * b_bytes + b_sub, &tmap_b, k0 + 64, U.y, full_bar(s));
                    pend_ph[s] = static_cast<int>(ph);
                }
                if (++s == S) { s = 0; ph ^= 1u; }
            }
        }
        // copies still in flight must land before the CTA exits
        if (lane == 0)
            for (int i = 0; i < S; ++i)
                if (pend_ph[i] >= 0) mbar_wait_drain(full_bar(i), static_cast<uint32_t>(pend_ph[i]), 200000000ull);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        // The whole warp runs the loop so descriptors and TMEM addresses stay
        // warp-uniform; elect.sync inside each tcgen05 instruction picks the lane
        // that issues it.  K steps are unrolled with compile-time offsets.
        int s = 0, a = 0;
        uint32_t ph = 0, aph = 0, acc_ph = 0;
        const uint64_t bdesc0 = sw128_kmajor_desc(b_sm);
        const uint32_t dg = tmem + d_col0;
        const uint32_t du = dg + p.BN;
        bool ok = true;
        for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
            const int4 U = p.units[u];
            const int sp = U.w >> 16;
            const int c0 = sp * KC / nsplit, c1 = (sp + 1) * KC / nsplit;
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(acce_bar, acc_ph ^ 1u, abort_flag, p.status, p.timeout_ns));
            if (!ok) break;
            for (int c = c0; c < c1; ++c) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(afull_bar(a), aph, abort_flag, p.status, p.timeout_ns));
                if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), ph, abort_flag, p.status, p.timeout_ns));
                if (!ok) break;
                tc_fence_after();
                const int ksteps = 2 * p.M.blocks_in_chunk(c);
                const uint64_t bd = bdesc0 + ((static_cast<uint64_t>(s) * b_bytes) >> 4);
                const uint32_t acol = tmem + a * A_COLS;
                const uint32_t acc0 = c > c0 ? 1u : 0u;
                const uint64_t bd1 = bd + (b_sub >> 4);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (i < ksteps) {
                        const uint32_t acc = i > 0 ? 1u : acc0;
                        const uint64_t bdi = (i < 4 ? bd : bd1) + 2 * (i & 3);
                        mma_f16_ts_warp(dg, acol + 8 * i, bdi, p.idesc, acc);
                        if (MODE == 0) mma_f16_ts_warp(du, acol + 64 + 8 * i, bdi, p.idesc, acc);
                    }
                }
                tc_commit_warp(aempty_bar(a));
                tc_commit_warp(empty_bar(s));
                if (++s == S) { s = 0; ph ^= 1u; }
                if (++a == NA) { a = 0; aph ^= 1u; }
            }
            if (!ok) break;
            tc_commit_warp(accf_bar);
            acc_ph ^= 1u;
        }
        tc_commit_warp(drain_bar);
        if (lane == 0) mbar_wait_drain(drain_bar, 0, 200000000ull);
        __syncwarp();
    } else {
        // ---------------------------------------------------------- decoders + epilogue
        const int q = warp & 3;               // TMEM lane quadrant (hardware rule: warp % 4)
        const int role = (warp - 2) >> 2;     // 0..3
        // MODE 0: matrix role>>1, blocks 2*(role&1) and 2*(role&1)+1 of each stage;
        // MODE 1: block `role` of each of two consecutive stages.
        const int mat = MODE == 0 ? (role >> 1) : 0;
        const int row = 32 * q + lane;        // weight row within the feature tile
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        constexpr int SPR = MODE == 0 ? 1 : 2;   // stages per decoder round
        int s = 0, a = 0;
        uint32_t ph = 0, aph = 0, acc_ph = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
            const int4 U = p.units[u];
            const int e = U.x, row0 = U.y, nvalid = U.z;
            const int ft = U.w & 0xFFFF, sp = U.w >> 16;
            const int c0 = sp * KC / nsplit, c1 = (sp + 1) * KC / nsplit;
            const int rf = min(128, p.N - ft * 128);
            const bool warp_rows = 32 * q < rf;
            const int n = ft * 128 + row;
            int rs_mine = 127, rs0 = 127, rs1 = 127;
            if (warp_rows) {
                if (MODE == 0) {
                    rs0 = p.rowscale[(static_cast<size_t>(e) * 2 + 0) * p.N + n];
                    rs1 = p.rowscale[(static_cast<size_t>(e) * 2 + 1) * p.N + n];
                    rs_mine = mat ? rs1 : rs0;
                } else {
                    rs0 = p.rowscale[static_cast<size_t>(e) * p.N + n];
                    rs_mine = rs0;
                }
            }
            for (int c = c0; c < c1 && ok; c += SPR) {
                const int g = min(SPR, c1 - c);       // stages this round
                uint4 cw[2];
                int sc[2];
                bool mine[2];
                int aslot[2];
                uint32_t tcol[2];
                // -- read this round's two blocks from shared memory
#pragma unroll
                for (int j = 0; j < SPR; ++j) {
                    if (j >= g) break;
                    const int nbc = p.M.blocks_in_chunk(c + j);
                    if (!__all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), ph, abort_flag, p.status, p.timeout_ns))) {
                        ok = false;
                        break;
                    }
                    const uint8_t* ws = smem_raw + (w_sm + s * W_STAGE - raw) + mat * 17 * nbc * rf;
#pragma unroll
                    for (int t = 0; t < (MODE == 0 ? 2 : 1); ++t) {
                        const int slot = MODE == 0 ? t : j;
                        const int hb = MODE == 0 ? 2 * (role & 1) + t : role;
                        mine[slot] = warp_rows && hb < nbc;
                        cw[slot] = make_uint4(0, 0, 0, 0);
                        sc[slot] = 127;
                        if (mine[slot]) {
                            cw[slot] = *reinterpret_cast<const uint4*>(ws + (hb * rf + row) * 16);
                            sc[slot] = ws[16 * nbc * rf + hb * rf + row];
                        }
                        tcol[slot] = static_cast<uint32_t>(mat * 64 + hb * 16);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(empty_bar(s));
                    if (++s == S) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                // -- claim the A slots
#pragma unroll
                for (int j = 0; j < SPR; ++j) {
                    if (j >= g) break;
                    if (!__all_sync(0xffffffffu, mbar_wait_bounded(aempty_bar(a), aph ^ 1u, abort_flag, p.status, p.timeout_ns))) {
                        ok = false;
                        break;
                    }
                    aslot[j] = a;
                    if (++a == NA) { a = 0; aph ^= 1u; }
                }
                if (!ok) break;
                if (MODE == 0) aslot[1] = aslot[0];
                tc_fence_after();
                // -- decode and store to tensor memory
                if (MODE == 0 && mine[0] && mine[1]) {
                    // the thread's two blocks are adjacent columns of one slot: one x32 store
                    uint32_t r[32];
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const uint32_t m1 = f16_pow2_bits(sc[b] - rs_mine);
                        const uint32_t m2 = m1 | (m1 << 16);
                        e2m1x8_to_f16x8(cw[b].x, m2, r[16 * b + 0], r[16 * b + 1], r[16 * b + 2], r[16 * b + 3]);
                        e2m1x8_to_f16x8(cw[b].y, m2, r[16 * b + 4], r[16 * b + 5], r[16 * b + 6], r[16 * b + 7]);
                        e2m1x8_to_f16x8(cw[b].z, m2, r[16 * b + 8], r[16 * b + 9], r[16 * b + 10], r[16 * b + 11]);
                        e2m1x8_to_f16x8(cw[b].w, m2, r[16 * b + 12], r[16 * b + 13], r[16 * b + 14], r[16 * b + 15]);
                    }
                    tmem_st32(tmem + lane_addr + aslot[0] * A_COLS + tcol[0], r);
                } else
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    if (MODE == 1 && b >= g) break;
                    if (mine[b]) {
                        uint32_t r[16];
                        const uint32_t m1 = f16_pow2_bits(sc[b] - rs_mine);
                        const uint32_t m2 = m1 | (m1 << 16);
                        e2m1x8_to_f16x8(cw[b].x, m2, r[0], r[1], r[2], r[3]);
                        e2m1x8_to_f16x8(cw[b].y, m2, r[4], r[5], r[6], r[7]);
                        e2m1x8_to_f16x8(cw[b].z, m2, r[8], r[9], r[10], r[11]);
                        e2m1x8_to_f16x8(cw[b].w, m2, r[12], r[13], r[14], r[15]);
                        tmem_st16(tmem + lane_addr + aslot[b] * A_COLS + tcol[b], r);
                    }
                }
                if (warp_rows) tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int j = 0; j < SPR; ++j)
                        if (j < g) mbar_arrive(afull_bar(aslot[j]));
                }
            }
            if (!ok) break;

            // ------------------------------------------------------ epilogue
            {
                const bool w_ok = mbar_wait_bounded(accf_bar, acc_ph, abort_flag, p.status, p.timeout_ns);
                if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
            }
            acc_ph ^= 1u;
            tc_fence_after();
            if (warp_rows) {
                const float f0 = pow2f(rs0 - 127);
                const float f1 = pow2f(rs1 - 127);
                for (int col = role * 8; col < p.BN; col += 32) {
                    if (col >= nvalid) break;
                    uint32_t g[8];
                    tmem_ld8(tmem + lane_addr + d_col0 + col, g);
                    if (MODE == 0) {
                        uint32_t v[8];
                        tmem_ld8(tmem + lane_addr + d_col0 + p.BN + col, v);
                        tmem_wait_ld();
                        if (nsplit == 1) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                if (col + j < nvalid) {
                                    const float gg = __uint_as_float(g[j]) * f0;
                                    const float uu = __uint_as_float(v[j]) * f1;
                                    p.H[static_cast<size_t>(row0 + col + j) * p.N + n] = to_half_sat(swish_f(gg) * uu);
                                }
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                if (col + j < nvalid) {
                                    float* gu = p.GU + static_cast<size_t>(row0 + col + j) * 2 * p.N;
                                    atomicAdd(gu + n, __uint_as_float(g[j]) * f0);
                                    atomicAdd(gu + p.N + n, __uint_as_float(v[j]) * f1);
                                }
                            }
                        }
                    } else {
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            if (col + j < nvalid) {
                                const int rr = row0 + col + j;
                                const int t = p.row_token[rr];
                                const float wv = p.row_weight[rr];
                                atomicAdd(p.yacc + static_cast<size_t>(t) * p.N + n, __uint_as_float(g[j]) * f0 * wv);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce_bar);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, GEMM_TMEM_COLS);
    }
}

}  // namespace moe
