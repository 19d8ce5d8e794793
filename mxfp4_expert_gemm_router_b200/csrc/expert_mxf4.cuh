// expert_mxf4.cuh -- grouped expert GEMMs on block-scaled MXFP4 tensor cores.
//
// Method (page "GPT-OSS-20B : Architecture MoE & Résumé du Model Card", §3.2 Les
// Experts): each expert is (Swish(x . W_gate) (.) (x . W_up)) . W_down with
// Swish(z) = z sigma(z); §2.1: the k expert outputs of a token are summed with
// the router weights; §4: the expert weights are MXFP4.
//
// The MMA is tcgen05.mma kind::mxf4 with 32-element block scaling: both
// operands are packed E2M1 in shared memory and every row carries one E8M0
// scale per 32 elements of K, held in tensor memory.  Orientation:
// D[feature, token] = W[feature, :] . X[token, :]^T with M = 128 weight rows
// (output features) as the A operand and N = BN grouped token rows as B.  The
// activations are three MXFP4 terms (mxq.cuh); one MMA per term accumulates
// into the same D, so the tensor core sums the terms.  The weights reach the
// tensor core exactly as stored, with no decode step: one bulk copy per K =
// 128 stage brings codes and scale atoms, a 3-D TMA box {BN rows x 16 B, 3
// terms, 4 blocks} brings the activation codes and a bulk copy their scale
// atoms (one per term).
// tcgen05.cp moves the scale atoms into a ring of tensor-memory slots; fp32
// accumulators stay in tensor memory (two buffers when they fit, so the
// epilogue of one unit overlaps the main loop of the next).
//
//   MODE 0 (gate/up): per stage gate and up chunks (17408 bytes), two
//     accumulators for the same 128 features; epilogue: H = Swish(g) * u for
//     32 tokens x 32 features per warp goes through a small shared-memory tile
//     (fp32, transposed) so that each lane then holds one token's 32-feature
//     block and encodes it as three MXFP4 terms straight into the down GEMM's
//     B operand; with a K split, fp32 partials are added into GU instead (and
//     h_encode_kernel encodes H).
//   MODE 1 (down): per stage the down chunk (8704 bytes), one accumulator;
//     epilogue: the row's weighted output w_row * d, stored once per grouped
//     row (combine_out_kernel sums a token's k rows), or, when K is split,
//     red.add into the fp32 output accumulator.
//
// Persistent kernel: one CTA per SM, units (expert | token tile, first row,
// valid rows, feature tile | K split) taken round-robin from a device-built
// list.  Warp roles: warp 0 TMA producer, warp 1 TMEM allocator and MMA issuer
// (warp-uniform loops, elect.sync issues), warps 2..9 epilogue (warp w reads
// TMEM lanes 32*(w%4).. ; the quarter's two warps alternate groups of token
// columns: 32 for the gate/up encode, 8 otherwise).  Every
// mbarrier wait is bounded; on a timeout the CTA raises an abort flag, all
// roles leave their loops, in-flight copies and MMAs are drained, TMEM is
// freed and the status word reports the timeout.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "mxq.cuh"
#include "quantize.cuh"
#include "routing.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int MXG_EPI_WARPS = 8;
constexpr int MXG_THREADS = (2 + MXG_EPI_WARPS) * 32;
constexpr int MXG_MAX_STAGES = 16;
constexpr int MXG_TMEM_COLS = 512;
constexpr int MXG_SF_COL0 = 448;      // scale-factor ring: MXG_SF_SLOTS slots of 32 columns
constexpr int MXG_SF_SLOTS = 2;       //   [A (gate) 4 | A (up) 4 | B term 0 4 | B term 1 4 | B term 2 4]
constexpr int MXG_SF_SLOT_COLS = 32;
constexpr int MXG_MAX_ACC = 2;
constexpr int MXG_MAX_BN = 128;
constexpr int MXG_MIN_SMEM = 120 * 1024;  // keeps one CTA (and one TMEM owner) per SM

struct MxgParams {
    const uint8_t* wpack;     // tiled MXFP4 weights (quantize.cuh layout)
    const int4* units;        // {expert | token tile << 8, first grouped row, valid rows, feature tile | split << 16}
    const int32_t* sched;
    TiledMatrix M;            // geometry of the (first) matrix streamed
    int N;                    // output features
    int K;                    // contraction length
    int BN;                   // token rows per tile (multiple of 16, at most 128)
    int stages;
    int nacc;                 // accumulator buffers (1 or 2)
    const uint8_t* sfb;       // B operand scale atoms [tiles][K chunks][3][512]
    int stacked;              // 1: the three terms are N = 3 * BN rows of one MMA (3 * BN <= 192)
    uint32_t idesc;           // M = 128, N = BN (or 3 * BN stacked), without scale-factor ids
    GroupedOperand Hd;        // MODE 0 output: H as the down GEMM's B operand
    float* GU;                // MODE 0 split partials [rows][2N]
    float* yacc;              // MODE 1, K split: output accumulator [T][N] (scatter-add)
    void* obuf;               // MODE 1, K not split: weighted output of each grouped row [rows][N], act dtype
    int obuf_bf16;            // obuf element type: 1 bf16, 0 fp32
    const int32_t* row_token; // MODE 1
    const float* row_weight;  // MODE 1
    int* status;
    uint64_t timeout_ns;
    uint32_t skip_first_copy; // test hook: producer skips its first copy
    int n_experts, T, tiles_cap;   // bounds of the unit fields (checked in the debug build)
};

// Debug build: a unit whose fields are out of range is skipped by every role
// (the same decision everywhere, so no wait is left unmatched) and recorded.
__device__ __forceinline__ bool mxg_unit_ok(const MxgParams& p, const int4& U, int nsplit, bool record) {
#ifdef MOE_DEBUG_CHECKS
    const int e = U.x & 0xFF, tile = U.x >> 8, ft = U.w & 0xFFFF, sp = U.w >> 16;
    const bool ok = e < p.n_experts && tile >= 0 && tile < p.tiles_cap && ft < p.M.tiles() && sp < nsplit &&
                    U.y >= 0 && U.z > 0 && U.z <= p.BN && U.y + U.z <= p.Hd.R;
    if (!ok && record) atomicOr(p.status, DEV_BOUNDS);
    return ok;
#else
    (void)p; (void)U; (void)nsplit; (void)record;
    return true;
#endif
}

// Weight bytes per stage (codes of 128 rows x 4 blocks + one scale atom, per
// matrix), B bytes per stage (4 blocks x terms x BN rows x 16 B per 16-byte
// chunk of a block), B scale atoms per stage (one per term), accumulator
// columns (rounded to 32).  AF = 1 (two MXFP8 terms): each matrix's codes land
// padded to 16 KB (16 codes in the low half of every 16 bytes, 128-byte
// swizzle, 1024-byte aligned), the scale atoms follow all the matrices' codes,
// and a stage is a whole number of KB.
__host__ __device__ constexpr int mxg_terms(int af) { return af ? MX8_TERMS : MXQ_TERMS; }
__host__ __device__ constexpr uint32_t mxg_w_stage(int mode, int af = 0) {
    return (mode == 0 ? 2u : 1u) * (af ? 16384u + 512u : 4u * 128 * 16 + 512);
}
__host__ __device__ constexpr uint32_t mxg_b_bytes(int BN, int af = 0) {
    return 4u * (af ? 2u : 1u) * mxg_terms(af) * BN * 16;
}
constexpr uint32_t MXG_SFB_BYTES = 512u * MXQ_TERMS;   // B atoms per (token tile, chunk) in global memory
// Stacked terms: one MMA per K step and matrix, N = terms * BN, reads the weight
// tile from shared memory once (separate per-term MMAs read it once per term,
// which makes shared-memory bandwidth, not the tensor pipe, the limit);
// needs terms * BN <= 192 so that the gate and up accumulators (2 x 192
// columns) and the scale-factor slots fit in tensor memory.
__host__ __device__ constexpr bool mxg_stacked(int BN, int af = 0) { return mxg_terms(af) * BN <= 192; }
// B scale atoms per stage: stacked, the operand rows t * BN + r in one atom per
// 128 rows (one or two); per term, one atom per term.
__host__ __device__ constexpr uint32_t mxg_sfb_stage(int BN, int af = 0) {
    return mxg_stacked(BN, af) ? 512u * ((mxg_terms(af) * BN + 127) / 128) : 512u * mxg_terms(af);
}
__host__ __device__ constexpr uint32_t mxg_stage_bytes(int mode, int BN, int af = 0) {
    return af ? (mxg_w_stage(mode, af) + mxg_b_bytes(BN, af) + mxg_sfb_stage(BN, af) + 1023u) & ~1023u
              : mxg_w_stage(mode, af) + mxg_b_bytes(BN, af) + mxg_sfb_stage(BN, af);
}
__host__ __device__ constexpr int mxg_mat_cols(int BN, int af = 0) {
    return (((mxg_stacked(BN, af) ? mxg_terms(af) : 1) * BN + 31) / 32) * 32;
}
__host__ __device__ constexpr int mxg_acc_cols(int mode, int BN, int af = 0) {
    return (mode == 0 ? 2 : 1) * mxg_mat_cols(BN, af);
}
__host__ inline int mxg_nacc(int mode, int BN, int af = 0) {
    return 2 * mxg_acc_cols(mode, BN, af) <= MXG_SF_COL0 ? 2 : 1;
}
// MODE 0 epilogue tiles: per epilogue warp 32 tokens x 32 features of fp32 H,
// rows padded to 33 so both the row writes and the column reads are
// conflict-free.  fp32 keeps H's full range and precision into the encoder.
constexpr int MXG_HT_STRIDE = 33;
constexpr uint32_t MXG_HT_BYTES = MXG_EPI_WARPS * 32 * MXG_HT_STRIDE * 4;
__host__ __device__ constexpr uint32_t mxg_extra_smem(int mode) { return mode == 0 ? MXG_HT_BYTES : 0u; }
__host__ inline size_t mxg_smem_bytes(int mode, int BN, int stages, int af = 0, int cps = 1) {
    const size_t b = 1024 + static_cast<size_t>(stages) * cps * mxg_stage_bytes(mode, BN, af) +
                     (2 * stages + 2 * MXG_MAX_ACC + 1) * 8 + 64 + mxg_extra_smem(mode);
    return b < static_cast<size_t>(MXG_MIN_SMEM) ? static_cast<size_t>(MXG_MIN_SMEM) : b;
}

// AF = 0: activations as three MXFP4 terms, kind::mxf4 (K = 64 per MMA).
// AF = 1: activations as two MXFP8 terms, kind::mxf8f6f4 (K = 32 per MMA); the
// weights (padded form) arrive through tmap_w, a 16U4_ALIGN16B tensor map
// over the weight array's 8704-byte parts, one 128 x 128 box per matrix and
// stage, and their scale atoms through bulk copies.
// STK: the terms stacked into one MMA (1) or one MMA per term (0).
// CP2 (MODE 1, AF 0, stacked tiles with 3 * BN <= 128): two K chunks per stage.
// SPL = 0: the schedule cannot split K for this launch (the host proves it from
// T), so the split-K epilogue paths are left out.
// Each is its own instantiation: larger loop bodies measurably slowed the
// down GEMM when configurations shared one kernel (the loops of the warp
// roles compete for the instruction cache).
template <int MODE, int AF, int STK, int CP2 = 0, int SPL = 1>
__global__ void __launch_bounds__(MXG_THREADS, 1)
expert_mxf4_kernel(const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_w,
                   const MxgParams p) {
    extern __shared__ uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr uint32_t W_STAGE = mxg_w_stage(MODE, AF);
    constexpr int TERMS = mxg_terms(AF);
    constexpr int NMAT = MODE == 0 ? 2 : 1;

    const int S = p.stages, BN = p.BN, NB3 = TERMS * p.BN;
    const uint32_t b_bytes = mxg_b_bytes(BN, AF);
    const uint32_t sf_bytes = mxg_sfb_stage(BN, AF);               // atoms used per stage
    // a stage holds one K chunk of 128, or two (MODE 1 with cps2): [weights][B codes][B atoms],
    // each region holding the chunks in order
    const uint32_t stage_bytes = mxg_stage_bytes(MODE, BN, AF) * (CP2 ? 2u : 1u);
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t bar0 = base + S * stage_bytes;                 // barriers (8-byte aligned)
    auto w_sm = [&](int s) { return base + s * stage_bytes; };    // stage: weights | B codes | B scale atoms
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    auto accf_bar = [&](int b) { return bar0 + 8u * (2 * S + b); };
    auto acce_bar = [&](int b) { return bar0 + 8u * (2 * S + MXG_MAX_ACC + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * S + 2 * MXG_MAX_ACC);
    uint8_t* ctl = smem_raw + (drain_bar + 8u - raw);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 16);
    float* htile_all = reinterpret_cast<float*>(ctl + 64);     // MODE 0 epilogue tiles
    const int mat_cols = mxg_mat_cols(BN, AF);
    const int acc_cols = (MODE == 0 ? 2 : 1) * mat_cols;
    const int NACC = p.nacc;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);   // the MMA commit of the stage
        }
        for (int b = 0; b < MXG_MAX_ACC; ++b) {
            mbar_init(accf_bar(b), 1);
            mbar_init(acce_bar(b), MXG_EPI_WARPS);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), MXG_TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_b);
        if (AF) prefetch_tmap(&tmap_w);
    }
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // everything above is local set-up; the unit list and the B operand come
    // from the preceding kernels
    pdl_wait();

    const int num_units = p.sched[MODE == 0 ? SCHED_UNITS_GU : SCHED_UNITS_DN];
    const int nsplit = SPL ? p.sched[MODE == 0 ? SCHED_SPLIT_GU : SCHED_SPLIT_DN] : 1;
    const int KC = p.M.chunks();
    const size_t expert_bytes = p.M.expert_bytes();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // Warp-uniform loop; one elected lane issues each copy.
        int s = 0;
        uint32_t ph = 0;
        int pend_ph[MXG_MAX_STAGES];
        for (int i = 0; i < MXG_MAX_STAGES; ++i) pend_ph[i] = -1;
        bool skip = p.skip_first_copy != 0;
        bool ok = true;
        for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
            const int4 U = p.units[u];
            if (!mxg_unit_ok(p, U, nsplit, true)) continue;
            const int e = U.x & 0xFF, tile = U.x >> 8;
            const int ft = U.w & 0xFFFF, sp = U.w >> 16;
            const int c0 = sp * KC / nsplit, c1 = (sp + 1) * KC / nsplit;
            const int rf = min(128, p.N - ft * 128);
            const uint8_t* we = p.wpack + static_cast<size_t>(e) * expert_bytes;
            for (int c = c0; c < c1; ++c) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, p.status, p.timeout_ns));
                if (!ok) break;
                if (skip) {
                    skip = false;  // test hook: this stage is never filled
                } else if (AF) {
                    // per matrix: the 128 x 128 code box (8192 global bytes, padded to
                    // 16 KB in shared memory) and its scale atom
                    const uint32_t st = w_sm(s);
                    mbar_arrive_expect_tx_warp(full_bar(s), NMAT * (8192u + 512u) + b_bytes + sf_bytes);
                    const size_t off = static_cast<size_t>(e) * expert_bytes + p.M.chunk_offset(ft, c, rf);
                    const int part = static_cast<int>(off / TiledMatrix::PAD_MAT);
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) {
                        tma_load_3d_warp(st + 16384u * m, &tmap_w, 0, 0, part + m, full_bar(s));
                        bulk_g2s_warp(st + 16384u * NMAT + 512u * m, p.wpack + off + m * TiledMatrix::PAD_MAT + 8192,
                                      512u, full_bar(s));
                    }
                    // rows U.y .. U.y + BN - 1 of every (16-byte chunk, term)
                    tma_load_3d_warp(st + W_STAGE, &tmap_b, 2 * U.y, 0, 8 * c, full_bar(s));
                    bulk_g2s_warp(st + W_STAGE + b_bytes, p.sfb + (static_cast<size_t>(tile) * KC + c) * MXG_SFB_BYTES,
                                  sf_bytes, full_bar(s));
                    pend_ph[s] = static_cast<int>(ph);
                } else if (CP2) {
                    // chunks c and c + 1 of the feature tile are adjacent (chunk c is full)
                    const int nch = min(2, c1 - c);
                    const uint32_t st = w_sm(s);
                    uint32_t wb = 0;
                    for (int j = 0; j < nch; ++j) wb += static_cast<uint32_t>(p.M.chunk_bytes(c + j, rf));
                    mbar_arrive_expect_tx_warp(full_bar(s), wb + nch * (b_bytes + sf_bytes));
                    bulk_g2s_warp(st, we + p.M.chunk_offset(ft, c, rf), wb, full_bar(s));
                    for (int j = 0; j < nch; ++j) {
                        tma_load_3d_warp(st + 2 * W_STAGE + j * b_bytes, &tmap_b, 2 * U.y, 0, 4 * (c + j), full_bar(s));
                        bulk_g2s_warp(st + 2 * W_STAGE + 2 * b_bytes + j * sf_bytes,
                                      p.sfb + (static_cast<size_t>(tile) * KC + c + j) * MXG_SFB_BYTES, sf_bytes,
                                      full_bar(s));
                    }
                    pend_ph[s] = static_cast<int>(ph);
                } else {
                    const uint32_t wb = static_cast<uint32_t>(p.M.chunk_bytes(c, rf));
                    const uint32_t st = w_sm(s);
                    mbar_arrive_expect_tx_warp(full_bar(s), wb + b_bytes + sf_bytes);
                    bulk_g2s_warp(st, we + p.M.chunk_offset(ft, c, rf), wb, full_bar(s));
                    // rows U.y .. U.y + BN - 1 of every (block, term): 8-byte elements 2 * U.y ..
                    tma_load_3d_warp(st + W_STAGE, &tmap_b, 2 * U.y, 0, 4 * c, full_bar(s));
                    bulk_g2s_warp(st + W_STAGE + b_bytes, p.sfb + (static_cast<size_t>(tile) * KC + c) * MXG_SFB_BYTES,
                                  sf_bytes, full_bar(s));
                    pend_ph[s] = static_cast<int>(ph);
                }
                if (++s == S) { s = 0; ph ^= 1u; }
                if (CP2) ++c;   // the stage took chunk c + 1 as well
            }
        }
        // copies still in flight must land before the CTA exits
        if (lane == 0)
            for (int i = 0; i < S; ++i)
                if (pend_ph[i] >= 0) mbar_wait_drain(full_bar(i), static_cast<uint32_t>(pend_ph[i]), 200000000ull);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        // Per stage: scale atoms to the next tensor-memory slot, then one MMA
        // per matrix for each pair of 32-blocks (K = 64), scale-factor id 0 or 2.
        int s = 0, sfs = 0, buf = 0;
        uint32_t ph = 0;
        uint32_t eph[MXG_MAX_ACC] = {0u, 0u};
        bool ok = true;
        for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
            const int4 U = p.units[u];
            if (!mxg_unit_ok(p, U, nsplit, false)) continue;
            const int ft = U.w & 0xFFFF, sp = U.w >> 16;
            const int c0 = sp * KC / nsplit, c1 = (sp + 1) * KC / nsplit;
            const int rf = min(128, p.N - ft * 128);
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(acce_bar(buf), eph[buf] ^ 1u, abort_flag, p.status, p.timeout_ns));
            if (!ok) break;
            eph[buf] ^= 1u;
            tc_fence_after();
            const uint32_t d0 = tmem + static_cast<uint32_t>(buf * acc_cols);
            for (int c = c0; c < c1; ++c) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), ph, abort_flag, p.status, p.timeout_ns));
                if (!ok) break;
                tc_fence_after();
                const int nbc = p.M.blocks_in_chunk(c);
                if constexpr (AF == 1) {
                    // one MMA per block (K = 32, scale byte i); A from the padded,
                    // swizzled 16 KB tile of each matrix, B [8 chunks][2 terms][BN][16 B]
                    const uint32_t ws = w_sm(s), bs = ws + W_STAGE, ss = bs + b_bytes;
                    const uint32_t wsf = ws + 16384u * NMAT;
                    const uint32_t sfc = tmem + MXG_SF_COL0 + MXG_SF_SLOT_COLS * sfs;
                    tc_cp_sf_warp(sfc, desc_noswz(wsf, 0, 128));
                    if (MODE == 0) tc_cp_sf_warp(sfc + 4, desc_noswz(wsf + 512, 0, 128));
                    if constexpr (STK != 0) {
                        tc_cp_sf_warp(sfc + 8, desc_noswz(ss, 0, 128));
                        if (NB3 > 128) tc_cp_sf_warp(sfc + 12, desc_noswz(ss + 512, 0, 128));
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            if (i < nbc) {
                                const uint32_t acc = (c > c0 || i > 0) ? 1u : 0u;
                                const uint32_t id = p.idesc | idesc_sf_ids(static_cast<uint32_t>(i));
                                const uint64_t bd = desc_noswz(bs + 2 * i * NB3 * 16, NB3 * 16, 128);
                                mma_mxf8f6f4_warp(d0, desc_sw128(ws + 32 * i), bd, id, sfc, sfc + 8, acc);
                                if (MODE == 0)
                                    mma_mxf8f6f4_warp(d0 + mat_cols, desc_sw128(ws + 16384 + 32 * i), bd, id, sfc + 4,
                                                      sfc + 8, acc);
                            }
                        }
                    } else {
#pragma unroll
                        for (int t = 0; t < TERMS; ++t) tc_cp_sf_warp(sfc + 8 + 4 * t, desc_noswz(ss + 512 * t, 0, 128));
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            if (i < nbc) {
                                const uint32_t id = p.idesc | idesc_sf_ids(static_cast<uint32_t>(i));
#pragma unroll
                                for (int t = 0; t < TERMS; ++t) {
                                    const uint32_t acc = (c > c0 || i > 0 || t > 0) ? 1u : 0u;
                                    const uint64_t bd = desc_noswz(bs + (2 * i * TERMS + t) * BN * 16, NB3 * 16, 128);
                                    mma_mxf8f6f4_warp(d0, desc_sw128(ws + 32 * i), bd, id, sfc, sfc + 8 + 4 * t, acc);
                                    if (MODE == 0)
                                        mma_mxf8f6f4_warp(d0 + mat_cols, desc_sw128(ws + 16384 + 32 * i), bd, id,
                                                          sfc + 4, sfc + 8 + 4 * t, acc);
                                }
                            }
                        }
                    }
                    tc_commit_warp(empty_bar(s));
                    if (++s == S) { s = 0; ph ^= 1u; }
                    if (++sfs == MXG_SF_SLOTS) sfs = 0;
                    continue;
                }
                if constexpr (CP2 != 0) {
                    // two K chunks per stage; tensor-memory columns: A atom of chunk j
                    // at 4 j, B atom of chunk j at 8 + 4 j (3 * BN <= 128: one atom each)
                    const int nch = min(2, c1 - c);
                    const uint32_t ws = w_sm(s), bs = ws + 2 * W_STAGE, ss = bs + 2 * b_bytes;
                    const uint32_t sfc = tmem + MXG_SF_COL0 + MXG_SF_SLOT_COLS * sfs;
                    uint32_t wj = ws;
                    for (int j = 0; j < nch; ++j) {
                        const int nbj = p.M.blocks_in_chunk(c + j);
                        const uint32_t cb = static_cast<uint32_t>(nbj * rf * 16);
                        tc_cp_sf_warp(sfc + 4 * j, desc_noswz(wj + cb, 0, 128));
                        tc_cp_sf_warp(sfc + 8 + 4 * j, desc_noswz(ss + j * sf_bytes, 0, 128));
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            if (2 * i < nbj) {
                                const uint32_t acc = (c > c0 || j > 0 || i > 0) ? 1u : 0u;
                                const uint32_t id = p.idesc | idesc_sf_ids(2u * i);
                                const uint64_t ad = desc_noswz(wj + 2 * i * rf * 16, rf * 16, 128);
                                const uint64_t bd = desc_noswz(bs + j * b_bytes + 2 * i * NB3 * 16, NB3 * 16, 128);
                                mma_mxf4_warp(d0, ad, bd, id, sfc + 4 * j, sfc + 8 + 4 * j, acc);
                            }
                        }
                        wj += cb + 512u;
                    }
                    tc_commit_warp(empty_bar(s));
                    if (++s == S) { s = 0; ph ^= 1u; }
                    if (++sfs == MXG_SF_SLOTS) sfs = 0;
                    ++c;   // the stage held chunk c + 1 as well
                    continue;
                }
                const uint32_t codes_b = static_cast<uint32_t>(nbc * rf * 16);
                const uint32_t mat_b = codes_b + 512u;
                const uint32_t ws = w_sm(s), bs = ws + W_STAGE, ss = bs + b_bytes;
                const uint32_t sfc = tmem + MXG_SF_COL0 + MXG_SF_SLOT_COLS * sfs;
                tc_cp_sf_warp(sfc, desc_noswz(ws + codes_b, 0, 128));
                if (MODE == 0) tc_cp_sf_warp(sfc + 4, desc_noswz(ws + mat_b + codes_b, 0, 128));
                if constexpr (STK != 0) {
                    // one MMA per K step and matrix: N = 3 * BN rows (term-major); the B
                    // scales of rows 0..127 in columns 8..11, of rows 128.. in 12..15
                    tc_cp_sf_warp(sfc + 8, desc_noswz(ss, 0, 128));
                    if (NB3 > 128) tc_cp_sf_warp(sfc + 12, desc_noswz(ss + 512, 0, 128));
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if (2 * i < nbc) {
                            const uint32_t acc = (c > c0 || i > 0) ? 1u : 0u;
                            const uint32_t id = p.idesc | idesc_sf_ids(2u * i);
                            const uint64_t ad = desc_noswz(ws + 2 * i * rf * 16, rf * 16, 128);
                            const uint64_t bd = desc_noswz(bs + 2 * i * NB3 * 16, NB3 * 16, 128);
                            mma_mxf4_warp(d0, ad, bd, id, sfc, sfc + 8, acc);
                            if (MODE == 0) mma_mxf4_warp(d0 + mat_cols, ad + (mat_b >> 4), bd, id, sfc + 4, sfc + 8, acc);
                        }
                    }
                } else {
#pragma unroll
                    for (int t = 0; t < MXQ_TERMS; ++t) tc_cp_sf_warp(sfc + 8 + 4 * t, desc_noswz(ss + 512 * t, 0, 128));
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if (2 * i < nbc) {
                            const uint32_t id = p.idesc | idesc_sf_ids(2u * i);
                            const uint64_t ad = desc_noswz(ws + 2 * i * rf * 16, rf * 16, 128);
#pragma unroll
                            for (int t = 0; t < MXQ_TERMS; ++t) {
                                // B of term t, blocks 2i and 2i+1: smem [block][term][row][16 B]
                                const uint32_t acc = (c > c0 || i > 0 || t > 0) ? 1u : 0u;
                                const uint64_t bd = desc_noswz(bs + (2 * i * MXQ_TERMS + t) * BN * 16, NB3 * 16, 128);
                                mma_mxf4_warp(d0, ad, bd, id, sfc, sfc + 8 + 4 * t, acc);
                                if (MODE == 0)
                                    mma_mxf4_warp(d0 + mat_cols, ad + (mat_b >> 4), bd, id, sfc + 4, sfc + 8 + 4 * t, acc);
                            }
                        }
                    }
                }
                tc_commit_warp(empty_bar(s));
                if (++s == S) { s = 0; ph ^= 1u; }
                if (++sfs == MXG_SF_SLOTS) sfs = 0;
            }
            if (!ok) break;
            tc_commit_warp(accf_bar(buf));
            if (++buf == NACC) buf = 0;
        }
        tc_commit_warp(drain_bar);
        if (lane == 0) mbar_wait_drain(drain_bar, 0, 200000000ull);
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;               // TMEM lane quarter (hardware rule: warp % 4)
        const int hh = (warp - 2) >> 2;       // which groups of 8 token columns
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        int buf = 0;
        uint32_t fph[MXG_MAX_ACC] = {0u, 0u};
        bool ok = true;
        for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
            const int4 U = p.units[u];
            if (!mxg_unit_ok(p, U, nsplit, false)) continue;
            const int tile = U.x >> 8, row0 = U.y, nvalid = U.z;
            const int ft = U.w & 0xFFFF;
            const int rf = min(128, p.N - ft * 128);
            const bool warp_rows = 32 * q < rf;
            const int n = ft * 128 + 32 * q + lane;
            {
                const bool w_ok = mbar_wait_bounded(accf_bar(buf), fph[buf], abort_flag, p.status, p.timeout_ns);
                if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
            }
            fph[buf] ^= 1u;
            tc_fence_after();
            bool released = false;   // the accumulator went back to the MMA warp early
            if (warp_rows) {
                const uint32_t d0 = tmem + lane_addr + static_cast<uint32_t>(buf * acc_cols);
                // accumulators of token columns r0 .. r0 + 7 for this lane's feature
                auto load8 = [&](int r0, float (&gs)[8], float (&us)[8]) {
                    if constexpr (STK != 0) {
                        // the term columns of each token are BN apart: add them
                        uint32_t g[TERMS][8], v[TERMS][8];
#pragma unroll
                        for (int t = 0; t < TERMS; ++t) {
                            tmem_ld8(d0 + t * BN + r0, g[t]);
                            if (MODE == 0) tmem_ld8(d0 + mat_cols + t * BN + r0, v[t]);
                        }
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            float a = 0.f, b = 0.f;
#pragma unroll
                            for (int t = 0; t < TERMS; ++t) {
                                a += __uint_as_float(g[t][j]);
                                if (MODE == 0) b += __uint_as_float(v[t][j]);
                            }
                            gs[j] = a;
                            us[j] = b;
                        }
                    } else {
                        uint32_t g[8], v[8];
                        tmem_ld8(d0 + r0, g);
                        if (MODE == 0) tmem_ld8(d0 + mat_cols + r0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            gs[j] = __uint_as_float(g[j]);
                            us[j] = MODE == 0 ? __uint_as_float(v[j]) : 0.f;
                        }
                    }
                };
                if (MODE == 0 && nsplit == 1) {
                    // Groups of 32 tokens alternate between the quarter's two warps
                    // (at most two groups each, BN <= 128).  First H of both groups
                    // is read out of the accumulator into registers, which then goes
                    // back to the MMA warp; the transposes and the encodes of H run
                    // while the next unit's MMAs do.
                    float hreg[2][32];
#pragma unroll
                    for (int gi = 0; gi < 2; ++gi) {
                        const int g0 = 32 * hh + 64 * gi;
#pragma unroll
                        for (int s8 = 0; s8 < 32; s8 += 8) {
                            if (g0 + s8 < nvalid) {
                                float gs[8], us[8];
                                load8(g0 + s8, gs, us);
#pragma unroll
                                for (int j = 0; j < 8; ++j) hreg[gi][s8 + j] = swish_f(gs[j]) * us[j];
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(acce_bar(buf));
                    released = true;
                    float* ht = htile_all + (warp - 2) * 32 * MXG_HT_STRIDE;
                    const int blk = 4 * ft + q;
                    uint8_t* atoms = scale_atom_base(p.Hd, tile, ft);
#pragma unroll
                    for (int gi = 0; gi < 2; ++gi) {
                        const int g0 = 32 * hh + 64 * gi;
                        if (g0 >= nvalid) break;
#pragma unroll
                        for (int c = 0; c < 32; ++c) ht[c * MXG_HT_STRIDE + lane] = hreg[gi][c];
                        __syncwarp();
                        const int r = g0 + lane;   // this lane's token: one 32-feature block of H
                        if (r < nvalid) {
                            float hv[32];
#pragma unroll
                            for (int c = 0; c < 32; ++c) hv[c] = ht[lane * MXG_HT_STRIDE + c];
                            uint32_t sb[MXQ_TERMS];
                            act_encode_store<AF>(hv, p.Hd.codes, p.Hd.R, blk, row0 + r, sb);
#pragma unroll
                            for (int t = 0; t < TERMS; ++t)
                                atoms[sf_atom_offset(t * p.Hd.term_rows + r, q)] = static_cast<uint8_t>(sb[t]);
                        }
                        __syncwarp();
                    }
                } else {
                    for (int r0 = 8 * hh; r0 < nvalid; r0 += 16) {
                        float gs[8], us[8];
                        load8(r0, gs, us);
                        const int nv = min(8, nvalid - r0);   // valid token columns in this group (warp-uniform)
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            if (j < nv) {
                                const int rr = row0 + r0 + j;
                                if (MODE == 0) {
                                    float* gu = p.GU + static_cast<size_t>(rr) * 2 * p.N;
                                    atomicAdd(gu + n, gs[j]);
                                    atomicAdd(gu + p.N + n, us[j]);
                                } else if (nsplit > 1) {
                                    const int tok = p.row_token[rr];
                                    if (MOE_IN_BOUNDS(tok >= 0 && tok < p.T, p.status))
                                        atomicAdd(p.yacc + static_cast<size_t>(tok) * p.N + n, gs[j] * p.row_weight[rr]);
                                } else {
                                    // the row's whole output: stored once, summed per token by the combine
                                    const float o = gs[j] * p.row_weight[rr];
                                    if (p.obuf_bf16)
                                        static_cast<__nv_bfloat16*>(p.obuf)[static_cast<size_t>(rr) * p.N + n] =
                                            __float2bfloat16_rn(o);
                                    else
                                        static_cast<float*>(p.obuf)[static_cast<size_t>(rr) * p.N + n] = o;
                                }
                            }
                        }
                    }
                }
            }
            if (!released) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acce_bar(buf));
            }
            if (++buf == NACC) buf = 0;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, MXG_TMEM_COLS);
    }
}

}  // namespace moe
