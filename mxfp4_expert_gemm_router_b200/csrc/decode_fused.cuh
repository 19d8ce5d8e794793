// decode_fused.cuh -- the whole layer in one persistent, cooperative launch
// for small batches (T <= 16 tokens).
//
// Method (page "GPT-OSS-20B : Architecture MoE & Résumé du Model Card"):
// §3.1 Le Routeur (scores = W_router . h, top-k, softmax over the selected
// scores), §3.2 Les Experts (SwiGLU FFN per selected expert), §2.1 (the k
// expert outputs summed with the routing weights), §4 (MXFP4 weights); with
// the optional pre-norm (page "GPT-OSS vs Qwen3 : comparaison détaillée",
// Adoption de RMSNorm) and the residual around the block.
//
// At decode sizes the layer is the weight stream of the touched experts (a
// few to a few tens of microseconds on B200); a chain of launches spends as
// long again in launch gaps, ramps and tails.  This kernel runs every step in
// one grid of one CTA per SM, all resident (cooperative launch):
//
//  1. Router, split over the grid: CTA b computes partial scores for
//     (expert, K split) units -- fp32 within 64-wide K chunks, fp64 across --
//     and the partial sums of x^2 for the pre-norm.  One grid barrier; then
//     every CTA sums the partials in split order (identical results in every
//     CTA), applies the RMS scaling and the bias, takes the top-k (warp
//     arg-max rounds, ties to the lower index) and the softmax, and lists the
//     touched experts in ascending order.
//  2. The B operand is every token of the batch (16 rows per term, the three
//     MXFP4 terms stacked: N = 48) for every expert.  Columns of tokens not
//     routed to an expert are computed and dropped: next to the weight stream
//     the MMA work is negligible, and one B operand for the whole K replaces
//     the grouping and the gather.  The grid encodes it once (each CTA a
//     share of the (block, token) items, into global memory); each CTA then
//     bulk-copies it into shared memory when every share is written.
//  3. Gate/up work comes in whole feature tiles (128 features of one touched
//     expert over all of K, gate and up: 23 chunks of 17,408 bytes at the
//     2880-wide shape), dealt round-robin over the CTAs; a CTA accumulates a
//     tile in tensor memory and its epilogue forms H = Swish(g) u for the
//     tokens routed to the expert straight from the accumulator, encodes it
//     as three MXFP4 terms (one 32-feature block per warp, one element per
//     lane) into the expert's H operand in global memory, and stamps the tile
//     with the launch's epoch.  Down work comes in items of two consecutive K
//     chunks of one feature tile of the down matrix (at most 17,408 bytes),
//     dealt in contiguous ranges sized so that every CTA streams the same
//     total number of bytes; a run of down items of the same (expert, tile) is
//     a piece.
//  4. A down piece over d_ff chunks [c0, c1) waits (bounded) for the stamps
//     of gate/up feature tiles c0 .. c1-1, bulk-copies that range of the
//     expert's H operand into shared memory, and the MMA warp runs.  Down
//     weight copies never wait: the producer streams them into the ring while
//     other CTAs finish their gate/up tiles.
//  5. Down epilogue: y_acc[t] += w[t, e] D[., t] for the tokens routed to e
//     (red.add).  The last CTA to finish writes y (cast; + x with the
//     residual).
//
// State across launches (epoch, grid-barrier and x-operand arrival counts)
// lives in device memory; every CTA arrives at each count exactly once per
// launch, so targets are (epoch + 1) * gridDim.x and nothing is reset.  The
// output accumulator alternates by the epoch's parity: each launch clears the
// other parity, so the buffer a launch accumulates into is always clear.
// Every wait (mbarrier phases, the grid barrier, the counts, the stamps) is
// bounded; on a timeout the CTA raises its abort flag and the status word,
// all roles leave their loops, copies and MMAs in flight are drained and the
// tensor memory is freed.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "mxq.cuh"
#include "quantize.cuh"
#include "routing.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int DF_MAX_T = 16;                 // token rows per term of the B operand
constexpr int DF_NB3 = MXQ_TERMS * DF_MAX_T; // 48 operand rows
constexpr int DF_EPI_WARPS = 8;
// warps: 0 weight producer, 1 MMA issuer, 2..9 epilogue, 10 H-operand issuer
constexpr int DF_HWARP = 2 + DF_EPI_WARPS;
constexpr int DF_THREADS = (3 + DF_EPI_WARPS) * 32;
constexpr int DF_EPI_THREADS = DF_EPI_WARPS * 32;
constexpr uint32_t DF_STAGE = 2u * (4u * 128 * 16 + 512);   // 17,408 bytes
constexpr int DF_MAX_STAGES = 8;
constexpr int DF_MAT_COLS = 64;              // accumulator columns per matrix (48 used)
constexpr int DF_ACC_COLS = 2 * DF_MAT_COLS; // gate and up
constexpr int DF_SF_COL0 = 448;
constexpr int DF_SF_SLOTS = 2;
constexpr int DF_SF_SLOT_COLS = 32;
constexpr uint32_t DF_B_BLOCK = DF_NB3 * 16;  // 768 bytes of B codes per 32-block
constexpr int DF_MAX_TOUCHED = DF_MAX_T * MAX_TOPK;   // touched experts <= T * k
// H ring slot of one down item (two K chunks): codes [2][4 blocks][48][16 B], then two scale atoms
constexpr uint32_t DF_HSLOT_CODES = 2u * 4u * DF_B_BLOCK;   // 6144
constexpr uint32_t DF_HSLOT = DF_HSLOT_CODES + 2u * 512u;   // 7168

struct DecodeState {
    uint32_t bar;      // grid-barrier arrivals: grows by gridDim.x per launch
    uint32_t epoch;    // launches completed
    uint32_t finish;   // CTAs finished in the current launch
    uint32_t xdone;    // CTAs that wrote their share of x's operand: grows by gridDim.x per launch
    uint32_t pad[4];
};

struct DecodeParams {
    const void* x;          // [T][d] act dtype
    void* y;                // [T][d] act dtype
    const void* wr;         // [E][d] act dtype
    const float* bias;      // [E] or null
    const float* gamma;     // [d] or null (no pre-norm)
    float eps;
    int residual;
    int T, d, f, E, k;
    TiledMatrix Mgu;        // gate + up (N = f, K = d), expert 0 at base
    TiledMatrix Mdn;        // down (N = d, K = f)
    int S;                  // router K splits
    int stages;             // weight-ring stages
    int nb_max;             // 32-blocks of the B buffer: max(d, f) / 32
    int kc_max;             // K chunks of the B buffer: max over both GEMMs
    DecodeState* st;
    double* part;           // [S][16][E] partial scores
    double* part_ss;        // [S][16] partial sums of x^2
    float* yacc;            // [2][16][d]
    uint8_t* xq;            // x as the B operand: codes [d/32][48][16 B], then scale atoms [KC_gu][512]
    uint8_t* hq;            // H per touched slot (stride hq_stride): codes [f/32][48][16 B], atoms [KC_dn][512]
    size_t hq_stride;
    uint32_t* hdone;        // [max_touched][F_gu][8] epoch + 1 once epilogue warp w wrote its part of the tile's H
    int32_t* topk_idx;      // [T][k] or null
    float* topk_w;          // [T][k] or null
    int32_t* counts;        // [E] or null
    int* status;
    uint64_t timeout_ns;
    uint32_t skip_first_copy;   // test hook: each producer skips its first copy
};

// Shared memory after the 1024-aligned weight ring and B buffer.
struct DecodeCtl {
    uint64_t full[DF_MAX_STAGES], empty[DF_MAX_STAGES];
    uint64_t hfull[DF_MAX_STAGES], hempty[DF_MAX_STAGES];
    uint64_t accf[2], acce[2], xready, xfree, drain;
    int abort_flag;
    uint32_t tmem;
    int last;
    int n_t;
    double inv_rms[DF_MAX_T];
    int tok_e[DF_MAX_T][MAX_TOPK];
    float tok_w[DF_MAX_T][MAX_TOPK];
    int slot_of[MAX_EXPERTS];
    int touched[DF_MAX_TOUCHED];
    float selw[DF_MAX_TOUCHED][DF_MAX_T];   // routing weight of token t for touched slot i (0: not routed)
};

__host__ __device__ inline uint32_t df_bbuf_bytes(int nb_max, int kc_max) {
    return static_cast<uint32_t>(nb_max) * DF_B_BLOCK + static_cast<uint32_t>(kc_max) * 512u;
}
// The B buffer holds x's operand during the gate/up work and the H ring (one
// slot per weight stage) during the down work.
__host__ __device__ inline uint32_t df_bregion_bytes(int stages, int nb_max, int kc_max) {
    const uint32_t a = df_bbuf_bytes(nb_max, kc_max), b = static_cast<uint32_t>(stages) * DF_HSLOT;
    return a > b ? a : b;
}
__host__ inline size_t df_smem_bytes(int stages, int nb_max, int kc_max) {
    return 1024 + static_cast<size_t>(stages) * DF_STAGE + df_bregion_bytes(stages, nb_max, kc_max) +
           sizeof(DecodeCtl) + 16;
}

// Bytes of the down item j (chunks 2j and 2j+1 of feature tile ft): contiguous in the tiled layout.
__device__ __forceinline__ uint32_t df_down_item_bytes(const TiledMatrix& M, int j, int rf) {
    const int c = 2 * j;
    uint32_t b = static_cast<uint32_t>(M.mat_bytes(c, rf));
    if (c + 1 < M.chunks()) b += static_cast<uint32_t>(M.mat_bytes(c + 1, rf));
    return b;
}

template <typename TA>
__global__ void __launch_bounds__(DF_THREADS, 1) decode_fused_kernel(const DecodeParams p) {
    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    const int T = p.T, d = p.d, f = p.f, E = p.E, k = p.k;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    const uint32_t ring = base;
    const uint32_t bbuf = base + static_cast<uint32_t>(p.stages) * DF_STAGE;      // B codes
    const uint32_t bsf = bbuf + static_cast<uint32_t>(p.nb_max) * DF_B_BLOCK;    // B scale atoms
    uint8_t* bbuf_ptr = base_ptr + static_cast<size_t>(p.stages) * DF_STAGE;
    DecodeCtl& C = *reinterpret_cast<DecodeCtl*>(bbuf_ptr + df_bregion_bytes(p.stages, p.nb_max, p.kc_max));
    volatile int* abort_flag = &C.abort_flag;
    const int S = p.stages;
    auto full_bar = [&](int s) { return smem_u32(&C.full[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&C.empty[s]); };

    const int F_gu = p.Mgu.tiles(), KC_gu = p.Mgu.chunks();
    const int F_dn = p.Mdn.tiles(), KC_dn = p.Mdn.chunks();
    const int NP = (KC_dn + 1) / 2;   // down items per feature tile
    const bool norm = p.gamma != nullptr;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&C.accf[b]), 1);
            mbar_init(smem_u32(&C.acce[b]), DF_EPI_WARPS);
        }
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&C.hfull[s]), 1);
            mbar_init(smem_u32(&C.hempty[s]), 1);   // the MMA commit of the H slot
        }
        mbar_init(smem_u32(&C.xready), 1);
        mbar_init(smem_u32(&C.xfree), 1);
        mbar_init(smem_u32(&C.drain), 1);
        C.abort_flag = 0;
        C.last = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&C.tmem), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = C.tmem;
    const uint32_t epoch = ld_acquire_u32(&p.st->epoch);
    const int par = static_cast<int>(epoch & 1u);
    float* yacc = p.yacc + static_cast<size_t>(par) * DF_MAX_T * d;

    // ---- clear the other parity's output accumulator (nothing in this launch
    // touches it; the next launch accumulates into it)
    {
        float4* y_other = reinterpret_cast<float4*>(p.yacc + static_cast<size_t>(1 - par) * DF_MAX_T * d);
        const long y4 = static_cast<long>(DF_MAX_T) * d / 4;
        for (long i = static_cast<long>(blockIdx.x) * DF_THREADS + tid; i < y4; i += static_cast<long>(G) * DF_THREADS)
            y_other[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // ---- this CTA's share of x's B operand (every token row, 16 per term; rows
    // past T are zero), written to global memory; xdone tells the grid.  x does
    // not depend on the routing: without the pre-norm the share is written
    // first, so the operand is complete by the time the routing is; with it
    // the share waits for the RMS of each token.
    const int nb_d = d / 32, nb_f = f / 32;
    auto x_share = [&](int first, int stride) {
        uint8_t* xcodes = p.xq;
        uint8_t* xatoms = p.xq + static_cast<size_t>(nb_d) * DF_B_BLOCK;
        const int items = nb_d * DF_MAX_T;
        const int i0 = static_cast<int>(static_cast<long>(items) * blockIdx.x / G);
        const int i1 = static_cast<int>(static_cast<long>(items) * (blockIdx.x + 1) / G);
        for (int itm = i0 + first; itm < i1; itm += stride) {
            const int b = itm / DF_MAX_T, t = itm % DF_MAX_T;
            uint4 codes[MXQ_TERMS] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u),
                                      make_uint4(0u, 0u, 0u, 0u)};
            uint32_t sb[MXQ_TERMS] = {0u, 0u, 0u};
            if (t < T) {
                float v[32];
                BlockLoader<TA>::load(static_cast<const TA*>(p.x) + static_cast<size_t>(t) * d + b * 32, v);
                if (norm) {
                    const float r = static_cast<float>(C.inv_rms[t]);
                    const float4* g4 = reinterpret_cast<const float4*>(p.gamma + b * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 g = g4[i];
                        v[4 * i] *= g.x * r;
                        v[4 * i + 1] *= g.y * r;
                        v[4 * i + 2] *= g.z * r;
                        v[4 * i + 3] *= g.w * r;
                    }
                }
                mxq_block_thread(v, codes, sb);
            }
#pragma unroll
            for (int tt = 0; tt < MXQ_TERMS; ++tt) {
                *reinterpret_cast<uint4*>(xcodes + (static_cast<size_t>(b) * DF_NB3 + tt * DF_MAX_T + t) * 16) =
                    codes[tt];
                xatoms[(b >> 2) * 512 + sf_atom_offset(tt * DF_MAX_T + t, b & 3)] = static_cast<uint8_t>(sb[tt]);
            }
        }
    };
    if (!norm) {
        x_share(tid, DF_THREADS);
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            atomicAdd(&p.st->xdone, 1u);
        }
    }

    // ---- 1. router partials over (expert, K split) units
    const TA* x = static_cast<const TA*>(p.x);
    const TA* wr = static_cast<const TA*>(p.wr);
    const int KCH = (d + ROUTER_KCHUNK - 1) / ROUTER_KCHUNK;
    {
        double* scratch = reinterpret_cast<double*>(base_ptr);   // the ring is free until the producer starts
        double* scratch_ss = scratch + DF_MAX_T * KCH;
        for (int u = blockIdx.x; u < E * p.S; u += G) {
            const int e = u / p.S, sp = u % p.S;
            const int j0 = sp * KCH / p.S, j1 = (sp + 1) * KCH / p.S, nj = j1 - j0;
            for (int it = tid; it < T * nj; it += DF_THREADS) {
                const int t = it / nj, j = j0 + it % nj;
                float acc = 0.f, sq = 0.f;
#pragma unroll
                for (int g8 = 0; g8 < ROUTER_KCHUNK / 8; ++g8) {
                    const int kk = j * ROUTER_KCHUNK + g8 * 8;
                    if (kk < d) {
                        Raw8<TA> xr, wv;
                        xr.load(x + static_cast<size_t>(t) * d + kk);
                        wv.load(wr + static_cast<size_t>(e) * d + kk);
                        if (norm) {
                            const float4 g0 = *reinterpret_cast<const float4*>(p.gamma + kk);
                            const float4 g1 = *reinterpret_cast<const float4*>(p.gamma + kk + 4);
                            const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float xv = xr.get(q);
                                sq = fmaf(xv, xv, sq);
                                acc = fmaf(xv * gv[q], wv.get(q), acc);
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; ++q) acc = fmaf(xr.get(q), wv.get(q), acc);
                        }
                    }
                }
                scratch[t * nj + (j - j0)] = static_cast<double>(acc);
                scratch_ss[t * nj + (j - j0)] = static_cast<double>(sq);
            }
            __syncthreads();
            if (tid < T) {
                double s = 0.0, ss = 0.0;
                for (int j = 0; j < nj; ++j) {
                    s += scratch[tid * nj + j];
                    ss += scratch_ss[tid * nj + j];
                }
                p.part[(static_cast<size_t>(sp) * DF_MAX_T + tid) * E + e] = s;
                if (norm && e == 0) p.part_ss[static_cast<size_t>(sp) * DF_MAX_T + tid] = ss;
            }
            __syncthreads();
        }
    }
    // grid barrier: every CTA arrives exactly once per launch
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        atomicAdd(&p.st->bar, 1u);
        const uint32_t target = (epoch + 1u) * static_cast<uint32_t>(G);
        spin_until_reached(&p.st->bar, target, abort_flag, p.status, p.timeout_ns);
    }
    __syncthreads();

    // ---- finish the routing in every CTA (identical order, identical results)
    {
        float* lg = reinterpret_cast<float*>(base_ptr);   // [16][E + 1]
        if (tid < T) {
            double ss = 0.0;
            if (norm)
                for (int sp = 0; sp < p.S; ++sp) ss += __ldcg(p.part_ss + static_cast<size_t>(sp) * DF_MAX_T + tid);
            C.inv_rms[tid] = norm ? 1.0 / sqrt(ss / static_cast<double>(d) + static_cast<double>(p.eps)) : 1.0;
        }
        for (int e = tid; e < E; e += DF_THREADS) {
            C.slot_of[e] = 0;
        }
        __syncthreads();
        for (int i = tid; i < T * E; i += DF_THREADS) {
            const int t = i / E, e = i % E;
            double s = 0.0;
            for (int sp = 0; sp < p.S; ++sp) s += __ldcg(p.part + (static_cast<size_t>(sp) * DF_MAX_T + t) * E + e);
            if (norm) s *= C.inv_rms[t];
            if (p.bias) s += p.bias[e];
            lg[t * (E + 1) + e] = static_cast<float>(s);
        }
        __syncthreads();
        const int ept = (E + 31) / 32;
        for (int t = warp; t < T; t += DF_THREADS / 32) {
            const float* row = lg + t * (E + 1);
            uint32_t taken = 0;
            float sel_v[MAX_TOPK];
            int sel_e[MAX_TOPK];
            for (int r = 0; r < k; ++r) {
                float bv = -INFINITY;
                int be = 0x7FFFFFFF;
                for (int i = 0; i < ept; ++i) {
                    const int e = lane + 32 * i;
                    if (e < E && !((taken >> i) & 1u)) {
                        const float v = row[e];
                        if (v > bv || (v == bv && e < be)) { bv = v; be = e; }
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, off);
                    if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
                }
                be = min(be, E - 1);   // a NaN score selects nothing: keep the index in range
                if ((be & 31) == lane) taken |= 1u << (be >> 5);
                sel_v[r] = bv;
                sel_e[r] = be;
            }
            if (lane == 0) {
                const float m = sel_v[0];
                float den = 0.f;
                for (int r = 0; r < k; ++r) den += expf(sel_v[r] - m);
                const float inv = 1.f / den;
                for (int r = 0; r < k; ++r) {
                    C.tok_e[t][r] = sel_e[r];
                    C.tok_w[t][r] = expf(sel_v[r] - m) * inv;
                }
            }
        }
        __syncthreads();
        // touched experts, ascending: mark, then one warp-wide exclusive scan
        if (tid < T * k) atomicOr(&C.slot_of[C.tok_e[tid / k][tid % k]], 1);
        __syncthreads();
        if (warp == 0) {
            int cnt = 0;
            for (int i = 0; i < ept; ++i) {
                const int e = lane * ept + i;
                if (e < E) cnt += C.slot_of[e];
            }
            int inc = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += n;
            }
            int pos = inc - cnt;
            for (int i = 0; i < ept; ++i) {
                const int e = lane * ept + i;
                if (e < E) {
                    if (C.slot_of[e]) {
                        C.touched[pos] = e;
                        C.slot_of[e] = pos++;
                    } else {
                        C.slot_of[e] = -1;
                    }
                }
            }
            if (lane == 31) C.n_t = inc;
        }
        __syncthreads();
        for (int i = tid; i < C.n_t * DF_MAX_T; i += DF_THREADS) C.selw[i / DF_MAX_T][i % DF_MAX_T] = 0.f;
        __syncthreads();
        if (tid < T * k) {
            const int t = tid / k, r = tid % k;
            C.selw[C.slot_of[C.tok_e[t][r]]][t] = C.tok_w[t][r];
        }
        if (blockIdx.x == 0) {
            if (p.topk_idx && tid < T * k) p.topk_idx[tid] = C.tok_e[tid / k][tid % k];
            if (p.topk_w && tid < T * k) p.topk_w[tid] = C.tok_w[tid / k][tid % k];
            if (p.counts)
                for (int e = tid; e < E; e += DF_THREADS) {
                    int c = 0;
                    for (int i = 0; i < T * k; ++i) c += (C.tok_e[i / k][i % k] == e);
                    p.counts[e] = c;
                }
        }
        __syncthreads();
    }
    const int n_t = C.n_t;
    // gate/up: whole tiles u = b, b + G, ...; down: a contiguous range of items
    // sized so that every CTA streams about the same number of bytes (a gate/up
    // chunk and a down item are both at most 17,408 bytes)
    const int NT = n_t * F_gu;
    const long ND = static_cast<long>(n_t) * F_dn * NP;
    long d_lo, d_hi;
    {
        const long q = NT / G, r = NT % G;
        const long W = static_cast<long>(NT) * KC_gu + ND;             // items of the whole launch
        const long defA = max(0L, W - static_cast<long>(G) * (q + 1) * KC_gu);   // CTAs b < r (one tile more)
        const long defB = max(0L, W - static_cast<long>(G) * q * KC_gu);
        const long tot = r * defA + (G - r) * defB;
        auto D = [&](long b) -> long {
            if (b <= 0 || tot == 0) return 0;
            if (b >= G) return ND;
            const long pre = b < r ? b * defA : r * defA + (b - r) * defB;
            return ND * pre / tot;
        };
        d_lo = D(blockIdx.x);
        d_hi = D(blockIdx.x + 1);
    }
    const size_t ebytes_gu = p.Mgu.expert_bytes(), ebytes_dn = p.Mdn.expert_bytes();
    const uint32_t idesc = idesc_mxf4(128, DF_NB3);

    if (warp == 0) {
        // -------------------------------------------------------------- producer
        int s = 0;
        uint32_t ph = 0;
        int pend_ph[DF_MAX_STAGES];
        for (int i = 0; i < DF_MAX_STAGES; ++i) pend_ph[i] = -1;
        bool skip = p.skip_first_copy != 0;
        bool ok = __all_sync(0xffffffffu, *abort_flag == 0);
        auto issue = [&](const uint8_t* src, uint32_t bytes) {
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, p.status, p.timeout_ns));
            if (!ok) return;
            if (skip) {
                skip = false;   // test hook: this stage is never filled
            } else {
                mbar_arrive_expect_tx_warp(full_bar(s), bytes);
                bulk_g2s_warp(ring + s * DF_STAGE, src, bytes, full_bar(s));
                pend_ph[s] = static_cast<int>(ph);
            }
            if (++s == S) { s = 0; ph ^= 1u; }
        };
        for (int u = blockIdx.x; u < NT && ok; u += G) {
            const int i = u / F_gu, ft = u % F_gu;
            const int rf = min(128, f - ft * 128);
            const uint8_t* we = p.Mgu.base + C.touched[i] * ebytes_gu;
            for (int c = 0; c < KC_gu && ok; ++c)
                issue(we + p.Mgu.chunk_offset(ft, c, rf), static_cast<uint32_t>(p.Mgu.chunk_bytes(c, rf)));
        }
        for (long jt = d_lo; jt < d_hi && ok; ++jt) {
            const int i = static_cast<int>(jt / (F_dn * NP));
            const int rem = static_cast<int>(jt % (F_dn * NP));
            const int ft = rem / NP, j = rem % NP;
            const int rf = min(128, d - ft * 128);
            issue(p.Mdn.base + C.touched[i] * ebytes_dn + p.Mdn.chunk_offset(ft, 2 * j, rf),
                  df_down_item_bytes(p.Mdn, j, rf));
        }
        if (lane == 0)
            for (int i = 0; i < S; ++i)
                if (pend_ph[i] >= 0) mbar_wait_drain(full_bar(i), static_cast<uint32_t>(pend_ph[i]), 200000000ull);
        __syncwarp();
    } else if (warp == 1) {
        // -------------------------------------------------------------- MMA issuer
        int s = 0, sfs = 0, buf = 0;
        uint32_t ph = 0;
        uint32_t eph[2] = {0u, 0u};
        bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&C.xready), 0, abort_flag, p.status, p.timeout_ns));
        // gate/up tiles
        for (int u = blockIdx.x; u < NT && ok; u += G) {
            const int ft = u % F_gu;
            const int rf = min(128, f - ft * 128);
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&C.acce[buf]), eph[buf] ^ 1u, abort_flag, p.status,
                                                           p.timeout_ns));
            if (!ok) break;
            eph[buf] ^= 1u;
            tc_fence_after();
            const uint32_t d0 = tmem + static_cast<uint32_t>(buf * DF_ACC_COLS);
            for (int c = 0; c < KC_gu; ++c) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), ph, abort_flag, p.status, p.timeout_ns));
                if (!ok) break;
                tc_fence_after();
                const int nbc = p.Mgu.blocks_in_chunk(c);
                const uint32_t codes_b = static_cast<uint32_t>(nbc * rf * 16), mat_b = codes_b + 512u;
                const uint32_t ws = ring + s * DF_STAGE;
                const uint32_t sfc = tmem + DF_SF_COL0 + DF_SF_SLOT_COLS * sfs;
                tc_cp_sf_warp(sfc, desc_noswz(ws + codes_b, 0, 128));
                tc_cp_sf_warp(sfc + 4, desc_noswz(ws + mat_b + codes_b, 0, 128));
                tc_cp_sf_warp(sfc + 8, desc_noswz(bsf + c * 512u, 0, 128));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (2 * h < nbc) {
                        const uint32_t acc = (c > 0 || h > 0) ? 1u : 0u;
                        const uint32_t id = idesc | idesc_sf_ids(2u * h);
                        const uint64_t ad = desc_noswz(ws + 2 * h * rf * 16, rf * 16, 128);
                        const uint64_t bd = desc_noswz(bbuf + (4 * c + 2 * h) * DF_B_BLOCK, DF_B_BLOCK, 128);
                        mma_mxf4_warp(d0, ad, bd, id, sfc, sfc + 8, acc);
                        mma_mxf4_warp(d0 + DF_MAT_COLS, ad + (mat_b >> 4), bd, id, sfc + 4, sfc + 8, acc);
                    }
                }
                tc_commit_warp(empty_bar(s));
                if (++s == S) { s = 0; ph ^= 1u; }
                if (++sfs == DF_SF_SLOTS) sfs = 0;
            }
            if (!ok) break;
            tc_commit_warp(smem_u32(&C.accf[buf]));
            buf ^= 1;
        }
        // down pieces: item k of this CTA takes weight stage s (the producer's
        // sequence) and H slot k % S (the H issuer's sequence)
        long jt = d_lo;
        int hs = 0;
        uint32_t hph = 0;
        while (ok && jt < d_hi) {
            const int i = static_cast<int>(jt / (F_dn * NP));
            const int ft = static_cast<int>((jt % (F_dn * NP)) / NP);
            const long piece_end = min(d_hi, static_cast<long>(i) * F_dn * NP + static_cast<long>(ft + 1) * NP);
            const int rf = min(128, d - ft * 128);
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&C.acce[buf]), eph[buf] ^ 1u, abort_flag, p.status,
                                                           p.timeout_ns));
            if (!ok) break;
            eph[buf] ^= 1u;
            tc_fence_after();
            const uint32_t d0 = tmem + static_cast<uint32_t>(buf * DF_ACC_COLS);
            bool first = true;
            for (; jt < piece_end; ++jt) {
                const int j = static_cast<int>(jt % NP);
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), ph, abort_flag, p.status, p.timeout_ns));
                if (ok)
                    ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&C.hfull[hs]), hph, abort_flag, p.status,
                                                                   p.timeout_ns));
                if (!ok) break;
                tc_fence_after();
                const uint32_t ws = ring + s * DF_STAGE;
                const uint32_t hsl = bbuf + hs * DF_HSLOT;
                const uint32_t sfc = tmem + DF_SF_COL0 + DF_SF_SLOT_COLS * sfs;
                uint32_t off = 0;
                for (int hc = 0; hc < 2; ++hc) {
                    const int c = 2 * j + hc;
                    if (c >= KC_dn) break;
                    const int nbc = p.Mdn.blocks_in_chunk(c);
                    const uint32_t codes_b = static_cast<uint32_t>(nbc * rf * 16);
                    tc_cp_sf_warp(sfc + 4 * hc, desc_noswz(ws + off + codes_b, 0, 128));
                    tc_cp_sf_warp(sfc + 8 + 4 * hc, desc_noswz(hsl + DF_HSLOT_CODES + hc * 512u, 0, 128));
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (2 * h < nbc) {
                            const uint32_t acc = first ? 0u : 1u;
                            first = false;
                            const uint32_t id = idesc | idesc_sf_ids(2u * h);
                            const uint64_t ad = desc_noswz(ws + off + 2 * h * rf * 16, rf * 16, 128);
                            const uint64_t bd = desc_noswz(hsl + (4 * hc + 2 * h) * DF_B_BLOCK, DF_B_BLOCK, 128);
                            mma_mxf4_warp(d0, ad, bd, id, sfc + 4 * hc, sfc + 8 + 4 * hc, acc);
                        }
                    }
                    off += codes_b + 512u;
                }
                tc_commit_warp(empty_bar(s));
                tc_commit_warp(smem_u32(&C.hempty[hs]));
                if (++s == S) { s = 0; ph ^= 1u; }
                if (++hs == S) { hs = 0; hph ^= 1u; }
                if (++sfs == DF_SF_SLOTS) sfs = 0;
            }
            if (!ok) break;
            tc_commit_warp(smem_u32(&C.accf[buf]));
            buf ^= 1;
        }
        tc_commit_warp(smem_u32(&C.drain));
        if (lane == 0) mbar_wait_drain(smem_u32(&C.drain), 0, 200000000ull);
        __syncwarp();
    } else if (warp < DF_HWARP) {
        // -------------------------------------------------------------- epilogue warps
        const int et = tid - 64;                 // 0 .. 255
        const int q = warp & 3;                  // TMEM lane quarter (hardware rule: warp % 4)
        const int hh = (warp - 2) >> 2;          // token columns 8 hh .. 8 hh + 7
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;

        // with the pre-norm, this CTA's share of x's operand now (see above)
        {
            if (norm) x_share(et, DF_EPI_THREADS);
            named_barrier(1, DF_EPI_THREADS);
            if (et == 0) {
                if (norm) {
                    __threadfence();
                    atomicAdd(&p.st->xdone, 1u);
                }
                // when every share is written, copy the operand (codes and scale
                // atoms) into shared memory; xready completes on the bytes
                const uint32_t target = (epoch + 1u) * static_cast<uint32_t>(G);
                if (spin_until_reached(&p.st->xdone, target, abort_flag, p.status, p.timeout_ns)) {
                    fence_proxy_async_global();
                    const uint32_t cb = static_cast<uint32_t>(nb_d) * DF_B_BLOCK,
                                   ab = static_cast<uint32_t>(KC_gu) * 512u;
                    mbar_arrive_expect_tx(smem_u32(&C.xready), cb + ab);
                    bulk_g2s(bbuf, p.xq, cb, smem_u32(&C.xready));
                    bulk_g2s(bsf, p.xq + cb, ab, smem_u32(&C.xready));
                }
            }
        }
        bool ok = named_barrier_and(1, DF_EPI_THREADS, *abort_flag == 0);

        int buf = 0;
        uint32_t fph[2] = {0u, 0u};
        // accumulator of token group hh: sum of the three stacked term columns
        auto load_acc = [&](uint32_t d0, float (&out)[8]) {
            uint32_t r[MXQ_TERMS][8];
#pragma unroll
            for (int tt = 0; tt < MXQ_TERMS; ++tt) tmem_ld8(d0 + lane_addr + tt * DF_MAX_T + 8 * hh, r[tt]);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                out[j] = __uint_as_float(r[0][j]) + __uint_as_float(r[1][j]) + __uint_as_float(r[2][j]);
        };

        // gate/up tiles: H of the tile's 128 features for every token row (zero
        // rows for tokens not routed to the expert) into the expert's H operand,
        // then the tile's stamp
        for (int u = blockIdx.x; u < NT && ok; u += G) {
            const int i = u / F_gu, ft = u % F_gu;
            const int rf = min(128, f - ft * 128);
            const bool w_ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&C.accf[buf]), fph[buf], abort_flag,
                                                                         p.status, p.timeout_ns));
            fph[buf] ^= 1u;
            tc_fence_after();
            if (w_ok && 32 * q < rf) {
                const uint32_t d0 = tmem + static_cast<uint32_t>(buf * DF_ACC_COLS);
                float g[8], uu[8];
                load_acc(d0, g);
                load_acc(d0 + DF_MAT_COLS, uu);
                const int b = 4 * ft + q;   // the warp's 32-feature block of H
                uint8_t* hcodes = p.hq + i * p.hq_stride;
                uint8_t* hatoms = hcodes + static_cast<size_t>(nb_f) * DF_B_BLOCK;
#pragma unroll 1
                for (int j = 0; j < 8; ++j) {
                    const int t = 8 * hh + j;
                    uint32_t w[MXQ_TERMS] = {0u, 0u, 0u}, sb[MXQ_TERMS] = {0u, 0u, 0u};
                    if (t < T && C.selw[i][t] != 0.f) mxq_block_warp(swish_f(g[j]) * uu[j], w, sb);
                    if (lane < 4) {
#pragma unroll
                        for (int tt = 0; tt < MXQ_TERMS; ++tt)
                            reinterpret_cast<uint32_t*>(hcodes + (static_cast<size_t>(b) * DF_NB3 + tt * DF_MAX_T + t) *
                                                                     16)[lane] = w[tt];
                    }
                    if (lane == 0) {
#pragma unroll
                        for (int tt = 0; tt < MXQ_TERMS; ++tt)
                            hatoms[(b >> 2) * 512 + sf_atom_offset(tt * DF_MAX_T + t, b & 3)] =
                                static_cast<uint8_t>(sb[tt]);
                    }
                }
            }
            tc_fence_before();
            // this warp's part of the tile's H is written: stamp it (each lane that
            // stored fences its own stores first)
            if (lane < 4) __threadfence();
            __syncwarp();
            if (w_ok && lane == 0) {
                mbar_arrive(smem_u32(&C.acce[buf]));
                atomicExch(&p.hdone[(static_cast<size_t>(i) * F_gu + ft) * DF_EPI_WARPS + (warp - 2)], epoch + 1u);
            }
            buf ^= 1;
            // every epilogue thread takes the same decision (no thread is left waiting)
            ok = named_barrier_and(1, DF_EPI_THREADS, w_ok);
        }
        // the x operand is no longer read (every gate/up MMA has completed): the
        // H issuer may reuse its space
        if (et == 0) mbar_arrive(smem_u32(&C.xfree));

        // down pieces: y_acc[t] += w[t, e] D for the tokens routed to the piece's expert
        long jt = d_lo;
        while (ok && jt < d_hi) {
            const int i = static_cast<int>(jt / (F_dn * NP));
            const int ft = static_cast<int>((jt % (F_dn * NP)) / NP);
            const long piece_end = min(d_hi, static_cast<long>(i) * F_dn * NP + static_cast<long>(ft + 1) * NP);
            const int rf = min(128, d - ft * 128);
            const bool w_ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&C.accf[buf]), fph[buf], abort_flag,
                                                                         p.status, p.timeout_ns));
            fph[buf] ^= 1u;
            tc_fence_after();
            if (w_ok && 32 * q < rf && 8 * hh < T) {
                const uint32_t d0 = tmem + static_cast<uint32_t>(buf * DF_ACC_COLS);
                float o[8];
                load_acc(d0, o);
                const int n = ft * 128 + 32 * q + lane;
                if (32 * q + lane < rf) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int t = 8 * hh + j;
                        const float w = t < T ? C.selw[i][t] : 0.f;
                        if (w != 0.f) atomicAdd(yacc + static_cast<size_t>(t) * d + n, w * o[j]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (w_ok && lane == 0) mbar_arrive(smem_u32(&C.acce[buf]));
            buf ^= 1;
            ok = named_barrier_and(1, DF_EPI_THREADS, w_ok);
            jt = piece_end;
        }
    } else {
        // -------------------------------------------------------------- H issuer
        // For down item k of this CTA (H slot k % S): once the slot is free and
        // the gate/up tiles of its two K chunks are stamped by all their
        // epilogue warps, copy that part of the expert's H operand (codes of 8
        // blocks, 2 scale atoms) into the slot; hfull completes on the bytes.
        int hs = 0;
        uint32_t hph = 0;
        int hpend[DF_MAX_STAGES];
        for (int i = 0; i < DF_MAX_STAGES; ++i) hpend[i] = -1;
        bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&C.xready), 0, abort_flag, p.status, p.timeout_ns));
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&C.xfree), 0, abort_flag, p.status, p.timeout_ns));
        for (long jt = d_lo; jt < d_hi && ok; ++jt) {
            const int i = static_cast<int>(jt / (F_dn * NP));
            const int j = static_cast<int>(jt % NP);
            const int c0 = 2 * j, c1 = min(KC_dn, c0 + 2);
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&C.hempty[hs]), hph ^ 1u, abort_flag, p.status,
                                                           p.timeout_ns));
            if (!ok) break;
            if (lane < (c1 - c0) * DF_EPI_WARPS) {
                // lane l polls the stamp of warp l % 8 of gate/up tile c0 + l / 8
                const int ft_g = c0 + lane / DF_EPI_WARPS, wq = lane % DF_EPI_WARPS;
                ok = spin_until_reached(&p.hdone[(static_cast<size_t>(i) * F_gu + ft_g) * DF_EPI_WARPS + wq], epoch + 1u,
                                        abort_flag, p.status, p.timeout_ns);
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (lane == 0) {
                // the stamps were read with acquire loads; order them before the
                // async-proxy reads of the copy
                fence_proxy_async_global();
                const uint8_t* hcodes = p.hq + i * p.hq_stride;
                const uint8_t* hatoms = hcodes + static_cast<size_t>(nb_f) * DF_B_BLOCK;
                const int b0 = 4 * c0, b1 = min(4 * c1, nb_f);
                const uint32_t cb = static_cast<uint32_t>(b1 - b0) * DF_B_BLOCK, ab = static_cast<uint32_t>(c1 - c0) * 512u;
                const uint32_t hsl = bbuf + hs * DF_HSLOT;
                mbar_arrive_expect_tx(smem_u32(&C.hfull[hs]), cb + ab);
                bulk_g2s(hsl, hcodes + static_cast<size_t>(b0) * DF_B_BLOCK, cb, smem_u32(&C.hfull[hs]));
                bulk_g2s(hsl + DF_HSLOT_CODES, hatoms + static_cast<size_t>(c0) * 512, ab, smem_u32(&C.hfull[hs]));
            }
            hpend[hs] = static_cast<int>(hph);
            if (++hs == S) { hs = 0; hph ^= 1u; }
        }
        // copies still in flight must land before the CTA exits
        if (lane == 0)
            for (int i = 0; i < S; ++i)
                if (hpend[i] >= 0) mbar_wait_drain(smem_u32(&C.hfull[i]), static_cast<uint32_t>(hpend[i]), 200000000ull);
        __syncwarp();
    }

    // ---- finish: free tensor memory; the last CTA writes y
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (tid == 0) {
        __threadfence();
        C.last = (atomicAdd(&p.st->finish, 1u) == static_cast<uint32_t>(G - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (!C.last) return;
    __threadfence();
    {
        const long n4 = static_cast<long>(T) * d / 4;
        for (long i4 = tid; i4 < n4; i4 += DF_THREADS) {
            float4 v = __ldcg(reinterpret_cast<const float4*>(yacc) + i4);
            if (p.residual) {
                float xv[4];
                if constexpr (sizeof(TA) == 2) {
                    const uint2 xr = reinterpret_cast<const uint2*>(p.x)[i4];
                    xv[0] = __uint_as_float(xr.x << 16);
                    xv[1] = __uint_as_float(xr.x & 0xFFFF0000u);
                    xv[2] = __uint_as_float(xr.y << 16);
                    xv[3] = __uint_as_float(xr.y & 0xFFFF0000u);
                } else {
                    const float4 xr = reinterpret_cast<const float4*>(p.x)[i4];
                    xv[0] = xr.x; xv[1] = xr.y; xv[2] = xr.z; xv[3] = xr.w;
                }
                v.x += xv[0]; v.y += xv[1]; v.z += xv[2]; v.w += xv[3];
            }
            if constexpr (sizeof(TA) == 2) {
                __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
                __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
                uint2 o;
                o.x = *reinterpret_cast<uint32_t*>(&a);
                o.y = *reinterpret_cast<uint32_t*>(&b);
                reinterpret_cast<uint2*>(p.y)[i4] = o;
            } else {
                reinterpret_cast<float4*>(p.y)[i4] = v;
            }
        }
        __syncthreads();
        if (tid == 0) {
            p.st->finish = 0u;
            __threadfence();
            atomicAdd(&p.st->epoch, 1u);
        }
    }
}

}  // namespace moe
