// routing.cuh -- router (scores, top-k, softmax over the selected scores), the
// expert histogram / prefix-sum schedule, the gather that groups token rows by
// expert, and the small finishing kernels.
//
// Method (page "GPT-OSS-20B : Architecture MoE & Résumé du Model Card", §3.1 Le
// Routeur): scores = W_router . h (+ optional bias), the top-k scores are
// selected (descending, ties to the lower expert index) and a softmax over the
// k selected scores gives weights summing to 1.  §2.1: the expert outputs are
// later combined with these weights.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "mxq.cuh"

namespace moe {

constexpr int ROUTER_TOKENS = 128;  // tokens per router tile
constexpr int ROUTER_THREADS = 256;
constexpr int ROUTER_KCHUNK = 64;
constexpr int MAX_EXPERTS = 256;
constexpr int MAX_TOPK = 8;

// Eight consecutive activation-dtype elements held raw in registers.
template <typename TA> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 v;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ void zero() { v = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ float get(int i) const {
        const uint32_t w = (&v.x)[i >> 1];
        return __uint_as_float((i & 1) ? (w & 0xFFFF0000u) : (w << 16));
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = *reinterpret_cast<const float4*>(p);
        b = *reinterpret_cast<const float4*>(p + 4);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ float get(int i) const {
        const float4& q = i < 4 ? a : b;
        const int j = i & 3;
        return j == 0 ? q.x : j == 1 ? q.y : j == 2 ? q.z : q.w;
    }
};

// Router tiles: ROUTER_TOKENS tokens x ROUTER_ETILE experts per CTA (grid.z
// covers the experts), K split over grid.y.  Dynamic shared memory: the x chunk
// transposed [64 k][128 tokens] and the router chunk [64 k][32 experts], fp32;
// the top-k tail reuses it for the scores of 32 tokens [32][E + 1].
constexpr int ROUTER_ETILE = 32;
constexpr int ROUTER_MAX_SPLITS = 8;
constexpr int ROUTER_SUB = 32;   // tokens per pass of the top-k tail at E = 256 (more when E is smaller)
__host__ __device__ constexpr size_t router_smem_bytes() {
    return sizeof(float) * (static_cast<size_t>(ROUTER_KCHUNK) * ROUTER_TOKENS +
                            static_cast<size_t>(ROUTER_KCHUNK) * ROUTER_ETILE);
}
static_assert(sizeof(float) * ROUTER_SUB * (MAX_EXPERTS + 1) <= router_smem_bytes(), "top-k scores must fit");

// Schedule slots.
enum : int {
    SCHED_UNITS_GU = 0,   // units of the gate/up GEMM
    SCHED_UNITS_DN = 1,   // units of the down GEMM
    SCHED_SPLIT_GU = 2,   // K splits of the gate/up GEMM (>1: partials + finish kernel)
    SCHED_SPLIT_DN = 3,   // K splits of the down GEMM
    SCHED_ROWS = 4,       // grouped rows = T*k
    SCHED_SLOTS = 8
};

struct RouterArgs {
    const void* x;         // [T][d] act dtype
    const void* wr;        // [E][d] act dtype
    const float* bias;     // [E] or null
    int T, d, E, k;
    int S;                 // K splits = gridDim.y
    double* part;          // [S][T][E] partial scores
    // optional pre-norm: scores of h = x * gamma / sqrt(mean(x^2) + eps)
    const float* gamma;    // [d] or null (no pre-norm)
    float eps;
    double* part_ss;       // [S][T] partial sums of x^2 (used with gamma)
    float* inv_rms;        // [T] 1 / sqrt(mean(x^2) + eps), written with gamma
    int* tile_cnt;         // [tiles] arrival counters (zero between launches)
    int* glob_cnt;         // [1] arrival counter (zero between launches)
    int32_t* idx_out;      // [T][k]
    float* w_out;          // [T][k]
    int32_t* local_rank;   // [T][k] rank of the pair among earlier pairs of its tile with the same expert
    int32_t* hist;         // [tiles][E] per-tile counts, turned into per-tile prefixes by the schedule
    // schedule
    int BN, F_gu, F_dn, KC_gu, KC_dn, nsm, split_rows_cap, max_units;
    int32_t* offsets;      // [E+1]
    int32_t* tile_base;    // [E] first token tile of each expert (tiles numbered over all experts), or null
    int32_t* counts_out;   // [E] or null
    int4* units_gu;
    int4* units_dn;
    int32_t* sched;
};

__device__ inline int pick_split(int base, int nsm, int KC) {
    if (base <= 0 || base >= nsm) return 1;
    int best = 1;
    float best_eff = 0.f;
    const int smax = min(8, max(1, KC / 4));
    for (int s = 1; s <= smax; ++s) {
        const int w = base * s;
        const float eff = static_cast<float>(w) / static_cast<float>(((w + nsm - 1) / nsm) * nsm);
        if (eff >= 0.9f) return s;
        if (eff > best_eff + 1e-6f) { best_eff = eff; best = s; }
    }
    return best;
}

// Run by the last router CTA to finish: per-expert totals and per-tile
// prefixes of the histogram (warp scans over tiles), group offsets and token
// tile bases (one warp-wide scan over experts), K splits and the unit counts of
// both expert GEMMs.  Units are ordered (expert, token tile, feature tile,
// split); token tiles are numbered consecutively over the experts.  The unit
// lists themselves are written by the next kernel (build_units), in parallel.
__device__ inline void schedule_block(const RouterArgs& a, int ntiles, int* cnt, int* off, int* tb, int* split_s) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    for (int e = warp; e < a.E; e += nwarps) {
        int carry = 0;
        // 256 tiles per round: the eight loads of a lane are issued together
        for (int r0 = 0; r0 < ntiles; r0 += 256) {
            int v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int b = r0 + 32 * i + lane;
                v[i] = (b < ntiles) ? __ldcg(a.hist + static_cast<size_t>(b) * a.E + e) : 0;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (r0 + 32 * i >= ntiles) break;   // warp-uniform
                const int b = r0 + 32 * i + lane;
                int inc = v[i];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int n = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += n;
                }
                if (b < ntiles) a.hist[static_cast<size_t>(b) * a.E + e] = carry + inc - v[i];
                carry += __shfl_sync(0xffffffffu, inc, 31);
            }
        }
        if (lane == 0) cnt[e] = carry;
    }
    __syncthreads();
    if (warp == 0) {
        // lane l owns experts [l*epl, (l+1)*epl): exclusive scans of rows and tiles
        const int epl = (a.E + 31) / 32;
        int rows = 0, tiles = 0;
        for (int i = 0; i < epl; ++i) {
            const int e = lane * epl + i;
            if (e < a.E) {
                rows += cnt[e];
                tiles += (cnt[e] + a.BN - 1) / a.BN;
            }
        }
        int rinc = rows, tinc = tiles;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int rn = __shfl_up_sync(0xffffffffu, rinc, o), tn = __shfl_up_sync(0xffffffffu, tinc, o);
            if (lane >= o) { rinc += rn; tinc += tn; }
        }
        int r = rinc - rows, tt = tinc - tiles;
        for (int i = 0; i < epl; ++i) {
            const int e = lane * epl + i;
            if (e < a.E) {
                off[e] = r;
                tb[e] = tt;
                r += cnt[e];
                tt += (cnt[e] + a.BN - 1) / a.BN;
            }
        }
        const int total_rows = __shfl_sync(0xffffffffu, rinc, 31), total_tiles = __shfl_sync(0xffffffffu, tinc, 31);
        if (lane == 0) {
            off[a.E] = total_rows;
            tb[a.E] = total_tiles;
            const int base_gu = total_tiles * a.F_gu, base_dn = total_tiles * a.F_dn;
            int sg = (total_rows <= a.split_rows_cap) ? pick_split(base_gu, a.nsm, a.KC_gu) : 1;
            int sd = pick_split(base_dn, a.nsm, a.KC_dn);
            while (sg > 1 && base_gu * sg > a.max_units) --sg;
            while (sd > 1 && base_dn * sd > a.max_units) --sd;
            split_s[0] = sg;
            split_s[1] = sd;
            a.sched[SCHED_UNITS_GU] = min(base_gu * sg, a.max_units);
            a.sched[SCHED_UNITS_DN] = min(base_dn * sd, a.max_units);
            a.sched[SCHED_SPLIT_GU] = sg;
            a.sched[SCHED_SPLIT_DN] = sd;
            a.sched[SCHED_ROWS] = total_rows;
        }
    }
    __syncthreads();
    for (int e = tid; e <= a.E; e += blockDim.x) a.offsets[e] = off[e];
    if (a.counts_out)
        for (int e = tid; e < a.E; e += blockDim.x) a.counts_out[e] = cnt[e];
    if (a.tile_base)
        for (int e = tid; e < a.E; e += blockDim.x) a.tile_base[e] = tb[e];
}

// Unit u of an expert GEMM's list (F feature tiles, S K splits): token tile
// u / (F S), feature tile (u / S) % F, split u % S; the tile's expert is the
// last e with tile_base[e] <= tile (an expert with no tiles shares its base
// with the next one).  {expert | tile << 8, first grouped row, rows, feature
// tile | split << 16}.
__device__ __forceinline__ int4 make_unit(int u, int F, int S, int E, int BN, const int32_t* tile_base,
                                          const int32_t* offsets) {
    const int tile = u / (F * S);
    const int rem = u - tile * F * S;
    const int ft = rem / S, sp = rem - ft * S;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_base[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int m = tile - tile_base[lo];
    const int cnt = offsets[lo + 1] - offsets[lo];
    return make_int4(lo | (tile << 8), offsets[lo] + m * BN, min(BN, cnt - m * BN), ft | (sp << 16));
}

// Both GEMMs' unit lists from the schedule, spread over a whole grid (thread
// `gtid` of `gthreads`): run by the kernel after the router.
__device__ inline void build_units(int gtid, int gthreads, const int32_t* sched, int E, int BN, int F_gu, int F_dn,
                                   const int32_t* tile_base, const int32_t* offsets, int4* units_gu, int4* units_dn) {
    const int n_gu = sched[SCHED_UNITS_GU], n_dn = sched[SCHED_UNITS_DN];
    const int S_gu = sched[SCHED_SPLIT_GU], S_dn = sched[SCHED_SPLIT_DN];
    for (int u = gtid; u < n_gu + n_dn; u += gthreads) {
        if (u < n_gu)
            units_gu[u] = make_unit(u, F_gu, S_gu, E, BN, tile_base, offsets);
        else
            units_dn[u - n_gu] = make_unit(u - n_gu, F_dn, S_dn, E, BN, tile_base, offsets);
    }
}

// The end of a router launch, run by every CTA once its partial scores (and
// partial sums of x^2) are written.  The last CTA of a token tile to finish
// (of `ctas_per_tile`) sums the S partials in split order (deterministic),
// scales by the inverse RMS, adds the bias, and for up to 128 tokens at a time
// selects the top-k (one thread per token; ties to the lower index) and
// applies the softmax over the k selected scores; it
// then ranks the tile's (token, slot) pairs within their expert and writes the
// tile histogram.  The last tile to finish builds the schedule
// (schedule_block).  `lg` (lg_bytes of shared memory) holds the scores of a
// pass.  Needs ROUTER_THREADS threads.
__device__ __forceinline__ void router_tail(const RouterArgs& a, int tile, int ntiles, int ctas_per_tile, float* lg,
                                            size_t lg_bytes) {
    __shared__ int hist_s[MAX_EXPERTS];
    __shared__ int es[ROUTER_TOKENS * MAX_TOPK];
    __shared__ int cnt_s[MAX_EXPERTS];
    __shared__ int off_s[MAX_EXPERTS + 1];
    __shared__ int tb_s[MAX_EXPERTS + 1];
    __shared__ int split_s[2];
    __shared__ int last_s;
    __shared__ double inv_s[ROUTER_TOKENS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, d = a.d, k = a.k;
    const int t0 = tile * ROUTER_TOKENS;
    const int ntok = min(ROUTER_TOKENS, a.T - t0);
    const bool norm = a.gamma != nullptr;
    __threadfence();
    __syncthreads();
    if (tid == 0) last_s = (atomicAdd(a.tile_cnt + tile, 1) == ctas_per_tile - 1);
    __syncthreads();
    if (!last_s) return;
    __threadfence();
    if (tid == 0) a.tile_cnt[tile] = 0;  // ready for the next launch

    for (int e = tid; e < E; e += ROUTER_THREADS) hist_s[e] = 0;
    if (tid < ntok) {
        double inv = 1.0;
        if (norm) {
            double pq[ROUTER_MAX_SPLITS];
#pragma unroll
            for (int sp = 0; sp < ROUTER_MAX_SPLITS; ++sp)
                pq[sp] = sp < a.S ? __ldcg(a.part_ss + static_cast<size_t>(sp) * a.T + t0 + tid) : 0.0;
            double sq = 0.0;
#pragma unroll
            for (int sp = 0; sp < ROUTER_MAX_SPLITS; ++sp) sq += pq[sp];
            inv = 1.0 / sqrt(sq / static_cast<double>(d) + static_cast<double>(a.eps));
            a.inv_rms[t0 + tid] = static_cast<float>(inv);
        }
        inv_s[tid] = inv;
    }
    const size_t pstride = static_cast<size_t>(a.T) * E;
    // tokens per pass: as many as the scores [sub][E + 1] fit in the staging
    // space (128 at E = 32, 64 at E = 128, 32 at E = 256)
    int sub_n = static_cast<int>(lg_bytes / (sizeof(float) * (E + 1))) & ~31;
    sub_n = min(ROUTER_TOKENS, max(ROUTER_SUB, sub_n));
    for (int sub = 0; sub < ntok; sub += sub_n) {
        const int nsub = min(sub_n, ntok - sub);
        __syncthreads();
        // scores = partials summed in split order (deterministic), x inverse RMS,
        // + bias; four scores per thread at a time, all their partials in flight
        for (int i0 = tid; i0 < nsub * E; i0 += 4 * ROUTER_THREADS) {
            double pv[4][ROUTER_MAX_SPLITS];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = i0 + m * ROUTER_THREADS;
                const double* pp = a.part + static_cast<size_t>(t0 + sub + i / E) * E + i % E;
#pragma unroll
                for (int sp = 0; sp < ROUTER_MAX_SPLITS; ++sp)
                    pv[m][sp] = (i < nsub * E && sp < a.S) ? __ldcg(pp + sp * pstride) : 0.0;
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = i0 + m * ROUTER_THREADS;
                if (i < nsub * E) {
                    double sv = 0.0;
#pragma unroll
                    for (int sp = 0; sp < ROUTER_MAX_SPLITS; ++sp) sv += pv[m][sp];
                    const int tl = i / E, e = i % E;
                    if (norm) sv *= inv_s[sub + tl];
                    if (a.bias) sv += a.bias[e];
                    lg[tl * (E + 1) + e] = static_cast<float>(sv);
                }
            }
        }
        __syncthreads();
        // top-k + softmax: G = 256 / (tokens rounded up to a power of two)
        // consecutive lanes per token (1 .. 8).  Lane g of a token takes experts
        // g, g + G, ... in ascending order, keeping its k best sorted by (score
        // desc, index asc): a candidate displaces an entry only if it is
        // larger, or equal with a lower index (ties go to the lower index; a
        // NaN never enters).  The G lists are then merged by k rounds of a
        // shuffle arg-max over the lanes' heads.
        int G = 1;
        while (G < 8 && G * 2 * nsub <= ROUTER_THREADS) G *= 2;
        const int tl = tid / G, g = tid % G;
        {
            const bool active = tl < nsub;
            const float* row = lg + (active ? tl : 0) * (E + 1);
            float sv[MAX_TOPK];
            int se[MAX_TOPK];
#pragma unroll
            for (int r = 0; r < MAX_TOPK; ++r) {
                sv[r] = -INFINITY;
                se[r] = 0x7FFFFFFF;
            }
            if (active) {
#pragma unroll 4
                for (int e = g; e < E; e += G) {
                    float cv = row[e];
                    int ce = e;
#pragma unroll
                    for (int r = 0; r < MAX_TOPK; ++r) {
                        if (r < k && (cv > sv[r] || (cv == sv[r] && ce < se[r]))) {
                            const float tv = sv[r];
                            const int te = se[r];
                            sv[r] = cv;
                            se[r] = ce;
                            cv = tv;
                            ce = te;
                        }
                    }
                }
            }
            // merge: round r takes the best head over the G lanes; its lane pops it
            float mv[MAX_TOPK];
            int me[MAX_TOPK];
#pragma unroll
            for (int r = 0; r < MAX_TOPK; ++r) {
                float bv = sv[0];
                int be = se[0];
                for (int o = 1; o < G; o <<= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                    if (ov > bv || (ov == bv && oe < be)) {
                        bv = ov;
                        be = oe;
                    }
                }
                mv[r] = bv;
                me[r] = be;
                if (se[0] == be) {   // experts are disjoint across the lanes: only the owner pops
#pragma unroll
                    for (int i = 0; i + 1 < MAX_TOPK; ++i) {
                        sv[i] = sv[i + 1];
                        se[i] = se[i + 1];
                    }
                    sv[MAX_TOPK - 1] = -INFINITY;
                    se[MAX_TOPK - 1] = 0x7FFFFFFF;
                }
            }
            if (active && g == 0) {
                const float m = mv[0];
                float den = 0.f;
#pragma unroll
                for (int r = 0; r < MAX_TOPK; ++r)
                    if (r < k) den += expf(mv[r] - m);
                const float inv = 1.f / den;
                const int t = t0 + sub + tl;
#pragma unroll
                for (int r = 0; r < MAX_TOPK; ++r) {
                    if (r < k) {
                        const int e = min(me[r], E - 1);   // a NaN score selects nothing: keep the index in range
                        a.idx_out[static_cast<size_t>(t) * k + r] = e;
                        a.w_out[static_cast<size_t>(t) * k + r] = expf(mv[r] - m) * inv;
                        es[(sub + tl) * k + r] = e;
                    }
                }
            }
        }
    }
    __syncthreads();
    // stable rank of each pair among the tile's earlier pairs with the same
    // expert, and the tile histogram: warp 0 walks the pairs in order, 32 at a
    // time; lanes with the same expert find one another with match_any.
    if (warp == 0) {
        for (int p0 = 0; p0 < ntok * k; p0 += 32) {
            const int p = p0 + lane;
            const bool valid = p < ntok * k;
            const int e = valid ? es[p] : -1 - lane;   // idle lanes form groups of their own
            const unsigned grp = __match_any_sync(0xffffffffu, e);
            const int before = __popc(grp & ((1u << lane) - 1u));
            if (valid) a.local_rank[static_cast<size_t>(t0) * k + p] = hist_s[e] + before;
            __syncwarp();
            if (valid && before == 0) hist_s[e] += __popc(grp);
            __syncwarp();
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += ROUTER_THREADS) a.hist[static_cast<size_t>(tile) * E + e] = hist_s[e];

    // the last tile builds the schedule
    __threadfence();
    __syncthreads();
    if (tid == 0) last_s = (atomicAdd(a.glob_cnt, 1) == ntiles - 1);
    __syncthreads();
    if (!last_s) return;
    __threadfence();
    if (tid == 0) *a.glob_cnt = 0;
    schedule_block(a, ntiles, cnt_s, off_s, tb_s, split_s);
}

// Grid (token tiles of 128, S splits of K, expert tiles of 32).  Each CTA
// accumulates the scores of its 128 tokens x 32 experts over its K range on
// the CUDA cores: each thread holds a 4-token x 4-expert register tile, fp32
// within a 64-wide K chunk staged in shared memory (products of bf16 or fp32
// inputs), fp64 across chunks; the next chunk is loaded into registers while
// the current one is multiplied.  With the pre-norm the staged router chunk is
// W_router * gamma (so the scores are of x * gamma) and the sum of x^2 per
// token is kept (by the expert tile 0 CTAs).  router_tail finishes.  The
// layers with bf16 activations use router_tc_kernel (tensor cores) instead;
// this kernel serves fp32 activations and the no-allocation entry point.
template <typename TA>
__global__ void __launch_bounds__(ROUTER_THREADS) router_kernel(const RouterArgs a) {
    extern __shared__ __align__(16) float rsm[];
    float* xs = rsm;                                        // [64 k][128 tokens]
    float* ws = xs + ROUTER_KCHUNK * ROUTER_TOKENS;         // [64 k][32 experts]
    float* lg = rsm;                                        // tail: [32 tokens][E + 1]
    __shared__ double ss_s[ROUTER_TOKENS];

    pdl_launch_dependents();
    const TA* x = static_cast<const TA*>(a.x);
    const TA* wr = static_cast<const TA*>(a.wr);
    const int tid = threadIdx.x;
    const int E = a.E, d = a.d;
    const int tile = blockIdx.x, split = blockIdx.y, e0 = blockIdx.z * ROUTER_ETILE;
    const int ntiles = gridDim.x;
    const int t0 = tile * ROUTER_TOKENS;
    const int ntok = min(ROUTER_TOKENS, a.T - t0);
    const int KCH = (d + ROUTER_KCHUNK - 1) / ROUTER_KCHUNK;
    const int kc0 = split * KCH / a.S, kc1 = (split + 1) * KCH / a.S;
    const bool norm = a.gamma != nullptr;

    // staging roles: x -- token tid % 128, K half tid / 128 (32 values);
    // router -- expert tid % 32, K eighth tid / 32 (8 values)
    const int xt = tid & (ROUTER_TOKENS - 1), xh = (tid >> 7) * 32;
    const int we = tid & 31, wk = (tid >> 5) * 8;
    // compute roles: tokens 4 tq .. 4 tq + 3, experts 4 eq .. 4 eq + 3
    const int tq = tid >> 3, eq = tid & 7;
    Raw8<TA> xr[4], wv;
    float4 g0 = make_float4(1.f, 1.f, 1.f, 1.f), g1 = g0;
    auto load_chunk = [&](int kc) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int kk = kc + xh + 8 * i;
            if (xt < ntok && kk < d) xr[i].load(x + static_cast<size_t>(t0 + xt) * d + kk);
            else xr[i].zero();
        }
        const int kk = kc + wk;
        if (e0 + we < E && kk < d) {
            wv.load(wr + static_cast<size_t>(e0 + we) * d + kk);
            if (norm) {
                g0 = *reinterpret_cast<const float4*>(a.gamma + kk);
                g1 = *reinterpret_cast<const float4*>(a.gamma + kk + 4);
            }
        } else {
            wv.zero();
        }
    };

    double tot[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) tot[i][j] = 0.0;
    double ss = 0.0;

    if (kc0 < kc1) load_chunk(kc0 * ROUTER_KCHUNK);
    for (int c = kc0; c < kc1; ++c) {
        const int kc = c * ROUTER_KCHUNK;
        __syncthreads();
        float sq = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float v = xr[i].get(j);
                sq = fmaf(v, v, sq);
                xs[(xh + 8 * i + j) * ROUTER_TOKENS + xt] = v;
            }
        ss += static_cast<double>(sq);
        {
            const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) ws[(wk + j) * ROUTER_ETILE + we] = norm ? wv.get(j) * gv[j] : wv.get(j);
        }
        __syncthreads();
        if (c + 1 < kc1) load_chunk(kc + ROUTER_KCHUNK);
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
        for (int kk = 0; kk < ROUTER_KCHUNK; ++kk) {
            const float4 xv = *reinterpret_cast<const float4*>(xs + kk * ROUTER_TOKENS + 4 * tq);
            const float4 wv4 = *reinterpret_cast<const float4*>(ws + kk * ROUTER_ETILE + 4 * eq);
            const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
            const float wa[4] = {wv4.x, wv4.y, wv4.z, wv4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xa[i], wa[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) tot[i][j] += static_cast<double>(acc[i][j]);
    }
    // partial scores of this split
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int tl = 4 * tq + i;
        if (tl < ntok) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = e0 + 4 * eq + j;
                if (e < E) a.part[(static_cast<size_t>(split) * a.T + t0 + tl) * E + e] = tot[i][j];
            }
        }
    }
    if (norm && blockIdx.z == 0) {
        // the token's two K halves are threads xt and xt + 128
        if (tid >= ROUTER_TOKENS) ss_s[xt] = ss;
        __syncthreads();
        if (tid < ROUTER_TOKENS && xt < ntok) a.part_ss[static_cast<size_t>(split) * a.T + t0 + xt] = ss + ss_s[xt];
    }
    router_tail(a, tile, ntiles, a.S * static_cast<int>(gridDim.z), lg, router_smem_bytes());
}

// One 32-element block of a token's activations as floats.
template <typename TA> struct BlockLoader;
template <> struct BlockLoader<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[32]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 q = reinterpret_cast<const uint4*>(p)[i];
            const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(b[j]);
                v[8 * i + 2 * j] = f.x;
                v[8 * i + 2 * j + 1] = f.y;
            }
        }
    }
};
template <> struct BlockLoader<float> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[32]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 q = reinterpret_cast<const float4*>(p)[i];
            v[4 * i] = q.x;
            v[4 * i + 1] = q.y;
            v[4 * i + 2] = q.z;
            v[4 * i + 3] = q.w;
        }
    }
};

// Where the grouped operands live.
struct GroupedOperand {
    uint8_t* codes;   // three MXFP4 terms [K/32][3][R][16 B]; two MXFP8 terms [K/16][2][R][16 B]
    uint8_t* scales;  // [tiles][KC][3 atoms][512]
    int R;            // row capacity
    int KC;           // chunks of 128 along K
    int term_rows;    // operand row of (term t, tile row r) = t * term_rows + r: 128 when each term
                      // is its own MMA (atom t), BN when the terms are stacked into one MMA
};

__device__ __forceinline__ uint8_t* scale_atom_base(const GroupedOperand& g, int tile, int chunk) {
    return g.scales + (static_cast<size_t>(tile) * g.KC + chunk) * MXQ_TERMS * 512;
}

// Grouping, part 1: one CTA per ROWS_TOKENS tokens.  The whole grid first
// writes both expert GEMMs' unit lists (build_units).  Pair p = t*k + j goes
// to grouped row offsets[e] + (rows of e in earlier router tiles) + (its rank
// within its router tile), so the rows of an expert are in (token, slot)
// order; the row's place in the expert's token tiles is (tile_base[e] +
// (row - offsets[e]) / BN, (row - offsets[e]) % BN).  One thread per pair
// records each row's token, routing weight and tile slot, and the pair's row.
// When the down GEMM splits K, all threads then initialise the tokens' rows
// of the fp32 output accumulator for its scatter-add (to x itself when the
// block's residual is fused, else to zero); when the gate/up GEMM splits K,
// they clear the pairs' fp32 partial-sum rows.
constexpr int ROWS_TOKENS = 8;
constexpr int ROWS_THREADS = 256;
template <typename TA>
__global__ void __launch_bounds__(ROWS_THREADS)
rows_kernel(const TA* __restrict__ x, const int32_t* idx, const float* w, const int32_t* local_rank,
            const int32_t* tile_prefix, const int32_t* offsets, const int32_t* tile_base, int T, int d, int E, int k,
            int BN, int32_t* __restrict__ row_token, float* __restrict__ row_weight, int32_t* __restrict__ row_slot,
            float* __restrict__ GU, int gu_ld, float* __restrict__ yacc, const int32_t* sched,
            int residual, int tiles_cap, int* status, int32_t* __restrict__ pair_row, int F_gu, int F_dn,
            int4* __restrict__ units_gu, int4* __restrict__ units_dn) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ int pos_s[ROWS_TOKENS * MAX_TOPK];
    const int t0 = blockIdx.x * ROWS_TOKENS;
    const int nt = min(ROWS_TOKENS, T - t0);
    const int tid = threadIdx.x;
    build_units(blockIdx.x * ROWS_THREADS + tid, gridDim.x * ROWS_THREADS, sched, E, BN, F_gu, F_dn, tile_base, offsets,
                units_gu, units_dn);
    if (tid < nt * k) {
        const int p = t0 * k + tid;
        const int t = p / k;
        const int e = idx[p];
        pos_s[tid] = -1;
        if (MOE_IN_BOUNDS(e >= 0 && e < E, status)) {
            const int loc = tile_prefix[static_cast<size_t>(t / ROUTER_TOKENS) * E + e] + local_rank[p];
            const int pos = offsets[e] + loc;
            const int tl = tile_base[e] + loc / BN;
            if (MOE_IN_BOUNDS(pos >= 0 && pos < T * k && tl >= 0 && tl < tiles_cap, status)) {
                row_token[pos] = t;
                row_weight[pos] = w[p];
                row_slot[pos] = tl * BN + loc % BN;
                pair_row[p] = pos;
                pos_s[tid] = pos;
            }
        }
    }
    // output accumulator rows: x (residual) or zero -- only when the down GEMM
    // splits K and adds partial sums (otherwise each grouped row's output is
    // stored once and combine_out_kernel sums them)
    const int d4 = d / 4;
    if (sched[SCHED_SPLIT_DN] > 1)
    for (int i = tid; i < nt * d4; i += ROWS_THREADS) {
        const int t = t0 + i / d4, c4 = i % d4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (residual) {
            if constexpr (sizeof(TA) == 2) {
                const uint2 r = reinterpret_cast<const uint2*>(x + static_cast<size_t>(t) * d)[c4];
                v = make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xFFFF0000u),
                                __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xFFFF0000u));
            } else {
                v = reinterpret_cast<const float4*>(x + static_cast<size_t>(t) * d)[c4];
            }
        }
        reinterpret_cast<float4*>(yacc + static_cast<size_t>(t) * d)[c4] = v;
    }
    if (sched[SCHED_SPLIT_GU] > 1) {
        __syncthreads();
        const int g4 = gu_ld / 4;
        for (int i = tid; i < nt * k * g4; i += ROWS_THREADS) {
            const int pos = pos_s[i / g4];
            if (pos >= 0)
                reinterpret_cast<float4*>(GU + static_cast<size_t>(pos) * gu_ld)[i % g4] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

// Grouping, part 2: the B operand of the gate/up GEMM.  One CTA per (token
// tile, K chunk of 128), chunk-major over the grid (blockIdx.x = tile), so the
// CTAs running together read one 128-wide column slice of x, which stays in
// L2 while every tile that needs it reads it.  Thread r encodes blocks
// 4c .. 4c+3 of the tile's row r (x of its token, times gamma / rms(x) with
// the pre-norm) in the operand format AF (three MXFP4 or two MXFP8 terms):
// the codes go straight to global memory
// (consecutive threads, consecutive rows: coalesced), the scale bytes into a
// shared-memory copy of the tile's scale atoms, which the CTA then writes
// whole (rows past the tile's valid rows get zero scale bytes).
constexpr int ENC_THREADS = 128;
template <typename TA, int AF>
__global__ void __launch_bounds__(ENC_THREADS)
encode_rows_kernel(const TA* __restrict__ x, const float* __restrict__ gamma, const float* inv_rms,
                   const int32_t* row_token, const int4* units_gu, const int32_t* sched, int F_gu, int d, GroupedOperand X, int T, int* status) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ __align__(16) uint8_t atoms[MXQ_TERMS * 512];
    const int tile = blockIdx.x, c = blockIdx.y;
    const int S = sched[SCHED_SPLIT_GU];
    const long u = static_cast<long>(tile) * F_gu * S;
    if (u >= sched[SCHED_UNITS_GU]) return;
    const int4 U = units_gu[u];
    const int row0 = U.y, nvalid = U.z;
    const int tid = threadIdx.x;
    for (int i = tid; i < MXQ_TERMS * 512 / 16; i += ENC_THREADS)
        reinterpret_cast<uint4*>(atoms)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    if (tid < nvalid && MOE_IN_BOUNDS(row0 >= 0 && row0 + nvalid <= X.R, status)) {
        const int row = row0 + tid;
        int t = row_token[row];
        if (!MOE_IN_BOUNDS(t >= 0 && t < T, status)) t = 0;
        const int nb = d / 32;
        const float r = gamma ? inv_rms[t] : 1.f;
        for (int q = 0; q < 4 && 4 * c + q < nb; ++q) {
            const int b = 4 * c + q;
            float v[32];
            BlockLoader<TA>::load(x + static_cast<size_t>(t) * d + b * 32, v);
            if (gamma) {
                const float4* g4 = reinterpret_cast<const float4*>(gamma + b * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 g = g4[i];
                    v[4 * i] *= g.x * r;
                    v[4 * i + 1] *= g.y * r;
                    v[4 * i + 2] *= g.z * r;
                    v[4 * i + 3] *= g.w * r;
                }
            }
            uint32_t sb[MXQ_TERMS];
            act_encode_store<AF>(v, X.codes, X.R, b, row, sb);
#pragma unroll
            for (int tt = 0; tt < ActFormat<AF>::TERMS; ++tt)
                atoms[sf_atom_offset(tt * X.term_rows + tid, q)] = static_cast<uint8_t>(sb[tt]);
        }
    }
    __syncthreads();
    uint4* dst = reinterpret_cast<uint4*>(scale_atom_base(X, tile, c));
    for (int i = tid; i < MXQ_TERMS * 512 / 16; i += ENC_THREADS) dst[i] = reinterpret_cast<const uint4*>(atoms)[i];
}

__device__ __forceinline__ float swish_f(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

constexpr int HENC_THREADS = 128;

// Split-K finish of the gate/up GEMM (only when the schedule split K): one
// thread per (grouped row, 32-feature block), consecutive threads taking
// consecutive blocks of a row, applies SwiGLU to the fp32 partial sums of g
// and u and encodes the block of H (format AF) into the down GEMM's
// B operand (the codes of each term, one scale byte per term into the scale
// atom of the row's token tile).
template <int AF>
__global__ void __launch_bounds__(HENC_THREADS)
h_encode_kernel(const float* GU, GroupedOperand Hd, int d_ff, int BN, const int32_t* row_slot, const int32_t* sched,
                int tiles_cap, int* status) {
    pdl_launch_dependents();
    pdl_wait();
    if (sched[SCHED_SPLIT_GU] <= 1) return;
    const int nb = d_ff / 32;
    const long item = static_cast<long>(blockIdx.x) * HENC_THREADS + threadIdx.x;
    if (item >= static_cast<long>(sched[SCHED_ROWS]) * nb) return;
    const int row = static_cast<int>(item / nb), b = static_cast<int>(item % nb);
    const int slot = row_slot[row];
    const int tile = slot / BN, rloc = slot % BN;
    if (!MOE_IN_BOUNDS(row < Hd.R && slot >= 0 && tile < tiles_cap, status)) return;
    float v[32];
    const float4* g = reinterpret_cast<const float4*>(GU + static_cast<size_t>(row) * 2 * d_ff + 32 * b);
    const float4* u = reinterpret_cast<const float4*>(GU + static_cast<size_t>(row) * 2 * d_ff + d_ff + 32 * b);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 gg = g[i], uu = u[i];
        v[4 * i] = swish_f(gg.x) * uu.x;
        v[4 * i + 1] = swish_f(gg.y) * uu.y;
        v[4 * i + 2] = swish_f(gg.z) * uu.z;
        v[4 * i + 3] = swish_f(gg.w) * uu.w;
    }
    uint32_t sb[MXQ_TERMS];
    act_encode_store<AF>(v, Hd.codes, Hd.R, b, row, sb);
    uint8_t* atoms = scale_atom_base(Hd, tile, b >> 2);
#pragma unroll
    for (int t = 0; t < ActFormat<AF>::TERMS; ++t)
        atoms[sf_atom_offset(t * Hd.term_rows + rloc, b & 3)] = static_cast<uint8_t>(sb[t]);
}

// The layer output.  When the down GEMM did not split K, each grouped row's
// weighted expert output w_j (H_row . W_down) was stored once (act dtype);
// y[t] = (x[t] with the residual) + the sum of token t's k rows, added in
// slot order j = 0 .. k-1 in fp32 (deterministic).  When it split K, the
// outputs were added into the fp32 accumulator (which started at x with the
// residual): y = that accumulator, cast.  One thread per 8 consecutive
// features of a token (16-byte loads and stores for bf16).
constexpr int COMBINE_THREADS = 256;
template <typename TA> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
        const uint4 q = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&b);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <> struct Vec8<float> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
        const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    static __device__ __forceinline__ void store(float* p, const float (&v)[8]) {
        reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
};
template <typename TA>
__global__ void __launch_bounds__(COMBINE_THREADS)
combine_out_kernel(const TA* obuf, const int32_t* pair_row, const float* yacc, const TA* __restrict__ x,
                   TA* __restrict__ y, int T, int d, int k, int residual, const int32_t* sched) {
    pdl_wait();
    const int d8 = d / 8;
    const bool split = sched[SCHED_SPLIT_DN] > 1;
    for (long i = blockIdx.x * static_cast<long>(COMBINE_THREADS) + threadIdx.x; i < static_cast<long>(T) * d8;
         i += static_cast<long>(gridDim.x) * COMBINE_THREADS) {
        const int t = static_cast<int>(i / d8), c = static_cast<int>(i % d8) * 8;
        float v[8];
        if (split) {
            Vec8<float>::load(yacc + static_cast<size_t>(t) * d + c, v);
        } else {
            if (residual) {
                Vec8<TA>::load(x + static_cast<size_t>(t) * d + c, v);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] = 0.f;
            }
            for (int j = 0; j < k; ++j) {
                float o[8];
                Vec8<TA>::load(obuf + static_cast<size_t>(pair_row[static_cast<size_t>(t) * k + j]) * d + c, o);
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] += o[q];
            }
        }
        Vec8<TA>::store(y + static_cast<size_t>(t) * d + c, v);
    }
}

}  // namespace moe
