// routing.cuh -- router (scores, top-k, softmax over the selected scores), the
// expert histogram / prefix-sum schedule, the permute-and-gather that groups
// token rows by expert, and the small finishing kernels.
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

namespace moe {

constexpr int ROUTER_TOKENS = 32;   // tokens per router / permute block
constexpr int ROUTER_THREADS = 256;
constexpr int ROUTER_KCHUNK = 64;
constexpr int MAX_EXPERTS = 256;
constexpr int MAX_TOPK = 8;

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Dynamic shared memory of router_kernel (floats): x chunk [32][65], router
// chunk [64][E], scores [32][E+1].
__host__ __device__ inline size_t router_smem_bytes(int E) {
    return sizeof(float) * (static_cast<size_t>(ROUTER_TOKENS) * (ROUTER_KCHUNK + 1) +
                            static_cast<size_t>(ROUTER_KCHUNK) * E + static_cast<size_t>(ROUTER_TOKENS) * (E + 1));
}

// One block scores 32 tokens against all E experts (fp32 accumulation over
// K-chunks staged in shared memory), then one warp per token selects the top-k
// with k rounds of warp arg-max and applies the softmax over the k selected
// scores.  Also writes the block's expert histogram and zeroes the rows of the
// output accumulator that the down GEMM adds into.
template <typename TA>
__global__ void __launch_bounds__(ROUTER_THREADS)
router_kernel(const TA* __restrict__ x, const TA* __restrict__ wr, const float* __restrict__ bias, int T, int d,
              int E, int k, int32_t* __restrict__ idx_out, float* __restrict__ w_out, int32_t* __restrict__ hist,
              float* __restrict__ zero_rows, int zero_ld) {
    extern __shared__ float rsm[];
    float* xs = rsm;                                     // [32][65]
    float* ws = xs + ROUTER_TOKENS * (ROUTER_KCHUNK + 1); // [64][E]
    float* lg = ws + ROUTER_KCHUNK * E;                   // [32][E+1]
    __shared__ int hist_s[MAX_EXPERTS];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * ROUTER_TOKENS;
    const int ntok = min(ROUTER_TOKENS, T - t0);
    const int EPT = (E + 31) / 32;  // experts per lane

    for (int e = tid; e < E; e += ROUTER_THREADS) hist_s[e] = 0;

    float acc[MAX_EXPERTS / 32][4];
#pragma unroll
    for (int i = 0; i < MAX_EXPERTS / 32; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int kc = 0; kc < d; kc += ROUTER_KCHUNK) {
        __syncthreads();
        for (int i = tid; i < ROUTER_TOKENS * ROUTER_KCHUNK; i += ROUTER_THREADS) {
            int t = i / ROUTER_KCHUNK, kk = i % ROUTER_KCHUNK;
            float v = 0.f;
            if (t < ntok && kc + kk < d) v = to_f32(x[static_cast<size_t>(t0 + t) * d + kc + kk]);
            xs[t * (ROUTER_KCHUNK + 1) + kk] = v;
        }
        for (int i = tid; i < E * ROUTER_KCHUNK; i += ROUTER_THREADS) {
            int e = i / ROUTER_KCHUNK, kk = i % ROUTER_KCHUNK;
            float v = 0.f;
            if (kc + kk < d) v = to_f32(wr[static_cast<size_t>(e) * d + kc + kk]);
            ws[kk * E + e] = v;
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < ROUTER_KCHUNK; ++kk) {
            float xv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) xv[j] = xs[(warp * 4 + j) * (ROUTER_KCHUNK + 1) + kk];
#pragma unroll
            for (int i = 0; i < MAX_EXPERTS / 32; ++i) {
                if (i < EPT) {
                    const int e = lane + 32 * i;
                    const float wv = (e < E) ? ws[kk * E + e] : 0.f;
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(wv, xv[j], acc[i][j]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < MAX_EXPERTS / 32; ++i) {
        if (i < EPT) {
            const int e = lane + 32 * i;
            if (e < E) {
                const float b = bias ? bias[e] : 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) lg[(warp * 4 + j) * (E + 1) + e] = acc[i][j] + b;
            }
        }
    }
    __syncthreads();

    // top-k + softmax: warp w handles tokens 4w .. 4w+3
    for (int j = 0; j < 4; ++j) {
        const int tl = warp * 4 + j;
        if (tl >= ntok) break;
        const float* row = lg + tl * (E + 1);
        uint32_t taken = 0;  // bit i: expert lane + 32 i already selected
        float sel_v[MAX_TOPK];
        int sel_e[MAX_TOPK];
        for (int r = 0; r < k; ++r) {
            float bv = -INFINITY;
            int be = 0x7FFFFFFF;
            for (int i = 0; i < EPT; ++i) {
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
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
            sel_v[r] = bv;
            sel_e[r] = be;
        }
        if (lane == 0) {
            const float m = sel_v[0];
            float den = 0.f;
            for (int r = 0; r < k; ++r) den += expf(sel_v[r] - m);
            const float inv = 1.f / den;
            const int t = t0 + tl;
            for (int r = 0; r < k; ++r) {
                idx_out[static_cast<size_t>(t) * k + r] = sel_e[r];
                w_out[static_cast<size_t>(t) * k + r] = expf(sel_v[r] - m) * inv;
                atomicAdd(&hist_s[sel_e[r]], 1);
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += ROUTER_THREADS) hist[static_cast<size_t>(blockIdx.x) * E + e] = hist_s[e];

    // zero the accumulator rows of this block's tokens (zero_ld % 4 == 0)
    if (zero_rows) {
        const int nvec = zero_ld / 4;
        for (int i = tid; i < ntok * nvec; i += ROUTER_THREADS) {
            const int t = i / nvec, v = i % nvec;
            reinterpret_cast<float4*>(zero_rows + static_cast<size_t>(t0 + t) * zero_ld)[v] =
                make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

// Schedule slots written by schedule_kernel.
enum : int {
    SCHED_UNITS_GU = 0,   // units of the gate/up GEMM
    SCHED_UNITS_DN = 1,   // units of the down GEMM
    SCHED_SPLIT_GU = 2,   // K splits of the gate/up GEMM (>1: partials + finish kernel)
    SCHED_SPLIT_DN = 3,   // K splits of the down GEMM
    SCHED_ROWS = 4,       // grouped rows = T*k
    SCHED_SLOTS = 8
};

struct ScheduleArgs {
    int32_t* hist;       // [nblk][E]: per-block counts in, per-block exclusive prefix out
    int nblk, E, BN;
    int F_gu, F_dn;      // 128-row feature tiles of the two GEMMs
    int KC_gu, KC_dn;    // 64-wide K chunks of the two GEMMs
    int nsm;
    int split_rows_cap;  // largest T*k for which the gate/up GEMM may split K
    int max_units;
    int32_t* offsets;    // [E+1]
    int32_t* counts_out; // [E] or null
    int4* units_gu;
    int4* units_dn;
    int32_t* sched;
};

__device__ inline int pick_split(int base, int nsm, int KC) {
    if (base <= 0 || base >= nsm) return 1;
    int best = 1;
    double best_eff = 0.0;
    const int smax = min(8, max(1, KC / 4));
    for (int s = 1; s <= smax; ++s) {
        const int w = base * s;
        const double eff = static_cast<double>(w) / (static_cast<double>((w + nsm - 1) / nsm) * nsm);
        if (eff >= 0.9) return s;
        if (eff > best_eff + 1e-9) { best_eff = eff; best = s; }
    }
    return best;
}

// Single block: per-expert totals and per-block prefixes of the router
// histogram (one warp per expert, warp scans over the blocks), exclusive scan
// of the totals into group offsets, choice of K splits, and the unit lists of
// both expert GEMMs ordered (expert, token tile, feature tile, split).
__global__ void __launch_bounds__(1024) schedule_kernel(ScheduleArgs a) {
    __shared__ int cnt[MAX_EXPERTS];
    __shared__ int off[MAX_EXPERTS + 1];
    __shared__ int split_s[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = warp; e < a.E; e += 32) {
        int carry = 0;
        for (int b0 = 0; b0 < a.nblk; b0 += 32) {
            const int b = b0 + lane;
            const int v = (b < a.nblk) ? a.hist[static_cast<size_t>(b) * a.E + e] : 0;
            int inc = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += n;
            }
            if (b < a.nblk) a.hist[static_cast<size_t>(b) * a.E + e] = carry + inc - v;
            carry += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) cnt[e] = carry;
    }
    __syncthreads();
    if (tid == 0) {
        int s = 0, base_gu = 0, base_dn = 0;
        for (int e = 0; e < a.E; ++e) {
            off[e] = s;
            s += cnt[e];
            const int mt = (cnt[e] + a.BN - 1) / a.BN;
            base_gu += mt * a.F_gu;
            base_dn += mt * a.F_dn;
        }
        off[a.E] = s;
        int sg = (s <= a.split_rows_cap) ? pick_split(base_gu, a.nsm, a.KC_gu) : 1;
        int sd = pick_split(base_dn, a.nsm, a.KC_dn);
        while (sg > 1 && base_gu * sg > a.max_units) --sg;
        while (sd > 1 && base_dn * sd > a.max_units) --sd;
        split_s[0] = sg;
        split_s[1] = sd;
        a.sched[SCHED_UNITS_GU] = min(base_gu * sg, a.max_units);
        a.sched[SCHED_UNITS_DN] = min(base_dn * sd, a.max_units);
        a.sched[SCHED_SPLIT_GU] = sg;
        a.sched[SCHED_SPLIT_DN] = sd;
        a.sched[SCHED_ROWS] = s;
    }
    __syncthreads();
    for (int e = tid; e <= a.E; e += blockDim.x) a.offsets[e] = off[e];
    if (a.counts_out)
        for (int e = tid; e < a.E; e += blockDim.x) a.counts_out[e] = cnt[e];
    for (int g = 0; g < 2; ++g) {
        const int F = g ? a.F_dn : a.F_gu;
        const int S = split_s[g];
        int4* units = g ? a.units_dn : a.units_gu;
        int ubase = 0;
        for (int e = 0; e < a.E; ++e) {
            const int n = cnt[e];
            const int mt = (n + a.BN - 1) / a.BN;
            const int nu = mt * F * S;
            for (int i = tid; i < nu; i += blockDim.x) {
                const int u = ubase + i;
                if (u >= a.max_units) break;
                const int m = i / (F * S);
                const int rem = i % (F * S);
                const int ft = rem / S, sp = rem % S;
                units[u] = make_int4(e, off[e] + m * a.BN, min(a.BN, n - m * a.BN), ft | (sp << 16));
            }
            ubase += nu;
        }
    }
}

__device__ __forceinline__ __half to_half_sat(float v) {
    v = fminf(fmaxf(v, -65504.f), 65504.f);
    return __float2half_rn(v);
}

template <typename TA> struct RowLoader;
template <> struct RowLoader<__nv_bfloat16> {
    // 8 consecutive elements -> 8 f16 (one 16-byte store)
    static __device__ __forceinline__ uint4 load8(const __nv_bfloat16* p) {
        const uint4 v = *reinterpret_cast<const uint4*>(p);
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
        uint4 o;
        __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(b[i]);
            h[i] = __halves2half2(to_half_sat(f.x), to_half_sat(f.y));
        }
        return o;
    }
};
template <> struct RowLoader<float> {
    static __device__ __forceinline__ uint4 load8(const float* p) {
        const float4 a = *reinterpret_cast<const float4*>(p);
        const float4 b = *reinterpret_cast<const float4*>(p + 4);
        uint4 o;
        __half2* h = reinterpret_cast<__half2*>(&o);
        h[0] = __halves2half2(to_half_sat(a.x), to_half_sat(a.y));
        h[1] = __halves2half2(to_half_sat(a.z), to_half_sat(a.w));
        h[2] = __halves2half2(to_half_sat(b.x), to_half_sat(b.y));
        h[3] = __halves2half2(to_half_sat(b.z), to_half_sat(b.w));
        return o;
    }
};

// Same token blocking as router_kernel.  Each (token, slot) pair of the block
// gets its grouped row: offsets[e] + (rows of e in earlier blocks) + (rank among
// earlier pairs of e in this block), so rows of an expert are in (token, slot)
// order.  The block then copies its token rows into the grouped activation
// matrix as f16 (16-byte vectors) and, when the gate/up GEMM splits K, zeroes
// the matching rows of its fp32 partial-sum buffer.
template <typename TA>
__global__ void __launch_bounds__(ROUTER_THREADS)
permute_kernel(const TA* __restrict__ x, const int32_t* __restrict__ idx, const float* __restrict__ w,
               const int32_t* __restrict__ hist_prefix, const int32_t* __restrict__ offsets, int T, int d, int E,
               int k, int32_t* __restrict__ row_token, float* __restrict__ row_weight, __half* __restrict__ Xp,
               float* __restrict__ GU, int gu_ld, const int32_t* __restrict__ sched) {
    __shared__ int es[ROUTER_TOKENS * MAX_TOPK];
    __shared__ int pos_s[ROUTER_TOKENS * MAX_TOPK];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * ROUTER_TOKENS;
    const int npairs = min(ROUTER_TOKENS, T - t0) * k;
    int e = -1;
    if (tid < npairs) {
        e = idx[static_cast<size_t>(t0) * k + tid];
        es[tid] = e;
    }
    __syncthreads();
    if (tid < npairs) {
        int rank = 0;
        for (int q = 0; q < tid; ++q) rank += (es[q] == e);
        const int pos = offsets[e] + hist_prefix[static_cast<size_t>(blockIdx.x) * E + e] + rank;
        pos_s[tid] = pos;
        row_token[pos] = t0 + tid / k;
        row_weight[pos] = w[static_cast<size_t>(t0) * k + tid];
    }
    __syncthreads();
    const bool split = sched[SCHED_SPLIT_GU] > 1;
    const int nvec = d / 8;
    for (int r = warp; r < npairs; r += ROUTER_THREADS / 32) {
        const int t = t0 + r / k;
        const int pos = pos_s[r];
        const TA* src = x + static_cast<size_t>(t) * d;
        uint4* dst = reinterpret_cast<uint4*>(Xp + static_cast<size_t>(pos) * d);
        for (int v = lane; v < nvec; v += 32) dst[v] = RowLoader<TA>::load8(src + v * 8);
        if (split) {
            float4* g = reinterpret_cast<float4*>(GU + static_cast<size_t>(pos) * gu_ld);
            for (int v = lane; v < gu_ld / 4; v += 32) g[v] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

__device__ __forceinline__ float swish_f(float z) { return z / (1.0f + __expf(-z)); }

// Split-K finish of the gate/up GEMM: H = Swish(G) * U from the fp32 partial
// sums (only when the schedule split K).
__global__ void swiglu_finish_kernel(const float* __restrict__ GU, __half* __restrict__ H, int d_ff,
                                     const int32_t* __restrict__ sched) {
    if (sched[SCHED_SPLIT_GU] <= 1) return;
    const int rows = sched[SCHED_ROWS];
    const size_t n = static_cast<size_t>(rows) * d_ff;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t r = i / d_ff, f = i % d_ff;
        const float g = GU[r * 2 * d_ff + f], u = GU[r * 2 * d_ff + d_ff + f];
        H[i] = to_half_sat(swish_f(g) * u);
    }
}

// fp32 accumulator -> bf16 output, 4 elements per thread-iteration.
__global__ void cast_out_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ y, size_t n4) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const float4 v = reinterpret_cast<const float4*>(acc)[i];
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
        __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
        uint2 o;
        o.x = *reinterpret_cast<uint32_t*>(&a);
        o.y = *reinterpret_cast<uint32_t*>(&b);
        reinterpret_cast<uint2*>(y)[i] = o;
    }
}

}  // namespace moe
