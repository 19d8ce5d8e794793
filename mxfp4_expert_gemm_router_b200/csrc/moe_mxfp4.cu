// moe_mxfp4.cu -- C ABI of the MoE feed-forward layer with MXFP4 experts
// (declarations and argument contracts in include/moe_mxfp4.h).
//
// A forward of at most 16 tokens is one cooperative launch of
// decode_fused_kernel (router, both expert GEMMs and the combine in one
// persistent grid).  Larger forwards are up to seven launches on the caller's
// stream; no host sync and no allocation either way:
//   router_tc_kernel     scores on the tensor cores (bf16 layers; router_kernel
//                        on the CUDA cores for fp32 ones), K split over the grid;
//                        top-k, softmax over the selected scores, per-tile
//                        histogram and ranks; its last CTA builds the schedule
//                        (expert offsets, K splits, unit counts)
//   rows_kernel          the unit lists; grouped rows (token, weight, tile
//                        slot); output accumulator initialised when K is split
//   encode_rows_kernel   the grouped rows of x encoded as the gate/up GEMM's B
//                        operand (three MXFP4 or two MXFP8 terms)
//   expert_mxf4<0>       gate/up GEMM on block-scaled tensor cores (kind::mxf4,
//                        or kind::mxf8f6f4 for two MXFP8 terms), SwiGLU epilogue
//                        encoding H for the down GEMM (fp32 partials instead
//                        when K is split)
//   h_encode_kernel      only when the gate/up GEMM may split K: SwiGLU + encoding
//   expert_mxf4<1>       down GEMM: each grouped row's weighted output stored
//                        once (a fp32 scatter-add when K is split)
//   combine_out_kernel   y = (x) + the sum of each token's k rows, in slot order
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <new>

#include "../../include/moe_mxfp4.h"
#include "decode_fused.cuh"
#include "expert_mxf4.cuh"
#include "quantize.cuh"
#include "router_tc.cuh"
#include "routing.cuh"

using namespace moe;

namespace {

constexpr int BN_OPTIONS = 8;  // BN = 16 * (i + 1): 16 .. 128
constexpr int SPLIT_ROWS_CAP = 2048;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

}  // namespace

struct moe_mxfp4 {
    moe_mxfp4_config_t cfg;
    int dev = 0, nsm = 0;
    int act_bytes = 2;
    int KC_gu = 0, KC_dn = 0, F_gu = 0, F_dn = 0;
    int TK = 0, nblk_max = 0, max_units = 0, gu_rows = 0;
    int af = 0;                // activation operand format: 0 three MXFP4 terms, 1 two MXFP8 terms
    size_t part_elems = 0;
    // weights
    uint8_t* w_gu = nullptr;   // tiled gate+up
    uint8_t* w_dn = nullptr;   // tiled down
    void* w_router = nullptr;
    float* bias = nullptr;
    bool has_bias = false, router_set = false;
    // optional steps adjacent to the block: pre-norm (gamma) and residual
    float* gamma = nullptr;    // [d_model]
    bool use_norm = false, residual = false;
    float eps = 0.f;
    int experts_quantized = 0;
    bool* expert_done = nullptr;
    // workspace
    int32_t* idx_ws = nullptr;
    float* w_ws = nullptr;
    int32_t* hist = nullptr;
    double* part = nullptr;
    double* part_ss = nullptr;   // router partial sums of x^2 (pre-norm)
    float* inv_rms = nullptr;    // [max_tokens] 1 / rms(x) (pre-norm)
    int* counters = nullptr;   // [nblk_max] tile counters + [1] global counter
    int32_t* local_rank = nullptr;
    int32_t* offsets = nullptr;
    int32_t* tile_base = nullptr;
    int32_t* sched = nullptr;
    int4* units_gu = nullptr;
    int4* units_dn = nullptr;
    int32_t* row_token = nullptr;
    float* row_weight = nullptr;
    int32_t* row_slot = nullptr;
    uint8_t* Xq = nullptr;     // x as three MXFP4 terms [d/32][3][TK][16]
    uint8_t* Hq = nullptr;     // H as three MXFP4 terms [d_ff/32][3][TK][16]
    uint8_t* sfx = nullptr;    // scale atoms of Xq per (token tile, K chunk)
    uint8_t* sfh = nullptr;    // scale atoms of Hq per (token tile, K chunk)
    size_t sfx_bytes = 0, sfh_bytes = 0, xq_bytes = 0, hq_bytes = 0;
    float* GU = nullptr;
    float* yacc = nullptr;      // fp32 output accumulator (down GEMM with split K)
    void* obuf = nullptr;       // weighted output of each grouped row (down GEMM without split K)
    int32_t* pair_row = nullptr;  // grouped row of each (token, slot) pair
    int* status = nullptr;
    void* x_stage = nullptr;
    void* y_stage = nullptr;
    int32_t* idx_stage = nullptr;
    float* w_stage = nullptr;
    // tensor maps per BN
    CUtensorMap tm_x[BN_OPTIONS];
    CUtensorMap tm_h[BN_OPTIONS];
    bool tm_ok[BN_OPTIONS] = {};
    CUtensorMap tm_wgu{}, tm_wdn{};
    // tensor-core router (bf16 layers): the weight planes and their map
    __nv_bfloat16* wr_planes = nullptr;   // [3][E][d]: gamma * W_router as hi, mid, lo (with the pre-norm)
    CUtensorMap tm_wr{};
    int router_P = 1;                     // planes the map covers (1: W_router itself, 3: the planes)   // two-MXFP8-term layers: the padded weights as 16U4_ALIGN16B boxes
    // fused decode path (forwards of at most DF_MAX_T tokens)
    bool df_ok = false, last_fused = false;
    int df_stages = 0, df_S = 0, df_nb_max = 0, df_kc_max = 0, df_max_touched = 0;
    size_t df_smem = 0;
    DecodeState* df_state = nullptr;
    double* df_part = nullptr;
    double* df_part_ss = nullptr;
    float* df_yacc = nullptr;
    uint8_t* df_xq = nullptr;
    uint8_t* df_hq = nullptr;
    size_t df_hq_stride = 0;
    uint32_t* df_hdone = nullptr;
    cudaStream_t last_stream = nullptr;
    // forward_host: copy streams and per-chunk events (copies overlap compute)
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_done = nullptr;
    cudaEvent_t ev_in[8] = {}, ev_out[8] = {};
    // debug build: the guard region after each device buffer
    uint8_t* guard_ptr[48] = {};
    int n_guards = 0;
    // profiling
    bool prof = false, prof_valid = false;
    cudaEvent_t ev[MOE_NUM_STAGES + 1] = {};
    bool stage_ran[MOE_NUM_STAGES] = {};
    uint64_t launches = 0;
};

// Kernel attributes belong to the current device's context, so they are set
// once per device, under a lock (create and the no-allocation router both call
// this).  The router's shared-memory limit is always the one for the largest
// expert count, so no caller ever lowers it below what another layer needs.
constexpr int MOE_MAX_DEVICES = 64;
static std::mutex g_attr_mutex;
static bool g_attrs_set[MOE_MAX_DEVICES] = {};

static bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Debug build: every device buffer of a handle is followed by MOE_GUARD_BYTES
// of a known pattern; moe_mxfp4_check_guards reports any that changed.
#ifdef MOE_DEBUG_CHECKS
constexpr size_t MOE_GUARD_BYTES = 4096;
#else
constexpr size_t MOE_GUARD_BYTES = 0;
#endif
constexpr unsigned char MOE_GUARD_BYTE = 0xA5;

// Launch with programmatic stream serialization when `pdl` is set: the kernel
// may start while the previous kernel in the stream finishes (it runs its
// local set-up, then waits in pdl_wait for the previous kernel's results).
// Used for decode-sized forwards, where launch latency and kernel ramp-up are
// a large share of the step; with large grids, dependents launched early only
// take residency from the running kernel.
template <typename... KArgs, typename... Args>
static void launch_pdl(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaLaunchKernelEx(&cfg, kernel, args...);
}

static moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                                   \
    do {                                                \
        cudaError_t _e = (expr);                        \
        if (_e != cudaSuccess) return MOE_ERR_CUDA;     \
    } while (0)

// One device allocation of a handle (at least 256 bytes), with the debug
// build's guard region after it.
static cudaError_t handle_alloc(moe_mxfp4* h, void** p, size_t bytes) {
    const size_t n = std::max<size_t>(bytes, 256);
    cudaError_t e = cudaMalloc(p, n + MOE_GUARD_BYTES);
    if (e != cudaSuccess || MOE_GUARD_BYTES == 0) return e;
    uint8_t* g = static_cast<uint8_t*>(*p) + n;
    if ((e = cudaMemset(g, MOE_GUARD_BYTE, MOE_GUARD_BYTES)) != cudaSuccess) return e;
    if (h->n_guards < static_cast<int>(sizeof(h->guard_ptr) / sizeof(h->guard_ptr[0])))
        h->guard_ptr[h->n_guards++] = g;
    return cudaSuccess;
}

static void free_all(moe_mxfp4* h) {
    void* ptrs[] = {h->w_gu, h->w_dn, h->w_router, h->bias, h->gamma, h->part_ss, h->inv_rms,
                    h->idx_ws, h->w_ws, h->hist,
                    h->part, h->counters, h->local_rank, h->offsets, h->tile_base, h->sched, h->units_gu,
                    h->units_dn, h->row_token, h->row_weight, h->row_slot, h->Xq, h->Hq, h->sfx, h->sfh,
                    h->GU, h->yacc, h->obuf, h->pair_row, h->status, h->x_stage, h->y_stage, h->idx_stage, h->w_stage,
                    h->df_state, h->df_part, h->df_part_ss, h->df_yacc, h->df_xq, h->df_hq, h->df_hdone,
                    h->wr_planes};
    for (void* p : ptrs)
        if (p) cudaFree(p);
    for (auto& e : h->ev)
        if (e) cudaEventDestroy(e);
    for (int i = 0; i < 8; ++i) {
        if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
        if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
    }
    if (h->ev_start) cudaEventDestroy(h->ev_start);
    if (h->ev_done) cudaEventDestroy(h->ev_done);
    if (h->s_in) cudaStreamDestroy(h->s_in);
    if (h->s_out) cudaStreamDestroy(h->s_out);
    delete[] h->expert_done;
}

// Token rows per tile: about three times the mean rows per expert, so that
// most experts need one tile (each tile streams the expert's weights once),
// rounded up to 16 and capped at 128.  Flags may force it.
static int choose_bn(int T, int k, int E, uint32_t flags) {
    const uint32_t forced = (flags & MOE_FLAG_TOKEN_TILE_MASK) >> MOE_FLAG_TOKEN_TILE_SHIFT;
    if (forced >= 1 && forced <= BN_OPTIONS) return 16 * static_cast<int>(forced);
    const long per_expert = (static_cast<long>(T) * k + E - 1) / E;
    const long want = std::min<long>(T, std::max<long>(1, 3 * per_expert));
    const int bn = static_cast<int>((want + 15) / 16) * 16;
    return std::max(16, std::min(MXG_MAX_BN, bn));
}

// Scale atoms per K chunk over all token tiles: an expert with n rows has
// ceil(n / BN) tiles, so at most TK / 16 + E tiles (the smallest tile), each
// with one atom per term.
static size_t max_tile_atoms(size_t TK, int E) { return (TK / 16 + E) * MXQ_TERMS; }

static TiledMatrix tiled(moe_mxfp4* h, int which) {
    const auto& c = h->cfg;
    TiledMatrix M;
    M.padded = h->af;
    if (which < 2) {
        M.base = h->w_gu;
        M.N = c.d_ff;
        M.K = c.d_model;
        M.NM = 2;
        M.sub = which;
    } else {
        M.base = h->w_dn;
        M.N = c.d_model;
        M.K = c.d_ff;
        M.NM = 1;
        M.sub = 0;
    }
    return M;
}

// K splits of the router: enough CTAs (token tiles x expert tiles x splits) to
// cover the SMs twice, at most ROUTER_MAX_SPLITS and one 64-wide K chunk per
// split (the last CTA of a token tile sums the splits' partials).
static int router_etiles(int E) { return (E + ROUTER_ETILE - 1) / ROUTER_ETILE; }
static int router_splits(int T, int d, int E, int nsm) {
    const int tiles = (T + ROUTER_TOKENS - 1) / ROUTER_TOKENS;
    const int kch = (d + ROUTER_KCHUNK - 1) / ROUTER_KCHUNK;
    const int ctas = tiles * router_etiles(E);
    const int want = (2 * nsm + ctas - 1) / ctas;
    return std::max(1, std::min(std::min(kch, ROUTER_MAX_SPLITS), want));
}

// CUDA-core router launch (fp32 activations and the no-allocation entry point).
template <typename TA>
static void launch_router(const RouterArgs& ra, dim3 grid, size_t smem, cudaStream_t stream) {
    router_kernel<TA><<<grid, ROUTER_THREADS, smem, stream>>>(ra);
}
template <typename TA>
static cudaError_t set_router_smem(int bytes) {
    return cudaFuncSetAttribute(router_kernel<TA>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// The handle's buffers live on the device that was current at create: calls
// that launch work require it to be current again.
static moe_status_t check_device(const moe_mxfp4* h) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return MOE_ERR_CUDA;
    return cur == h->dev ? MOE_OK : MOE_ERR_INVALID_ARG;
}

static cudaError_t ensure_kernel_attrs(int dev) {
    if (dev < 0 || dev >= MOE_MAX_DEVICES) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    if (g_attrs_set[dev]) return cudaSuccess;
    const int rsm = static_cast<int>(router_smem_bytes());
    cudaError_t e;
    const void* gemms[] = {
        reinterpret_cast<const void*>(expert_mxf4_kernel<0, 0, 0>), reinterpret_cast<const void*>(expert_mxf4_kernel<0, 0, 1>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<1, 0, 0>), reinterpret_cast<const void*>(expert_mxf4_kernel<1, 0, 1>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<1, 0, 1, 1>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<0, 1, 0>), reinterpret_cast<const void*>(expert_mxf4_kernel<0, 1, 1>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<1, 1, 0>), reinterpret_cast<const void*>(expert_mxf4_kernel<1, 1, 1>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<0, 0, 0, 0, 0>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<1, 0, 0, 0, 0>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<0, 1, 0, 0, 0>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<1, 1, 0, 0, 0>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<0, 0, 1, 0, 0>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<1, 0, 1, 0, 0>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<1, 0, 1, 1, 0>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<0, 1, 1, 0, 0>),
        reinterpret_cast<const void*>(expert_mxf4_kernel<1, 1, 1, 0, 0>)};
    for (const void* k : gemms)
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024))) return e;
    if ((e = set_router_smem<float>(rsm))) return e;
    {
        const int tsm = static_cast<int>(rtc_smem_bytes(3));
        if ((e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tsm))) return e;
    }
    if ((e = set_router_smem<__nv_bfloat16>(rsm))) return e;
    if ((e = cudaFuncSetAttribute(decode_fused_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  227 * 1024)))
        return e;
    if ((e = cudaFuncSetAttribute(decode_fused_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  227 * 1024)))
        return e;
    g_attrs_set[dev] = true;
    return cudaSuccess;
}

static int stages_for(int mode, int BN, int af, int cps = 1) {
    const size_t budget = 227 * 1024 - 1024 - 512 - mxg_extra_smem(mode);
    int s = static_cast<int>(budget / (static_cast<size_t>(cps) * mxg_stage_bytes(mode, BN, af)));
    return std::max(2, std::min(MXG_MAX_STAGES, s));
}

extern "C" {

const char* moe_mxfp4_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_NOT_QUANTIZED: return "weights or router not set";
        case MOE_ERR_TIMEOUT: return "device pipeline wait timed out";
        case MOE_ERR_BOUNDS: return "a debug-build bounds check failed or a guard region changed";
    }
    return "unknown status";
}

const char* moe_mxfp4_stage_name(int32_t stage) {
    static const char* names[MOE_NUM_STAGES] = {"router_topk_schedule", "gather", "gate_up_swiglu",
                                                 "h_encode", "down", "combine_out", "fused_decode"};
    return (stage >= 0 && stage < MOE_NUM_STAGES) ? names[stage] : "unknown";
}

int64_t moe_mxfp4_expert_param_count(const moe_mxfp4_config_t* cfg) {
    if (!cfg) return -1;
    return 3LL * cfg->d_model * cfg->d_ff;
}

int64_t moe_mxfp4_expert_weight_bytes(const moe_mxfp4_config_t* cfg) {
    if (!cfg) return -1;
    return moe_mxfp4_expert_param_count(cfg) * 17 / 32;
}

uint64_t moe_mxfp4_launch_count(const moe_mxfp4_t* h) { return h ? h->launches : 0; }

static moe_status_t make_weight_tmaps(moe_mxfp4* h);

moe_status_t moe_mxfp4_create(const moe_mxfp4_config_t* cfg, moe_mxfp4_t** out) {
    if (!cfg || !out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    const moe_mxfp4_config_t c = *cfg;
    if (c.d_model <= 0 || c.d_ff <= 0 || c.n_experts <= 0 || c.top_k <= 0 || c.max_tokens <= 0)
        return MOE_ERR_INVALID_ARG;
    if (c.act_dtype != MOE_DTYPE_F32 && c.act_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (c.d_model % 32 || c.d_ff % 32 || c.n_experts > MAX_EXPERTS || c.top_k > std::min(MAX_TOPK, c.n_experts) ||
        c.d_model > 16384 || c.d_ff > 16384 || static_cast<long>(c.max_tokens) * c.top_k > (1L << 26))
        return MOE_ERR_UNSUPPORTED;
    if (!get_encode_fn()) return MOE_ERR_CUDA;

    moe_mxfp4* h = new (std::nothrow) moe_mxfp4();
    if (!h) return MOE_ERR_CUDA;
    h->cfg = c;
    h->act_bytes = c.act_dtype == MOE_DTYPE_BF16 ? 2 : 4;
    auto fail = [&](moe_status_t s) {
        free_all(h);
        delete h;
        return s;
    };
    if (cudaGetDevice(&h->dev) != cudaSuccess) return fail(MOE_ERR_CUDA);
    if (cudaDeviceGetAttribute(&h->nsm, cudaDevAttrMultiProcessorCount, h->dev) != cudaSuccess)
        return fail(MOE_ERR_CUDA);
    const int E = c.n_experts, d = c.d_model, f = c.d_ff, k = c.top_k;
    h->KC_gu = (d / 32 + 3) / 4;   // 128-wide chunks of the gate/up GEMM
    h->KC_dn = (f / 32 + 3) / 4;   // 128-wide chunks of the down GEMM
    h->F_gu = (f + 127) / 128;
    h->F_dn = (d + 127) / 128;
    h->TK = c.max_tokens * k;
    h->nblk_max = (c.max_tokens + ROUTER_TOKENS - 1) / ROUTER_TOKENS;
    {
        // every unit of the unsplit schedule fits: at most TK / 16 + E token
        // tiles (the smallest tile) times the feature tiles; K splits are only
        // chosen while the split list still fits
        const long tiles = static_cast<long>(h->TK) / 16 + E + 2;
        const long F = std::max(h->F_gu, h->F_dn);
        h->max_units = static_cast<int>(tiles * F + 8L * h->nsm + 64);
    }
    h->gu_rows = std::min(h->TK, SPLIT_ROWS_CAP);
    // partial scores [S][T][E]: S * T <= ROUTER_TOKENS * (S * tiles) <= ROUTER_TOKENS * (2 nsm + tiles)
    h->part_elems = static_cast<size_t>(ROUTER_TOKENS) * (2 * h->nsm + h->nblk_max + 1) * E;
    h->expert_done = new (std::nothrow) bool[E]();
    if (!h->expert_done) return fail(MOE_ERR_CUDA);

    const size_t TK = h->TK;
    h->af = (c.flags & MOE_FLAG_ACT_MXF8X2) ? 1 : 0;
    // operand codes per row and block: 3 terms x 16 B, or 2 terms x 32 B
    const size_t block_code_bytes = h->af ? 2 * 32 : MXQ_TERMS * 16;
    h->xq_bytes = static_cast<size_t>(d / 32) * block_code_bytes * TK;
    h->hq_bytes = static_cast<size_t>(f / 32) * block_code_bytes * TK;
    h->sfx_bytes = max_tile_atoms(TK, E) * h->KC_gu * 512;
    h->sfh_bytes = max_tile_atoms(TK, E) * h->KC_dn * 512;
    const size_t gu_bytes = static_cast<size_t>(E) * tiled(h, 0).expert_bytes();
    const size_t dn_bytes = static_cast<size_t>(E) * tiled(h, 2).expert_bytes();
    struct A { void** p; size_t bytes; };
    A allocs[] = {
        {reinterpret_cast<void**>(&h->w_gu), gu_bytes},
        {reinterpret_cast<void**>(&h->w_dn), dn_bytes},
        {&h->w_router, static_cast<size_t>(E) * d * h->act_bytes},
        {reinterpret_cast<void**>(&h->bias), sizeof(float) * E},
        {reinterpret_cast<void**>(&h->idx_ws), sizeof(int32_t) * TK},
        {reinterpret_cast<void**>(&h->w_ws), sizeof(float) * TK},
        {reinterpret_cast<void**>(&h->hist), sizeof(int32_t) * static_cast<size_t>(h->nblk_max) * E},
        {reinterpret_cast<void**>(&h->part), sizeof(double) * h->part_elems},
        {reinterpret_cast<void**>(&h->part_ss), sizeof(double) * (h->part_elems / E + 64)},
        {reinterpret_cast<void**>(&h->inv_rms), sizeof(float) * c.max_tokens},
        {reinterpret_cast<void**>(&h->gamma), sizeof(float) * d},
        {reinterpret_cast<void**>(&h->counters), sizeof(int) * (h->nblk_max + 1)},
        {reinterpret_cast<void**>(&h->local_rank), sizeof(int32_t) * TK},
        {reinterpret_cast<void**>(&h->offsets), sizeof(int32_t) * (E + 1)},
        {reinterpret_cast<void**>(&h->tile_base), sizeof(int32_t) * E},
        {reinterpret_cast<void**>(&h->sched), sizeof(int32_t) * SCHED_SLOTS},
        {reinterpret_cast<void**>(&h->units_gu), sizeof(int4) * h->max_units},
        {reinterpret_cast<void**>(&h->units_dn), sizeof(int4) * h->max_units},
        {reinterpret_cast<void**>(&h->row_token), sizeof(int32_t) * TK},
        {reinterpret_cast<void**>(&h->row_weight), sizeof(float) * TK},
        {reinterpret_cast<void**>(&h->row_slot), sizeof(int32_t) * TK},
        {reinterpret_cast<void**>(&h->Xq), h->xq_bytes},
        {reinterpret_cast<void**>(&h->Hq), h->hq_bytes},
        {reinterpret_cast<void**>(&h->sfx), h->sfx_bytes},
        {reinterpret_cast<void**>(&h->sfh), h->sfh_bytes},
        {reinterpret_cast<void**>(&h->GU), sizeof(float) * h->gu_rows * 2 * f},
        {reinterpret_cast<void**>(&h->yacc), sizeof(float) * static_cast<size_t>(c.max_tokens) * d},
        {&h->obuf, TK * d * static_cast<size_t>(h->act_bytes)},
        {reinterpret_cast<void**>(&h->pair_row), sizeof(int32_t) * TK},
        {reinterpret_cast<void**>(&h->status), sizeof(int) * 4},
        {&h->x_stage, static_cast<size_t>(c.max_tokens) * d * h->act_bytes},
        {reinterpret_cast<void**>(&h->wr_planes), 3 * static_cast<size_t>(E) * d * sizeof(__nv_bfloat16)},
        {&h->y_stage, static_cast<size_t>(c.max_tokens) * d * h->act_bytes},
        {reinterpret_cast<void**>(&h->idx_stage), sizeof(int32_t) * TK},
        {reinterpret_cast<void**>(&h->w_stage), sizeof(float) * TK},
    };
    // test hook: the fail_at-th device allocation (1-based) fails as if cudaMalloc had
    const uint32_t fail_at = (c.flags & MOE_FLAG_TEST_FAIL_ALLOC_MASK) >> MOE_FLAG_TEST_FAIL_ALLOC_SHIFT;
    uint32_t n_alloc = 0;
    for (auto& a : allocs) {
        if (++n_alloc == fail_at) return fail(MOE_ERR_CUDA);
        if (handle_alloc(h, a.p, a.bytes) != cudaSuccess) return fail(MOE_ERR_CUDA);
    }
    // Operand buffers start as zeros: codes, scale atoms and the weights' padding
    // are then always finite (an E2M1 code is never NaN; scale bytes written by
    // the kernels are at most 253, never the E8M0 NaN 0xFF), so operand rows a
    // tile reads past its expert's rows only feed accumulator columns that the
    // epilogue drops.  The status word starts clear.
    if (cudaMemset(h->Xq, 0, h->xq_bytes) != cudaSuccess || cudaMemset(h->Hq, 0, h->hq_bytes) != cudaSuccess ||
        cudaMemset(h->sfx, 0, h->sfx_bytes) != cudaSuccess || cudaMemset(h->sfh, 0, h->sfh_bytes) != cudaSuccess ||
        cudaMemset(h->w_gu, 0, gu_bytes) != cudaSuccess || cudaMemset(h->w_dn, 0, dn_bytes) != cudaSuccess ||
        cudaMemset(h->status, 0, sizeof(int) * 4) != cudaSuccess ||
        cudaMemset(h->counters, 0, sizeof(int) * (h->nblk_max + 1)) != cudaSuccess ||
        cudaMemset(h->bias, 0, sizeof(float) * E) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
        return fail(MOE_ERR_CUDA);

    if (ensure_kernel_attrs(h->dev) != cudaSuccess) return fail(MOE_ERR_CUDA);
    if (h->af && make_weight_tmaps(h) != MOE_OK) return fail(MOE_ERR_CUDA);

    // fused decode path: one persistent grid for forwards of at most DF_MAX_T
    // tokens, when its shared-memory plan fits (the whole-K B operand plus at
    // least two weight stages) and one CTA per SM can be resident
    {
        h->df_nb_max = std::max(d, f) / 32;
        h->df_kc_max = std::max(h->KC_gu, h->KC_dn);
        const size_t fixed = df_smem_bytes(0, h->df_nb_max, h->df_kc_max);
        const long st = (227L * 1024 - static_cast<long>(fixed)) / static_cast<long>(DF_STAGE);
        h->df_stages = static_cast<int>(std::min<long>(st, DF_MAX_STAGES));
        // the router's scratch (2 x 16 x K chunks doubles) and logits live in the ring
        const size_t router_scratch = 2 * DF_MAX_T * sizeof(double) * ((d + ROUTER_KCHUNK - 1) / ROUTER_KCHUNK);
        const size_t logits = DF_MAX_T * sizeof(float) * (E + 1);
        // (the fused kernel reads three-MXFP4-term operands only)
        if (!h->af && h->df_stages >= 2 &&
            std::max(router_scratch, logits) <= static_cast<size_t>(h->df_stages) * DF_STAGE) {
            h->df_smem = df_smem_bytes(h->df_stages, h->df_nb_max, h->df_kc_max);
            const int kch = (d + ROUTER_KCHUNK - 1) / ROUTER_KCHUNK;
            h->df_S = std::max(1, std::min(h->nsm / E, kch));
            h->df_max_touched = std::min(E, DF_MAX_T * k);
            int per_sm = 0;
            cudaError_t oe =
                c.act_dtype == MOE_DTYPE_BF16
                    ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_kernel<__nv_bfloat16>,
                                                                    DF_THREADS, h->df_smem)
                    : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_kernel<float>, DF_THREADS,
                                                                    h->df_smem);
            if (oe != cudaSuccess) return fail(MOE_ERR_CUDA);
            if (per_sm >= 1) {
                const size_t ya_bytes_df = sizeof(float) * 2 * DF_MAX_T * static_cast<size_t>(d);
                const size_t stamp_bytes = sizeof(uint32_t) * h->df_max_touched * h->F_gu * DF_EPI_WARPS;
                const size_t xq_bytes = static_cast<size_t>(d / 32) * DF_B_BLOCK + static_cast<size_t>(h->KC_gu) * 512;
                h->df_hq_stride = static_cast<size_t>(f / 32) * DF_B_BLOCK + static_cast<size_t>(h->KC_dn) * 512;
                A dfa[] = {
                    {reinterpret_cast<void**>(&h->df_state), sizeof(DecodeState)},
                    {reinterpret_cast<void**>(&h->df_part), sizeof(double) * h->df_S * DF_MAX_T * E},
                    {reinterpret_cast<void**>(&h->df_part_ss), sizeof(double) * h->df_S * DF_MAX_T},
                    {reinterpret_cast<void**>(&h->df_yacc), ya_bytes_df},
                    {reinterpret_cast<void**>(&h->df_xq), xq_bytes},
                    {reinterpret_cast<void**>(&h->df_hq), h->df_hq_stride * h->df_max_touched},
                    {reinterpret_cast<void**>(&h->df_hdone), stamp_bytes},
                };
                for (auto& a : dfa) {
                    if (++n_alloc == fail_at) return fail(MOE_ERR_CUDA);
                    if (handle_alloc(h, a.p, a.bytes) != cudaSuccess) return fail(MOE_ERR_CUDA);
                    if (cudaMemset(*a.p, 0, std::max<size_t>(a.bytes, 256)) != cudaSuccess) return fail(MOE_ERR_CUDA);
                }
                if (cudaDeviceSynchronize() != cudaSuccess) return fail(MOE_ERR_CUDA);
                h->df_ok = true;
            }
        }
    }
    for (auto& e : h->ev)
        if (cudaEventCreate(&e) != cudaSuccess) return fail(MOE_ERR_CUDA);
    if (cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_start, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_done, cudaEventDisableTiming) != cudaSuccess)
        return fail(MOE_ERR_CUDA);
    for (int i = 0; i < 8; ++i)
        if (cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming) != cudaSuccess)
            return fail(MOE_ERR_CUDA);
    *out = h;
    return MOE_OK;
}

void moe_mxfp4_destroy(moe_mxfp4_t* h) {
    if (!h) return;
    cudaDeviceSynchronize();
    free_all(h);
    delete h;
}


// Quantise experts [e0, e0+ne) of one matrix from fp32 [ne][K][N].
static moe_status_t quantize_matrix(moe_mxfp4* h, int which, const float* W, int e0, int ne, cudaStream_t s) {
    TiledMatrix M = tiled(h, which);
    M.base += static_cast<size_t>(e0) * M.expert_bytes();
    const dim3 blk(128);
    const dim3 grid((M.N + 127) / 128, M.nb(), ne);
    quantize_kernel<<<grid, blk, 0, s>>>(W, static_cast<size_t>(M.K) * M.N, M);
    h->launches++;
    return cuda_status(cudaGetLastError());
}

// The tensor-core router's weight operand (bf16 layers): W_router itself, or
// with the pre-norm gamma * W_router as three bf16 planes; and its map, a 3-D
// view {d, E, planes} read in boxes {64, 32, planes} with the 128-byte swizzle.
static moe_status_t prepare_router_tc(moe_mxfp4* h, cudaStream_t stream) {
    const auto& c = h->cfg;
    if (c.act_dtype != MOE_DTYPE_BF16 || !h->router_set) return MOE_OK;
    const int E = c.n_experts, d = c.d_model;
    void* src = h->w_router;
    h->router_P = 1;
    if (h->use_norm) {
        const long n = static_cast<long>(E) * d;
        const int blocks = static_cast<int>(std::min<long>(4L * h->nsm, (n + 255) / 256));
        router_planes_kernel<<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(h->w_router), h->gamma,
                                                          h->wr_planes, E, d);
        h->launches++;
        MOE_TRY(cudaGetLastError());
        src = h->wr_planes;
        h->router_P = 3;
    }
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return MOE_ERR_CUDA;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(E), static_cast<cuuint64_t>(h->router_P)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(E) * d * 2};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(ROUTER_KCHUNK), static_cast<cuuint32_t>(ROUTER_ETILE),
                         static_cast<cuuint32_t>(h->router_P)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&h->tm_wr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, src, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_mxfp4_set_router(moe_mxfp4_t* h, const void* w_router, const float* router_bias,
                                  cudaStream_t stream) {
    if (!h || !w_router) return MOE_ERR_INVALID_ARG;
    const auto& c = h->cfg;
    MOE_TRY(cudaMemcpyAsync(h->w_router, w_router, static_cast<size_t>(c.n_experts) * c.d_model * h->act_bytes,
                            cudaMemcpyDeviceToDevice, stream));
    if (router_bias) {
        MOE_TRY(cudaMemcpyAsync(h->bias, router_bias, sizeof(float) * c.n_experts, cudaMemcpyDeviceToDevice, stream));
    } else {
        MOE_TRY(cudaMemsetAsync(h->bias, 0, sizeof(float) * c.n_experts, stream));
    }
    h->has_bias = router_bias != nullptr;
    h->router_set = true;
    h->last_stream = stream;
    return prepare_router_tc(h, stream);
}

moe_status_t moe_mxfp4_set_norm_residual(moe_mxfp4_t* h, const float* gamma, float eps, int32_t residual,
                                        cudaStream_t stream) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 1e30f || !aligned_to(gamma, 4)) return MOE_ERR_INVALID_ARG;
    if (gamma)
        MOE_TRY(cudaMemcpyAsync(h->gamma, gamma, sizeof(float) * h->cfg.d_model, cudaMemcpyDeviceToDevice, stream));
    h->use_norm = gamma != nullptr;
    h->eps = eps;
    h->residual = residual != 0;
    h->last_stream = stream;
    return prepare_router_tc(h, stream);
}

moe_status_t moe_mxfp4_quantize_expert(moe_mxfp4_t* h, int32_t e, const float* w_gate, const float* w_up,
                                       const float* w_down, cudaStream_t stream) {
    if (!h || !w_gate || !w_up || !w_down) return MOE_ERR_INVALID_ARG;
    if (e < 0 || e >= h->cfg.n_experts) return MOE_ERR_INVALID_ARG;
    if (!aligned_to(w_gate, 4) || !aligned_to(w_up, 4) || !aligned_to(w_down, 4)) return MOE_ERR_INVALID_ARG;
    moe_status_t st;
    if ((st = quantize_matrix(h, 0, w_gate, e, 1, stream)) != MOE_OK) return st;
    if ((st = quantize_matrix(h, 1, w_up, e, 1, stream)) != MOE_OK) return st;
    if ((st = quantize_matrix(h, 2, w_down, e, 1, stream)) != MOE_OK) return st;
    if (!h->expert_done[e]) {
        h->expert_done[e] = true;
        h->experts_quantized++;
    }
    h->last_stream = stream;
    return MOE_OK;
}

moe_status_t moe_mxfp4_quantize_weights(moe_mxfp4_t* h, const float* w_gate, const float* w_up,
                                        const float* w_down, const void* w_router, const float* router_bias,
                                        cudaStream_t stream) {
    if (!h || !w_gate || !w_up || !w_down || !w_router) return MOE_ERR_INVALID_ARG;
    if (!aligned_to(w_gate, 4) || !aligned_to(w_up, 4) || !aligned_to(w_down, 4)) return MOE_ERR_INVALID_ARG;
    const int E = h->cfg.n_experts;
    moe_status_t st;
    if ((st = quantize_matrix(h, 0, w_gate, 0, E, stream)) != MOE_OK) return st;
    if ((st = quantize_matrix(h, 1, w_up, 0, E, stream)) != MOE_OK) return st;
    if ((st = quantize_matrix(h, 2, w_down, 0, E, stream)) != MOE_OK) return st;
    for (int e = 0; e < E; ++e) h->expert_done[e] = true;
    h->experts_quantized = E;
    return moe_mxfp4_set_router(h, w_router, router_bias, stream);
}

moe_status_t moe_mxfp4_export_weights(const moe_mxfp4_t* hc, int32_t which, uint8_t* codes, uint8_t* scales,
                                      cudaStream_t stream) {
    if (!hc || !codes || !scales || which < 0 || which > 2) return MOE_ERR_INVALID_ARG;
    if (!aligned_to(codes, 16)) return MOE_ERR_INVALID_ARG;   // codes are written 16 bytes at a time
    moe_mxfp4* h = const_cast<moe_mxfp4*>(hc);
    TiledMatrix M = tiled(h, which);
    const dim3 grid((M.N + 127) / 128, M.K / 32, h->cfg.n_experts);
    export_kernel<<<grid, 128, 0, stream>>>(M, codes, scales);
    h->launches++;
    return cuda_status(cudaGetLastError());
}

// 3-D maps over the activation operands, read as 8-byte elements so that the
// innermost box dimension is one contiguous run of BN rows (BN * 16 bytes).
// Three MXFP4 terms, [K/32 blocks][3 terms][TK rows x 16 B]: box {2 BN, 3
// terms, 4 blocks} lands in shared memory as [4 blocks][3 terms][BN rows][16 B].
// Two MXFP8 terms, [K/16 chunks][2 terms][TK rows x 16 B]: box {2 BN, 2 terms,
// 8 chunks} lands as [8 chunks][2 terms][BN rows][16 B].  Either is the
// unswizzled K-major layout of each term's operand.  Rows past TK and blocks
// past K read as zeros.
static moe_status_t ensure_tmaps(moe_mxfp4* h, int BN) {
    const int i = BN / 16 - 1;
    if (h->tm_ok[i]) return MOE_OK;
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return MOE_ERR_CUDA;
    const auto& c = h->cfg;
    const cuuint64_t R = static_cast<cuuint64_t>(h->TK);
    const cuuint32_t terms = h->af ? 2 : MXQ_TERMS, cpb = h->af ? 2 : 1;
    for (int which = 0; which < 2; ++which) {
        const cuuint64_t nch = (which == 0 ? c.d_model : c.d_ff) / 32 * cpb;
        cuuint64_t dims[3] = {2 * R, terms, nch};
        cuuint64_t strides[2] = {R * 16, R * 16 * terms};
        cuuint32_t box[3] = {static_cast<cuuint32_t>(2 * BN), terms, 4 * cpb};
        cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(which == 0 ? &h->tm_x[i] : &h->tm_h[i], CU_TENSOR_MAP_DATA_TYPE_UINT64, 3,
                         which == 0 ? static_cast<void*>(h->Xq) : static_cast<void*>(h->Hq), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return MOE_ERR_CUDA;
    }
    h->tm_ok[i] = true;
    return MOE_OK;
}

// Two-MXFP8-term layers keep the weights in the padded form: parts of 8704
// bytes (codes [128 rows][64 B] + a scale atom).  The map views the array as
// {128 four-bit elements, 128 rows, parts} with the 16U4_ALIGN16B type and the
// 128-byte swizzle: a {128, 128, 1} box is one matrix's codes of a chunk,
// landing as the 16 KB padded, swizzled A operand of kind::mxf8f6f4.
static moe_status_t make_weight_tmaps(moe_mxfp4* h) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return MOE_ERR_CUDA;
    for (int which = 0; which < 2; ++which) {
        const TiledMatrix M = tiled(h, which == 0 ? 0 : 2);
        const cuuint64_t parts = static_cast<cuuint64_t>(h->cfg.n_experts) * M.expert_bytes() / TiledMatrix::PAD_MAT;
        cuuint64_t dims[3] = {128, 128, parts};
        cuuint64_t strides[2] = {64, TiledMatrix::PAD_MAT};
        cuuint32_t box[3] = {128, 128, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(which == 0 ? &h->tm_wgu : &h->tm_wdn, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, M.base, dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

moe_status_t moe_mxfp4_forward(moe_mxfp4_t* h, const void* x, int32_t T, void* y, int32_t* topk_idx,
                               float* topk_w, int32_t* expert_counts, cudaStream_t stream) {
    if (!h) return MOE_ERR_INVALID_ARG;
    const auto& c = h->cfg;
    if (T < 0) return MOE_ERR_INVALID_ARG;
    if (T > c.max_tokens) return MOE_ERR_UNSUPPORTED;
    if (T > 0 && (!x || !y)) return MOE_ERR_INVALID_ARG;
    // the kernels read x and write y 16 bytes at a time and the routing outputs 4
    if (!aligned_to(x, 16) || !aligned_to(y, 16) || !aligned_to(topk_idx, 4) || !aligned_to(topk_w, 4) ||
        !aligned_to(expert_counts, 4))
        return MOE_ERR_INVALID_ARG;
    if (!h->router_set || h->experts_quantized < c.n_experts) return MOE_ERR_NOT_QUANTIZED;
    if (moe_status_t ds = check_device(h)) return ds;
    h->last_stream = stream;
    if (T == 0) return MOE_OK;
    const int E = c.n_experts, d = c.d_model, f = c.d_ff, k = c.top_k;
    const int BN = choose_bn(T, k, E, c.flags);
    moe_status_t st = ensure_tmaps(h, BN);
    if (st != MOE_OK) return st;
    const int nblk = (T + ROUTER_TOKENS - 1) / ROUTER_TOKENS;
    int32_t* idx = topk_idx ? topk_idx : h->idx_ws;
    float* wts = topk_w ? topk_w : h->w_ws;
    const bool bf16 = c.act_dtype == MOE_DTYPE_BF16;
    float* acc = h->yacc;
    const bool prof = h->prof;
    for (int i = 0; i < MOE_NUM_STAGES; ++i) h->stage_ran[i] = false;
    // While the stream is being captured into a CUDA graph, the stage events
    // become event-record nodes of the graph (recorded at every replay).
    unsigned ev_flags = cudaEventRecordDefault;
    if (prof) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
            ev_flags = cudaEventRecordExternal;
    }
    auto mark = [&](int i) {
        if (prof) cudaEventRecordWithFlags(h->ev[i], stream, ev_flags);
    };

    const uint64_t tmo = static_cast<uint64_t>(c.wait_timeout_ms > 0 ? c.wait_timeout_ms : 2000) * 1000000ull;
    // at most DF_MAX_T tokens: the whole layer in one cooperative launch
    if (h->df_ok && T <= DF_MAX_T && !(c.flags & (MOE_FLAG_UNFUSED_DECODE | MOE_FLAG_TOKEN_TILE_MASK))) {
        DecodeParams dp{};
        dp.x = x;
        dp.y = y;
        dp.wr = h->w_router;
        dp.bias = h->has_bias ? h->bias : nullptr;
        dp.gamma = h->use_norm ? h->gamma : nullptr;
        dp.eps = h->eps;
        dp.residual = h->residual ? 1 : 0;
        dp.T = T;
        dp.d = d;
        dp.f = f;
        dp.E = E;
        dp.k = k;
        dp.Mgu = tiled(h, 0);
        dp.Mdn = tiled(h, 2);
        dp.S = h->df_S;
        dp.stages = h->df_stages;
        dp.nb_max = h->df_nb_max;
        dp.kc_max = h->df_kc_max;
        dp.st = h->df_state;
        dp.part = h->df_part;
        dp.part_ss = h->df_part_ss;
        dp.yacc = h->df_yacc;
        dp.xq = h->df_xq;
        dp.hq = h->df_hq;
        dp.hq_stride = h->df_hq_stride;
        dp.hdone = h->df_hdone;
        dp.topk_idx = topk_idx;
        dp.topk_w = topk_w;
        dp.counts = expert_counts;
        dp.status = h->status;
        dp.timeout_ns = tmo;
        dp.skip_first_copy = (c.flags & MOE_FLAG_TEST_SKIP_FIRST_COPY) ? 1u : 0u;
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(h->nsm);
        lc.blockDim = dim3(DF_THREADS);
        lc.dynamicSmemBytes = h->df_smem;
        lc.stream = stream;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the grid barrier and counters rely on it
        at[0].val.cooperative = 1;
        lc.attrs = at;
        lc.numAttrs = 1;
        mark(6);
        if (bf16)
            cudaLaunchKernelEx(&lc, decode_fused_kernel<__nv_bfloat16>, dp);
        else
            cudaLaunchKernelEx(&lc, decode_fused_kernel<float>, dp);
        mark(7);
        h->stage_ran[6] = true;
        h->last_fused = true;
        h->prof_valid = prof;
        h->launches += 1;
        return cuda_status(cudaGetLastError());
    }
    h->last_fused = false;

    // 0: router + top-k + softmax + schedule
    mark(0);
    RouterArgs ra{};
    ra.x = x;
    ra.wr = h->w_router;
    ra.bias = h->has_bias ? h->bias : nullptr;
    ra.T = T;
    ra.d = d;
    ra.E = E;
    ra.k = k;
    ra.S = router_splits(T, d, E, h->nsm);
    ra.part = h->part;
    ra.gamma = h->use_norm ? h->gamma : nullptr;
    ra.eps = h->eps;
    ra.part_ss = h->part_ss;
    ra.inv_rms = h->inv_rms;
    ra.tile_cnt = h->counters;
    ra.glob_cnt = h->counters + h->nblk_max;
    ra.idx_out = idx;
    ra.w_out = wts;
    ra.local_rank = h->local_rank;
    ra.hist = h->hist;
    ra.BN = BN;
    ra.F_gu = h->F_gu;
    ra.F_dn = h->F_dn;
    ra.KC_gu = h->KC_gu;
    ra.KC_dn = h->KC_dn;
    ra.nsm = h->nsm;
    ra.split_rows_cap = h->gu_rows;
    ra.max_units = h->max_units;
    ra.offsets = h->offsets;
    ra.tile_base = h->tile_base;
    ra.counts_out = expert_counts;
    ra.units_gu = h->units_gu;
    ra.units_dn = h->units_dn;
    ra.sched = h->sched;
    if (bf16) {
        // tensor-core scores: x's map is made per call (its pointer and T change)
        EncodeTiledFn enc = get_encode_fn();
        if (!enc) return MOE_ERR_CUDA;
        CUtensorMap tm_x;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
        cuuint32_t box[2] = {static_cast<cuuint32_t>(ROUTER_KCHUNK), static_cast<cuuint32_t>(ROUTER_TOKENS)};
        cuuint32_t estr[2] = {1, 1};
        if (enc(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
        const int Z = router_etiles(E), P = h->router_P;
        const dim3 tgrid(static_cast<unsigned>(nblk * ra.S * Z));
        const size_t tsm = rtc_smem_bytes(P);
        router_tc_kernel<<<tgrid, RTC_THREADS, tsm, stream>>>(tm_x, h->tm_wr, ra, Z, P, h->status, tmo);
    } else {
        launch_router<float>(ra, dim3(nblk, ra.S, router_etiles(E)), router_smem_bytes(), stream);
    }
    h->stage_ran[0] = true;
    // 1: gather into grouped rows
    mark(1);
    const bool pdl = static_cast<long>(T) * k <= h->gu_rows;
    const int af = h->af;
    const bool stacked = mxg_stacked(BN, af);
    GroupedOperand Xop{h->Xq, h->sfx, h->TK, h->KC_gu, stacked ? BN : 128};
    GroupedOperand Hop{h->Hq, h->sfh, h->TK, h->KC_dn, stacked ? BN : 128};
    const float* gam = h->use_norm ? h->gamma : nullptr;
    const dim3 rgrid_rows((T + ROWS_TOKENS - 1) / ROWS_TOKENS);
    const int tiles_cap = static_cast<int>(max_tile_atoms(h->TK, E) / MXQ_TERMS);   // token tiles the atoms hold
    // token tiles: at most ceil(T k / BN) plus one ragged tile per expert
    const dim3 egrid(static_cast<unsigned>((static_cast<long>(T) * k + BN - 1) / BN + E), h->KC_gu);
    if (bf16) {
        launch_pdl(pdl, rows_kernel<__nv_bfloat16>, rgrid_rows, dim3(ROWS_THREADS), 0, stream,
                   static_cast<const __nv_bfloat16*>(x), static_cast<const int32_t*>(idx),
                   static_cast<const float*>(wts), static_cast<const int32_t*>(h->local_rank),
                   static_cast<const int32_t*>(h->hist), static_cast<const int32_t*>(h->offsets),
                   static_cast<const int32_t*>(h->tile_base), T, d, E, k, BN, h->row_token, h->row_weight,
                   h->row_slot, h->GU, 2 * f, acc, static_cast<const int32_t*>(h->sched), h->residual ? 1 : 0,
                   tiles_cap, h->status, h->pair_row, h->F_gu, h->F_dn,
                   h->units_gu, h->units_dn);
        launch_pdl(pdl, af ? encode_rows_kernel<__nv_bfloat16, 1> : encode_rows_kernel<__nv_bfloat16, 0>, egrid, dim3(ENC_THREADS), 0, stream,
                   static_cast<const __nv_bfloat16*>(x), gam, static_cast<const float*>(h->inv_rms),
                   static_cast<const int32_t*>(h->row_token), static_cast<const int4*>(h->units_gu),
                   static_cast<const int32_t*>(h->sched), h->F_gu, d, Xop, T, h->status);
    } else {
        launch_pdl(pdl, rows_kernel<float>, rgrid_rows, dim3(ROWS_THREADS), 0, stream, static_cast<const float*>(x),
                   static_cast<const int32_t*>(idx), static_cast<const float*>(wts),
                   static_cast<const int32_t*>(h->local_rank), static_cast<const int32_t*>(h->hist),
                   static_cast<const int32_t*>(h->offsets), static_cast<const int32_t*>(h->tile_base), T, d, E, k,
                   BN, h->row_token, h->row_weight, h->row_slot, h->GU, 2 * f, acc,
                   static_cast<const int32_t*>(h->sched), h->residual ? 1 : 0, tiles_cap, h->status, h->pair_row, h->F_gu, h->F_dn,
                   h->units_gu, h->units_dn);
        launch_pdl(pdl, af ? encode_rows_kernel<float, 1> : encode_rows_kernel<float, 0>, egrid, dim3(ENC_THREADS), 0, stream, static_cast<const float*>(x),
                   gam, static_cast<const float*>(h->inv_rms), static_cast<const int32_t*>(h->row_token),
                   static_cast<const int4*>(h->units_gu), static_cast<const int32_t*>(h->sched), h->F_gu, d, Xop, T,
                   h->status);
    }
    h->launches += 1;   // stage 1 is two launches
    h->stage_ran[1] = true;
    // 2: gate/up GEMM + SwiGLU
    mark(2);
    MxgParams gp{};
    gp.wpack = h->w_gu;
    gp.units = h->units_gu;
    gp.sched = h->sched;
    gp.M = tiled(h, 0);
    gp.N = f;
    gp.K = d;
    gp.BN = BN;
    gp.stages = stages_for(0, BN, af);
    gp.nacc = mxg_nacc(0, BN, af);
    gp.sfb = h->sfx;
    gp.stacked = stacked ? 1 : 0;
    gp.idesc = af ? idesc_mxf8f6f4_e2m1_e4m3(128, (stacked ? MX8_TERMS : 1) * BN)
                  : idesc_mxf4(128, (stacked ? MXQ_TERMS : 1) * BN);
    gp.Hd = Hop;
    gp.GU = h->GU;
    gp.yacc = nullptr;
    gp.row_token = h->row_token;
    gp.row_weight = h->row_weight;
    gp.status = h->status;
    gp.timeout_ns = tmo;
    gp.skip_first_copy = (c.flags & MOE_FLAG_TEST_SKIP_FIRST_COPY) ? 1u : 0u;
    gp.n_experts = E;
    gp.T = T;
    gp.tiles_cap = tiles_cap;
    const int grid = h->nsm;
    // The schedule splits a GEMM's K only while its units (at least ceil(rows /
    // BN) token tiles x its feature tiles) leave SMs idle, and the gate/up K
    // only for at most gu_rows grouped rows: past those bounds the kernel
    // without the split-K epilogue runs.
    const long rows_all = static_cast<long>(T) * k;
    const bool gu_nosplit = rows_all > h->gu_rows || ((rows_all + BN - 1) / BN) * h->F_gu >= h->nsm;
    const bool dn_nosplit = ((rows_all + BN - 1) / BN) * h->F_dn >= h->nsm;
    auto gu_kernel =
        af ? (stacked ? (gu_nosplit ? expert_mxf4_kernel<0, 1, 1, 0, 0> : expert_mxf4_kernel<0, 1, 1>)
                      : (gu_nosplit ? expert_mxf4_kernel<0, 1, 0, 0, 0> : expert_mxf4_kernel<0, 1, 0>))
           : (stacked ? (gu_nosplit ? expert_mxf4_kernel<0, 0, 1, 0, 0> : expert_mxf4_kernel<0, 0, 1>)
                      : (gu_nosplit ? expert_mxf4_kernel<0, 0, 0, 0, 0> : expert_mxf4_kernel<0, 0, 0>));
    launch_pdl(pdl, gu_kernel, dim3(grid), dim3(MXG_THREADS),
               mxg_smem_bytes(0, BN, gp.stages, af), stream, h->tm_x[BN / 16 - 1], h->tm_wgu, gp);
    h->stage_ran[2] = true;
    // 3: split-K finish (a no-op unless the schedule split K): SwiGLU + H encoding.
    // The schedule splits the gate/up K only for at most gu_rows grouped rows,
    // fewer units than SMs and a split limit above 1; the units are at least
    // ceil(rows / BN) token tiles x F_gu feature tiles, so the launch is left
    // out whenever that bound already rules a split out.
    mark(3);
    const long grows = static_cast<long>(T) * k;
    const bool may_split = grows <= h->gu_rows && ((grows + BN - 1) / BN) * h->F_gu < h->nsm &&
                           std::min(8, std::max(1, h->KC_gu / 4)) > 1;
    if (may_split) {
        const long items = static_cast<long>(T) * k * (f / 32);
        const int blocks = static_cast<int>((items + HENC_THREADS - 1) / HENC_THREADS);
        launch_pdl(pdl, af ? h_encode_kernel<1> : h_encode_kernel<0>, dim3(blocks), dim3(HENC_THREADS), 0, stream, static_cast<const float*>(h->GU),
                   Hop, f, BN, static_cast<const int32_t*>(h->row_slot), static_cast<const int32_t*>(h->sched), tiles_cap,
                   h->status);
        h->stage_ran[3] = true;
    }
    // 4: down GEMM + weighted scatter-combine
    mark(4);
    MxgParams dp = gp;
    dp.wpack = h->w_dn;
    dp.units = h->units_dn;
    dp.M = tiled(h, 2);
    dp.N = d;
    dp.K = f;
    // small stacked tiles: two K chunks (17,408 weight bytes) per down stage, as
    // many bytes per stage round trip as a gate/up stage
    const bool cp2 = af == 0 && stacked && MXQ_TERMS * BN <= 128;
    dp.stages = stages_for(1, BN, af, cp2 ? 2 : 1);
    dp.nacc = mxg_nacc(1, BN, af);
    dp.sfb = h->sfh;
    dp.GU = nullptr;
    dp.yacc = acc;
    dp.obuf = h->obuf;
    dp.obuf_bf16 = bf16 ? 1 : 0;
    dp.skip_first_copy = 0;
    auto dn_kernel =
        af ? (stacked ? (dn_nosplit ? expert_mxf4_kernel<1, 1, 1, 0, 0> : expert_mxf4_kernel<1, 1, 1>)
                      : (dn_nosplit ? expert_mxf4_kernel<1, 1, 0, 0, 0> : expert_mxf4_kernel<1, 1, 0>))
           : (cp2 ? (dn_nosplit ? expert_mxf4_kernel<1, 0, 1, 1, 0> : expert_mxf4_kernel<1, 0, 1, 1>)
                  : (stacked ? (dn_nosplit ? expert_mxf4_kernel<1, 0, 1, 0, 0> : expert_mxf4_kernel<1, 0, 1>)
                             : (dn_nosplit ? expert_mxf4_kernel<1, 0, 0, 0, 0> : expert_mxf4_kernel<1, 0, 0>)));
    launch_pdl(pdl, dn_kernel,
               dim3(grid), dim3(MXG_THREADS), mxg_smem_bytes(1, BN, dp.stages, af, cp2 ? 2 : 1), stream,
               h->tm_h[BN / 16 - 1], h->tm_wdn, dp);
    h->stage_ran[4] = true;
    // 5: the output: the sum of each token's k rows (+ x), or the cast accumulator
    mark(5);
    {
        const size_t n8 = static_cast<size_t>(T) * d / 8;
        const int blocks = static_cast<int>(
            std::min<size_t>(4 * static_cast<size_t>(h->nsm), (n8 + COMBINE_THREADS - 1) / COMBINE_THREADS));
        if (bf16)
            launch_pdl(pdl, combine_out_kernel<__nv_bfloat16>, dim3(std::max(1, blocks)), dim3(COMBINE_THREADS), 0,
                       stream, static_cast<const __nv_bfloat16*>(h->obuf), static_cast<const int32_t*>(h->pair_row),
                       static_cast<const float*>(h->yacc), static_cast<const __nv_bfloat16*>(x),
                       static_cast<__nv_bfloat16*>(y), T, d, k, h->residual ? 1 : 0,
                       static_cast<const int32_t*>(h->sched));
        else
            launch_pdl(pdl, combine_out_kernel<float>, dim3(std::max(1, blocks)), dim3(COMBINE_THREADS), 0, stream,
                       static_cast<const float*>(h->obuf), static_cast<const int32_t*>(h->pair_row),
                       static_cast<const float*>(h->yacc), static_cast<const float*>(x), static_cast<float*>(y), T, d,
                       k, h->residual ? 1 : 0, static_cast<const int32_t*>(h->sched));
        h->stage_ran[5] = true;
    }
    mark(6);
    mark(7);   // the record's end event (stage 6, the fused path, did not run)
    h->prof_valid = prof;
    for (int i = 0; i < MOE_NUM_STAGES; ++i) h->launches += h->stage_ran[i] ? 1 : 0;
    return cuda_status(cudaGetLastError());
}

moe_status_t moe_mxfp4_forward_host(moe_mxfp4_t* h, const void* x_host, int32_t T, void* y_host,
                                    int32_t* topk_idx_host, float* topk_w_host, cudaStream_t stream) {
    if (!h) return MOE_ERR_INVALID_ARG;
    const auto& c = h->cfg;
    if (T < 0) return MOE_ERR_INVALID_ARG;
    if (T > c.max_tokens) return MOE_ERR_UNSUPPORTED;
    if (T > 0 && (!x_host || !y_host)) return MOE_ERR_INVALID_ARG;
    if (moe_status_t ds = check_device(h)) return ds;
    if (T == 0) return MOE_OK;
    const size_t row_bytes = static_cast<size_t>(c.d_model) * h->act_bytes;
    // Large batches run as up to 8 chunks of at least FH_MIN_CHUNK tokens: the
    // copy of chunk i+1 in and of chunk i-1 out overlap the forward of chunk i
    // (the rows of a forward are independent, so chunking changes nothing in
    // the result beyond fp32 summation order).  The forwards themselves run in
    // order on `stream`; the copies on the handle's two copy streams.
    constexpr int FH_MIN_CHUNK = 4096;
    const int nch = std::max(1, std::min(8, T / FH_MIN_CHUNK));
    const int chunk = (T + nch - 1) / nch;
    auto* xs = static_cast<uint8_t*>(h->x_stage);
    auto* ys = static_cast<uint8_t*>(h->y_stage);
    const uint8_t* xh = static_cast<const uint8_t*>(x_host);
    uint8_t* yh = static_cast<uint8_t*>(y_host);
    const int k = c.top_k;
    // the copy streams start after the work already queued on `stream`
    MOE_TRY(cudaEventRecord(h->ev_start, stream));
    MOE_TRY(cudaStreamWaitEvent(h->s_in, h->ev_start, 0));
    MOE_TRY(cudaStreamWaitEvent(h->s_out, h->ev_start, 0));
    for (int i = 0; i < nch; ++i) {
        const int t0 = i * chunk, n = std::min(chunk, T - t0);
        if (n <= 0) break;
        const size_t off = static_cast<size_t>(t0) * row_bytes, bytes = static_cast<size_t>(n) * row_bytes;
        MOE_TRY(cudaMemcpyAsync(xs + off, xh + off, bytes, cudaMemcpyHostToDevice, h->s_in));
        MOE_TRY(cudaEventRecord(h->ev_in[i], h->s_in));
        MOE_TRY(cudaStreamWaitEvent(stream, h->ev_in[i], 0));
        moe_status_t st = moe_mxfp4_forward(h, xs + off, n, ys + off, h->idx_stage + static_cast<size_t>(t0) * k,
                                            h->w_stage + static_cast<size_t>(t0) * k, nullptr, stream);
        if (st != MOE_OK) {
            cudaStreamSynchronize(h->s_in);
            return st;
        }
        MOE_TRY(cudaEventRecord(h->ev_out[i], stream));
        MOE_TRY(cudaStreamWaitEvent(h->s_out, h->ev_out[i], 0));
        MOE_TRY(cudaMemcpyAsync(yh + off, ys + off, bytes, cudaMemcpyDeviceToHost, h->s_out));
        const size_t tk = static_cast<size_t>(n) * k, tk0 = static_cast<size_t>(t0) * k;
        if (topk_idx_host)
            MOE_TRY(cudaMemcpyAsync(topk_idx_host + tk0, h->idx_stage + tk0, tk * sizeof(int32_t),
                                    cudaMemcpyDeviceToHost, h->s_out));
        if (topk_w_host)
            MOE_TRY(cudaMemcpyAsync(topk_w_host + tk0, h->w_stage + tk0, tk * sizeof(float), cudaMemcpyDeviceToHost,
                                    h->s_out));
    }
    // `stream` ends after the last copy out
    MOE_TRY(cudaEventRecord(h->ev_done, h->s_out));
    MOE_TRY(cudaStreamWaitEvent(stream, h->ev_done, 0));
    MOE_TRY(cudaStreamSynchronize(stream));
    return MOE_OK;
}

moe_status_t moe_mxfp4_get_grouping(const moe_mxfp4_t* hc, int32_t* offsets, int32_t* row_token, float* row_weight,
                                    cudaStream_t stream) {
    if (!hc || !offsets) return MOE_ERR_INVALID_ARG;
    moe_mxfp4* h = const_cast<moe_mxfp4*>(hc);
    if (h->last_fused) return MOE_ERR_UNSUPPORTED;   // the fused decode path builds no grouping
    const auto& c = h->cfg;
    MOE_TRY(cudaMemcpyAsync(offsets, h->offsets, sizeof(int32_t) * (c.n_experts + 1), cudaMemcpyDeviceToDevice, stream));
    // rows in use = offsets[E]; copy the full capacity bound the caller sized for T*k
    int32_t rows = 0;
    MOE_TRY(cudaMemcpyAsync(&rows, h->sched + SCHED_ROWS, sizeof(int32_t), cudaMemcpyDeviceToHost, stream));
    MOE_TRY(cudaStreamSynchronize(stream));
    if (row_token && rows > 0)
        MOE_TRY(cudaMemcpyAsync(row_token, h->row_token, sizeof(int32_t) * rows, cudaMemcpyDeviceToDevice, stream));
    if (row_weight && rows > 0)
        MOE_TRY(cudaMemcpyAsync(row_weight, h->row_weight, sizeof(float) * rows, cudaMemcpyDeviceToDevice, stream));
    return MOE_OK;
}

moe_status_t moe_mxfp4_get_status(moe_mxfp4_t* h) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (h->last_stream) {
        MOE_TRY(cudaStreamSynchronize(h->last_stream));
    } else {
        MOE_TRY(cudaDeviceSynchronize());
    }
    int s = 0;
    MOE_TRY(cudaMemcpy(&s, h->status, sizeof(int), cudaMemcpyDeviceToHost));
    MOE_TRY(cudaMemset(h->status, 0, sizeof(int)));
    return (s & DEV_BOUNDS) ? MOE_ERR_BOUNDS : (s & DEV_TIMEOUT) ? MOE_ERR_TIMEOUT : MOE_OK;
}

moe_status_t moe_mxfp4_check_guards(moe_mxfp4_t* h) {
    if (!h) return MOE_ERR_INVALID_ARG;
#ifndef MOE_DEBUG_CHECKS
    return MOE_ERR_UNSUPPORTED;
#else
    MOE_TRY(cudaDeviceSynchronize());
    unsigned char buf[MOE_GUARD_BYTES];
    for (int i = 0; i < h->n_guards; ++i) {
        MOE_TRY(cudaMemcpy(buf, h->guard_ptr[i], MOE_GUARD_BYTES, cudaMemcpyDeviceToHost));
        for (size_t j = 0; j < MOE_GUARD_BYTES; ++j)
            if (buf[j] != MOE_GUARD_BYTE) return MOE_ERR_BOUNDS;
    }
    return MOE_OK;
#endif
}

moe_status_t moe_mxfp4_test_write_guard(moe_mxfp4_t* h, int32_t i) {
    if (!h || i < 0) return MOE_ERR_INVALID_ARG;
#ifndef MOE_DEBUG_CHECKS
    return MOE_ERR_UNSUPPORTED;
#else
    if (i >= h->n_guards) return MOE_ERR_INVALID_ARG;
    MOE_TRY(cudaDeviceSynchronize());
    MOE_TRY(cudaMemset(h->guard_ptr[i] + MOE_GUARD_BYTES / 2, 0, 1));
    return MOE_OK;
#endif
}

moe_status_t moe_mxfp4_set_profiling(moe_mxfp4_t* h, int32_t enable) {
    if (!h) return MOE_ERR_INVALID_ARG;
    h->prof = enable != 0;
    // turning profiling on starts a new record; turning it off keeps the last
    // one readable (e.g. the stage events of a graph captured while it was on)
    if (h->prof) h->prof_valid = false;
    return MOE_OK;
}

moe_status_t moe_mxfp4_kernel_times(moe_mxfp4_t* h, float* ms, int32_t n) {
    if (!h || !ms || n < 0) return MOE_ERR_INVALID_ARG;
    if (!h->prof_valid) return MOE_ERR_INVALID_ARG;
    MOE_TRY(cudaEventSynchronize(h->ev[MOE_NUM_STAGES]));
    for (int i = 0; i < std::min<int>(n, MOE_NUM_STAGES); ++i) {
        float t = 0.f;
        if (h->stage_ran[i]) MOE_TRY(cudaEventElapsedTime(&t, h->ev[i], h->ev[i + 1]));
        ms[i] = t;
    }
    return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Routing with no device allocation (moe_mxfp4_route_noalloc).
//
// The router kernel's scratch -- partial scores, tile and global arrival
// counters, per-tile histograms and ranks, offsets and schedule slots -- lives
// in one file-scope static device array.  Host code must not pass the array's
// name to a kernel (on the host it is only a stand-in symbol); the device
// address comes from cudaGetSymbolAddress, looked up once per device.
namespace {

constexpr int NOALLOC_MAX_SPLITS = 8;
constexpr size_t NOALLOC_PART_BYTES = sizeof(double) * NOALLOC_MAX_SPLITS * MOE_ROUTE_NOALLOC_MAX_TOKENS *
                                      MOE_ROUTE_NOALLOC_MAX_EXPERTS;
constexpr int NOALLOC_MAX_TILES = (MOE_ROUTE_NOALLOC_MAX_TOKENS + ROUTER_TOKENS - 1) / ROUTER_TOKENS;
// byte offsets inside the array (each 256-byte aligned)
constexpr size_t NA_OFF_PART = 0;
constexpr size_t NA_OFF_HIST = NA_OFF_PART + NOALLOC_PART_BYTES;
constexpr size_t NA_OFF_RANK = NA_OFF_HIST + 4096 * 4;
constexpr size_t NA_OFF_CNT = NA_OFF_RANK + sizeof(int32_t) * MOE_ROUTE_NOALLOC_MAX_TOKENS * MAX_TOPK;
constexpr size_t NA_OFF_OFFS = NA_OFF_CNT + 256;
constexpr size_t NA_OFF_SCHED = NA_OFF_OFFS + 4096;
constexpr size_t NA_END = NA_OFF_SCHED + 256;
static_assert(NOALLOC_MAX_TILES * MOE_ROUTE_NOALLOC_MAX_EXPERTS * 4 <= 4096 * 4, "histogram region too small");
static_assert(NOALLOC_MAX_TILES + 1 <= 64, "counter region too small");
static_assert(NA_END <= MOE_ROUTE_NOALLOC_SCRATCH_BYTES, "scratch array too small");

__device__ __align__(256) unsigned char g_route_scratch[MOE_ROUTE_NOALLOC_SCRATCH_BYTES];

struct NoallocDevice {
    bool ready = false;
    unsigned char* scratch = nullptr;  // device address of g_route_scratch on this device
    int nsm = 0;
};
constexpr int NOALLOC_MAX_DEVICES = MOE_MAX_DEVICES;
NoallocDevice g_noalloc[NOALLOC_MAX_DEVICES];
std::mutex g_noalloc_mutex;

moe_status_t noalloc_setup(int dev, NoallocDevice** out) {
    if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoallocDevice& nd = g_noalloc[dev];
    if (!nd.ready) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
        int nsm = 0;
        if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
        // the same per-device attributes as a layer's (never a lower router limit)
        if (ensure_kernel_attrs(dev) != cudaSuccess) return MOE_ERR_CUDA;
        nd.scratch = static_cast<unsigned char*>(ptr);
        nd.nsm = nsm;
        nd.ready = true;
    }
    *out = &nd;
    return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_mxfp4_route_noalloc(const void* x, const void* w_router, const float* router_bias,
                                                int32_t T, int32_t d_model, int32_t n_experts, int32_t top_k,
                                                int32_t act_dtype, int32_t* topk_idx, float* topk_w,
                                                int32_t* expert_counts, cudaStream_t stream) {
    if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (T <= 0 || d_model <= 0 || n_experts <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
    if (act_dtype != MOE_DTYPE_F32 && act_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (T > MOE_ROUTE_NOALLOC_MAX_TOKENS || n_experts > MOE_ROUTE_NOALLOC_MAX_EXPERTS ||
        top_k > std::min(MAX_TOPK, static_cast<int>(n_experts)) || d_model % 32 || d_model > 16384)
        return MOE_ERR_UNSUPPORTED;
    // the router reads x and w_router 16 bytes at a time
    if (!aligned_to(x, 16) || !aligned_to(w_router, 16) || !aligned_to(router_bias, 4) || !aligned_to(topk_idx, 4) ||
        !aligned_to(topk_w, 4) || !aligned_to(expert_counts, 4))
        return MOE_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    NoallocDevice* nd = nullptr;
    moe_status_t st = noalloc_setup(dev, &nd);
    if (st != MOE_OK) return st;
    unsigned char* sc = nd->scratch;
    const int tiles = (T + ROUTER_TOKENS - 1) / ROUTER_TOKENS;
    int* counters = reinterpret_cast<int*>(sc + NA_OFF_CNT);
    // the arrival counters must start at zero (a previous call may have been cut short)
    if (cudaMemsetAsync(counters, 0, sizeof(int) * (tiles + 1), stream) != cudaSuccess) return MOE_ERR_CUDA;
    RouterArgs ra{};
    ra.x = x;
    ra.wr = w_router;
    ra.bias = router_bias;
    ra.T = T;
    ra.d = d_model;
    ra.E = n_experts;
    ra.k = top_k;
    ra.S = std::min(NOALLOC_MAX_SPLITS, router_splits(T, d_model, n_experts, nd->nsm));
    ra.part = reinterpret_cast<double*>(sc + NA_OFF_PART);
    ra.tile_cnt = counters;
    ra.glob_cnt = counters + tiles;
    ra.idx_out = topk_idx;
    ra.w_out = topk_w;
    ra.local_rank = reinterpret_cast<int32_t*>(sc + NA_OFF_RANK);
    ra.hist = reinterpret_cast<int32_t*>(sc + NA_OFF_HIST);
    // no expert GEMMs follow: zero feature tiles, so the schedule step only
    // totals the histogram (expert_counts) and emits no units
    ra.BN = 16;
    ra.F_gu = 0;
    ra.F_dn = 0;
    ra.KC_gu = 1;
    ra.KC_dn = 1;
    ra.nsm = nd->nsm;
    ra.split_rows_cap = 0;
    ra.max_units = 0;
    ra.offsets = reinterpret_cast<int32_t*>(sc + NA_OFF_OFFS);
    ra.tile_base = nullptr;
    ra.counts_out = expert_counts;
    ra.units_gu = nullptr;
    ra.units_dn = nullptr;
    ra.sched = reinterpret_cast<int32_t*>(sc + NA_OFF_SCHED);
    const dim3 grid(tiles, ra.S, router_etiles(n_experts));
    const size_t smem = router_smem_bytes();
    if (act_dtype == MOE_DTYPE_BF16)
        launch_router<__nv_bfloat16>(ra, grid, smem, stream);
    else
        launch_router<float>(ra, grid, smem, stream);
    return cuda_status(cudaGetLastError());
}
