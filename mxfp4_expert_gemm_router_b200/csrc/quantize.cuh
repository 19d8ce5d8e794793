// quantize.cuh -- MXFP4 quantisation of expert weights into the layout the
// expert GEMMs stream, plus the export back to the canonical layout.
//
// Format (page "GPT-OSS-20B : Architecture MoE & Résumé du Model Card", §4
// Quantification MXFP4: 4.25 bits per parameter; the Microscaling format cited
// there): blocks of 32 weights along the contraction axis share one E8M0
// scale 2^(s-127); each weight is an E2M1 code (sign, 2 exponent bits, 1
// mantissa bit).  Block rule: exponent floor(log2(max|w|)) - 2 clamped to
// [-127, 127]; elements round to the nearest E2M1 magnitude with ties to the
// even code, magnitudes above 6 saturate, the sign bit is kept; an all-zero
// block gets scale byte 127.
//
// Streamed layout ("tiled"), the A operand of the block-scaled MMA: rows
// (output features) are cut into 128-row feature tiles (the last one holds the
// remainder rf) and each row's nb = K/32 blocks into chunks of 4 blocks (K =
// 128; the last chunk may hold fewer, nbc).  For each (tile, chunk) the NM
// interleaved matrices (gate and up, or down alone) follow one another, each as
//     codes  [nbc blocks][rf rows][16 B]   (even element in the low nibble)
//     scales one 512-byte atom: row r, block h at 16*(r%32) + 4*(r/32) + h
// so that one bulk copy brings a chunk into shared memory where the codes are
// a K-major, unswizzled canonical operand (8-row core matrices of 128 B) and
// the atom is what tcgen05.cp moves into tensor memory.  Codes take exactly
// 4 bits per parameter; the scale atoms add 8 bits per 32 parameters, plus
// padding where a tile has fewer than 128 rows or a chunk fewer than 4 blocks
// (0.26 % for the 2880 x 2880 experts).  Padding bytes stay zero (a finite
// scale, 2^-127).
//
// Padded form (the layers whose activations are two MXFP8 terms, read by the
// kind::mxf8f6f4 MMA): every tile has 128 rows and every chunk 4 blocks (zero
// padding), and a matrix's part of a chunk is codes [128 rows][64 B] (row-major:
// the row's 128 elements of the chunk) + the same scale atom, 8704 bytes.
// All parts have one size, so the array is a 3-D tensor {128 elements, 128
// rows, parts} that a tensor map of the 16U4_ALIGN16B type reads, writing
// each group of 16 codes into the low half of 16 bytes of shared memory: the
// layout that MMA kind wants for E2M1.  Padding costs 2.2 % rows and 2.2 %
// blocks for the 2880 x 2880 experts.
#pragma once
#include <cstdint>

namespace moe {

struct TiledMatrix {
    uint8_t* base;   // expert 0 of the packed array
    int N, K;        // rows, contraction length (K % 32 == 0)
    int NM;          // matrices interleaved per chunk (2: gate+up, 1: down)
    int sub;         // which matrix of the chunk this one is (0 or 1)
    int padded;      // 1: the row-major, padded form (below), 0: the compact form
    static constexpr int BPC = 4;   // 32-blocks per chunk
    static constexpr size_t PAD_MAT = 128 * 64 + 512;   // padded form: one matrix's part of a chunk
    __host__ __device__ int nb() const { return K / 32; }
    __host__ __device__ int chunks() const { return (nb() + BPC - 1) / BPC; }
    __host__ __device__ int tiles() const { return (N + 127) / 128; }
    __host__ __device__ int blocks_in_chunk(int c) const { return min(BPC, nb() - c * BPC); }
    // bytes of one matrix's part of a chunk: codes + one scale atom
    __host__ __device__ size_t mat_bytes(int c, int rf) const {
        return padded ? PAD_MAT : static_cast<size_t>(blocks_in_chunk(c)) * rf * 16 + 512;
    }
    __host__ __device__ size_t chunk_bytes(int c, int rf) const { return NM * mat_bytes(c, rf); }
    __host__ __device__ size_t tile_offset(int ft) const {
        if (padded) return static_cast<size_t>(ft) * chunks() * NM * PAD_MAT;
        return static_cast<size_t>(ft) * NM * (static_cast<size_t>(128) * 16 * nb() + 512 * static_cast<size_t>(chunks()));
    }
    // byte offset, within one expert, of feature tile ft's chunk c (all NM matrices)
    __host__ __device__ size_t chunk_offset(int ft, int c, int rf) const {
        if (padded) return tile_offset(ft) + static_cast<size_t>(c) * NM * PAD_MAT;
        return tile_offset(ft) + static_cast<size_t>(c) * NM * (static_cast<size_t>(BPC) * rf * 16 + 512);
    }
    __host__ __device__ size_t expert_bytes() const {
        if (padded) return static_cast<size_t>(tiles()) * chunks() * NM * PAD_MAT;
        return static_cast<size_t>(NM) *
               (static_cast<size_t>(N) * 16 * nb() + 512 * static_cast<size_t>(chunks()) * tiles());
    }
    // byte offsets (within one expert) of block b of row n of this matrix
    __host__ __device__ void locate(int n, int b, size_t& code_off, size_t& scale_off) const {
        const int ft = n >> 7, r = n & 127;
        const int rf = min(128, N - (ft << 7));
        const int c = b / BPC, h = b % BPC;
        const int nbc = blocks_in_chunk(c);
        const size_t base_m = chunk_offset(ft, c, rf) + static_cast<size_t>(sub) * mat_bytes(c, rf);
        const size_t sf = 16 * (r & 31) + 4 * (r >> 5) + h;
        if (padded) {
            code_off = base_m + static_cast<size_t>(r) * 64 + h * 16;
            scale_off = base_m + 128 * 64 + sf;
        } else {
            code_off = base_m + static_cast<size_t>(h * rf + r) * 16;
            scale_off = base_m + static_cast<size_t>(nbc) * rf * 16 + sf;
        }
    }
};

__device__ __forceinline__ int floor_log2_pos(float a) {
    const uint32_t u = __float_as_uint(a);
    const int ex = static_cast<int>((u >> 23) & 0xFF);
    if (ex != 0) return ex - 127;
    return (31 - __clz(static_cast<int>(u & 0x7FFFFF))) - 149;  // subnormal
}

// E2M1 magnitude code of a >= 0: nearest of {0,.5,1,1.5,2,3,4,6}; at a midpoint
// the even code wins; above 6 saturates.
__device__ __forceinline__ uint32_t e2m1_code_of(float a) {
    return a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
         : a <= 2.5f ? 4u : a < 3.5f ? 5u : a <= 5.0f ? 6u : 7u;
}

// One thread per (row n, block b) of expert blockIdx.z.  W is [K][N] fp32 per
// expert (y = x . W); consecutive threads take consecutive n so the reads of
// each of the 32 block elements are coalesced.
__global__ void quantize_kernel(const float* __restrict__ W, size_t w_expert_stride, TiledMatrix M) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = blockIdx.y;
    const int e = blockIdx.z;
    if (n >= M.N || b >= M.nb()) return;
    size_t co, so;
    M.locate(n, b, co, so);
    uint8_t* dst = M.base + static_cast<size_t>(e) * M.expert_bytes();
    const float* src = W + static_cast<size_t>(e) * w_expert_stride + static_cast<size_t>(b) * 32 * M.N + n;
    float v[32];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        v[i] = src[static_cast<size_t>(i) * M.N];
        amax = fmaxf(amax, fabsf(v[i]));
    }
    uint4 out = make_uint4(0, 0, 0, 0);
    uint32_t scale = 127;
    if (amax > 0.f) {
        int ex = floor_log2_pos(amax) - 2;
        ex = ex < -127 ? -127 : (ex > 127 ? 127 : ex);
        scale = static_cast<uint32_t>(ex + 127);
        const float inv = __int_as_float((127 - ex) << 23);  // 2^-ex, exact (ex in [-127, 125])
        uint32_t words[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            uint32_t c = e2m1_code_of(fabsf(v[i] * inv));
            if (__float_as_uint(v[i]) >> 31) c |= 8u;
            words[i >> 3] |= c << (4 * (i & 7));
        }
        out = make_uint4(words[0], words[1], words[2], words[3]);
    }
    *reinterpret_cast<uint4*>(dst + co) = out;
    dst[so] = static_cast<uint8_t>(scale);
}

// Tiled -> canonical: codes [E][N][K/2], scales [E][N][K/32].
__global__ void export_kernel(TiledMatrix M, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = blockIdx.y;
    const int e = blockIdx.z;
    const int nb = M.nb();
    if (n >= M.N || b >= nb) return;
    size_t co, so;
    M.locate(n, b, co, so);
    const uint8_t* src = M.base + static_cast<size_t>(e) * M.expert_bytes();
    const size_t row = static_cast<size_t>(e) * M.N + n;
    *reinterpret_cast<uint4*>(codes + row * (M.K / 2) + static_cast<size_t>(b) * 16) =
        *reinterpret_cast<const uint4*>(src + co);
    scales[row * nb + b] = src[so];
}

}  // namespace moe
