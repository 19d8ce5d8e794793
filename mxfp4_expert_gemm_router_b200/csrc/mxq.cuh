// mxq.cuh -- activations as sums of three MXFP4 terms, the operand format the
// block-scaled expert GEMMs read.
//
// The expert weights are MXFP4 (page "GPT-OSS-20B : Architecture MoE & Résumé
// du Model Card", §4 Quantification MXFP4: E2M1 values in blocks of 32 with
// one shared E8M0 scale).  The tensor cores' block-scaled MMA multiplies two
// MXFP4 operands, so the activations (x for gate/up, the SwiGLU output H for
// down) are encoded in the same format.  One MXFP4 term keeps about two
// significant bits, far too coarse for the layer's accuracy, so a block v of
// 32 values is written as v ~= q1 + q2 + q3: q1 encodes v, q2 encodes the
// residual v - q1, q3 the residual v - q1 - q2, each with its own scale.  The
// GEMM either issues one MMA per term into the same accumulator (the tensor
// core adds the three products) or, for small token tiles, stacks the terms
// as 3 * BN rows of one MMA and adds the three accumulator columns itself.  Measured on the oracle's weights (double
// precision emulation), the layer error of the 3-term encoding is about 0.25 %
// of max|y| (2 terms: about 3 %).
//
// Scale rule of a term: the smallest power of two 2^e with max|v| <= 6 * 2^e,
// so no element saturates; elements round to the nearest E2M1 value with ties
// to the even code (the hardware conversion).
//
// Operand layouts in global memory (R = row capacity, NB = K / 32 blocks):
//   codes   [NB][3 terms][R rows][16 B]   (element 2i of the block in the low nibble of byte i)
//   scales  per (token tile, K chunk of 128): three 512-byte atoms; row r of
//           the tile, term t, block q (0..3) of the chunk at byte
//           sf_atom_offset(t * R_t + r, q), R_t = 128 (terms as separate MMAs,
//           atom t) or BN (terms stacked, 3 * BN <= 128 rows in atom 0).
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "sm100_ptx.cuh"

namespace moe {

constexpr int MXQ_TERMS = 3;

// Byte of the scale of operand row n (n < 256) and block q (0..3) within the
// scale atoms of one K chunk: atom n / 128, then 16 * (n % 32) + 4 * ((n / 32) % 4) + q.
// tcgen05.cp 32x128b.warpx4 copies an atom into 4 tensor-memory columns of lanes
// 0..31 (replicated over the lane quarters); the MMA reads row n's scales at
// column n / 32, byte q (+ the sf id).
__host__ __device__ constexpr uint32_t sf_atom_offset(int n, int q) {
    return static_cast<uint32_t>((n >> 7) * 512 + 16 * (n & 31) + 4 * ((n >> 5) & 3) + q);
}

// Exponent e of the scale 2^e of a term whose largest magnitude has bits
// `amax_bits`: the smallest e with amax <= 6 * 2^e.  amax = m 2^E0 with m in
// [1, 2): e = E0 - 2 when m <= 1.5, else E0 - 1.  -127 for zero or subnormal
// amax (the E8M0 minimum).
__device__ __forceinline__ int mxq_exp(uint32_t amax_bits) {
    const int ex = static_cast<int>(amax_bits >> 23);
    if (ex == 0) return -127;
    const int e = ex - 129 + ((amax_bits & 0x7FFFFFu) > 0x400000u ? 1 : 0);
    return e < -127 ? -127 : e;
}
// 2^-e for e in [-127, 126] and 2^e for e in [-127, 127], exact.
__device__ __forceinline__ float mxq_inv(int e) { return __int_as_float((127 - e) << 23); }
__device__ __forceinline__ float mxq_scale(int e) {
    return e > -127 ? __int_as_float((127 + e) << 23) : __int_as_float(0x00400000);
}

// One thread encodes one block of 32 values (v is overwritten with the final
// residual).  codes[t] = the 16 code bytes of term t, sbyte[t] = its E8M0 byte.
__device__ __forceinline__ void mxq_block_thread(float (&v)[32], uint4 (&codes)[MXQ_TERMS],
                                                 uint32_t (&sbyte)[MXQ_TERMS]) {
#pragma unroll
    for (int t = 0; t < MXQ_TERMS; ++t) {
        float am = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(v[i]));
        const int e = mxq_exp(__float_as_uint(am));
        sbyte[t] = static_cast<uint32_t>(e + 127);
        const float inv = mxq_inv(e), sc = mxq_scale(e);
        uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t byte = e2m1x2_from_f32(v[2 * i] * inv, v[2 * i + 1] * inv);
            w[i >> 2] |= byte << (8 * (i & 3));
            if (t + 1 < MXQ_TERMS) {
                const uint32_t h2 = e2m1x2_to_f16x2(byte);
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
                v[2 * i] -= f.x * sc;
                v[2 * i + 1] -= f.y * sc;
            }
        }
        codes[t] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// One block of 32 values held one per lane (lane = element) encoded as three
// MXFP4 terms by the whole warp, with the same rule and rounding as
// mxq_block_thread.  Lanes 0..3 return word `lane` of each term's 16 code
// bytes in w[t]; every lane returns the E8M0 bytes in sbyte[t].
__device__ __forceinline__ void mxq_block_warp(float v, uint32_t (&w)[MXQ_TERMS], uint32_t (&sbyte)[MXQ_TERMS]) {
    const int lane = threadIdx.x & 31;
    const bool even = (lane & 1) == 0;
#pragma unroll
    for (int t = 0; t < MXQ_TERMS; ++t) {
        float am = fabsf(v);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        const int e = mxq_exp(__float_as_uint(am));
        sbyte[t] = static_cast<uint32_t>(e + 127);
        const float q = v * mxq_inv(e);
        const float qn = __shfl_xor_sync(0xffffffffu, q, 1);
        // both lanes of a pair form the byte of elements (2i, 2i+1)
        const uint32_t byte = even ? e2m1x2_from_f32(q, qn) : e2m1x2_from_f32(qn, q);
        if (t + 1 < MXQ_TERMS) {
            const uint32_t h2 = e2m1x2_to_f16x2(byte);
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
            v -= (even ? f.x : f.y) * mxq_scale(e);
        }
        // word m holds bytes 4m .. 4m+3, i.e. the bytes of lanes 8m, 8m+2, 8m+4, 8m+6
        const int m = lane & 3;
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) word |= (__shfl_sync(0xffffffffu, byte, 8 * m + 2 * j) & 0xFFu) << (8 * j);
        w[t] = word;
    }
}


// ---------------------------------------------------------------- 2 x MXFP8
// The alternative operand format: a block of 32 values as q1 + q2, two MXFP8
// terms (E4M3 elements: 4 exponent and 3 mantissa bits, largest finite 448;
// one E8M0 scale per term and block), read by the kind::mxf8f6f4 MMA against
// the same MXFP4 weights.  Scale rule of a term: the smallest power of two
// 2^e with max|v| <= 448 * 2^e (no element saturates); elements round to the
// nearest E4M3 value with ties to even (the hardware conversion).  Two terms
// keep about eight significant bits per element.
//
// Operand codes in global memory: [K/16 chunks][2 terms][R rows][16 B], chunk
// 2b + j holding elements 16j .. 16j+15 of block b (one byte per element);
// the scale atoms are laid out as for the three-term format (atom t per term,
// or rows t * BN + r when the terms are stacked).
constexpr int MX8_TERMS = 2;

// Exponent e of a term whose largest magnitude has bits `amax_bits`: amax =
// m 2^E0 with m in [1, 2); e = E0 - 8 when m <= 1.75, else E0 - 7.  -127 for
// zero or subnormal amax.
__device__ __forceinline__ int mx8_exp(uint32_t amax_bits) {
    const int ex = static_cast<int>(amax_bits >> 23);
    if (ex == 0) return -127;
    const int e = ex - 135 + ((amax_bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return e < -127 ? -127 : e;
}

// One thread encodes one block of 32 values (v is overwritten with the final
// residual).  codes[t][j] = the 16 code bytes of chunk j of term t.
__device__ __forceinline__ void mx8_block_thread(float (&v)[32], uint4 (&codes)[MX8_TERMS][2],
                                                 uint32_t (&sbyte)[MX8_TERMS]) {
#pragma unroll
    for (int t = 0; t < MX8_TERMS; ++t) {
        float am = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(v[i]));
        const int e = mx8_exp(__float_as_uint(am));
        sbyte[t] = static_cast<uint32_t>(e + 127);
        const float inv = mxq_inv(e), sc = mxq_scale(e);
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t pair = e4m3x2_from_f32(v[2 * i] * inv, v[2 * i + 1] * inv);
            if (i & 1)
                w[i >> 1] |= pair << 16;
            else
                w[i >> 1] = pair;
            if (t + 1 < MX8_TERMS) {
                const uint32_t h2 = e4m3x2_to_f16x2(pair);
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
                v[2 * i] -= f.x * sc;
                v[2 * i + 1] -= f.y * sc;
            }
        }
        codes[t][0] = make_uint4(w[0], w[1], w[2], w[3]);
        codes[t][1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

// Activation operand formats: AF = 0, three MXFP4 terms (16 code bytes per
// block and term); AF = 1, two MXFP8 terms (32 bytes per block and term).
template <int AF> struct ActFormat;
template <> struct ActFormat<0> {
    static constexpr int TERMS = MXQ_TERMS;
    static constexpr int CPB = 1;   // 16-byte chunks per block and term
};
template <> struct ActFormat<1> {
    static constexpr int TERMS = MX8_TERMS;
    static constexpr int CPB = 2;
};

// Encode one block b (32 values along K) of operand row `row` in format AF:
// the codes go to `codes` ([K/32 * CPB chunks][TERMS][R][16 B]), the scale
// bytes to sb[0 .. TERMS-1].
template <int AF>
__device__ __forceinline__ void act_encode_store(float (&v)[32], uint8_t* codes, int R, int b, int row,
                                                 uint32_t (&sb)[MXQ_TERMS]) {
    if constexpr (AF == 0) {
        uint4 c[MXQ_TERMS];
        mxq_block_thread(v, c, sb);
#pragma unroll
        for (int t = 0; t < MXQ_TERMS; ++t)
            *reinterpret_cast<uint4*>(codes + ((static_cast<size_t>(b) * MXQ_TERMS + t) * R + row) * 16) = c[t];
    } else {
        uint4 c[MX8_TERMS][2];
        uint32_t s2[MX8_TERMS];
        mx8_block_thread(v, c, s2);
        sb[0] = s2[0];
        sb[1] = s2[1];
        sb[2] = 0u;
#pragma unroll
        for (int t = 0; t < MX8_TERMS; ++t)
#pragma unroll
            for (int j = 0; j < 2; ++j)
                *reinterpret_cast<uint4*>(codes + ((static_cast<size_t>(2 * b + j) * MX8_TERMS + t) * R + row) * 16) =
                    c[t][j];
    }
}

}  // namespace moe
