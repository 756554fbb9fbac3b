// Pieces shared by the 1-CTA and CTA-pair block-scaled FP4 GEMM kernels:
// the tile order and the epilogue (accumulator drain, bf16 output, optional
// fused next-layer NVFP4 quantization of Y).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "gemm.h"
#include "nvfp4_math.cuh"
#include "ptx.cuh"

namespace nvfp4 {

struct TileCoord {
    int m_blk, n_blk;
};

// Tile t -> (m, n) block, walking groups of kGroupM row-blocks with m fastest
// inside a group, so concurrently running CTAs share B (weight) tiles and a
// group's A rows stay in L2.
constexpr int kGroupM = 8;
__device__ __forceinline__ TileCoord tile_coord(int t, int tiles_m, int tiles_n) {
    const int per_group = kGroupM * tiles_n;
    const int g = t / per_group;
    const int first_m = g * kGroupM;
    const int gsz = min(tiles_m - first_m, kGroupM);
    const int r = t - g * per_group;
    TileCoord c;
    c.m_blk = first_m + r % gsz;
    c.n_blk = r / gsz;
    return c;
}

// GELU of the fused FFN epilogue, g(h) = 0.5 h (1 + erf(h / sqrt 2)), from
// erfc(u), u = |h| / sqrt 2, by Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (Hastings' rational approximation,
// |error of erf| <= 1.5e-7):
//   erfc(u) ~ t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-u^2),
//   t = 1 / (1 + p u).
// Both signs in one expression without cancellation:
//   g = max(h, 0) - |h| erfc(|h| / sqrt 2) / 2,
// (h >= 0: h - h c / 2; h < 0: h c / 2).  Folded at compile time: p / sqrt 2
// (t straight from |h|), the 1/2 into the coefficients, and exp(-u^2) =
// 2^(h^2 * (-log2(e) / 2)).  The reciprocal and the power of two are the PTX
// approximations rcp.approx and ex2.approx (relative errors ~2^-23 and
// ~2^-22); the total error stays far below the bf16 rounding of the output.
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Abramowitz & Stegun 7.1.26, published coefficients.
constexpr float kAsP = 0.3275911f, kAsA1 = 0.254829592f, kAsA2 = -0.284496736f,
                kAsA3 = 1.421413741f, kAsA4 = -1.453152027f, kAsA5 = 1.061405429f;

__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// GELU of two values with the packed f32x2 operations of sm_100 (two fp32
// FMAs or products, each rounded as its scalar form, per instruction): the
// result is bit-identical to the scalar arrangement g = fma(-|h|, c/2,
// max(h, 0)) with c/2 = (t * poly) * e, because the -1/2 is folded into the
// coefficients (negating every coefficient negates every rounded
// intermediate exactly).
__device__ __forceinline__ float2 gelu_erf2(float2 h) {
    constexpr float p_h = kAsP * 0.70710678118654752f;  // t = 1 / (1 + p_h |h|)
    constexpr float n1 = -0.5f * kAsA1, n2 = -0.5f * kAsA2, n3 = -0.5f * kAsA3,
                    n4 = -0.5f * kAsA4, n5 = -0.5f * kAsA5;
    constexpr float k_e = -0.72134752044448170f;  // -log2(e) / 2
    const float2 ah = make_float2(fabsf(h.x), fabsf(h.y));
    const float2 den = __ffma2_rn(splat2(p_h), ah, splat2(1.0f));
    const float2 t = make_float2(rcp_approx(den.x), rcp_approx(den.y));
    float2 q = __ffma2_rn(t, splat2(n5), splat2(n4));
    q = __ffma2_rn(t, q, splat2(n3));
    q = __ffma2_rn(t, q, splat2(n2));
    q = __ffma2_rn(t, q, splat2(n1));
    q = __fmul2_rn(t, q);  // -erfc(|h|/sqrt 2) / 2 before the exponential
    const float2 arg = __fmul2_rn(__fmul2_rn(h, h), splat2(k_e));
    const float2 neg_half_c = __fmul2_rn(q, make_float2(ex2_approx(arg.x), ex2_approx(arg.y)));
    return __ffma2_rn(ah, neg_half_c, make_float2(fmaxf(h.x, 0.0f), fmaxf(h.y, 0.0f)));
}

// Scales 32 fp32 accumulator values by alpha (packed pairs), applies the
// activation (kGelu) and rounds to 16 packed bf16x2.
template <bool kGelu>
__device__ __forceinline__ void cvt_32(const uint32_t (&r)[32], float alpha, uint32_t *pk) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float2 h = __fmul2_rn(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])),
                              splat2(alpha));
        if (kGelu) h = gelu_erf2(h);
        const __nv_bfloat162 b = __floats2bfloat162_rn(h.x, h.y);
        pk[i] = *reinterpret_cast<const uint32_t *>(&b);
    }
}

// Reads NC (64 or 128) fp32 accumulator columns of this warp's 32 TMEM lanes
// (taddr = lane base + first column) into NC / 2 packed bf16x2 at pk (alpha,
// activation kGelu, rounding).  Two 32-column loads are in flight at a time.
template <int NC, bool kGelu>
__device__ __forceinline__ void drain_cols(uint32_t taddr, float alpha, uint32_t *pk) {
    static_assert(NC == 64 || NC == 128, "64 or 128 columns");
#pragma unroll
    for (int ch = 0; ch < NC / 32; ch += 2) {
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(taddr + ch * 32, r0);
        tmem_ld_32x32b_x32(taddr + ch * 32 + 32, r1);
        tmem_ld_wait();
        tmem_regs_ready(r0);
        tmem_regs_ready(r1);
        cvt_32<kGelu>(r0, alpha, pk + 16 * ch);
        cvt_32<kGelu>(r1, alpha, pk + 16 * ch + 16);
    }
}

// Writes one row's NC (64 or 128) bf16 outputs (columns n0..n0+NC-1 of row
// m) and, when the GEMM fuses the next layer's quantization, their codes and
// block scales (blocks of 16 along N with S_enc = s_enc_y).  Rows at or
// beyond M write no Y and no codes; rows in [M, pad128(M)) write zero scales
// (the layout's padding); rows beyond that write nothing.
template <int NC>
__device__ __forceinline__ void store_row(const GemmParams &p, const uint32_t (&pk)[NC / 2],
                                          int64_t m, int64_t n0, float s_enc_y,
                                          const float *inv_tab, uint32_t &amax_bits,
                                          bool write_y = true) {
    const bool row_ok = m < p.M;
    if (row_ok && p.y != nullptr && write_y) {
        uint8_t *yrow = p.y + (m * p.N + n0) * 2;
        if (n0 + NC <= p.N && (p.N & 15) == 0 && (reinterpret_cast<uintptr_t>(p.y) & 31) == 0) {
#pragma unroll
            for (int g = 0; g < NC / 16; ++g)
                stg256(yrow + 32 * g, pk[8 * g], pk[8 * g + 1], pk[8 * g + 2], pk[8 * g + 3],
                       pk[8 * g + 4], pk[8 * g + 5], pk[8 * g + 6], pk[8 * g + 7]);
        } else {
#pragma unroll
            for (int g = 0; g < NC / 8; ++g)
                if (n0 + 8 * g < p.N)
                    *reinterpret_cast<uint4 *>(yrow + 16 * g) =
                        make_uint4(pk[4 * g], pk[4 * g + 1], pk[4 * g + 2], pk[4 * g + 3]);
        }
    }
    if (p.yq == nullptr) return;
    const int64_t rows_pad = (p.M + 127) & ~int64_t(127);
    if (m >= rows_pad) return;
    const int64_t nb_y = p.N / 16;
    const int64_t nb4_y = (nb_y + 3) / 4;
#pragma unroll
    for (int q4 = 0; q4 < NC / 64; ++q4) {  // groups of 4 blocks (64 columns)
        uint32_t sf_word = 0;
        uint32_t cw[8];  // the group's 32 bytes of codes
        const int64_t nblk0 = (n0 >> 4) + 4 * q4;
        uint8_t *qrow = p.yq + m * (p.N / 2) + nblk0 * 8;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int bi = 4 * q4 + b;  // block within the NC columns
            const bool ok_blk = row_ok && nblk0 + b < nb_y;
            const uint4 v0 = make_uint4(pk[8 * bi], pk[8 * bi + 1], pk[8 * bi + 2], pk[8 * bi + 3]);
            const uint4 v1 =
                make_uint4(pk[8 * bi + 4], pk[8 * bi + 5], pk[8 * bi + 6], pk[8 * bi + 7]);
            const uint32_t mb = max(absmax_bf16x8(v0), absmax_bf16x8(v1));
            const BlockScale bs = block_scale(__uint_as_float(mb << 16), s_enc_y, inv_tab);
            cw[2 * b] = quantize_bf16x8(v0, bs.inv);
            cw[2 * b + 1] = quantize_bf16x8(v1, bs.inv);
            if (ok_blk) amax_bits = max(amax_bits, mb);
            sf_word |= (ok_blk ? bs.sf : 0u) << (8 * b);
        }
        // One 32-byte store (a whole sector) when the four blocks are in range
        // and the address is 32-byte aligned, else one 8-byte store per block.
        if (row_ok && nblk0 + 3 < nb_y && (reinterpret_cast<uintptr_t>(qrow) & 31) == 0) {
            stg256(qrow, cw[0], cw[1], cw[2], cw[3], cw[4], cw[5], cw[6], cw[7]);
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if (row_ok && nblk0 + b < nb_y)
                    *reinterpret_cast<uint2 *>(qrow + 8 * b) = make_uint2(cw[2 * b], cw[2 * b + 1]);
        }
        if (nblk0 < nb4_y * 4)
            *reinterpret_cast<uint32_t *>(p.ysf + sf_offset(m, nblk0, nb4_y)) = sf_word;
    }
}

// The epilogue of 64 accumulator columns (columns n0..n0+63 of row m) held
// in registers as raw fp32 (r0: the first 32, r1: the next 32), one block of
// 16 columns at a time: alpha, activation, bf16 rounding, the bf16 Y store
// and the fused quantize of that block, so each block's registers are free
// again before the next block starts (with the 64 raw values pinned in an
// 80-register budget, converting all 64 columns first left no room for
// independent work).  Same arithmetic per element, and the same outputs, as
// cvt_32 on both halves followed by store_row<64>.
template <bool kGelu>
__device__ __forceinline__ void store_blocks_64(const GemmParams &p, const uint32_t (&r0)[32],
                                                const uint32_t (&r1)[32], float alpha, int64_t m,
                                                int64_t n0, float s_enc_y, const float *inv_tab,
                                                uint32_t &amax_bits) {
    const bool row_ok = m < p.M;
    const bool want_y = row_ok && p.y != nullptr;
    uint8_t *yrow = want_y ? p.y + (m * p.N + n0) * 2 : nullptr;
    const bool y_fast = n0 + 64 <= p.N && (p.N & 15) == 0 &&
                        (reinterpret_cast<uintptr_t>(p.y) & 31) == 0;
    const int64_t rows_pad = (p.M + 127) & ~int64_t(127);
    const bool want_q = p.yq != nullptr && m < rows_pad;
    const int64_t nb_y = p.N / 16;
    const int64_t nblk0 = n0 >> 4;
    uint32_t cw[8];
    uint32_t sf_word = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t(&r)[32] = b < 2 ? r0 : r1;
        const int base = (b & 1) * 16;
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float2 h = __fmul2_rn(make_float2(__uint_as_float(r[base + 2 * i]),
                                              __uint_as_float(r[base + 2 * i + 1])),
                                  splat2(alpha));
            if (kGelu) h = gelu_erf2(h);
            const __nv_bfloat162 bb = __floats2bfloat162_rn(h.x, h.y);
            pk[i] = *reinterpret_cast<const uint32_t *>(&bb);
        }
        if (want_y) {
            if (y_fast) {
                stg256(yrow + 32 * b, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
            } else {
                if (n0 + 16 * b < p.N)
                    *reinterpret_cast<uint4 *>(yrow + 32 * b) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                if (n0 + 16 * b + 8 < p.N)
                    *reinterpret_cast<uint4 *>(yrow + 32 * b + 16) =
                        make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
        if (want_q) {
            const bool ok_blk = row_ok && nblk0 + b < nb_y;
            const uint4 v0 = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            const uint4 v1 = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            const uint32_t mb = max(absmax_bf16x8(v0), absmax_bf16x8(v1));
            const BlockScale bs = block_scale(__uint_as_float(mb << 16), s_enc_y, inv_tab);
            cw[2 * b] = quantize_bf16x8(v0, bs.inv);
            cw[2 * b + 1] = quantize_bf16x8(v1, bs.inv);
            if (ok_blk) amax_bits = max(amax_bits, mb);
            sf_word |= (ok_blk ? bs.sf : 0u) << (8 * b);
        }
    }
    if (!want_q) return;
    uint8_t *qrow = p.yq + m * (p.N / 2) + nblk0 * 8;
    if (row_ok && nblk0 + 3 < nb_y && (reinterpret_cast<uintptr_t>(qrow) & 31) == 0) {
        stg256(qrow, cw[0], cw[1], cw[2], cw[3], cw[4], cw[5], cw[6], cw[7]);
    } else {
#pragma unroll
        for (int b = 0; b < 4; ++b)
            if (row_ok && nblk0 + b < nb_y)
                *reinterpret_cast<uint2 *>(qrow + 8 * b) = make_uint2(cw[2 * b], cw[2 * b + 1]);
    }
    const int64_t nb4_y = (nb_y + 3) / 4;
    if (nblk0 < nb4_y * 4)
        *reinterpret_cast<uint32_t *>(p.ysf + sf_offset(m, nblk0, nb4_y)) = sf_word;
}

// Warp-reduces the fused output's |Y| maximum and folds it into amax_y.
__device__ __forceinline__ void flush_amax_y(const GemmParams &p, uint32_t amax_bits, int lane) {
    if (p.yq == nullptr || p.amax_y == nullptr) return;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        amax_bits = max(amax_bits, __shfl_xor_sync(0xFFFFFFFFu, amax_bits, o));
    if (lane == 0 && amax_bits != 0)
        atomicMax(reinterpret_cast<unsigned *>(p.amax_y), amax_bits << 16);
}

}  // namespace nvfp4
