// NVFP4 two-level microblock quantization arithmetic on the device: the FP32
// per-tensor scale and the per-16-element E4M3 block scale ("英伟达B200狂飙
// 10.2倍！AI绘图告别龟速！", section "NVFP4量化：在精度与速度之间寻得最佳平衡"),
// with E2M1 elements.  Every fp32 step is one IEEE round-to-nearest-even
// operation (__fdiv_rn / __fmul_rn), in a fixed order, so the codes are
// reproducible bit for bit:
//   S_enc = 2688 / amax (1 if amax == 0, FLT_MAX if not finite)
//   s     = (a_b / 6) * S_enc ;  sf = E4M3_rn_satfinite(s)
//   inv   = sf == 0 ? 0 : min(S_enc / sf, FLT_MAX)
//   q     = E2M1_rn_satfinite(x * inv), sign kept
// Conversions use the sm_100 cvt.rn.satfinite instructions.
#pragma once

#include <cfloat>
#include <cstdint>

namespace nvfp4 {

__device__ __forceinline__ float tensor_encode_scale(float amax) {
    if (amax == 0.0f) return 1.0f;
    float s = __fdiv_rn(2688.0f, amax);
    if (!isfinite(s)) s = FLT_MAX;
    return s;
}

// E4M3 code (low byte) of a non-negative fp32 value, round-to-nearest-even,
// saturating to 448.
__device__ __forceinline__ uint32_t e4m3_encode(float s) {
    uint32_t r;
    asm("{\n\t.reg .b16 h;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h, %1, %2;\n\t"
        "cvt.u32.u16 %0, h;\n\t}\n"
        : "=r"(r)
        : "f"(0.0f), "f"(s));
    return r & 0xFFu;
}

// Value of an unsigned E4M3 code (bias 7; exponent field 0 = subnormal).
__device__ __forceinline__ float e4m3_decode(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20))
             : __fmul_rn(static_cast<float>(m), 0.001953125f /* 2^-9 */);
}

struct BlockScale {
    uint32_t sf;  // E4M3 code
    float inv;    // multiplier taking x to E2M1 code space
};

// RN_fp32(a / 6) for every bf16 value a (subnormals included), computed as
// the double product a * RN64(1/6) rounded once to fp32.  Why it equals the
// IEEE fp32 quotient: a = M * 2^k with k >= -133, so a / 6 measured in units
// of its fp32 ulp (or of the subnormal spacing 2^-149) is an integer multiple
// of 1/3: it lies 0, 1/3 or 2/3 of a unit above a representable value, at
// least 1/6 unit from every rounding midpoint, while the double product is
// within 2^-52 relative of a / 6 (far below 1/6 unit); both round to the same
// fp32 value.  (The argument uses a's form; the fp32 product a * RN32(1/6)
// is not enough and differs for thousands of bf16 values.)
__device__ __forceinline__ float div6_short(float a) {
    return __double2float_rn(static_cast<double>(a) * (1.0 / 6.0));
}

// The block multiplier S_enc / sf depends only on the launch's S_enc and the
// 8-bit E4M3 code, so each CTA tabulates it once for the 127 finite
// non-negative codes (cvt ... satfinite never yields 0x7F):
//   inv[c] = sf_c == 0 ? 0 : min(S_enc / sf_c, FLT_MAX)   (IEEE division)
// Called by all threads of the CTA; the caller syncs before use.
__device__ __forceinline__ void fill_inv_table(float *tab, float s_enc) {
    for (int c = threadIdx.x; c < 128; c += blockDim.x) {
        const float sfv = e4m3_decode(static_cast<uint32_t>(c));
        float inv = 0.0f;
        if (sfv != 0.0f) {
            inv = __fdiv_rn(s_enc, sfv);
            if (!isfinite(inv)) inv = FLT_MAX;
        }
        tab[c] = inv;
    }
}

// Block scale with the multiplier computed directly (for per-row tensor
// scales, where one table per row would not pay off); same arithmetic as
// fill_inv_table.
__device__ __forceinline__ BlockScale block_scale_direct(float a_b, float s_enc) {
    const float s = __fmul_rn(div6_short(a_b), s_enc);
    BlockScale b;
    b.sf = e4m3_encode(s);
    const float sfv = e4m3_decode(b.sf);
    float inv = 0.0f;
    if (sfv != 0.0f) {
        inv = __fdiv_rn(s_enc, sfv);
        if (!isfinite(inv)) inv = FLT_MAX;
    }
    b.inv = inv;
    return b;
}

// Block scale of a 16-element block with amax a_b (a bf16 value):
//   s = (a_b / 6) * S_enc ; sf = E4M3_rn_satfinite(s) ; inv = tab[sf]
__device__ __forceinline__ BlockScale block_scale(float a_b, float s_enc, const float *inv_tab) {
    const float s = __fmul_rn(div6_short(a_b), s_enc);
    BlockScale b;
    b.sf = e4m3_encode(s);
    b.inv = inv_tab[b.sf];
    return b;
}

// Packs 8 fp32 values (already multiplied by inv) into 8 E2M1 codes, element
// 2j in the low nibble of byte j.  cvt...e2m1x2 puts its first source
// operand in the upper nibble.
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4,
                                           float v5, float v6, float v7) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}\n"
        : "=r"(r)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return r;
}

// |x| maximum of the 8 bf16 values in a 16-byte word, as bf16 bits (the
// magnitude order of non-NaN bf16 equals the unsigned order of bits&0x7FFF).
__device__ __forceinline__ uint32_t absmax_bf16x8(uint4 v) {
    uint32_t m = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    return max(m & 0xFFFFu, m >> 16);
}

// 16 bf16 values (32 bytes) held as 8 words.
struct BF16x16 {
    uint32_t w[8];
};

__device__ __forceinline__ BF16x16 ldg_stream_32B(const void *p) {
    BF16x16 v;
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]),
                   "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7])
                 : "l"(p));
    return v;
}

// 32 bytes at p: one 256-bit load when p is 32-byte aligned, else two
// 128-bit loads (the ABI only guarantees 16-byte alignment).
__device__ __forceinline__ BF16x16 ldg_32B(const uint8_t *p, bool aligned32) {
    if (aligned32) return ldg_stream_32B(p);
    BF16x16 v;
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint4 b = __ldg(reinterpret_cast<const uint4 *>(p + 16));
    v.w[0] = a.x; v.w[1] = a.y; v.w[2] = a.z; v.w[3] = a.w;
    v.w[4] = b.x; v.w[5] = b.y; v.w[6] = b.z; v.w[7] = b.w;
    return v;
}

__device__ __forceinline__ uint32_t absmax_bf16x16(const BF16x16 &v) {
    uint32_t m = __vmaxu2(v.w[0] & 0x7FFF7FFFu, v.w[1] & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w[2] & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w[3] & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w[4] & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w[5] & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w[6] & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w[7] & 0x7FFF7FFFu);
    return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// E2M1 codes of 8 bf16 values times inv.
// (The products are packed f32x2 multiplies, each half rounded as __fmul_rn.)
__device__ __forceinline__ uint32_t quantize_bf16x8(uint4 v, float inv) {
    const float2 i2 = make_float2(inv, inv);
    const float2 p0 = __fmul2_rn(make_float2(bf16_lo(v.x), bf16_hi(v.x)), i2);
    const float2 p1 = __fmul2_rn(make_float2(bf16_lo(v.y), bf16_hi(v.y)), i2);
    const float2 p2 = __fmul2_rn(make_float2(bf16_lo(v.z), bf16_hi(v.z)), i2);
    const float2 p3 = __fmul2_rn(make_float2(bf16_lo(v.w), bf16_hi(v.w)), i2);
    return e2m1x8(p0.x, p0.y, p1.x, p1.y, p2.x, p2.y, p3.x, p3.y);
}

// Byte offset of the block scale (row r, block c) in the 128x4-tiled layout
// whose rows hold kb4 = ceil(kb/4) tiles.
// T is int64_t, or uint32_t where the caller has checked every offset < 2^31.
template <typename T>
__device__ __forceinline__ T sf_offset(T r, T c, T kb4) {
    return ((r >> 7) * kb4 + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

}  // namespace nvfp4
