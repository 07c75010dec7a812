// Encoding helpers of the block-scaled FP4 activation forms shared by the grouped FFN's
// quantisers and the router (which writes decode activation rows itself): E2M1 and E4M3
// conversions, the four-plane MXFP4 decomposition, and the byte positions of a row in a
// tile of 128-byte rows (128-byte swizzle) and in a scale atom.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {

// E4M3 byte of 2^k, -9 <= k <= 8 (k < -6: subnormal).
__device__ __forceinline__ uint8_t e4m3_pow2(int k) {
    return k >= -6 ? (uint8_t)((k + 7) << 3) : (uint8_t)(1u << (k + 9));
}

__device__ __forceinline__ uint32_t atom_offset(int row, int j) { return (row & 31) * 16 + (row >> 5) * 4 + j; }

// Byte offset of 16-byte chunk c of row R in a tile of 128-byte rows with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_chunk(int R, int c) { return R * 128 + ((c ^ (R & 7)) << 4); }

// E2M1 rounding (nearest, ties to even, saturating at 6) of the pairs
// (v[2i], v[2i+1]), i < 4, by the hardware conversion: the returned word holds
// v[j] in bits 4j..4j+3 (low nibble = lower index); q[j] gets the rounded values.
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8], float (&q)[8]) {
    uint32_t w, h[4];
    asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t0, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t1, %8, %7;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t2, %10, %9;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t3, %12, %11;\n\t"
        "mov.b32 %0, {t0, t1, t2, t3};\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, t0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, t1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, t2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %4, t3;\n\t}"
        : "=r"(w), "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[i]));
        q[2 * i] = f.x;
        q[2 * i + 1] = f.y;
    }
    return w;
}

// The same for one pair: the byte holds lo in bits 0-3 and hi in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi, float *qlo, float *qhi) {
    uint32_t w, h;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %3, %2;\n\t"
        "mov.b32 %0, {t, 0, 0, 0};\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, t;\n\t}"
        : "=r"(w), "=r"(h)
        : "f"(lo), "f"(hi));
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
    *qlo = f.x;
    *qhi = f.y;
    return w;
}

// E2M1 codes (nearest, ties to even, saturating at 6) of the pair (lo, hi): one byte,
// lo in bits 0-3.
__device__ __forceinline__ uint32_t e2m1x2_code(float lo, float hi) {
    uint32_t w;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
        "mov.b32 %0, {t, 0, 0, 0};\n\t}"
        : "=r"(w)
        : "f"(lo), "f"(hi));
    return w;
}

// E4M3 code of v (nearest, ties to even, saturating at 448), in the low byte.
__device__ __forceinline__ uint32_t e4m3_code(float v) {
    uint32_t w;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\t"
        "cvt.u32.u16 %0, t;\n\t}"
        : "=r"(w)
        : "f"(v), "f"(0.0f));
    return w & 0xFFu;
}

// Value of an E4M3 code (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.u16.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h)
        : "r"(code & 0xFFu));
    return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

// Biased E8M0 exponent s of plane 0 for a block with maximum magnitude amax:
// s - 127 = floor(log2(amax)) - 1, so every |x| 2^-(s-127) < 4. Kept in
// [10, 253] so that the finest plane (s - 9) is a valid exponent and every
// plane unit and its inverse are normal floats.
__device__ __forceinline__ int mx_plane0_exp(float amax) {
    if (!(amax > 0.0f)) return 127;
    const int s = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 1;
    return s < 10 ? 10 : (s > 253 ? 253 : s);
}

__device__ __forceinline__ float exp2_biased(int s) { return __uint_as_float((uint32_t)s << 23); }   // 2^(s-127)
__device__ __forceinline__ float exp2_neg_biased(int s) { return __uint_as_float((uint32_t)(254 - s) << 23); }

// The four planes of 8 consecutive values of one 32-block with plane-0
// exponent s: out[p] holds the codes of plane p, value i in bits 4i..4i+3
// (low nibble = lower K index). The residual updates are exact in fp32.
__device__ __forceinline__ void mx_planes8(const float (&v)[8], int s, uint32_t (&out)[kMxPlanes]) {
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = v[i];
#pragma unroll
    for (int pl = 0; pl < kMxPlanes; ++pl) {
        const int sp = s - 3 * pl;
        const float inv = exp2_neg_biased(sp), unit = exp2_biased(sp);
        float t[8], q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = r[i] * inv;
        out[pl] = e2m1x8(t, q);
#pragma unroll
        for (int i = 0; i < 8; ++i) r[i] = fmaf(-q[i], unit, r[i]);
    }
}

}  // namespace moe
