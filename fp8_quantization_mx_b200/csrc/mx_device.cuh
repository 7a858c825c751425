// Device building blocks of the MX block-32 kernels (sm_100a).
//
// Work decomposition shared by every kernel: the bf16 input is viewed as a
// flat array of 32-byte "slices" of 16 elements, one per lane. Because every
// row length is a multiple of 32 (of 128 with Macro Block Scaling), a 32-element
// MX block is exactly 2 consecutive slices and a 128-element macro block 8, in
// the flat order, whatever the row length. A warp reads 32 consecutive slices
// per step (1 KiB contiguous, one 32-byte load per lane), so lanes 2q, 2q+1
// hold block q of the step and lanes 8h..8h+7 hold macro block h.
//
// Numerics, per block (OCP Microscaling as restated by "[vLLM] MXFP8/MXFP4"
// (MX format table) and "Unveiling the Potential of Quantization with MXFP4"
// (2.A, 2.B)):
//  * amax is the largest |x| of the block: a max of absolute values on packed
//    bf16 pairs (NaN-propagating), then the sign cleared; as an integer the
//    result orders finite values, then Inf, then NaN, so a non-finite block is
//    one whose amax bits reach 0x7F80;
//  * the E8M0 byte comes from the amax exponent field and mantissa bits with
//    integer arithmetic only;
//  * x * 2^-E is exact in bf16 whenever it is at least 2^-126 (a power-of-two
//    scaling of an 8-bit significand), and anything smaller rounds to a signed
//    zero code anyway, so the scaled pairs feed the hardware conversions
//    cvt.rn.satfinite.{e2m1x2,e4m3x2,e5m2x2,e3m2x2,e2m3x2}.f32 (round to
//    nearest even, saturate) or, for INT8, an fma-based integer rounding;
//  * with a macro factor f = (256 + k) / 256 the quotient x / (f 2^E) is not
//    exact in float; it is bracketed by two products with 1/f rounded down
//    and up, both bounds go through the hardware conversion, and the only way
//    they can disagree is an exact tie, where the even code wins (see
//    enc_mbs_cvt_16);
//  * decoding (fake-quant, error, dequantize): a byte-permute table for E2M1
//    (integer only), the hardware cvt.rn.f16x2.{e4m3x2,e5m2x2,e3m2x2,e2m3x2}
//    for the other float elements and an integer-to-float step for INT8 (all
//    exact), then an exact float product with the scale.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mxk {

constexpr int kFmtE2M1 = 0;
constexpr int kFmtE4M3 = 1;
constexpr int kFmtE5M2 = 2;
constexpr int kFmtE3M2 = 3;
constexpr int kFmtE2M3 = 4;
constexpr int kFmtInt8 = 5;
// 16-element blocks, E2M1 elements: MXFP4 at block 16 (E8M0 scale) and
// NVFP4 (E4M3 scale), the comparison formats of the MXFP4/NVFP4 gap analysis.
constexpr int kFmtE2M1B16 = 6;
constexpr int kFmtNvfp4 = 7;
constexpr int kFloor = 0, kCeil = 1, kOasRule = 2, kOas = 3;
constexpr int kMbsNone = 0, kMbsStatic = 1, kMbsDynamic = 2;
constexpr unsigned kFull = 0xFFFFFFFFu;

constexpr uint16_t kNaNbf16 = 0x7FC0;
constexpr uint32_t kNaNf32 = 0x7FC00000u;

// 16 bf16 values: w[i] holds elements 2i (low half) and 2i+1 (high half).
struct V16 {
  uint32_t w[8];
};
// 16 floats.
struct F16 {
  float v[16];
};

// ------------------------------------------------------------- memory ops --

// Streaming 32-byte load: read-only path, not kept in L1, 256-byte L2 prefetch.
__device__ __forceinline__ V16 ld_stream32(const void* p) {
  V16 r;
  asm volatile(
      "ld.global.nc.L1::no_allocate.L2::256B.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]), "=r"(r.w[5]),
        "=r"(r.w[6]), "=r"(r.w[7])
      : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Streaming (evict-first) stores of outputs nobody re-reads in this kernel.
__device__ __forceinline__ void st_stream8(void* p, uint2 v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ void st_stream16(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_stream32(void* p, const V16& v) {
  asm volatile("st.global.cs.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
               "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]),
               "r"(v.w[6]), "r"(v.w[7])
               : "memory");
}

// ------------------------------------------------------------ bf16 / bits --

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Element i of a V16 as a float (exact).
__device__ __forceinline__ float elem(const V16& v, int i) {
  return (i & 1) ? bf_hi(v.w[i >> 1]) : bf_lo(v.w[i >> 1]);
}

// Per-half max of |a|, |b| (sign of the result = xor of the signs; NaN wins).
__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Largest |x| bit pattern among the 16 bf16 values of a slice.
__device__ __forceinline__ uint32_t amax_bits16(const V16& v) {
  const uint32_t a = max_abs_bf16x2(max_abs_bf16x2(v.w[0], v.w[1]), max_abs_bf16x2(v.w[2], v.w[3]));
  const uint32_t b = max_abs_bf16x2(max_abs_bf16x2(v.w[4], v.w[5]), max_abs_bf16x2(v.w[6], v.w[7]));
  const uint32_t m = max_abs_bf16x2(a, b) & 0x7FFF7FFFu;
  return max(m & 0xFFFFu, m >> 16);
}

// Max over the two lanes of a block, and over the eight lanes of a macro block.
__device__ __forceinline__ uint32_t pair_max(uint32_t a) {
  return max(a, __shfl_xor_sync(kFull, a, 1));
}
__device__ __forceinline__ uint32_t oct_max(uint32_t a) {
  a = max(a, __shfl_xor_sync(kFull, a, 2));
  return max(a, __shfl_xor_sync(kFull, a, 4));
}

// 2^E as a float for E in [-149, 127] (subnormal below -126).
__device__ __forceinline__ float pow2f(int E) {
  return E >= -126 ? __uint_as_float(static_cast<uint32_t>(E + 127) << 23)
                   : __uint_as_float(1u << (E + 149));
}

// 2^-E for an E8M0 byte b = E + 127 in [0, 254]: a normal float, except
// 2^-127 (b = 254, reached only by INT8, whose emax is 0), a subnormal.
__device__ __forceinline__ float inv_scale_from_byte(int b) {
  return b <= 253 ? __uint_as_float(static_cast<uint32_t>(254 - b) << 23) : __uint_as_float(0x00400000u);
}

// 2^-E as a bf16x2 pair for b in [0, 254] (2^-127 is the bf16 subnormal 0x0040).
__device__ __forceinline__ uint32_t inv_scale_bf16x2(int b) {
  return b <= 253 ? static_cast<uint32_t>(254 - b) * 0x00800080u : 0x00400040u;
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// acc + h * h for the low (high) bf16 half h of w, in f32: the product is
// exact and the sum rounds once (mixed-precision fma of sm_100).
__device__ __forceinline__ float sq_acc_lo(uint32_t w, float acc) {
  float d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.bf16 %0, l, l, %2;\n\t}"
      : "=f"(d)
      : "r"(w), "f"(acc));
  return d;
}
__device__ __forceinline__ float sq_acc_hi(uint32_t w, float acc) {
  float d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.bf16 %0, h, h, %2;\n\t}"
      : "=f"(d)
      : "r"(w), "f"(acc));
  return d;
}

// Two fused multiply-adds in one instruction (sm_100 packed fp32): each half
// is an IEEE fma rounded to nearest even, exactly as fmaf.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n"
      " .reg .b64 ra, rb, rc, rd;\n"
      " mov.b64 ra, {%2, %3};\n"
      " mov.b64 rb, {%4, %5};\n"
      " mov.b64 rc, {%6, %7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n"
      " mov.b64 {%0, %1}, rd;\n"
      "}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// Two products in one instruction (sm_100 packed fp32): each half is an IEEE
// product rounded to nearest even, exactly as a * b.
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n"
      " .reg .b64 ra, rb, rd;\n"
      " mov.b64 ra, {%2, %3};\n"
      " mov.b64 rb, {%4, %5};\n"
      " mul.rn.f32x2 rd, ra, rb;\n"
      " mov.b64 {%0, %1}, rd;\n"
      "}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// lo[i] = e[i] * L and hi[i] = e[i] * H for N (even) values, two per
// instruction: the two ends of a reciprocal bracket.
template <int N>
__device__ __forceinline__ void bracket_products(const float* e, float L, float H, float* lo, float* hi) {
  const float2 l2 = make_float2(L, L), h2 = make_float2(H, H);
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float2 p = make_float2(e[2 * i], e[2 * i + 1]);
    const float2 a = fmul2(p, l2), b = fmul2(p, h2);
    lo[2 * i] = a.x;
    lo[2 * i + 1] = a.y;
    hi[2 * i] = b.x;
    hi[2 * i + 1] = b.y;
  }
}

// ------------------------------------------------------- element encoding --

// Two bf16x2 words (4 scaled values, element order) -> 4 E2M1 codes in the low
// 16 bits, element i in nibble i. cvt.rn.satfinite.e2m1x2.f32 d, a, b puts a
// in the upper nibble and b in the lower one.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const uint32_t s[4]) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(bf_lo(s[0])), "f"(bf_hi(s[0])), "f"(bf_lo(s[1])), "f"(bf_hi(s[1])),
        "f"(bf_lo(s[2])), "f"(bf_hi(s[2])), "f"(bf_lo(s[3])), "f"(bf_hi(s[3])));
  return r;
}

// Four bf16x2 words -> eight E4M3 bytes, element i in byte i.
__device__ __forceinline__ uint2 cvt_e4m3x8(const uint32_t s[4]) {
  uint2 r;
  asm("{\n\t.reg .b16 h0, h1, h2, h3;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h0, %3, %2;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h1, %5, %4;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h2, %7, %6;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h3, %9, %8;\n\t"
      "mov.b32 %0, {h0, h1};\n\t"
      "mov.b32 %1, {h2, h3};\n\t}"
      : "=r"(r.x), "=r"(r.y)
      : "f"(bf_lo(s[0])), "f"(bf_hi(s[0])), "f"(bf_lo(s[1])), "f"(bf_hi(s[1])),
        "f"(bf_lo(s[2])), "f"(bf_hi(s[2])), "f"(bf_lo(s[3])), "f"(bf_hi(s[3])));
  return r;
}

// The slice scaled by 2^-E (byte b), as bf16x2 words.
__device__ __forceinline__ V16 scale_slice(const V16& x, int b) {
  const uint32_t m = inv_scale_bf16x2(b);
  V16 s;
#pragma unroll
  for (int i = 0; i < 8; ++i) s.w[i] = mul_bf16x2(x.w[i], m);
  return s;
}

// 16 E2M1 codes of a scaled slice: nibble i of the result = element i.
__device__ __forceinline__ uint2 enc_e2m1_16(const V16& s) {
  return make_uint2(cvt_e2m1x8(&s.w[0]), cvt_e2m1x8(&s.w[4]));
}

// Codes of a block holding NaN/Inf: E2M1 has no NaN, so only the sign
// survives; E4M3 elements become S.1111.111, the NaN code.
__device__ __forceinline__ uint2 nonfinite_e2m1_16(const V16& x) {
  uint32_t r[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    r[i >> 2] |= ((x.w[i] >> 15) & 1u) << (8 * (i & 3) + 3);
    r[i >> 2] |= ((x.w[i] >> 31) & 1u) << (8 * (i & 3) + 7);
  }
  return make_uint2(r[0], r[1]);
}
__device__ __forceinline__ uint4 nonfinite_e4m3_16(const V16& x) {
  uint32_t r[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t a = x.w[2 * j], b = x.w[2 * j + 1];
    r[j] = (((a >> 15) & 1u) << 7 | 0x7Fu) | ((((a >> 31) & 1u) << 7 | 0x7Fu) << 8) |
           ((((b >> 15) & 1u) << 7 | 0x7Fu) << 16) | ((((b >> 31) & 1u) << 7 | 0x7Fu) << 24);
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

// ------------------------------------------------------- element decoding --
//
// E2M1 is decoded with integer operations only. (Feeding the register output
// of cvt.rn.satfinite.e2m1x2.f32 straight into cvt.rn.f16x2.e2m1x2 gave
// zeros on sm_100a in this build, while the same decode of codes loaded from
// memory was right; a table lookup avoids depending on that register path.
// The E4M3 pair of conversions showed no such problem in either path.)

// A table of the 8 E2M1 magnitudes as bf16 bit patterns, split into their
// high and low bytes, four entries per 32-bit word (index 0..3, 4..7), for
// byte-permute lookups.
struct E2m1Table {
  uint32_t hi0, hi1, lo0, lo1;
};
// Unscaled magnitudes 0 .5 1 1.5 2 3 4 6.
__device__ __forceinline__ E2m1Table e2m1_unscaled() {
  return E2m1Table{0x3F3F3F00u, 0x40404040u, 0xC0800000u, 0xC0804000u};
}

// The magnitudes times 2^E, for E in [-125, 125]: every nonzero product is a
// normal bf16 whose bit pattern is the unscaled one plus E in the exponent
// field (E * 128), added to both 16-bit halves of a packed pair at once (no
// half crosses zero or 0x7F80 in that range); code 0 stays 0.
__device__ __forceinline__ E2m1Table e2m1_table(int E) {
  const uint32_t both = static_cast<uint32_t>(E * (128 * 65537));   // E*128 in each half
  const uint32_t p01 = 0x3F000000u + static_cast<uint32_t>(E * (128 << 16));   // 0, 0.5
  const uint32_t p23 = 0x3FC03F80u + both;                                   // 1, 1.5
  const uint32_t p45 = 0x40404000u + both;                                   // 2, 3
  const uint32_t p67 = 0x40C04080u + both;                                   // 4, 6
  E2m1Table t;
  t.hi0 = __byte_perm(p01, p23, 0x7531);
  t.lo0 = __byte_perm(p01, p23, 0x6420);
  t.hi1 = __byte_perm(p45, p67, 0x7531);
  t.lo1 = __byte_perm(p45, p67, 0x6420);
  return t;
}

// Four E2M1 codes (nibbles 0..3 of c) -> two words of bf16x2 bit patterns.
__device__ __forceinline__ uint2 e2m1x4_to_bf16(uint32_t c, const E2m1Table& t) {
  const uint32_t sel = c & 0x7777u;                        // magnitude indices
  const uint32_t hi = __byte_perm(t.hi0, t.hi1, sel);
  const uint32_t lo = __byte_perm(t.lo0, t.lo1, sel);
  uint32_t w0 = __byte_perm(lo, hi, 0x5140);               // elements 0, 1
  uint32_t w1 = __byte_perm(lo, hi, 0x7362);               // elements 2, 3
  w0 |= ((c << 12) & 0x8000u) | ((c << 24) & 0x80000000u);  // sign bits 3, 7
  w1 |= ((c << 4) & 0x8000u) | ((c << 16) & 0x80000000u);   // sign bits 11, 15
  return make_uint2(w0, w1);
}

// Four E2M1 codes -> the magnitudes of their values (signs dropped).
__device__ __forceinline__ uint2 e2m1x4_mag_bf16(uint32_t c, const E2m1Table& t) {
  const uint32_t sel = c & 0x7777u;
  const uint32_t hi = __byte_perm(t.hi0, t.hi1, sel);
  const uint32_t lo = __byte_perm(t.lo0, t.lo1, sel);
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}
__device__ __forceinline__ V16 e2m1x16_mag_bf16(uint2 codes) {
  const E2m1Table t = e2m1_unscaled();
  V16 r;
  const uint32_t c[2] = {codes.x, codes.y};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint2 a = e2m1x4_mag_bf16(c[h] & 0xFFFFu, t);
    const uint2 b = e2m1x4_mag_bf16(c[h] >> 16, t);
    r.w[4 * h + 0] = a.x;
    r.w[4 * h + 1] = a.y;
    r.w[4 * h + 2] = b.x;
    r.w[4 * h + 3] = b.y;
  }
  return r;
}

// 16 E2M1 codes -> their values (unscaled, or scaled by the table) as bf16.
__device__ __forceinline__ V16 e2m1x16_to_bf16(uint2 codes, const E2m1Table& t) {
  V16 r;
  const uint32_t c[2] = {codes.x, codes.y};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint2 a = e2m1x4_to_bf16(c[h] & 0xFFFFu, t);
    const uint2 b = e2m1x4_to_bf16(c[h] >> 16, t);
    r.w[4 * h + 0] = a.x;
    r.w[4 * h + 1] = a.y;
    r.w[4 * h + 2] = b.x;
    r.w[4 * h + 3] = b.y;
  }
  return r;
}

__device__ __forceinline__ uint2 e2m1x4_to_bf16(uint32_t c) {
  return e2m1x4_to_bf16(c, e2m1_unscaled());
}
__device__ __forceinline__ V16 e2m1x16_to_bf16(uint2 codes) {
  return e2m1x16_to_bf16(codes, e2m1_unscaled());
}

// E8M0 bytes whose E2M1 products are all normal bf16 values: E in [-125, 125].
__device__ __forceinline__ bool e2m1_table_scale_ok(int b) { return b >= 2 && b <= 252; }

// Eight E4M3fn bytes (byte i = element i) -> four f16x2 words, exact (every
// E4M3 value is an f16 value; S.1111.111 becomes an f16 NaN). This hardware
// decode is exact for E4M3 both from memory and from the encoder's registers.
__device__ __forceinline__ void e4m3x8_to_f16x2(uint32_t lo, uint32_t hi, uint32_t h[4]) {
  asm("{\n\t.reg .b16 p0, p1, p2, p3;\n\t"
      "mov.b32 {p0, p1}, %4;\n\t"
      "mov.b32 {p2, p3}, %5;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, p0;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, p1;\n\t"
      "cvt.rn.f16x2.e4m3x2 %2, p2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %3, p3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(lo), "r"(hi));
}

__device__ __forceinline__ float f16_lo(uint32_t h) {
  float f;
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %1;\n\tcvt.f32.f16 %0, a;\n\t}" : "=f"(f) : "r"(h));
  return f;
}
__device__ __forceinline__ float f16_hi(uint32_t h) {
  float f;
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %1;\n\tcvt.f32.f16 %0, b;\n\t}" : "=f"(f) : "r"(h));
  return f;
}

// Decoded values times p (a power of two): exact floats, overflow to +-inf.
__device__ __forceinline__ F16 dec_e2m1_16(uint2 codes, float p) {
  const V16 b = e2m1x16_to_bf16(codes);
  F16 r;
#pragma unroll
  for (int i = 0; i < 16; ++i) r.v[i] = elem(b, i) * p;
  return r;
}
__device__ __forceinline__ F16 dec_e4m3_16(uint4 codes, float p) {
  uint32_t h[8];
  e4m3x8_to_f16x2(codes.x, codes.y, &h[0]);
  e4m3x8_to_f16x2(codes.z, codes.w, &h[4]);
  F16 r;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    r.v[2 * i] = f16_lo(h[i]) * p;
    r.v[2 * i + 1] = f16_hi(h[i]) * p;
  }
  return r;
}

// Two floats -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ------------------------------------------------------- one-byte formats --
//
// E4M3, E5M2, E3M2 and E2M3 codes come from the hardware converters
// cvt.rn.satfinite.{e4m3x2,e5m2x2,e3m2x2,e2m3x2}.f32 (round to nearest even,
// saturating, sign kept; an FP6 code sits in the low 6 bits of its byte) and
// decode through cvt.rn.f16x2.{...}x2 (every such value is an f16 value). An
// INT8 code is RNE(64 s) of the scaled value s clamped to +-127/64, two's
// complement, so that the element reads i * 2^-6.

#define MXK_CVT_BYTES_X8(NAME, TYPE)                                                 \
  __device__ __forceinline__ uint2 NAME(const uint32_t s[4]) {                     \
    uint2 r;                                                                        \
    asm("{\n\t.reg .b16 h0, h1, h2, h3;\n\t"                                       \
        "cvt.rn.satfinite." TYPE ".f32 h0, %3, %2;\n\t"                             \
        "cvt.rn.satfinite." TYPE ".f32 h1, %5, %4;\n\t"                             \
        "cvt.rn.satfinite." TYPE ".f32 h2, %7, %6;\n\t"                             \
        "cvt.rn.satfinite." TYPE ".f32 h3, %9, %8;\n\t"                             \
        "mov.b32 %0, {h0, h1};\n\t"                                                 \
        "mov.b32 %1, {h2, h3};\n\t}"                                                \
        : "=r"(r.x), "=r"(r.y)                                                      \
        : "f"(bf_lo(s[0])), "f"(bf_hi(s[0])), "f"(bf_lo(s[1])), "f"(bf_hi(s[1])),   \
          "f"(bf_lo(s[2])), "f"(bf_hi(s[2])), "f"(bf_lo(s[3])), "f"(bf_hi(s[3])));  \
    return r;                                                                       \
  }
MXK_CVT_BYTES_X8(cvt_e5m2x8, "e5m2x2")
MXK_CVT_BYTES_X8(cvt_e3m2x8, "e3m2x2")
MXK_CVT_BYTES_X8(cvt_e2m3x8, "e2m3x2")
#undef MXK_CVT_BYTES_X8

// INT8 codes of four bf16x2 words of scaled values: 64 s (exact) clamped to
// +-127, plus 1.5 * 2^23 in one fma, leaves RNE(64 s) in the low mantissa
// bits, so the low byte is the two's complement code.
__device__ __forceinline__ uint2 cvt_int8x8(const uint32_t s[4]) {
  uint32_t t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float v = (i & 1) ? bf_hi(s[i >> 1]) : bf_lo(s[i >> 1]);
    const float c = fminf(fmaxf(v, -1.984375f), 1.984375f);
    t[i] = __float_as_uint(fmaf(c, 64.0f, 12582912.0f));
  }
  return make_uint2(__byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410),
                    __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410));
}

template <int FMT>
__device__ __forceinline__ uint2 cvt_bytes_x8(const uint32_t s[4]) {
  if constexpr (FMT == kFmtE4M3) return cvt_e4m3x8(s);
  else if constexpr (FMT == kFmtE5M2) return cvt_e5m2x8(s);
  else if constexpr (FMT == kFmtE3M2) return cvt_e3m2x8(s);
  else if constexpr (FMT == kFmtE2M3) return cvt_e2m3x8(s);
  else return cvt_int8x8(s);
}

// 16 one-byte codes of a scaled slice: byte i = element i.
template <int FMT>
__device__ __forceinline__ uint4 enc_bytes_16(const V16& s) {
  const uint2 a = cvt_bytes_x8<FMT>(&s.w[0]);
  const uint2 b = cvt_bytes_x8<FMT>(&s.w[4]);
  return make_uint4(a.x, a.y, b.x, b.y);
}

// Codes of a block holding NaN/Inf: the FP8 NaN S.1111.111 / S.11111.11
// (0x7F with the sign); FP6 has no NaN, so only the sign (bit 5); INT8 has
// neither NaN nor -0: 0.
template <int FMT>
__device__ __forceinline__ uint4 nonfinite_bytes_16(const V16& x) {
  if constexpr (FMT == kFmtE4M3 || FMT == kFmtE5M2) {
    return nonfinite_e4m3_16(x);
  } else if constexpr (FMT == kFmtInt8) {
    return make_uint4(0, 0, 0, 0);
  } else {
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t a = x.w[2 * j], b = x.w[2 * j + 1];
      r[j] = (((a >> 15) & 1u) << 5) | (((a >> 31) & 1u) << 13) | (((b >> 15) & 1u) << 21) |
             (((b >> 31) & 1u) << 29);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
  }
}

#define MXK_BYTES_TO_F16X2(NAME, TYPE)                                         \
  __device__ __forceinline__ void NAME(uint32_t lo, uint32_t hi, uint32_t h[4]) { \
    asm("{\n\t.reg .b16 p0, p1, p2, p3;\n\t"                                   \
        "mov.b32 {p0, p1}, %4;\n\t"                                            \
        "mov.b32 {p2, p3}, %5;\n\t"                                            \
        "cvt.rn.f16x2." TYPE " %0, p0;\n\t"                                    \
        "cvt.rn.f16x2." TYPE " %1, p1;\n\t"                                    \
        "cvt.rn.f16x2." TYPE " %2, p2;\n\t"                                    \
        "cvt.rn.f16x2." TYPE " %3, p3;\n\t}"                                   \
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])                       \
        : "r"(lo), "r"(hi));                                                   \
  }
MXK_BYTES_TO_F16X2(e5m2x8_to_f16x2, "e5m2x2")
MXK_BYTES_TO_F16X2(e3m2x8_to_f16x2, "e3m2x2")
MXK_BYTES_TO_F16X2(e2m3x8_to_f16x2, "e2m3x2")
#undef MXK_BYTES_TO_F16X2

// Decoded values of 16 one-byte codes times p (a power of two): exact floats
// (INT8: i * 2^-6 * p, exact down to 2^-149), overflow to +-inf, NaN codes NaN.
template <int FMT>
__device__ __forceinline__ F16 dec_bytes_16(uint4 codes, float p) {
  if constexpr (FMT == kFmtE4M3) {
    return dec_e4m3_16(codes, p);
  } else if constexpr (FMT == kFmtInt8) {
    F16 r;
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    const float q = p * 0.015625f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int v = static_cast<int>(w[i >> 2] << (24 - 8 * (i & 3))) >> 24;   // sign-extended
      r.v[i] = (__int_as_float(0x4B400000 + v) - 12582912.0f) * q;
    }
    return r;
  } else {
    F16 r;
    uint32_t h[8];
    if constexpr (FMT == kFmtE5M2) {
      e5m2x8_to_f16x2(codes.x, codes.y, &h[0]);
      e5m2x8_to_f16x2(codes.z, codes.w, &h[4]);
    } else if constexpr (FMT == kFmtE3M2) {
      e3m2x8_to_f16x2(codes.x, codes.y, &h[0]);
      e3m2x8_to_f16x2(codes.z, codes.w, &h[4]);
    } else {
      e2m3x8_to_f16x2(codes.x, codes.y, &h[0]);
      e2m3x8_to_f16x2(codes.z, codes.w, &h[4]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      r.v[2 * i] = f16_lo(h[i]) * p;
      r.v[2 * i + 1] = f16_hi(h[i]) * p;
    }
    return r;
  }
}

// -------------------------------------------------------- scale selection --

// oas_m7: OAS can prefer the coarser exponent E1 + 1 only when the block max,
// scaled by 2^-E1, exceeds the midpoint between maxv and the first value of
// the coarser grid above it, 2 * (the element after maxv / 2): below that
// every element rounds to a value at least as close on the finer grid
// (maxv / 2 is an element, so maxv is on both grids, and the coarser grid
// below maxv is a subset of the finer one). In significand terms: M7 above
// oas_m7.
template <int FMT>
struct Elem;
template <>
struct Elem<kFmtE2M1> {
  static constexpr int emax = 2;          // 6 = 1.5 * 2^2
  static constexpr float maxv = 6.0f;
  static constexpr int ceil_m7 = 64;      // significand above 1.5 overflows 4m <= 6
  static constexpr int oas_m7 = 96;       // OAS band: scaled max above 7 (see below)
  static constexpr int min_log2 = -1;     // smallest magnitude 1/2
};
template <>
struct Elem<kFmtE4M3> {
  static constexpr int emax = 8;          // 448 = 1.75 * 2^8
  static constexpr float maxv = 448.0f;
  static constexpr int ceil_m7 = 96;      // significand above 1.75 overflows 256m <= 448
  static constexpr int oas_m7 = 104;      // scaled max above 464
  static constexpr int min_log2 = -9;     // smallest magnitude 2^-9
};
template <>
struct Elem<kFmtE5M2> {
  static constexpr int emax = 15;         // 57344 = 1.75 * 2^15
  static constexpr float maxv = 57344.0f;
  static constexpr int ceil_m7 = 96;
  static constexpr int oas_m7 = 112;      // scaled max above 61440
  static constexpr int min_log2 = -16;
};
template <>
struct Elem<kFmtE3M2> {
  static constexpr int emax = 4;          // 28 = 1.75 * 2^4
  static constexpr float maxv = 28.0f;
  static constexpr int ceil_m7 = 96;
  static constexpr int oas_m7 = 112;      // scaled max above 30
  static constexpr int min_log2 = -4;
};
template <>
struct Elem<kFmtE2M3> {
  static constexpr int emax = 2;          // 7.5 = 1.875 * 2^2
  static constexpr float maxv = 7.5f;
  static constexpr int ceil_m7 = 112;     // significand above 1.875 overflows
  static constexpr int oas_m7 = 120;      // scaled max above 7.75
  static constexpr int min_log2 = -3;
};
template <>
struct Elem<kFmtInt8> {
  static constexpr int emax = 0;          // i * 2^-6, |i| <= 127: 127/64 < 2
  static constexpr float maxv = 1.984375f;
  static constexpr int ceil_m7 = 126;     // significand 1 + 127/128 overflows 127/64
  static constexpr int oas_m7 = 127;      // (no OAS for INT8)
  static constexpr int min_log2 = -6;
};

// E8M0 byte of a finite block from its amax bits for the rules decided by the
// amax alone (FLOOR, CEIL, OAS_RULE); OAS starts from FLOOR. A subnormal or
// zero amax has exponent field 0 and always clamps to byte 0 (E = -127); the
// top clamp (E = 127, byte 254) is reachable only with emax 0 (INT8).
template <int FMT, int RULE>
__device__ __forceinline__ int rule_byte(uint32_t amax) {
  const int ex = static_cast<int>(amax >> 7);
  // a subnormal amax is below 2^-126: E = -127 under every rule (and its
  // mantissa bits are not a normalised significand, so the tests below would
  // misread them when emax is 0)
  if (ex == 0) return 0;
  const int m7 = static_cast<int>(amax & 0x7F);
  int b = ex - Elem<FMT>::emax;
  if (RULE == kCeil) b += (m7 > Elem<FMT>::ceil_m7) ? 1 : 0;
  if (RULE == kOasRule) b += (m7 > 96) ? 1 : 0;
  return min(max(b, 0), 254);
}

// OAS evaluation of one lane's 16 elements (E2M1, no macro factor): the codes
// under both candidates, E1 (byte b1) and E2 = E1 + 1, and the exact
// difference of their squared errors in units of 2^-10 of the E1 scale,
//   delta = sum over the elements of (d1^2 - d2^2) = sum (d1 - d2)(d1 + d2),
// with s = x 2^-E1, d1 = s - q1, d2 = s - 2 q2 (q the code values). Where
// both codes are zero, d1 == d2 and the term is exactly 0. Elsewhere s has
// 2^-9 resolution, d1 - d2 = 2 q2 - q1 (a multiple of 1/2, at most 8) and
// d1 + d2 (a multiple of 2^-9, below 4) multiply exactly, and the running sum
// of 16 such terms (multiples of 2^-10, each below 4) stays exact in float.
struct OasEval {
  uint2 c1, c2;
  int delta;
};
__device__ __forceinline__ OasEval oas_eval16(const V16& x, int b1) {
  const V16 s1 = scale_slice(x, b1);
  const V16 s2 = scale_slice(x, b1 + 1);
  OasEval r;
  r.c1 = enc_e2m1_16(s1);
  r.c2 = enc_e2m1_16(s2);
  const V16 q1 = e2m1x16_to_bf16(r.c1);
  const V16 q2 = e2m1x16_to_bf16(r.c2);
  // d1 = s - q1, d2 = s - 2 q2, sum of (d1 - d2)(d1 + d2), two elements per
  // packed fma; every value and partial sum is an exact multiple of 2^-9
  // below 2^6, so the order does not matter
  const float2 m1 = make_float2(-1.0f, -1.0f), p1 = make_float2(1.0f, 1.0f);
  const float2 m2 = make_float2(-2.0f, -2.0f);
  float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const float2 s = make_float2(bf_lo(s1.w[w]), bf_hi(s1.w[w]));
    const float2 d1 = ffma2(make_float2(bf_lo(q1.w[w]), bf_hi(q1.w[w])), m1, s);
    const float2 d2 = ffma2(make_float2(bf_lo(q2.w[w]), bf_hi(q2.w[w])), m2, s);
    acc = ffma2(ffma2(d2, m1, d1), ffma2(d2, p1, d1), acc);
  }
  r.delta = __float2int_rn((acc.x + acc.y) * 1024.0f);   // an integer below 2^16: exact
  return r;
}

// OAS evaluation of one lane's 16 elements for a one-byte float format
// (E4M3, E5M2, E3M2, E2M3): the codes under both candidates, E1 (byte b1) and
// E2 = E1 + 1, and the exact difference of their squared errors,
//   delta = sum (d1^2 - d2^2) = sum (D1 - D2)(D1 + D2)   in units of U^2,
// with s = x 2^-E1, d1 = s - q1, d2 = s - 2 q2 (q the code values) and
// D = d / U, U = 2^(min_log2 - 9) (in units of the E1 scale). An element that
// rounds differently under the two candidates has |s| of at least half the
// smallest magnitude, so s (8 significant bits) and both grid values are
// multiples of U and D1, D2 are exact integers below 2^41; an element that
// rounds to the same value gives D1 == D2 whatever its size. The products
// reach 2^82 for E5M2, so its sum is kept in 128-bit integers; for E4M3,
// E3M2 and E2M3, |D| < 2^(emax + 11 - min_log2) <= 2^28, every product stays
// below 2^58 and a lane's sum of 16 below 2^62: 64-bit integers hold them.
// The integer held exactly by a float v with |v| < 2^22 (no conversion unit:
// adding 1.5 * 2^23 puts v in the low mantissa bits).
__device__ __forceinline__ int small_int(float v) {
  return __float_as_int(v + 12582912.0f) - 0x4B400000;
}

struct OasEvalBytes {
  uint4 c1, c2;
  __int128 delta;
};
template <bool kWide> struct OasAcc { using T = long long; };
template <> struct OasAcc<true> { using T = __int128; };
template <int FMT>
__device__ __forceinline__ OasEvalBytes oas_eval_bytes16(const V16& x, int b1) {
  const V16 s1 = scale_slice(x, b1);
  const V16 s2 = scale_slice(x, b1 + 1);
  OasEvalBytes r;
  r.c1 = enc_bytes_16<FMT>(s1);
  r.c2 = enc_bytes_16<FMT>(s2);
  const F16 q1 = dec_bytes_16<FMT>(r.c1, 1.0f);
  const F16 q2 = dec_bytes_16<FMT>(r.c2, 2.0f);   // E2 values in units of the E1 scale
  const float unit = pow2f(9 - Elem<FMT>::min_log2);
  using Acc = typename OasAcc<FMT == kFmtE5M2>::T;
  Acc acc = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float si = elem(s1, i);
    long long D1, D2;
    if constexpr (Elem<FMT>::emax + 11 - Elem<FMT>::min_log2 <= 22) {
      // E3M2, E2M3: |D| < 2^22, so the float add of small_int extracts it
      D1 = small_int((si - q1.v[i]) * unit);
      D2 = small_int((si - q2.v[i]) * unit);
    } else if constexpr (Elem<FMT>::emax + 11 - Elem<FMT>::min_log2 <= 31) {
      // E4M3: |D| < 2^28 fits the 32-bit converter
      D1 = __float2int_rn((si - q1.v[i]) * unit);
      D2 = __float2int_rn((si - q2.v[i]) * unit);
    } else {
      D1 = __float2ll_rn((si - q1.v[i]) * unit);
      D2 = __float2ll_rn((si - q2.v[i]) * unit);
    }
    acc += static_cast<Acc>(D1 - D2) * static_cast<Acc>(D1 + D2);
  }
  r.delta = acc;
  return r;
}

// The sum of a 128-bit value over a lane pair.
__device__ __forceinline__ __int128 pair_sum_i128(__int128 v) {
  const unsigned long long lo = static_cast<unsigned long long>(v);
  const long long hi = static_cast<long long>(v >> 64);
  const unsigned long long olo = __shfl_xor_sync(kFull, lo, 1);
  const long long ohi = __shfl_xor_sync(kFull, hi, 1);
  return v + ((static_cast<__int128>(ohi) << 64) | static_cast<__int128>(olo));
}

// ------------------------------------------------ macro-factor arithmetic --

// Normalised 8-bit significand (128..255) of a nonzero finite bf16 magnitude.
__device__ __forceinline__ int norm_significand(uint32_t a) {
  if (a >> 7) return 128 | static_cast<int>(a & 0x7F);
  const int m = static_cast<int>(a & 0x7F);
  return m << (__clz(m) - 24);
}

// MBS-Static factor: with p such that 6 * 2^p <= A < 12 * 2^p, the smallest k
// with 6 (256 + k) 2^p >= 256 A. Writing A = S 2^(e-7) (S the 8-bit
// significand) this is k = ceil(c S / 3) - 256 with c = 4 when S >= 192
// (A / 2^p in [6, 8)) and c = 8 otherwise (A / 2^p in [8, 12)); k never
// reaches 256 for a bf16 A.
__device__ __forceinline__ int mbs_static_k(uint32_t A) {
  if (A == 0 || A >= 0x7F80u) return 0;
  const int S = norm_significand(A);
  const int c = S >= 192 ? 4 : 8;
  return (c * S + 2) / 3 - 256;
}

// E8M0 byte of a sub-block under factor k: floor(log2(amax / f)) - 2 + up,
// where dividing by f lowers the exponent by one exactly when the amax
// significand 1 + m7/128 is below f = 1 + k/256, i.e. 2 m7 < k. up = 0 gives
// the FLOOR byte, up = 1 the next coarser one (the OAS candidate).
__device__ __forceinline__ int mbs_byte(uint32_t amax, int k, int up) {
  const int ex = static_cast<int>(amax >> 7);
  if (ex == 0) return 0;
  const int m7 = static_cast<int>(amax & 0x7F);
  return max(ex - 2 + up - ((2 * m7 < k) ? 1 : 0), 0);
}

// Eight floats -> eight E2M1 codes, element i in nibble i.
__device__ __forceinline__ uint32_t cvt_e2m1_f8(const float* v) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// Bracket of 1/f for f = (256 + k) / 256: L <= 1/f <= H, both within 2^-20.
struct FactorBracket {
  float f, L, H;
};
// 1/f from the hardware reciprocal (PTX rcp.approx: at most 1 ulp from 1/f,
// i.e. within 2^-23 relatively for f in [1, 2)); the 2^-20 margins on either
// side keep L below and H above 1/f after their own rounding, and both within
// 2^-19 of it.
__device__ __forceinline__ FactorBracket factor_bracket(int k) {
  FactorBracket r;
  r.f = static_cast<float>(256 + k) * 0.00390625f;   // exact
  float inv;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(r.f));
  r.L = inv * 0.99999904632568359375f;   // 1 - 2^-20
  r.H = inv * 1.00000095367431640625f;   // 1 + 2^-20
  return r;
}

// OAS under a macro factor: the coarser candidate can only win when the block
// max, in units of f 2^E1 (byte b1), exceeds 7 -- below that every element's
// error on the finer grid is no larger (the grids are those of plain OAS
// scaled by f). amax * 2^-E1 and 7 f are exact floats.
__device__ __forceinline__ bool mbs_oas_band(uint32_t amax, int b1, int k) {
  const float s = __uint_as_float(amax << 16) * inv_scale_from_byte(b1);
  return s > 7.0f * static_cast<float>(256 + k) * 0.00390625f;
}

// Of two nibble-packed code words that agree except where an element's codes
// are adjacent (c, c+1), keep the even code of each such pair: those bits
// differ in bit 0, and the odd one of the pair is the one with bit 0 set.
__device__ __forceinline__ uint32_t even_of_adjacent(uint32_t lo, uint32_t hi) {
  const uint32_t diff = lo ^ hi;
  const uint32_t take_hi = (lo & diff & 0x11111111u) * 0xFu;   // nibbles where lo is odd
  return lo ^ (diff & take_hi);
}

// MBS codes of 16 elements under factor k and exponent byte b, rounded
// exactly with the hardware converter. The quotient q = s / f (s = x 2^-E
// exact, f = (256 + k) / 256) is not exact in float, but it is bracketed: with
// L <= 1/f <= H (within 2^-20 of 1/f, with margin for float rounding),
// fl(s L) <= |q| <= fl(s H) in magnitude. Rounding to the grid is monotone,
// so both bounds give the code of q unless the bracket holds a grid midpoint.
// It can hold one only when q is exactly that midpoint: s has 8 significant
// bits and mid * f is a multiple of 2^-10, so a q that is not a midpoint lies
// at least 2^-10 / 10 (relatively) away from every one, far outside the
// 2^-19 bracket. At a tie the bounds give the two adjacent codes, and the
// even one is the round-to-nearest-even result.
__device__ __forceinline__ uint2 enc_mbs_cvt_16(const V16& x, int b, int k) {
  const FactorBracket fb = factor_bracket(k);
  // 2^-E folded into the bracket: for a finite block E <= 125 (b <= 252), so
  // L 2^-E and H 2^-E are normal floats, exact, and x (L 2^-E) rounds as
  // (x 2^-E) L does wherever x 2^-E is a normal number; below that (an
  // element under 2^-126 of the scale) both give a zero code of x's sign
  const float p = inv_scale_from_byte(b);
  float e[16], lo[16], hi[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) e[i] = elem(x, i);
  bracket_products<16>(e, fb.L * p, fb.H * p, lo, hi);
  return make_uint2(even_of_adjacent(cvt_e2m1_f8(lo), cvt_e2m1_f8(hi)),
                    even_of_adjacent(cvt_e2m1_f8(lo + 8), cvt_e2m1_f8(hi + 8)));
}

// Codes of 8 non-negative scaled values under the bracket L <= 1/f <= H (see
// enc_mbs_cvt_16), and their E2M1 magnitudes as floats.
__device__ __forceinline__ uint32_t mbs_codes8(const float* s8, float L, float H) {
  float lo[8], hi[8];
  bracket_products<8>(s8, L, H, lo, hi);
  return even_of_adjacent(cvt_e2m1_f8(lo), cvt_e2m1_f8(hi));
}
// ---------------------------------------------------------------- NVFP4 --
//
// The block scale is amax / 6 rounded to E4M3 (ties to even, saturating):
// the IEEE quotient amax / 6 in float lies exactly on an E4M3 midpoint when
// the real one does (then it is a short dyadic number) and otherwise at least
// 2^-12 (relatively) from every midpoint, far beyond its 2^-24 rounding, so
// the hardware E4M3 conversion of it is the correctly rounded scale. Returns
// the E4M3 byte; the NaN byte 0x7F for a non-finite block.
__device__ __forceinline__ int nvfp4_scale_byte(uint32_t amax) {
  if (amax >= 0x7F80u) return 0x7F;
  const float q = __fdiv_rn(__uint_as_float(amax << 16), 6.0f);
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(q));
  return h & 0xFF;
}
// The value of an E4M3 byte as a float (exact; NaN for S.1111.111).
__device__ __forceinline__ float e4m3_value(int byte) {
  uint32_t h;
  const uint16_t b = static_cast<uint16_t>(byte);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(b));
  return f16_lo(h);
}

// E2M1 codes of x / s for a positive E4M3 scale value s: as with the macro
// factor, x / s is bracketed by two products with 1/s moved 2^-20 down and up
// (1/s from the hardware reciprocal, within 1 ulp) and both bounds are
// converted. x (8 significant bits) and mid * s (a midpoint of the grid times
// a 4-bit s) differ, unless equal, by at least 2^-8 of x, so the bounds
// disagree only at an exact tie, where the even code is kept.
__device__ __forceinline__ uint2 enc_e2m1_div_16(const V16& x, float s) {
  float inv;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(s));
  const float L = inv * 0.99999904632568359375f;   // 1 - 2^-20
  const float H = inv * 1.00000095367431640625f;   // 1 + 2^-20
  float e[16], lo[16], hi[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) e[i] = elem(x, i);
  bracket_products<16>(e, L, H, lo, hi);
  return make_uint2(even_of_adjacent(cvt_e2m1_f8(lo), cvt_e2m1_f8(hi)),
                    even_of_adjacent(cvt_e2m1_f8(lo + 8), cvt_e2m1_f8(hi + 8)));
}

__device__ __forceinline__ void e2m1x8_values(uint32_t codes, float* v) {
  const uint2 a = e2m1x4_to_bf16(codes & 0xFFFFu);
  const uint2 b = e2m1x4_to_bf16(codes >> 16);
  v[0] = bf_lo(a.x); v[1] = bf_hi(a.x); v[2] = bf_lo(a.y); v[3] = bf_hi(a.y);
  v[4] = bf_lo(b.x); v[5] = bf_hi(b.x); v[6] = bf_lo(b.y); v[7] = bf_hi(b.y);
}

// OAS evaluation of one lane's 16 elements under factor k: codes for E1
// (byte b1) and E2 = E1 + 1 and the exact difference of the squared errors,
// in units of 2^-18 of the E1 scale: sum of D1^2 - D2^2 with D = 512 d,
// d1 = s - q1 f and d2 = s - 2 q2 f (s = x 2^-E1, q the code values). Where
// both codes are zero, d1 == d2 and the term cancels; elsewhere s and q f are
// multiples of 2^-9, so each d is exact (below 4 in magnitude) and each D an
// integer below 2^11: the int32 sum is exact.
__device__ __forceinline__ OasEval oas_eval_mbs16(const V16& x, int b1, int k) {
  const FactorBracket fb = factor_bracket(k);
  const V16 s1 = scale_slice(x, b1);
  float s[16], h[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s[2 * i] = bf_lo(s1.w[i]);
    s[2 * i + 1] = bf_hi(s1.w[i]);
    const float2 hh = fmul2(make_float2(s[2 * i], s[2 * i + 1]), make_float2(0.5f, 0.5f));
    h[2 * i] = hh.x;
    h[2 * i + 1] = hh.y;
  }
  OasEval r;
  {
    float lo[16], hi[16], lo2[16], hi2[16];
    bracket_products<16>(s, fb.L, fb.H, lo, hi);
    bracket_products<16>(h, fb.L, fb.H, lo2, hi2);
    r.c1 = make_uint2(even_of_adjacent(cvt_e2m1_f8(lo), cvt_e2m1_f8(hi)),
                      even_of_adjacent(cvt_e2m1_f8(lo + 8), cvt_e2m1_f8(hi + 8)));
    r.c2 = make_uint2(even_of_adjacent(cvt_e2m1_f8(lo2), cvt_e2m1_f8(hi2)),
                      even_of_adjacent(cvt_e2m1_f8(lo2 + 8), cvt_e2m1_f8(hi2 + 8)));
  }
  const V16 q1 = e2m1x16_to_bf16(r.c1);
  const V16 q2 = e2m1x16_to_bf16(r.c2);
  // D = 512 (s - q f), two elements per packed fma; the second fma scales
  // by 512 (exact) and adds 1.5 * 2^23, which leaves the integer D in the
  // low mantissa bits (as small_int)
  const float2 nf1 = make_float2(-fb.f, -fb.f), nf2 = make_float2(-2.0f * fb.f, -2.0f * fb.f);
  const float2 k512 = make_float2(512.0f, 512.0f), kmag = make_float2(12582912.0f, 12582912.0f);
  int acc = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const float2 sp = make_float2(s[2 * w], s[2 * w + 1]);
    const float2 t1 = ffma2(make_float2(bf_lo(q1.w[w]), bf_hi(q1.w[w])), nf1, sp);
    const float2 t2 = ffma2(make_float2(bf_lo(q2.w[w]), bf_hi(q2.w[w])), nf2, sp);
    const float2 u1 = ffma2(t1, k512, kmag), u2 = ffma2(t2, k512, kmag);
    const int a0 = __float_as_int(u1.x) - 0x4B400000, a1 = __float_as_int(u1.y) - 0x4B400000;
    const int b0 = __float_as_int(u2.x) - 0x4B400000, b1v = __float_as_int(u2.y) - 0x4B400000;
    acc += a0 * a0 - b0 * b0 + a1 * a1 - b1v * b1v;
  }
  r.delta = acc;
  return r;
}

}  // namespace mxk
