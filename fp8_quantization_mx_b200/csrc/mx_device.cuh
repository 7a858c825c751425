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
//    cvt.rn.satfinite.{e2m1x2,e4m3x2}.f32 (round to nearest even, saturate);
//  * with a macro factor f = (256 + k) / 256 the quotient x / (f 2^E) is not
//    exact, so s = |x| 2^-E (exact, below 16) is compared with the grid
//    midpoints times f (exact); equality goes to the even code;
//  * decoding (fake-quant, error, dequantize): a byte-permute table for E2M1
//    (integer only) and the hardware cvt.rn.f16x2.e4m3x2 for E4M3 (exact),
//    then an exact float product with the scale.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mxk {

constexpr int kFmtE2M1 = 0;
constexpr int kFmtE4M3 = 1;
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

// 2^-E for an E8M0 byte b = E + 127 in [0, 253]: always a normal float.
__device__ __forceinline__ float inv_scale_from_byte(int b) {
  return __uint_as_float(static_cast<uint32_t>(254 - b) << 23);
}

// 2^-E as a bf16x2 pair for b in [0, 253] (a normal bf16).
__device__ __forceinline__ uint32_t inv_scale_bf16x2(int b) {
  return static_cast<uint32_t>(254 - b) * 0x00800080u;
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
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
// 16 E4M3 bytes of a scaled slice: byte i = element i.
__device__ __forceinline__ uint4 enc_e4m3_16(const V16& s) {
  const uint2 a = cvt_e4m3x8(&s.w[0]);
  const uint2 b = cvt_e4m3x8(&s.w[4]);
  return make_uint4(a.x, a.y, b.x, b.y);
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

// E2M1 magnitudes 0 .5 1 1.5 2 3 4 6 as bf16 bit patterns, split into their
// high and low bytes, four entries per 32-bit word (index 0..3, 4..7).
constexpr uint32_t kE2m1Hi0 = 0x3F3F3F00u, kE2m1Hi1 = 0x40404040u;
constexpr uint32_t kE2m1Lo0 = 0xC0800000u, kE2m1Lo1 = 0xC0804000u;

// Four E2M1 codes (nibbles 0..3 of c) -> two words of bf16x2 bit patterns.
__device__ __forceinline__ uint2 e2m1x4_to_bf16(uint32_t c) {
  const uint32_t sel = c & 0x7777u;                        // magnitude indices
  const uint32_t hi = __byte_perm(kE2m1Hi0, kE2m1Hi1, sel);
  const uint32_t lo = __byte_perm(kE2m1Lo0, kE2m1Lo1, sel);
  uint32_t w0 = __byte_perm(lo, hi, 0x5140);               // elements 0, 1
  uint32_t w1 = __byte_perm(lo, hi, 0x7362);               // elements 2, 3
  w0 |= ((c << 12) & 0x8000u) | ((c << 24) & 0x80000000u);  // sign bits 3, 7
  w1 |= ((c << 4) & 0x8000u) | ((c << 16) & 0x80000000u);   // sign bits 11, 15
  return make_uint2(w0, w1);
}

// 16 E2M1 codes -> the 16 unscaled values as bf16 bit patterns.
__device__ __forceinline__ V16 e2m1x16_to_bf16(uint2 codes) {
  V16 r;
  const uint32_t c[2] = {codes.x, codes.y};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint2 a = e2m1x4_to_bf16(c[h] & 0xFFFFu);
    const uint2 b = e2m1x4_to_bf16(c[h] >> 16);
    r.w[4 * h + 0] = a.x;
    r.w[4 * h + 1] = a.y;
    r.w[4 * h + 2] = b.x;
    r.w[4 * h + 3] = b.y;
  }
  return r;
}

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

// -------------------------------------------------------- scale selection --

template <int FMT>
struct Elem;
template <>
struct Elem<kFmtE2M1> {
  static constexpr int emax = 2;          // 6 = 1.5 * 2^2
  static constexpr float maxv = 6.0f;
  static constexpr int ceil_m7 = 64;      // significand above 1.5 overflows 4m <= 6
};
template <>
struct Elem<kFmtE4M3> {
  static constexpr int emax = 8;          // 448 = 1.75 * 2^8
  static constexpr float maxv = 448.0f;
  static constexpr int ceil_m7 = 96;      // significand above 1.75 overflows 256m <= 448
};

// E8M0 byte of a finite block from its amax bits for the rules decided by the
// amax alone (FLOOR, CEIL, OAS_RULE); OAS starts from FLOOR. A subnormal or
// zero amax has exponent field 0 and always clamps to byte 0 (E = -127).
template <int FMT, int RULE>
__device__ __forceinline__ int rule_byte(uint32_t amax) {
  const int ex = static_cast<int>(amax >> 7);
  const int m7 = static_cast<int>(amax & 0x7F);
  int b = ex - Elem<FMT>::emax;
  if (RULE == kCeil) b += (m7 > Elem<FMT>::ceil_m7) ? 1 : 0;
  if (RULE == kOasRule) b += (m7 > 96) ? 1 : 0;
  return max(b, 0);
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
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float s = elem(s1, i);
    const float d1 = s - elem(q1, i);
    const float d2 = fmaf(-2.0f, elem(q2, i), s);
    acc = fmaf(d1 - d2, d1 + d2, acc);
  }
  r.delta = __float2int_rn(acc * 1024.0f);   // an integer below 2^16: exact
  return r;
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

// Grid midpoints of E2M1 times f = (256 + k) / 256, for rounding the scaled
// magnitude s = |x| 2^-E (which is below 16, so it never overflows). Each
// threshold mid * (256 + k) / 256 has at most 12 significant bits: exact.
struct Thresholds {
  float t[7];
};
__device__ __forceinline__ Thresholds mbs_thresholds(int k) {
  const float f = static_cast<float>(256 + k) * 0.00390625f;   // (256 + k) / 256
  Thresholds T;
  T.t[0] = 0.25f * f; T.t[1] = 0.75f * f; T.t[2] = 1.25f * f; T.t[3] = 1.75f * f;
  T.t[4] = 2.5f * f;  T.t[5] = 3.5f * f;  T.t[6] = 5.0f * f;
  return T;
}

// Magnitude code 0..7 of s = |x| 2^-E under the factor f. At a midpoint
// between an even and an odd code the even one wins: strictly above is needed
// to leave an even code, reaching the midpoint suffices to leave an odd one.
__device__ __forceinline__ int mbs_round(float s, const Thresholds& T) {
  return (s > T.t[0]) + (s >= T.t[1]) + (s > T.t[2]) + (s >= T.t[3]) + (s > T.t[4]) +
         (s >= T.t[5]) + (s > T.t[6]);
}

// E2M1 magnitude (in units of 0.5) of code c: 0 1 2 3 4 6 8 12.
__device__ __forceinline__ int e2m1_halves(int c) { return (0xC8643210u >> (4 * c)) & 0xF; }

// 16 codes under factor k and exponent byte b (b in [0, 253]).
__device__ __forceinline__ uint2 enc_mbs_16(const V16& x, int b, const Thresholds& T) {
  const float m = inv_scale_from_byte(b);   // 2^-E, exact
  uint32_t r[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t sign = (x.w[i >> 1] >> ((i & 1) ? 31 : 15)) & 1u;
    const uint32_t c = static_cast<uint32_t>(mbs_round(fabsf(elem(x, i)) * m, T)) | (sign << 3);
    r[i >> 3] |= c << (4 * (i & 7));
  }
  return make_uint2(r[0], r[1]);
}

// Exact OAS comparison of one lane's 16 elements under factor k: candidates
// E1 (byte b1) and E1 + 1. D = 512 s - h (256 + k) with s = |x| 2^-E1 and h
// the code magnitude in units of 0.5 (doubled for the coarser candidate): an
// integer below 2^12 for every element that does not round to zero under both.
__device__ __forceinline__ int oas_delta_mbs16(const V16& x, int b1, const Thresholds& T,
                                               int k) {
  const float inv1 = inv_scale_from_byte(b1);
  const float fk = static_cast<float>(256 + k);
  int acc = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float s = fabsf(elem(x, i)) * inv1;
    const int c1 = mbs_round(s, T);
    const int c2 = mbs_round(s * 0.5f, T);
    const float d1 = s * 512.0f - static_cast<float>(e2m1_halves(c1)) * fk;
    const float d2 = s * 512.0f - static_cast<float>(2 * e2m1_halves(c2)) * fk;
    const int i1 = __float2int_rn(d1), i2 = __float2int_rn(d2);
    acc += i1 * i1 - i2 * i2;
  }
  return acc;
}

}  // namespace mxk
