// Device building blocks of the MX block-32 kernels (sm_100a).
//
// Work decomposition shared by every kernel: the bf16 input is viewed as a
// flat array of 16-byte "chunks" of 8 elements. Because every row length is a
// multiple of 32 (of 128 with Macro Block Scaling), a 32-element MX block is
// exactly 4 consecutive chunks and a 128-element macro block 16, in the flat
// order, whatever the row length. A warp reads 32 consecutive chunks per step
// (512 contiguous bytes, one 16-byte load per lane), so lanes 4q..4q+3 hold
// block q of the step and lanes 16h..16h+15 hold macro block h.
//
// Numerics, per block (OCP Microscaling as restated by "[vLLM] MXFP8/MXFP4"
// (MX format table) and "Unveiling the Potential of Quantization with MXFP4"
// (2.A, 2.B)):
//  * amax is the largest |x| of the block, taken on the bf16 bit patterns with
//    the sign cleared (an integer compare orders finite values, then Inf, then
//    NaN, so a non-finite block is one whose amax bits reach 0x7F80);
//  * the E8M0 byte is computed from the amax exponent field and mantissa bits
//    with integer arithmetic only;
//  * x * 2^-E is an exact float product (E is a power of two and the product
//    never needs more than the 8 significant bits x already has), so the
//    hardware conversions cvt.rn.satfinite.{e2m1x2,e4m3x2}.f32 see the exact
//    scaled value and round it to nearest-even with saturation;
//  * with a macro factor f = (256 + k) / 256 the scaled value x / (f 2^E) is not
//    exact in float, so it is rounded by comparing 256 |x| 2^-E (exact) with
//    the grid midpoints times (256 + k) (exact); equality goes to the even code.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace mxk {

constexpr int kFmtE2M1 = 0;
constexpr int kFmtE4M3 = 1;
constexpr int kFloor = 0, kCeil = 1, kOasRule = 2, kOas = 3;
constexpr int kMbsNone = 0, kMbsStatic = 1, kMbsDynamic = 2;

constexpr uint16_t kNaNbf16 = 0x7FC0;
constexpr uint32_t kNaNf32 = 0x7FC00000u;

// ------------------------------------------------------------- memory ops --

// Streaming 16-byte load: read-only path, not kept in L1, 256-byte L2 prefetch.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ld_stream4(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

// Streaming (evict-first) stores of outputs nobody re-reads in this kernel.
__device__ __forceinline__ void st_stream4(void* p, uint32_t v) {
  asm volatile("st.global.cs.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_stream8(void* p, uint2 v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ void st_stream16(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// ------------------------------------------------------------ bf16 / bits --

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Largest |x| bit pattern among 8 bf16 values.
__device__ __forceinline__ uint32_t amax_bits8(const uint4& v) {
  const uint32_t m = max_u16x2(max_u16x2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                               max_u16x2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ uint32_t quad_max(uint32_t a) {
  a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
  a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
  return a;
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

// ------------------------------------------------------- element encoding --

// Eight scaled values -> eight E2M1 codes, element i in nibble i.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float a0, float a1, float a2, float a3, float a4,
                                               float a5, float a6, float a7) {
  uint32_t r;
  // cvt.rn.satfinite.e2m1x2.f32 d, hi, lo: the second operand lands in the
  // upper nibble, the third in the lower one.
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
  return r;
}

// Eight scaled values -> eight E4M3 bytes, element i in byte i.
__device__ __forceinline__ uint2 cvt_e4m3x8(float a0, float a1, float a2, float a3, float a4,
                                            float a5, float a6, float a7) {
  uint2 r;
  asm("{\n\t.reg .b16 h0, h1, h2, h3;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h0, %3, %2;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h1, %5, %4;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h2, %7, %6;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h3, %9, %8;\n\t"
      "mov.b32 %0, {h0, h1};\n\t"
      "mov.b32 %1, {h2, h3};\n\t}"
      : "=r"(r.x), "=r"(r.y)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
  return r;
}

// The 8 bf16 of a chunk, each multiplied by m (exact for a power of two m).
struct F8 {
  float v[8];
};
__device__ __forceinline__ F8 scaled8(const uint4& x, float m) {
  F8 r;
  r.v[0] = bf_lo(x.x) * m; r.v[1] = bf_hi(x.x) * m;
  r.v[2] = bf_lo(x.y) * m; r.v[3] = bf_hi(x.y) * m;
  r.v[4] = bf_lo(x.z) * m; r.v[5] = bf_hi(x.z) * m;
  r.v[6] = bf_lo(x.w) * m; r.v[7] = bf_hi(x.w) * m;
  return r;
}

__device__ __forceinline__ uint32_t enc_e2m1_8(const F8& s) {
  return cvt_e2m1x8(s.v[0], s.v[1], s.v[2], s.v[3], s.v[4], s.v[5], s.v[6], s.v[7]);
}
__device__ __forceinline__ uint2 enc_e4m3_8(const F8& s) {
  return cvt_e4m3x8(s.v[0], s.v[1], s.v[2], s.v[3], s.v[4], s.v[5], s.v[6], s.v[7]);
}

// Sign-only codes of a block holding NaN/Inf (E2M1: no NaN exists, so only the
// sign survives; E4M3: S.1111.111, the NaN code).
__device__ __forceinline__ uint32_t nonfinite_e2m1_8(const uint4& x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t r = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    r |= ((w[j] >> 15) & 1u) << (8 * j + 3);
    r |= ((w[j] >> 31) & 1u) << (8 * j + 7);
  }
  return r;
}
__device__ __forceinline__ uint2 nonfinite_e4m3_8(const uint4& x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    b[j] = (((w[j] >> 15) & 1u) << 7 | 0x7Fu) | ((((w[j] >> 31) & 1u) << 7 | 0x7Fu) << 8);
  return make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
}

// ------------------------------------------------------- element decoding --
//
// Decoding is done with integer operations only. (Feeding the register output
// of cvt.rn.satfinite.e2m1x2.f32 straight into cvt.rn.f16x2.e2m1x2 gave
// zeros on sm_100a in this build, while the same decode of codes loaded from
// memory was right; a table lookup avoids depending on that register path.)

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

// Eight E2M1 codes (nibble i = element i) -> eight bf16 values (unscaled).
__device__ __forceinline__ uint4 e2m1x8_to_bf16(uint32_t codes) {
  const uint2 a = e2m1x4_to_bf16(codes & 0xFFFFu);
  const uint2 b = e2m1x4_to_bf16(codes >> 16);
  return make_uint4(a.x, a.y, b.x, b.y);
}

// E2M1 codes -> unscaled values as floats (exact).
__device__ __forceinline__ F8 dec_e2m1_8(uint32_t codes) {
  const uint4 b = e2m1x8_to_bf16(codes);
  F8 r;
  r.v[0] = bf_lo(b.x); r.v[1] = bf_hi(b.x);
  r.v[2] = bf_lo(b.y); r.v[3] = bf_hi(b.y);
  r.v[4] = bf_lo(b.z); r.v[5] = bf_hi(b.z);
  r.v[6] = bf_lo(b.w); r.v[7] = bf_hi(b.w);
  return r;
}

// One E4M3fn byte -> float (S.1111.111 -> NaN; subnormals m * 2^-9).
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const uint32_t ef = (c >> 3) & 15u, m = c & 7u;
  float v = ef ? __uint_as_float(((ef + 120u) << 23) | (m << 20))
               : static_cast<float>(m) * 0.001953125f;        // m * 2^-9, exact
  if (ef == 15u && m == 7u) v = __uint_as_float(kNaNf32);
  return (c & 0x80u) ? -v : v;
}

__device__ __forceinline__ F8 dec_e4m3_8(uint2 codes) {
  F8 r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r.v[i] = e4m3_to_f32((codes.x >> (8 * i)) & 0xFFu);
    r.v[4 + i] = e4m3_to_f32((codes.y >> (8 * i)) & 0xFFu);
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

// Exact OAS comparison for one lane's 8 elements (E2M1, no macro factor):
// returns sum over the elements of (D1^2 - D2^2) with D = 512 * (s - q), s the
// value scaled by the finer candidate 2^-E1 and q its dequantized value in the
// same units under each candidate (E2 = E1 + 1). Elements that quantize to
// zero under both have D1 == D2 and cancel; every other D is an integer below
// 2^11, so the int32 sum over a block is exact.
__device__ __forceinline__ int oas_delta8(const uint4& x, float inv1) {
  const F8 s1 = scaled8(x, inv1);
  F8 s2;
#pragma unroll
  for (int i = 0; i < 8; ++i) s2.v[i] = s1.v[i] * 0.5f;
  const F8 q1 = dec_e2m1_8(enc_e2m1_8(s1));
  const F8 q2 = dec_e2m1_8(enc_e2m1_8(s2));
  int acc = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int d1 = __float2int_rn((s1.v[i] - q1.v[i]) * 512.0f);
    const int d2 = __float2int_rn((s1.v[i] - 2.0f * q2.v[i]) * 512.0f);
    acc += d1 * d1 - d2 * d2;
  }
  return acc;
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

// E8M0 byte of a sub-block under factor k (FLOOR): floor(log2(amax / f)) - 2,
// where dividing by f lowers the exponent by one exactly when the amax
// significand 1 + m7/128 is below f = 1 + k/256, i.e. 2 m7 < k.
__device__ __forceinline__ int mbs_floor_byte(uint32_t amax, int k) {
  const int ex = static_cast<int>(amax >> 7);
  if (ex == 0) return 0;
  const int m7 = static_cast<int>(amax & 0x7F);
  return max(ex - 2 - ((2 * m7 < k) ? 1 : 0), 0);
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

// Eight codes under factor k and exponent byte b (b in [0, 253]).
__device__ __forceinline__ uint32_t enc_mbs_8(const uint4& x, int b, const Thresholds& T) {
  const float m = inv_scale_from_byte(b);   // 2^-E, exact
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t r = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float tlo = fabsf(bf_lo(w[j])) * m;
    const float thi = fabsf(bf_hi(w[j])) * m;
    const uint32_t clo = static_cast<uint32_t>(mbs_round(tlo, T)) | (((w[j] >> 15) & 1u) << 3);
    const uint32_t chi = static_cast<uint32_t>(mbs_round(thi, T)) | (((w[j] >> 31) & 1u) << 3);
    r |= (clo | (chi << 4)) << (8 * j);
  }
  return r;
}

// Exact OAS comparison of one lane's 8 elements under factor k: candidates
// E1 (byte b1) and E1 + 1. D = 512 s - h (256 + k) with s = |x| 2^-E1 and h
// the code magnitude in units of 0.5 (doubled for the coarser candidate): an
// integer below 2^12 for every element that does not round to zero under both.
__device__ __forceinline__ int oas_delta_mbs8(const uint4& x, int b1, const Thresholds& T,
                                              int k) {
  const float inv1 = inv_scale_from_byte(b1);
  const float fk = static_cast<float>(256 + k);
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  int acc = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t word = w[j >> 1];
    const float s = fabsf((j & 1) ? bf_hi(word) : bf_lo(word)) * inv1;
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
