// MX block-32 quantization: the plain CPU oracle.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product library links, includes or
// calls this file; only the tests, the smoke check and the benchmark's CPU
// baseline load it. It shares no code, header, table or helper with the CUDA
// path under fp8_quantization_mx_b200/csrc.
//
// It is deliberately slow and scalar: every value is decoded from its field
// definition into a double, every rounding is an exhaustive nearest-grid search
// over the representable magnitudes, and every scale is found by the rule the
// sources state, written out with exact comparisons. Nothing here is blocked,
// fused or reordered beyond the definitions.
//
// Sources (titles of the pages this restates):
//  [AX]  "[Axolotl] MXFP4 quantization support" (PR #3375 analysis), section 2
//        "Quantization config": block_size must be 32; float4_e2m1fn_x2 packs
//        two E2M1 codes (2-bit exponent, 1-bit mantissa) per byte. Section 3:
//        activations and weights go through the same fake-quantizer.
//  [VL]  "[vLLM] MXFP8/MXFP4: microscaling format quantization": "MXFP8: block-32
//        scaling" (block 32, uint8 scale per block, contiguous rows), "MXFP4:
//        4-bit MoE" (uint8 storage, two FP4 values per byte, last dim halved),
//        and the MX format table (E2M1 / E4M3 elements, E8M0 scale, block 32).
//  [UP]  "Unveiling the Potential of Quantization with MXFP4: Strategies for
//        Quantization Error Reduction": technical summary section 1 (E8M0 holds
//        powers of two 2^k only), section 2.A Overflow-Aware Scaling (FP4 max
//        6.0; a block max at 3.0-3.5 under the no-overflow scale may instead be
//        mapped to 6.0-7.0, decided from mantissa bits), section 2.B Macro Block
//        Scaling (a 1x128 macro block with an 8-bit-mantissa factor; Static =
//        cheap approximation, Dynamic = LUT search for minimum SSE), sections 3-4
//        (QSNR as the error figure).
//  [BQ]  "BATQuant: Outlier-resilient MXFP4 Quantization via Learnable
//        Block-wise Optimization", technical summary section 2 (methodology):
//        (a) a block-diagonal affine transform whose blocks match the MX block
//        (32 elements), (b) each block's matrix the Kronecker product of a
//        block-private matrix B_j and a globally shared matrix A (GPK),
//        (c) block-wise learnable clipping thresholds beta^min, beta^max.
//  The scale rule 2^(floor(log2 amax) - emax) and round-to-nearest-even with
//  saturation are the OCP Microscaling definition that [AX] and [VL] point to.
//
// Readings where the pages are silent (each is listed with its reason in the
// design notes): zero block -> scale byte 0; a block holding NaN/Inf -> scale
// byte 0xFF and element codes that carry only the sign; the E8M0 exponent is
// clamped to [-127, 127]; even element index -> low nibble; OAS candidates are
// {FLOOR, FLOOR+1}, tie -> FLOOR; MBS factor f = 1 + k/256 with k in [0, 255];
// a macro block holding NaN/Inf uses k = 0; the straight-through mask is
// |x| <= maxv * X (inclusive) with X the block's effective scale.
//
// Parity pins: every function here is checked by tests that do not re-type its
// formula (library decoders from ml_dtypes/torch, exact rational brute force,
// hand-worked blocks, and invariants). MBS has no numeric example on the pages,
// so its readings are pinned by invariants and brute force only.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

constexpr int kFmtE2M1 = 0;
constexpr int kFmtE4M3 = 1;
constexpr int kFmtE5M2 = 2;
constexpr int kFmtE3M2 = 3;
constexpr int kFmtE2M3 = 4;
constexpr int kFmtInt8 = 5;
// The comparison formats of [UP] section 1's gap analysis: E2M1 elements in
// 16-element blocks, with an E8M0 scale (MXFP4 at block 16) or an E4M3 scale
// (NVFP4).
constexpr int kFmtE2M1B16 = 6;
constexpr int kFmtNvfp4 = 7;

constexpr int kScaleFloor = 0;
constexpr int kScaleCeil = 1;
constexpr int kScaleOasRule = 2;
constexpr int kScaleOas = 3;
constexpr int kMbsStatic = 1;   // value of (scaling >> 4)
constexpr int kMbsDynamic = 2;

constexpr int kBlock = 32;       // [AX] section 2, [VL] MXFP8
constexpr int kMacro = 128;      // [UP] section 2.B: 1x128 macro block

int g_threads = 1;

// ---------------------------------------------------------------- formats --

// bf16: 1 sign, 8 exponent (bias 127), 7 mantissa bits.
double decode_bf16(uint16_t b) {
  const int sign = b >> 15;
  const int ef = (b >> 7) & 0xFF;
  const int mf = b & 0x7F;
  double v;
  if (ef == 0xFF) {
    v = mf ? std::numeric_limits<double>::quiet_NaN()
           : std::numeric_limits<double>::infinity();
  } else if (ef == 0) {
    v = std::ldexp(static_cast<double>(mf), -126 - 7);
  } else {
    v = std::ldexp(1.0 + mf / 128.0, ef - 127);
  }
  return sign ? -v : v;
}

// Round a double to the nearest bf16 (ties to even significand), overflow to
// infinity. NaN becomes the canonical quiet NaN 0x7FC0.
uint16_t encode_bf16_rne(double v) {
  if (std::isnan(v)) return 0x7FC0;
  const uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  const double a = std::fabs(v);
  if (std::isinf(a)) return sign | 0x7F80;
  if (a == 0.0) return sign;
  int e2;
  std::frexp(a, &e2);              // a = m * 2^e2, m in [0.5, 1)
  int e = e2 - 1;                  // floor(log2 a)
  if (e < -126) e = -126;          // subnormal range shares the 2^-126 quantum scale
  const double quantum = std::ldexp(1.0, e - 7);
  double r = a / quantum;          // exact: a power-of-two division
  double fl = std::floor(r);
  double frac = r - fl;
  double q;
  if (frac > 0.5) q = fl + 1;
  else if (frac < 0.5) q = fl;
  else q = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1;
  const double rounded = q * quantum;
  if (rounded == 0.0) return sign;             // below half the smallest subnormal
  if (rounded >= std::ldexp(1.0, 128)) return sign | 0x7F80;
  // Encode the exactly representable value by its fields.
  int re2;
  std::frexp(rounded, &re2);
  int re = re2 - 1;
  uint16_t bits;
  if (re < -126) {
    bits = static_cast<uint16_t>(rounded / std::ldexp(1.0, -133));
  } else {
    const double mant = rounded / std::ldexp(1.0, re) - 1.0;   // in [0, 1)
    bits = static_cast<uint16_t>(((re + 127) << 7) | static_cast<int>(mant * 128.0));
  }
  return sign | bits;
}

// E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa; no Inf/NaN ([AX] section 2,
// [VL] table, [UP] 2.A: max 6.0).
double decode_e2m1(int code) {
  const int sign = (code >> 3) & 1;
  const int ef = (code >> 1) & 3;
  const int mf = code & 1;
  const double v = ef == 0 ? 0.5 * mf : std::ldexp(1.0 + mf / 2.0, ef - 1);
  return sign ? -v : v;
}

// E4M3 "fn": 1 sign, 4 exponent (bias 7), 3 mantissa; no Inf; S.1111.111 is
// NaN ([VL] table, MXFP8 elements).
double decode_e4m3(int code) {
  const int sign = (code >> 7) & 1;
  const int ef = (code >> 3) & 15;
  const int mf = code & 7;
  double v;
  if (ef == 15 && mf == 7) v = std::numeric_limits<double>::quiet_NaN();
  else if (ef == 0) v = std::ldexp(mf / 8.0, -6);
  else v = std::ldexp(1.0 + mf / 8.0, ef - 7);
  return sign ? -v : v;
}

// E5M2: 1 sign, 5 exponent (bias 15), 2 mantissa, IEEE-style: exponent 31
// is Inf (mantissa 0) or NaN ([VL] MX table, MXFP8 elements E4M3/E5M2).
double decode_e5m2(int code) {
  const int sign = (code >> 7) & 1;
  const int ef = (code >> 2) & 31;
  const int mf = code & 3;
  double v;
  if (ef == 31) v = mf ? std::numeric_limits<double>::quiet_NaN() : std::numeric_limits<double>::infinity();
  else if (ef == 0) v = std::ldexp(mf / 4.0, -14);
  else v = std::ldexp(1.0 + mf / 4.0, ef - 15);
  return sign ? -v : v;
}

// FP6 elements of MXFP6 ([VL] MX table: E3M2 / E2M3), no Inf/NaN: 1 sign bit
// (bit 5), then the exponent and mantissa fields.
// E3M2: 3 exponent (bias 3), 2 mantissa.
double decode_e3m2(int code) {
  const int sign = (code >> 5) & 1;
  const int ef = (code >> 2) & 7;
  const int mf = code & 3;
  const double v = ef == 0 ? std::ldexp(mf / 4.0, -2) : std::ldexp(1.0 + mf / 4.0, ef - 3);
  return sign ? -v : v;
}
// E2M3: 2 exponent (bias 1), 3 mantissa.
double decode_e2m3(int code) {
  const int sign = (code >> 5) & 1;
  const int ef = (code >> 3) & 3;
  const int mf = code & 7;
  const double v = ef == 0 ? mf / 8.0 : std::ldexp(1.0 + mf / 8.0, ef - 1);
  return sign ? -v : v;
}

// MXINT8 elements ([VL] MX table: INT8): an 8-bit two's complement integer i
// read as i * 2^-6, so that the largest power of two it holds is 2^0 as for
// the float elements; magnitudes up to 127/64 (the code -128 is never
// produced: saturation is symmetric).
double decode_int8(int code) {
  const int i = code >= 128 ? code - 256 : code;
  return std::ldexp(static_cast<double>(i), -6);
}

// E8M0: an unsigned biased exponent, the value 2^(b-127); 0xFF is NaN
// ([VL] table; [UP] section 1: scale factors are powers of two only).
double decode_e8m0(int b) {
  if (b == 0xFF) return std::numeric_limits<double>::quiet_NaN();
  return std::ldexp(1.0, b - 127);
}

double element_value(int code, int fmt) {
  switch (fmt) {
    case kFmtE2M1: return decode_e2m1(code);
    case kFmtE4M3: return decode_e4m3(code);
    case kFmtE5M2: return decode_e5m2(code);
    case kFmtE3M2: return decode_e3m2(code);
    case kFmtE2M3: return decode_e2m3(code);
    default: return decode_int8(code);
  }
}

// Non-negative magnitudes are the codes 0 .. n-1 in increasing order (E4M3
// stops before its NaN, E5M2 before Inf).
int num_magnitude_codes(int fmt) {
  switch (fmt) {
    case kFmtE2M1: return 8;
    case kFmtE4M3: return 127;
    case kFmtE5M2: return 124;
    case kFmtE3M2:
    case kFmtE2M3: return 32;
    default: return 128;
  }
}
int sign_bit(int fmt) {
  switch (fmt) {
    case kFmtE2M1: return 0x8;
    case kFmtE3M2:
    case kFmtE2M3: return 0x20;
    default: return 0x80;
  }
}
// Code of the magnitude index c with the sign of v (INT8: two's complement,
// which has no negative zero).
int signed_code(int c, bool negative, int fmt) {
  if (fmt == kFmtInt8) return negative ? ((256 - c) & 0xFF) : c;
  return negative ? (c | sign_bit(fmt)) : c;
}
double magnitude(int fmt, int c) { return element_value(c, fmt); }

// The element format, block size and code packing of an API format.
int elem_fmt(int fmt) { return (fmt == kFmtE2M1B16 || fmt == kFmtNvfp4) ? kFmtE2M1 : fmt; }
int block_size(int fmt) { return (fmt == kFmtE2M1B16 || fmt == kFmtNvfp4) ? 16 : kBlock; }
bool packed_fp4(int fmt) { return elem_fmt(fmt) == kFmtE2M1; }
double max_value(int fmt) { return magnitude(fmt, num_magnitude_codes(fmt) - 1); }
// The smallest nonzero magnitude.
double min_magnitude(int fmt) { return magnitude(fmt, 1); }

// floor(log2 a) for finite a > 0.
int floor_log2(double a) {
  int e2;
  std::frexp(a, &e2);
  return e2 - 1;
}
int emax_elem(int fmt) { return floor_log2(max_value(fmt)); }   // 2 (E2M1), 8 (E4M3)

int clamp_exp(int E) { return std::min(127, std::max(-127, E)); }

// Nearest representable element to v / X, X = the block's effective scale,
// found by scanning every finite magnitude. Ties go to the even code (the one
// whose mantissa LSB is 0). Values past the largest magnitude land on it
// (saturation). The sign of v is kept, so small negatives give -0.
//
// Saturation is decided first: past the largest grid value every distance is
// almost the same large number, and for a value far past it the distances
// agree to the last bit of a double, so the scan could not tell them apart.
// Below it, the two grid values around |v| are within a factor of two of it
// (or one of them is zero), so their distances are exact and ties are seen.
int round_element(double v, double X, int fmt) {
  const double a = std::fabs(v);
  const int top = num_magnitude_codes(fmt) - 1;
  if (a >= X * magnitude(fmt, top)) return signed_code(top, std::signbit(v), fmt);
  int best = 0;
  double best_d = std::fabs(a - X * magnitude(fmt, 0));
  for (int c = 1; c < num_magnitude_codes(fmt); ++c) {
    const double d = std::fabs(a - X * magnitude(fmt, c));
    if (d < best_d || (d == best_d && (c % 2 == 0))) {
      best = c;
      best_d = d;
    }
  }
  return signed_code(best, std::signbit(v), fmt);
}

bool block_has_nonfinite(const double* x, int n) {
  for (int i = 0; i < n; ++i)
    if (!std::isfinite(x[i])) return true;
  return false;
}

double block_amax(const double* x, int n) {
  double m = 0.0;
  for (int i = 0; i < n; ++i) m = std::max(m, std::fabs(x[i]));
  return m;
}

// The integer e' with f * 2^e' <= a < f * 2^(e'+1), i.e. floor(log2(a / f)),
// found with exact comparisons (f * 2^e is exact in double).
int floor_log2_over(double a, double f) {
  int e = floor_log2(a);
  while (f * std::ldexp(1.0, e) > a) --e;
  while (f * std::ldexp(1.0, e + 1) <= a) ++e;
  return e;
}

// Exact comparison of the two candidate SSEs of an OAS decision: the real
// sums compared, not their rounded values. Elements whose dequantized value
// is the same under both scales add the same term to both sums and drop out.
// Every remaining element has |x| of at least half the smallest nonzero
// magnitude times X1, so x (8 significant bits), y1 and y2 are all integer
// multiples of U = min_magnitude * 2^(E1 - 9), where 2^E1 is the power of
// two in X1 = f * 2^E1 (y carries f = F / 256 with F an integer). Each
// difference is then an exact integer D below 2^44 units, and the sum of
// D1^2 - D2^2 is accumulated exactly in 128-bit integers. Returns true when
// the coarser scale X2 has the strictly smaller SSE.
bool coarser_scale_wins(const double* x, int n, double X1, double X2, int fmt) {
  const double U = std::ldexp(min_magnitude(fmt), floor_log2(X1) - 9);
  __int128 delta = 0;   // (SSE(X1) - SSE(X2)) / U^2 over the differing elements
  for (int i = 0; i < n; ++i) {
    const double y1 = element_value(round_element(x[i], X1, fmt), fmt) * X1;
    const double y2 = element_value(round_element(x[i], X2, fmt), fmt) * X2;
    if (y1 == y2) continue;
    const auto D1 = static_cast<int64_t>((x[i] - y1) / U);   // exact integers
    const auto D2 = static_cast<int64_t>((x[i] - y2) / U);
    delta += static_cast<__int128>(D1) * D1 - static_cast<__int128>(D2) * D2;
  }
  return delta > 0;
}

// Scale exponent of one finite 32-element block for the base rules, with the
// block's values already divided by nothing (f = 1) or by the macro factor f
// (MBS). Returns the clamped E; amax == 0 gives -127.
int block_exponent(const double* x, int n, int fmt, int rule, double f) {
  const double amax = block_amax(x, n);
  if (amax == 0.0) return -127;
  const int emax = emax_elem(fmt);
  const double maxv = max_value(fmt);
  const int e = floor_log2_over(amax, f);        // floor(log2(amax / f))
  switch (rule) {
    case kScaleFloor:
      // OCP rule: 2^(floor(log2 amax) - emax); amax may exceed maxv * X and
      // then saturates.
      return clamp_exp(e - emax);
    case kScaleCeil: {
      // [UP] 2.A, the "existing" no-overflow scale: the smallest power of two
      // X with amax <= maxv * X.
      int E = e - emax - 1;
      while (amax > maxv * f * std::ldexp(1.0, E)) ++E;
      return clamp_exp(E);
    }
    case kScaleOasRule: {
      // [UP] 2.A: take the no-overflow scale; if the block max then sits in
      // 3.0-3.5 (of the 6.0 range), halve the scale so it maps to 6.0-7.0 and
      // lets the largest values clamp.
      int Ec = e - emax - 1;
      while (amax > maxv * f * std::ldexp(1.0, Ec)) ++Ec;
      // normalized max = amax / (f 2^Ec), compared exactly against 3.0 / 3.5
      const double Xc = f * std::ldexp(1.0, Ec);
      const bool in_band = amax > 3.0 * Xc && amax <= 3.5 * Xc;
      return clamp_exp(in_band ? Ec - 1 : Ec);
    }
    case kScaleOas: {
      // Per-block choice by minimum block squared error between the
      // overflow-allowing OCP exponent and the next coarser one; a tie keeps
      // the finer one.
      const int E1 = clamp_exp(e - emax);
      const int E2 = clamp_exp(e - emax + 1);
      if (E1 == E2) return E1;
      const double X1 = f * std::ldexp(1.0, E1);
      const double X2 = f * std::ldexp(1.0, E2);
      return coarser_scale_wins(x, n, X1, X2, fmt) ? E2 : E1;
    }
  }
  return clamp_exp(e - emax);
}

// Macro factor f = 1 + k/256: "a high-precision scale with an 8-bit mantissa"
// ([UP] 2.B); its exponent is absorbed by the sub-block E8M0 bytes.
double macro_factor(int k) { return 1.0 + k / 256.0; }

// MBS-Static: the smallest factor that maps the macro-block maximum A to at
// most maxv: with p the integer where maxv*2^p <= A < maxv*2^(p+1), the
// smallest k with maxv * f * 2^p >= A; if only k = 256 would do, k = 0.
int mbs_static_k(const double* x, int n, int fmt) {
  const double A = block_amax(x, n);
  if (A == 0.0) return 0;
  const double maxv = max_value(fmt);
  int p = floor_log2(A) - emax_elem(fmt) - 1;
  while (maxv * std::ldexp(1.0, p + 1) <= A) ++p;
  for (int k = 0; k < 256; ++k)
    if (maxv * macro_factor(k) * std::ldexp(1.0, p) >= A) return k;
  return 0;
}

struct BlockResult {
  int scale_byte;
  double X;            // effective scale f * 2^E, or the NVFP4 scale (NaN for a non-finite block)
  int codes[kBlock];
};

// NVFP4 block ([UP] section 1: E4M3 scale factors with mantissa bits, block
// 16): the scale is amax / 6 rounded to the nearest E4M3 value (ties to
// even, saturating at 448) and the elements are x / s rounded onto the E2M1
// grid. amax / 6 is exact in double wherever it sits on an E4M3 midpoint and
// at least 2^-12 (relatively) away from every midpoint otherwise, so its one
// double rounding cannot move the E4M3 choice. A scale of 0 (amax below
// 2^-10 * 6 / 2) leaves only the signs.
BlockResult quantize_block_nvfp4(const double* x) {
  BlockResult r{};
  const int n = 16;
  if (block_has_nonfinite(x, n)) {
    r.scale_byte = 0x7F;   // the E4M3 NaN
    r.X = std::numeric_limits<double>::quiet_NaN();
    for (int i = 0; i < n; ++i) r.codes[i] = std::signbit(x[i]) ? sign_bit(kFmtE2M1) : 0;
    return r;
  }
  r.scale_byte = round_element(block_amax(x, n) / 6.0, 1.0, kFmtE4M3);
  r.X = decode_e4m3(r.scale_byte);
  for (int i = 0; i < n; ++i) {
    if (r.X == 0.0) r.codes[i] = std::signbit(x[i]) ? sign_bit(kFmtE2M1) : 0;
    else r.codes[i] = round_element(x[i], r.X, kFmtE2M1);
  }
  return r;
}

// Quantize one block (32 elements, 16 for the block-16 formats) with base
// rule `rule` under macro factor f.
BlockResult quantize_block(const double* x, int api_fmt, int rule, double f) {
  if (api_fmt == kFmtNvfp4) return quantize_block_nvfp4(x);
  const int fmt = elem_fmt(api_fmt);
  const int n = block_size(api_fmt);
  BlockResult r{};
  if (block_has_nonfinite(x, n)) {
    r.scale_byte = 0xFF;
    r.X = std::numeric_limits<double>::quiet_NaN();
    for (int i = 0; i < n; ++i) {
      const int s = std::signbit(x[i]) ? sign_bit(fmt) : 0;
      // The FP8 elements of a NaN-scale block are NaN (E4M3 S.1111.111, E5M2
      // S.11111.11); E2M1 and FP6 have no NaN, so only the sign is kept;
      // INT8 has neither NaN nor -0: 0.
      if (fmt == kFmtE4M3 || fmt == kFmtE5M2) r.codes[i] = s | 0x7F;
      else if (fmt == kFmtInt8) r.codes[i] = 0;
      else r.codes[i] = s;
    }
    return r;
  }
  const int E = block_exponent(x, n, fmt, rule, f);
  r.scale_byte = E + 127;
  r.X = f * std::ldexp(1.0, E);
  for (int i = 0; i < n; ++i) r.codes[i] = round_element(x[i], r.X, fmt);
  return r;
}

// Sum of squared errors of a 128-element macro block quantized with factor k,
// accumulated in double in element order 0..127 (each d and d*d is exact; the
// running sum rounds in this fixed order).
double macro_sse(const double* x, int fmt, int rule, int k) {
  const double f = macro_factor(k);
  const int bs = block_size(fmt);   // 32, or 16 for MXFP4 at block 16
  double sse = 0.0;
  for (int b = 0; b < kMacro / bs; ++b) {
    const BlockResult r = quantize_block(x + b * bs, fmt, rule, f);
    for (int i = 0; i < bs; ++i) {
      const double y = element_value(r.codes[i], elem_fmt(fmt)) * r.X;
      const double d = x[b * bs + i] - y;
      sse = sse + d * d;
    }
  }
  return sse;
}

// MBS-Dynamic: every k in the 256-entry factor table; the smallest SSE wins,
// and a tie keeps the smaller k ([UP] 2.B: LUT search for minimum SSE).
int mbs_dynamic_k(const double* x, int fmt, int rule) {
  int best_k = 0;
  double best = macro_sse(x, fmt, rule, 0);
  for (int k = 1; k < 256; ++k) {
    const double s = macro_sse(x, fmt, rule, k);
    if (s < best) {
      best = s;
      best_k = k;
    }
  }
  return best_k;
}

// Pick the macro factor for a 128-element macro block (k = 0 without MBS, or
// when the macro block holds a NaN/Inf).
int macro_k(const double* x, int fmt, int rule, int mbs) {
  if (mbs == 0) return 0;
  if (block_has_nonfinite(x, kMacro)) return 0;
  return mbs == kMbsStatic ? mbs_static_k(x, kMacro, elem_fmt(fmt)) : mbs_dynamic_k(x, fmt, rule);
}

// Decoded row of bf16 values.
void decode_row(const uint16_t* src, int64_t cols, double* dst) {
  for (int64_t c = 0; c < cols; ++c) dst[c] = decode_bf16(src[c]);
}

// Run f(row_begin, row_end) over [0, rows) split across g_threads threads.
template <typename F>
void parallel_rows(int64_t rows, F f) {
  const int nt = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(g_threads, rows)));
  if (nt == 1) {
    f(int64_t(0), rows);
    return;
  }
  std::vector<std::thread> pool;
  const int64_t per = (rows + nt - 1) / nt;
  for (int t = 0; t < nt; ++t) {
    const int64_t b = t * per, e = std::min(rows, b + per);
    if (b >= e) break;
    pool.emplace_back([=] { f(b, e); });
  }
  for (auto& th : pool) th.join();
}

struct RowQuant {
  std::vector<int> codes;        // [cols]
  std::vector<int> scale_bytes;  // [cols / 32]
  std::vector<int> ks;           // [cols / 128] (MBS only)
  std::vector<double> X;         // [cols / 32]
};

// Quantize a decoded row: macro factors first (MBS), then each 32-block.
RowQuant quantize_row(const double* x, int64_t cols, int fmt, int scaling) {
  const int rule = scaling & 0xF;
  const int mbs = scaling >> 4;
  const int bs = block_size(fmt);
  RowQuant q;
  q.codes.resize(cols);
  q.scale_bytes.resize(cols / bs);
  q.X.resize(cols / bs);
  if (mbs) q.ks.resize(cols / kMacro);
  for (int64_t b = 0; b < cols / bs; ++b) {
    double f = 1.0;
    if (mbs) {
      const int64_t m = b / (kMacro / bs);
      if (b % (kMacro / bs) == 0) q.ks[m] = macro_k(x + m * kMacro, fmt, rule, mbs);
      f = macro_factor(q.ks[m]);
    }
    const BlockResult r = quantize_block(x + b * bs, fmt, rule, f);
    q.scale_bytes[b] = r.scale_byte;
    q.X[b] = r.X;
    for (int i = 0; i < bs; ++i) q.codes[b * bs + i] = r.codes[i];
  }
  return q;
}

// Dequantized value of one element as an exact double (NaN for a NaN scale or
// a NaN element).
double dequant_value(int code, int scale_byte, int k, int fmt) {
  // NVFP4: the scale byte is an E4M3 value (NaN for S.1111.111)
  if (fmt == kFmtNvfp4) return element_value(code, kFmtE2M1) * decode_e4m3(scale_byte);
  if (scale_byte == 0xFF) return std::numeric_limits<double>::quiet_NaN();
  return element_value(code, elem_fmt(fmt)) * macro_factor(k) * decode_e8m0(scale_byte);
}

// ------------------------------------------------------------- BATQuant --
//
// [BQ] section 2: the activation row x is multiplied on the right by the
// block-diagonal matrix diag(P_0, P_1, ...), one 32x32 block P_j per MX
// block j of the row, with P_j = B_j (x) A: A is a x a and shared by every
// block, B_j is b x b and private to column block j, a * b = 32. Indexing
// the block's 32 elements as i = p * a + q (p < b, q < a), the Kronecker
// entry is P_j[p*a+q][r*a+s] = B_j[p][r] * A[q][s], so
//   y[r*a+s] = sum_p B_j[p][r] * Z[p][s],  Z[p][s] = sum_q x[p*a+q] * A[q][s]
// (the two small products the decomposition exists for). The block's values
// are then clipped to [beta^min_j * min(y), beta^max_j * max(y)] and the
// result, rounded to bf16, is what the MX quantizer sees.
//
// Readings (the pages fix neither precision nor order): fp32 arithmetic,
// each sum an fma chain in ascending index order starting from -0 (so a
// one-term sum is the rounded product), except that a sum whose index runs
// over both 16-element halves of the block is the fp32 sum of the chains of
// the two halves (lower half + upper half). That is the stage-2 sum for
// b >= 2 and the stage-1 sum for a = 32. The clip is t = y < lo ? lo : y,
// then t > hi ? hi : t, with lo = fl(beta^min * min y), hi = fl(beta^max *
// max y); a block whose transformed values are not all finite is not
// clipped (its scale is the NaN byte either way). No thresholds given: no
// clipping.

float fma_chain(const float* u, int su, const float* v, int sv, int n) {
  float acc = -0.0f;
  for (int t = 0; t < n; ++t) acc = std::fmaf(u[t * su], v[t * sv], acc);
  return acc;
}

void bat_block(const float* x, int a, const float* A, const float* Bj, const float* beta_min,
               const float* beta_max, float* y) {
  const int b = kBlock / a;
  float Z[kBlock];   // Z[p * a + s]
  for (int p = 0; p < b; ++p)
    for (int s = 0; s < a; ++s) {
      if (a == kBlock) {
        Z[s] = fma_chain(x, 1, A + s, a, 16) + fma_chain(x + 16, 1, A + 16 * a + s, a, 16);
      } else {
        Z[p * a + s] = fma_chain(x + p * a, 1, A + s, a, a);
      }
    }
  for (int r = 0; r < b; ++r)
    for (int s = 0; s < a; ++s) {
      const int h = b / 2;
      if (b == 1) {
        y[s] = fma_chain(Bj, 1, Z + s, a, 1);
      } else {
        y[r * a + s] = fma_chain(Bj + r, b, Z + s, a, h) +
                       fma_chain(Bj + h * b + r, b, Z + h * a + s, a, h);
      }
    }
  if (!beta_min) return;
  float mn = y[0], mx = y[0];
  for (int i = 0; i < kBlock; ++i) {
    if (!std::isfinite(y[i])) return;
    if (y[i] < mn) mn = y[i];
    if (y[i] > mx) mx = y[i];
  }
  const float lo = *beta_min * mn, hi = *beta_max * mx;
  for (int i = 0; i < kBlock; ++i) {
    const float t = y[i] < lo ? lo : y[i];
    y[i] = t > hi ? hi : t;
  }
}

uint32_t float_bits(float v) {
  uint32_t u;
  std::memcpy(&u, &v, 4);
  return u;
}

// Canonical NaN outputs of the dequantizing functions.
constexpr uint16_t kNaNbf16 = 0x7FC0;
constexpr uint32_t kNaNf32 = 0x7FC00000u;

}  // namespace

extern "C" {

void oracle_set_threads(int n) { g_threads = n < 1 ? 1 : n; }
int oracle_get_threads(void) { return g_threads; }

double oracle_decode_bf16(uint16_t b) { return decode_bf16(b); }
uint16_t oracle_encode_bf16_rne(double v) { return encode_bf16_rne(v); }
double oracle_decode_e2m1(int code) { return decode_e2m1(code); }
double oracle_decode_e4m3(int code) { return decode_e4m3(code); }
double oracle_decode_e8m0(int b) { return decode_e8m0(b); }
double oracle_decode_element(int code, int fmt) { return element_value(code, fmt); }
int oracle_round_element(double v, double X, int fmt) { return round_element(v, X, fmt); }

// round_element over an array (one X for all), for exhaustive checks.
void oracle_round_array(const double* v, int64_t n, double X, int fmt, int32_t* codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = round_element(v[i], X, fmt);
}

// Scale byte of one 32-element bf16 block for a base rule, factor f = 1 + k/256.
int oracle_block_scale(const uint16_t* x32, int fmt, int rule, int k) {
  double x[kBlock];
  decode_row(x32, kBlock, x);
  return quantize_block(x, fmt, rule, macro_factor(k)).scale_byte;
}

// Macro factor byte k of one 128-element bf16 macro block.
int oracle_macro_k(const uint16_t* x128, int fmt, int scaling) {
  double x[kMacro];
  decode_row(x128, kMacro, x);
  return macro_k(x, fmt, scaling & 0xF, scaling >> 4);
}

// Codes (FP4: two per byte, even element in the low nibble; FP8, FP6 and
// INT8: one per byte, FP6 in the low 6 bits), E8M0 scale bytes
// [rows, cols/32], and MBS factor bytes [rows, cols/128].
void oracle_quantize(const uint16_t* x, int64_t rows, int64_t cols, int fmt, int scaling,
                     uint8_t* codes, uint8_t* scales, uint8_t* macro) {
  parallel_rows(rows, [&](int64_t r0, int64_t r1) {
    std::vector<double> row(cols);
    for (int64_t r = r0; r < r1; ++r) {
      decode_row(x + r * cols, cols, row.data());
      const RowQuant q = quantize_row(row.data(), cols, fmt, scaling);
      const int64_t nb = cols / block_size(fmt);
      for (int64_t b = 0; b < nb; ++b) scales[r * nb + b] = static_cast<uint8_t>(q.scale_bytes[b]);
      if (macro && (scaling >> 4))
        for (int64_t m = 0; m < cols / kMacro; ++m)
          macro[r * (cols / kMacro) + m] = static_cast<uint8_t>(q.ks[m]);
      if (packed_fp4(fmt)) {
        for (int64_t c = 0; c < cols; c += 2)
          codes[r * (cols / 2) + c / 2] =
              static_cast<uint8_t>(q.codes[c] | (q.codes[c + 1] << 4));
      } else {
        for (int64_t c = 0; c < cols; ++c) codes[r * cols + c] = static_cast<uint8_t>(q.codes[c]);
      }
    }
  });
}

// ŷ = value(code) * f * 2^(scale-127), written as bf16 (one round to nearest
// even) or as float (exact); canonical NaN for NaN scales/elements.
void oracle_dequantize(const uint8_t* codes, const uint8_t* scales, const uint8_t* macro,
                       int64_t rows, int64_t cols, int fmt, int out_fp32, void* out) {
  parallel_rows(rows, [&](int64_t r0, int64_t r1) {
    for (int64_t r = r0; r < r1; ++r) {
      for (int64_t c = 0; c < cols; ++c) {
        int code;
        if (packed_fp4(fmt)) {
          const uint8_t byte = codes[r * (cols / 2) + c / 2];
          code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        } else {
          code = codes[r * cols + c];
        }
        const int bs = block_size(fmt);
        const int sb = scales[r * (cols / bs) + c / bs];
        const int k = macro ? macro[r * (cols / kMacro) + c / kMacro] : 0;
        const double v = dequant_value(code, sb, k, fmt);
        if (out_fp32) {
          const uint32_t bits = std::isnan(v) ? kNaNf32 : float_bits(static_cast<float>(v));
          static_cast<uint32_t*>(out)[r * cols + c] = bits;
        } else {
          static_cast<uint16_t*>(out)[r * cols + c] = std::isnan(v) ? kNaNbf16 : encode_bf16_rne(v);
        }
      }
    }
  });
}

// QAT forward ([AX] sections 2-3): quantize then dequantize, bf16 out.
void oracle_fake_quant_fwd(const uint16_t* x, int64_t rows, int64_t cols, int fmt, int scaling,
                           uint16_t* y, uint8_t* scales_out) {
  parallel_rows(rows, [&](int64_t r0, int64_t r1) {
    std::vector<double> row(cols);
    for (int64_t r = r0; r < r1; ++r) {
      decode_row(x + r * cols, cols, row.data());
      const RowQuant q = quantize_row(row.data(), cols, fmt, scaling);
      const int bs = block_size(fmt);
      for (int64_t c = 0; c < cols; ++c) {
        const int64_t b = c / bs;
        const int k = (scaling >> 4) ? q.ks[c / kMacro] : 0;
        const double v = dequant_value(q.codes[c], q.scale_bytes[b], k, fmt);
        y[r * cols + c] = std::isnan(v) ? kNaNbf16 : encode_bf16_rne(v);
      }
      if (scales_out)
        for (int64_t b = 0; b < cols / bs; ++b)
          scales_out[r * (cols / bs) + b] = static_cast<uint8_t>(q.scale_bytes[b]);
    }
  });
}

// Straight-through backward: the gradient passes where |x| <= maxv * X (X the
// block's effective scale, as in the forward), else +0; NaN x gives +0.
void oracle_fake_quant_bwd(const uint16_t* x, const uint16_t* gy, int64_t rows, int64_t cols,
                           int fmt, int scaling, uint16_t* gx) {
  const double maxv = max_value(elem_fmt(fmt));
  parallel_rows(rows, [&](int64_t r0, int64_t r1) {
    std::vector<double> row(cols);
    for (int64_t r = r0; r < r1; ++r) {
      decode_row(x + r * cols, cols, row.data());
      const RowQuant q = quantize_row(row.data(), cols, fmt, scaling);
      for (int64_t c = 0; c < cols; ++c) {
        const double X = q.X[c / block_size(fmt)];   // NaN for a non-finite block
        const bool pass = std::fabs(row[c]) <= maxv * X;
        gx[r * cols + c] = pass ? gy[r * cols + c] : 0;
      }
    }
  });
}

// Error statistics ([UP] sections 3-4, QSNR): d = x - ŷ with ŷ the dequantized
// value as a float; per-block SSE (may be NULL) and totals {sum d^2, sum x^2}.
void oracle_block_error(const uint16_t* x, int64_t rows, int64_t cols, int fmt, int scaling,
                        double* block_sse, double* totals) {
  const int nt = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(g_threads, rows)));
  std::vector<double> part_d(nt, 0.0), part_x(nt, 0.0);
  const int64_t per = (rows + nt - 1) / nt;
  std::vector<std::thread> pool;
  auto work = [&](int t) {
    const int64_t r0 = t * per, r1 = std::min(rows, r0 + per);
    std::vector<double> row(cols);
    double sd = 0.0, sx = 0.0;
    for (int64_t r = r0; r < r1; ++r) {
      decode_row(x + r * cols, cols, row.data());
      const RowQuant q = quantize_row(row.data(), cols, fmt, scaling);
      const int bsz = block_size(fmt);
      for (int64_t b = 0; b < cols / bsz; ++b) {
        double bs = 0.0;
        for (int i = 0; i < bsz; ++i) {
          const int64_t c = b * bsz + i;
          const int k = (scaling >> 4) ? q.ks[c / kMacro] : 0;
          // ŷ as a float: exact, except that a value past the float range is
          // infinite (only reachable for amax in the top binade of bf16)
          const double y = static_cast<float>(dequant_value(q.codes[c], q.scale_bytes[b], k, fmt));
          const double d = row[c] - y;
          bs += d * d;
          sx += row[c] * row[c];
        }
        sd += bs;
        if (block_sse) block_sse[r * (cols / bsz) + b] = bs;
      }
    }
    part_d[t] = sd;
    part_x[t] = sx;
  };
  for (int t = 0; t < nt; ++t) pool.emplace_back(work, t);
  for (auto& th : pool) th.join();
  double sd = 0.0, sx = 0.0;
  for (int t = 0; t < nt; ++t) {
    sd += part_d[t];
    sx += part_x[t];
  }
  totals[0] = sd;
  totals[1] = sx;
}

// [BQ] section 2 apply step: the transformed, clipped rows as bf16 (round
// to nearest even; NaN as the canonical 0x7FC0). A is [a, a] and B is
// [cols / 32, b, b], both row-major float; beta_min / beta_max are
// [cols / 32] or both NULL. Also returns the fp32 values before the bf16
// rounding when y_f32 is not NULL.
void oracle_bat_apply(const uint16_t* x, int64_t rows, int64_t cols, int a, const float* A,
                      const float* B, const float* beta_min, const float* beta_max, uint16_t* y,
                      float* y_f32) {
  const int b = kBlock / a;
  parallel_rows(rows, [&](int64_t r0, int64_t r1) {
    std::vector<double> row(cols);
    for (int64_t r = r0; r < r1; ++r) {
      decode_row(x + r * cols, cols, row.data());
      for (int64_t j = 0; j < cols / kBlock; ++j) {
        float xb[kBlock], yb[kBlock];
        for (int i = 0; i < kBlock; ++i) xb[i] = static_cast<float>(row[j * kBlock + i]);
        bat_block(xb, a, A, B + j * b * b, beta_min ? beta_min + j : nullptr,
                  beta_max ? beta_max + j : nullptr, yb);
        for (int i = 0; i < kBlock; ++i) {
          y[r * cols + j * kBlock + i] = encode_bf16_rne(yb[i]);
          if (y_f32) y_f32[r * cols + j * kBlock + i] = yb[i];
        }
      }
    }
  });
}

}  // extern "C"
