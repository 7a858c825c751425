// The per-slice MX quantizer shared by the streaming kernels: the layout of
// their arguments, the scale decision of one 32-element block held by a lane
// pair (16 elements per lane), and the per-slice step of quantize, fake-quant
// forward/backward and block error. Included by every source that streams
// bf16 rows through the quantizer.

#pragma once

#include "mx_device.cuh"
#include "mx_launch.h"

namespace mxk {

struct StreamArgs {
  const uint8_t* x;   // bf16 input, 32 bytes per slice
  const uint8_t* gy;  // bf16 upstream gradient (backward only)
  int64_t nslices;    // elements / 16
  uint8_t* codes;     // FP4: 8 bytes per slice; FP8: 16 bytes per slice
  uint8_t* scales;    // one byte per block (slice >> 1)
  uint8_t* macro;     // one byte per macro block (slice >> 3)
  uint8_t* out;       // bf16 y (forward) or grad_x (backward), 32 bytes per slice
  float* block_sse;   // one float per block (error)
  double* totals;     // {sum d^2, sum x^2} (error)
  ScaleMap smap;      // where each block's scale byte goes
};

// Byte offset of block b's scale under the map (see ScaleMap). The row index
// r = b / bpr comes from the rounded reciprocal: b < 2^35 and both roundings
// are relative 2^-53, so the estimate is off by at most one, which the
// remainder test corrects.
__device__ __forceinline__ int64_t scale_offset(const ScaleMap& m, int64_t b) {
  if (m.bpr == 0) return b;
  int64_t r = __double2ll_rz(static_cast<double>(b) * m.inv);
  int64_t j = b - r * m.bpr;
  if (j < 0) {
    --r;
    j += m.bpr;
  } else if (j >= m.bpr) {
    ++r;
    j -= m.bpr;
  }
  return ((r >> 7) * m.nct + (j >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (j & 3);
}

constexpr int kOpQuant = 0, kOpFakeFwd = 1, kOpFakeBwd = 2, kOpError = 3;

// Build-time tuning knobs (defaults measured on B200): threads per block, and
// the persistent grid size in multiples of the resident capacity (0: one warp
// tile per warp, no grid-stride reuse).
#ifndef MX_THREADS
#define MX_THREADS 256
#endif
#ifndef MX_GRID_WAVES
#define MX_GRID_WAVES 0
#endif
constexpr int kThreads = MX_THREADS;

// Per-block scale state as both lanes of the block see it.
struct BlockScale {
  int byte;          // E8M0 byte (255 for a non-finite block)
  int k;             // macro factor index (0 without MBS)
  bool nonfinite;
  bool have_codes;   // codes below already hold this lane's codes (OAS)
  uint4 codes;       // E2M1 in .x/.y, one-byte formats in all four words
};

// Scale decision for the block holding `v`; pa = the block amax bits. Every
// lane of the warp must call it (the OAS branch is warp-uniform).
template <int FMT, int RULE, int MBS>
__device__ __forceinline__ BlockScale decide_scale(const V16& v, uint32_t pa, int k) {
  BlockScale s;
  s.nonfinite = pa >= 0x7F80u;
  s.k = k;
  s.have_codes = false;
  s.codes = make_uint4(0, 0, 0, 0);
  if (MBS == kMbsNone) {
    s.byte = rule_byte<FMT, RULE>(pa);
    if constexpr (RULE == kOas && FMT == kFmtE2M1) {
      const int b2 = max(static_cast<int>(pa >> 7) - 1, 0);
      // for a max significand <= 1.75 the finer grid is element-wise no worse
      const bool need = !s.nonfinite && (pa & 0x7F) > 96 && b2 != s.byte;
      if (__any_sync(kFull, need)) {
        const OasEval e = oas_eval16(v, s.byte);
        const int d = e.delta + __shfl_xor_sync(kFull, e.delta, 1);
        const bool up = need && d > 0;
        if (up) s.byte = b2;
        const uint2 c = up ? e.c2 : e.c1;   // the codes of the chosen scale
        s.codes = make_uint4(c.x, c.y, 0, 0);
        s.have_codes = true;
      }
    } else if constexpr (RULE == kOas) {
      // One-byte float formats: only a block max past the band (oas_m7) can
      // prefer the coarser scale.
      const int b2 = max(static_cast<int>(pa >> 7) - Elem<FMT>::emax + 1, 0);
      const bool need = !s.nonfinite && (pa & 0x7F) > Elem<FMT>::oas_m7 && b2 != s.byte;
      if (__any_sync(kFull, need)) {
        const OasEvalBytes e = oas_eval_bytes16<FMT>(v, s.byte);
        const __int128 d = pair_sum_i128(e.delta);
        const bool up = need && d > 0;
        if (up) s.byte = b2;
        s.codes = up ? e.c2 : e.c1;
        s.have_codes = true;
      }
    }
  } else {
    s.byte = mbs_byte(pa, k, 0);
    if (RULE == kOas) {
      const int b2 = mbs_byte(pa, k, 1);
      // as without MBS, the finer candidate is element-wise no worse unless
      // the scaled block max exceeds 7 f (both sides of the test are exact)
      const bool need = !s.nonfinite && b2 != s.byte && mbs_oas_band(pa, s.byte, k);
      if (__any_sync(kFull, need)) {
        const OasEval e = oas_eval_mbs16(v, s.byte, k);
        const int d = e.delta + __shfl_xor_sync(kFull, e.delta, 1);
        const bool up = need && d > 0;
        if (up) s.byte = b2;
        const uint2 c = up ? e.c2 : e.c1;   // the codes of the chosen scale
        s.codes = make_uint4(c.x, c.y, 0, 0);
        s.have_codes = true;
      }
    }
  }
  if (s.nonfinite) s.byte = 255;
  return s;
}

// E2M1 codes of one lane's 16 elements (8 bytes, nibble i = element i).
template <int MBS>
__device__ __forceinline__ uint2 codes_fp4(const V16& v, const BlockScale& s) {
  if (s.nonfinite) return nonfinite_e2m1_16(v);
  if (s.have_codes) return make_uint2(s.codes.x, s.codes.y);
  if (MBS == kMbsNone) return enc_e2m1_16(scale_slice(v, s.byte));
  return enc_mbs_cvt_16(v, s.byte, s.k);
}

// Codes of one lane's 16 elements: E2M1 in .x/.y, one-byte formats in all
// four words.
template <int FMT, int MBS>
__device__ __forceinline__ uint4 lane_codes(const V16& v, const BlockScale& s) {
  if constexpr (FMT == kFmtE2M1) {
    const uint2 c = codes_fp4<MBS>(v, s);
    return make_uint4(c.x, c.y, 0, 0);
  } else {
    if (s.nonfinite) return nonfinite_bytes_16<FMT>(v);
    if (s.have_codes) return s.codes;
    return enc_bytes_16<FMT>(scale_slice(v, s.byte));
  }
}

// Dequantized values (exact floats, signed) of a finite block's 16 elements
// from their codes.
template <int FMT, int MBS>
__device__ __forceinline__ F16 block_values(const uint4& codes, const BlockScale& s) {
  const int E = s.byte - 127;
  if (FMT == kFmtE2M1) {
    // MBS: value * (256 + k) 2^(E-8) -- the multiplier has 9 significant bits
    // and the product at most 11, both exact in float
    const float p = MBS == kMbsNone ? pow2f(E) : static_cast<float>(256 + s.k) * pow2f(E - 8);
    return dec_e2m1_16(make_uint2(codes.x, codes.y), p);
  }
  return dec_bytes_16<FMT>(codes, pow2f(E));
}

template <int OP, int FMT, int RULE, int MBS>
__device__ __forceinline__ void process_slice(const StreamArgs& a, const V16& v, const V16& g,
                                              int64_t c, bool valid, int lane, uint32_t pa, int k,
                                              double& sd, double& sx) {
  const BlockScale s = decide_scale<FMT, RULE, MBS>(v, pa, k);
  // codes for every lane before any divergent branch (see codes_fp4)
  uint4 codes = make_uint4(0, 0, 0, 0);
  // block error of plain E2M1: the slice is scaled once, for the codes (as
  // codes_fp4 scales it) and for the error arithmetic below
  constexpr bool kScaleOnce = OP == kOpError && FMT == kFmtE2M1 && MBS == kMbsNone;
  V16 scaled;
  if constexpr (kScaleOnce) {
    scaled = scale_slice(v, s.nonfinite ? 127 : s.byte);
    uint2 c;
    if (s.nonfinite) c = nonfinite_e2m1_16(v);
    else if (s.have_codes) c = make_uint2(s.codes.x, s.codes.y);
    else c = enc_e2m1_16(scaled);
    codes = make_uint4(c.x, c.y, 0, 0);
  } else if (OP != kOpFakeBwd) {
    codes = lane_codes<FMT, MBS>(v, s);
  }

  if (OP == kOpQuant) {
    if (FMT == kFmtE2M1) {
      if (valid) st_stream8(a.codes + 8 * c, make_uint2(codes.x, codes.y));
    } else {
      if (valid) st_stream16(a.codes + 16 * c, codes);
    }
    if (valid && (lane & 1) == 0) a.scales[scale_offset(a.smap, c >> 1)] = static_cast<uint8_t>(s.byte);
    if (MBS != kMbsNone && valid && (lane & 7) == 0) a.macro[c >> 3] = static_cast<uint8_t>(s.k);
    return;
  }

  if (OP == kOpFakeFwd) {
    V16 o;
    if (s.nonfinite) {
#pragma unroll
      for (int i = 0; i < 8; ++i) o.w[i] = (static_cast<uint32_t>(kNaNbf16) << 16) | kNaNbf16;
    } else if (FMT == kFmtE2M1 && MBS == kMbsNone && e2m1_table_scale_ok(s.byte)) {
      // the products are normal bf16 values: a table of the scaled magnitudes
      o = e2m1x16_to_bf16(make_uint2(codes.x, codes.y), e2m1_table(s.byte - 127));
    } else {
      const F16 y = block_values<FMT, MBS>(codes, s);
#pragma unroll
      for (int i = 0; i < 8; ++i) o.w[i] = pack_bf16x2(y.v[2 * i], y.v[2 * i + 1]);
    }
    if (valid) st_stream32(a.out + 32 * c, o);
    if (a.scales && valid && (lane & 1) == 0) a.scales[scale_offset(a.smap, c >> 1)] = static_cast<uint8_t>(s.byte);
    return;
  }

  if (OP == kOpFakeBwd) {
    V16 o;
    // |x| <= maxv * X, X = f 2^E: the limit is exact in float (inf past range)
    const int E = s.byte - 127;
    const float lim = MBS == kMbsNone ? Elem<FMT>::maxv * pow2f(E)
                                      : 6.0f * static_cast<float>(256 + s.k) * pow2f(E - 8);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool plo = !s.nonfinite && fabsf(bf_lo(v.w[i])) <= lim;
      const bool phi = !s.nonfinite && fabsf(bf_hi(v.w[i])) <= lim;
      o.w[i] = (plo ? (g.w[i] & 0xFFFFu) : 0u) | (phi ? (g.w[i] & 0xFFFF0000u) : 0u);
    }
    if (valid) st_stream32(a.out + 32 * c, o);
    return;
  }

  if (OP == kOpError) {
    // In units of the block scale X = 2^E: s = x 2^-E (exact while it is a
    // normal bf16; below that, errors of at most 2^-134 are negligible by
    // the bound on Sd below) and the grid value g (code value, times f
    // under MBS) are exact floats, and so is ds = s - g (s has 8
    // significant bits, g at most 11, and g != 0 only when |s| is within a
    // small factor of |g|). ds^2 and s^2 are summed in
    // float, four fma chains of four per lane and then pairwise, so the
    // block's sum of the 32 ds^2 carries a relative error of at most 7 u
    // (u = 2^-24; all terms are non-negative) and the result, Sd 2^(2E)
    // rounded to float, at most 8 u. Terms that underflow in float
    // (ds < 2^-63) add absolute errors below 2^-144 in these units, so this
    // holds while Sd >= 2^-90; the final rounding is relative only while
    // the result is a normal float. Blocks outside those bounds (and those
    // whose dequantized values pass the float range) take the exact path:
    // d = x - y in float, d^2 summed in double.
    const int bs = s.nonfinite ? 127 : s.byte;
    const int E = bs - 127;
    const double p2 = __longlong_as_double(static_cast<long long>(2 * E + 1023) << 52);
    V16 sl;
    if constexpr (kScaleOnce) sl = scaled;
    else sl = scale_slice(v, bs);
    float ad[4] = {0.0f, 0.0f, 0.0f, 0.0f}, ax[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (FMT == kFmtE2M1 && MBS == kMbsNone) {
      // |s| - |g| (the code keeps the sign of s) is exact in bf16 too: for s
      // in [2^e, 2^(e+1)) the grid step is 2^(e-1), so |d| <= 2^(e-2) (or
      // below 2 when s saturates to 6) and d is a multiple of 2^(e-7)
      const V16 g = e2m1x16_mag_bf16(make_uint2(codes.x, codes.y));
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t d = sub_bf16x2(sl.w[i] & 0x7FFF7FFFu, g.w[i]);
        ad[(2 * i) & 3] = sq_acc_lo(d, ad[(2 * i) & 3]);
        ad[(2 * i + 1) & 3] = sq_acc_hi(d, ad[(2 * i + 1) & 3]);
        ax[(2 * i) & 3] = sq_acc_lo(sl.w[i], ax[(2 * i) & 3]);
        ax[(2 * i + 1) & 3] = sq_acc_hi(sl.w[i], ax[(2 * i + 1) & 3]);
      }
    } else {
      const F16 g = FMT == kFmtE2M1
                        ? dec_e2m1_16(make_uint2(codes.x, codes.y),
                                      static_cast<float>(256 + s.k) * 0.00390625f)
                        : dec_bytes_16<FMT>(codes, 1.0f);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float si = elem(sl, i);
        const float di = si - g.v[i];
        ad[i & 3] = fmaf(di, di, ad[i & 3]);
        ax[i & 3] = fmaf(si, si, ax[i & 3]);
      }
    }
    const float ld = (ad[0] + ad[1]) + (ad[2] + ad[3]);
    const float lx = (ax[0] + ax[1]) + (ax[2] + ax[3]);
    const float Sd = ld + __shfl_xor_sync(kFull, ld, 1);
    double q = static_cast<double>(Sd) * p2;
    double bd = static_cast<double>(ld) * p2;
    double bx = static_cast<double>(lx) * p2;
    const bool exact = !s.nonfinite && pa != 0 && !(Sd >= 0x1p-90f && q >= 0x1p-120 && q < 0x1p120);
    if (__any_sync(kFull, exact)) {
      const F16 y = block_values<FMT, MBS>(codes, s);
      double ed = 0.0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const double d = static_cast<double>(elem(v, i) - y.v[i]);   // exact in float
        ed = fma(d, d, ed);
      }
      const double eq = ed + __shfl_xor_sync(kFull, ed, 1);
      if (exact) {
        bd = ed;
        q = eq;
      }
    }
    if (s.nonfinite) {
      // the dequantized block is NaN; x^2 (possibly inf) still feeds the total
      bd = q = __int_as_float(0x7FC00000);
      bx = 0.0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const double xi = elem(v, i);
        bx = fma(xi, xi, bx);
      }
    }
    if (valid) {
      if (a.block_sse && (lane & 1) == 0) a.block_sse[c >> 1] = static_cast<float>(q);
      sd += bd;
      sx += bx;
    }
  }
}

}  // namespace mxk
