// MX block-32 kernels for sm_100a: quantize, fake-quant forward/backward and
// block error (one streaming template), MBS-Dynamic (search + the same ops),
// and dequantize.
//
// Every kernel is a grid-stride loop over "warp tiles" of 32*U consecutive
// 32-byte slices (U slices per lane; all loads of a tile are issued before
// any arithmetic, so each lane keeps U x 32 bytes in flight). By default the
// grid has one warp per tile and the block scheduler refills the SMs (measured
// faster on B200 than a persistent grid); the error kernel keeps a persistent
// grid so that its per-CTA atomics stay few.
// Shared memory holds only the block lists of the two-phase OAS quantize
// kernel and the magnitudes and per-k sums of the MBS-Dynamic sweep; no
// kernel waits on a flag.
//
// Sources restated: "[vLLM] MXFP8/MXFP4: microscaling format quantization"
// (MX format table; MXFP8 block-32 scaling; MXFP4 packing), "[Axolotl] MXFP4
// quantization support" (2-3: block 32, fake-quant of activations and
// weights), "Unveiling the Potential of Quantization with MXFP4" (2.A OAS,
// 2.B MBS, 3-4 QSNR).

#include "mx_stream.cuh"

namespace mxk {

// The 16-element-block formats (MXFP4 at block 16, NVFP4): a lane's slice
// is one whole block, so nothing is exchanged between lanes and the block
// index is the slice index.
template <int OP, int FMT, int RULE, int MBS>
__device__ __forceinline__ void process_slice16(const StreamArgs& a, const V16& v, const V16& g,
                                                int64_t c, bool valid, int lane, int k,
                                                double& sd, double& sx) {
  const uint32_t am = amax_bits16(v);
  const bool nonfinite = am >= 0x7F80u;
  int byte;
  float scale;   // the block's scale value, f 2^E under MBS (0 leaves only the signs)
  uint2 codes = make_uint2(0, 0);
  if constexpr (FMT == kFmtNvfp4) {
    byte = nvfp4_scale_byte(am);
    scale = nonfinite ? 0.0f : e4m3_value(byte);
    if (OP != kOpFakeBwd)
      codes = (nonfinite || scale == 0.0f) ? nonfinite_e2m1_16(v) : enc_e2m1_div_16(v, scale);
  } else {
    // MXFP4 at block 16: the base rules, or under a macro factor k the
    // exponent of amax / f (and OAS on x / f), exactly as at block 32
    byte = MBS == kMbsNone ? rule_byte<kFmtE2M1, RULE>(am) : mbs_byte(am, k, 0);
    bool have = false;
    if constexpr (RULE == kOas) {
      const int b2 = MBS == kMbsNone ? max(static_cast<int>(am >> 7) - 1, 0) : mbs_byte(am, k, 1);
      const bool band = MBS == kMbsNone ? (am & 0x7F) > Elem<kFmtE2M1>::oas_m7
                                        : mbs_oas_band(am, byte, k);
      const bool need = !nonfinite && band && b2 != byte;
      if (__any_sync(kFull, need)) {
        const OasEval e = MBS == kMbsNone ? oas_eval16(v, byte) : oas_eval_mbs16(v, byte, k);
        const bool up = need && e.delta > 0;   // the lane holds the whole block
        if (up) byte = b2;
        codes = up ? e.c2 : e.c1;
        have = true;
      }
    }
    if (nonfinite) byte = 255;
    scale = MBS == kMbsNone ? pow2f(byte - 127) : static_cast<float>(256 + k) * pow2f(byte - 127 - 8);
    if (OP != kOpFakeBwd && !have) {
      if (nonfinite) codes = nonfinite_e2m1_16(v);
      else if (MBS == kMbsNone) codes = enc_e2m1_16(scale_slice(v, byte));
      else codes = enc_mbs_cvt_16(v, byte, k);
    }
    if (OP != kOpFakeBwd && have && nonfinite) codes = nonfinite_e2m1_16(v);
  }

  if (OP == kOpQuant) {
    if (valid) {
      st_stream8(a.codes + 8 * c, codes);
      a.scales[scale_offset(a.smap, c)] = static_cast<uint8_t>(byte);
      if (MBS != kMbsNone && (lane & 7) == 0) a.macro[c >> 3] = static_cast<uint8_t>(k);
    }
    return;
  }
  if (OP == kOpFakeBwd) {
    // |x| <= 6 s (exact in float); nothing passes in a NaN/Inf block
    const float lim = 6.0f * scale;
    V16 o;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool plo = !nonfinite && fabsf(bf_lo(v.w[i])) <= lim;
      const bool phi = !nonfinite && fabsf(bf_hi(v.w[i])) <= lim;
      o.w[i] = (plo ? (g.w[i] & 0xFFFFu) : 0u) | (phi ? (g.w[i] & 0xFFFF0000u) : 0u);
    }
    if (valid) st_stream32(a.out + 32 * c, o);
    return;
  }
  // values q * s: exact floats (at most 2 + 4 significant bits)
  const F16 y = dec_e2m1_16(codes, scale);
  if (OP == kOpFakeFwd) {
    V16 o;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o.w[i] = nonfinite ? ((static_cast<uint32_t>(kNaNbf16) << 16) | kNaNbf16)
                         : pack_bf16x2(y.v[2 * i], y.v[2 * i + 1]);
    }
    if (valid) {
      st_stream32(a.out + 32 * c, o);
      if (a.scales) a.scales[scale_offset(a.smap, c)] = static_cast<uint8_t>(byte);
    }
    return;
  }
  if (OP == kOpError) {
    // d = x - y exact in float; d^2 summed in double (one lane, one block)
    double bd = 0.0, bx = 0.0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float xf = elem(v, i);
      const double d = static_cast<double>(xf - y.v[i]);
      bd = fma(d, d, bd);
      bx = fma(static_cast<double>(xf), static_cast<double>(xf), bx);
    }
    if (nonfinite) bd = __int_as_float(0x7FC00000);
    if (valid) {
      if (a.block_sse) a.block_sse[c] = static_cast<float>(bd);
      sd += bd;
      sx += bx;
    }
  }
}

// Sum of the per-lane error partials into totals: warp, then CTA (NW warps),
// then one double atomic per CTA.
template <int NW = kThreads / 32>
__device__ __forceinline__ void reduce_totals(double sd, double sx, double* totals) {
  __shared__ double red[2][NW];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sd += __shfl_xor_sync(kFull, sd, o);
    sx += __shfl_xor_sync(kFull, sx, o);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = sd;
    red[1][w] = sx;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double td = 0.0, tx = 0.0;
    for (int i = 0; i < NW; ++i) {
      td += red[0][i];
      tx += red[1][i];
    }
    atomicAdd(totals, td);
    atomicAdd(totals + 1, tx);
  }
}

template <int OP, int FMT, int RULE, int MBS, int U>
__global__ void __launch_bounds__(kThreads) stream_kernel(StreamArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  double sd = 0.0, sx = 0.0;
  for (int64_t tile = warp; tile * 32 * U < a.nslices; tile += nwarps) {
    const int64_t base = tile * 32 * U + lane;
    V16 v[U], g[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t c = base + 32 * j;
#pragma unroll
      for (int i = 0; i < 8; ++i) v[j].w[i] = g[j].w[i] = 0;
      if (c < a.nslices) {
        v[j] = ld_stream32(a.x + 32 * c);
        if (OP == kOpFakeBwd) g[j] = ld_stream32(a.gy + 32 * c);
      }
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t c = base + 32 * j;
      if constexpr (FMT == kFmtE2M1B16 || FMT == kFmtNvfp4) {
        int k = 0;
        // the macro max: over the lane pair, then over the 8 lanes
        if (MBS == kMbsStatic) k = mbs_static_k(oct_max(pair_max(amax_bits16(v[j]))));
        process_slice16<OP, FMT, RULE, MBS>(a, v[j], g[j], c, c < a.nslices, lane, k, sd, sx);
      } else {
        const uint32_t pa = pair_max(amax_bits16(v[j]));
        int k = 0;
        if (MBS == kMbsStatic) k = mbs_static_k(oct_max(pa));
        process_slice<OP, FMT, RULE, MBS>(a, v[j], g[j], c, c < a.nslices, lane, pa, k, sd, sx);
      }
    }
  }
  if (OP == kOpError) reduce_totals(sd, sx, a.totals);
}

// ------------------------------------------------------ OAS quantize path --

// OAS quantize in two phases per CTA tile: MXFP4 without MBS or with
// MBS-Static, and the one-byte float formats. Phase 1 handles every block
// whose finer exponent is already the answer (scaled max inside the band of
// Elem<FMT>::oas_m7 -- under MBS: at most 7f --, the two candidates equal, or
// NaN/Inf) exactly as the single-rule kernel does, and appends the other
// blocks (a fifth or fewer for Gaussian data) to a shared-memory list, with
// their macro factor. Phase 2 evaluates only the listed blocks, two lanes per
// block and full warps, re-reading their 64 bytes (just loaded, so from L2).
// Without the split every warp that holds one such block pays for the exact
// SSE comparison on all of its lanes.
// Output of one lane's slice once its block's codes and scale byte are
// decided: the codes (quantize) or the dequantized bf16 values (fake-quant
// forward), and the scale byte (quantize; fake-quant when asked for). The
// even lane of the block's lane pair writes the byte.
template <int OP, int FMT, int MBS>
__device__ __forceinline__ void emit_slice(const StreamArgs& a, int64_t c, int lane, uint4 codes,
                                           int byte, int k, bool nonfinite) {
  if constexpr (OP == kOpQuant) {
    if (FMT == kFmtE2M1) st_stream8(a.codes + 8 * c, make_uint2(codes.x, codes.y));
    else st_stream16(a.codes + 16 * c, codes);
  } else {
    V16 o;
    if (nonfinite) {
#pragma unroll
      for (int i = 0; i < 8; ++i) o.w[i] = (static_cast<uint32_t>(kNaNbf16) << 16) | kNaNbf16;
    } else if (FMT == kFmtE2M1 && MBS == kMbsNone && e2m1_table_scale_ok(byte)) {
      o = e2m1x16_to_bf16(make_uint2(codes.x, codes.y), e2m1_table(byte - 127));
    } else {
      BlockScale s;
      s.byte = byte;
      s.k = k;
      s.nonfinite = false;
      s.have_codes = true;
      s.codes = codes;
      const F16 y = block_values<FMT, MBS>(codes, s);
#pragma unroll
      for (int i = 0; i < 8; ++i) o.w[i] = pack_bf16x2(y.v[2 * i], y.v[2 * i + 1]);
    }
    st_stream32(a.out + 32 * c, o);
  }
  if ((OP == kOpQuant || a.scales) && (lane & 1) == 0)
    a.scales[scale_offset(a.smap, c >> 1)] = static_cast<uint8_t>(byte);
}

// OAS quantize and fake-quant forward in two phases per CTA tile: MXFP4
// without MBS or with MBS-Static, and the one-byte float formats. Phase 1
// handles every block whose finer exponent is already the answer (scaled
// max inside the band of Elem<FMT>::oas_m7 -- under MBS: at most 7f --, the
// two candidates equal, or NaN/Inf) exactly as the single-rule kernel does,
// and appends the other blocks (a fifth or fewer for Gaussian data) to a
// shared-memory list, with their macro factor. Phase 2 evaluates only the
// listed blocks, two lanes per block and full warps, re-reading their 64
// bytes (just loaded, so from L2). Without the split every warp that holds
// one such block pays for the exact SSE comparison on all of its lanes.
template <int OP, int FMT, int MBS, int U>
__global__ void __launch_bounds__(kThreads) oas_kernel(StreamArgs a) {
  constexpr int kWarps = kThreads / 32;
  constexpr int kTileSlices = kWarps * 32 * U;
  // listed blocks: first-slice offset in the low 16 bits, macro k above
  __shared__ uint32_t list[kTileSlices / 2];
  __shared__ int count;
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const int64_t tile0 = static_cast<int64_t>(blockIdx.x) * kTileSlices;
  if (threadIdx.x == 0) count = 0;
  __syncthreads();

  // phase 1
  V16 v[U];
#pragma unroll
  for (int j = 0; j < U; ++j) {
    const int64_t c = tile0 + w * 32 * U + 32 * j + lane;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[j].w[i] = 0;
    if (c < a.nslices) v[j] = ld_stream32(a.x + 32 * c);
  }
#pragma unroll
  for (int j = 0; j < U; ++j) {
    const int64_t c = tile0 + w * 32 * U + 32 * j + lane;
    const bool valid = c < a.nslices;
    const uint32_t pa = pair_max(amax_bits16(v[j]));
    const bool nonfinite = pa >= 0x7F80u;
    int k = 0, b1, b2;
    bool band;
    if (MBS == kMbsNone) {
      b1 = rule_byte<FMT, kFloor>(pa);
      b2 = max(static_cast<int>(pa >> 7) - Elem<FMT>::emax + 1, 0);
      band = (pa & 0x7F) > Elem<FMT>::oas_m7;
    } else {
      k = mbs_static_k(oct_max(pa));
      b1 = mbs_byte(pa, k, 0);
      b2 = mbs_byte(pa, k, 1);
      band = mbs_oas_band(pa, b1, k);
    }
    const bool need = valid && !nonfinite && band && b2 != b1;
    if (valid && !need) {
      uint4 codes;
      if constexpr (FMT == kFmtE2M1) {
        uint2 c2;
        if (nonfinite) c2 = nonfinite_e2m1_16(v[j]);
        else if (MBS == kMbsNone) c2 = enc_e2m1_16(scale_slice(v[j], b1));
        else c2 = enc_mbs_cvt_16(v[j], b1, k);
        codes = make_uint4(c2.x, c2.y, 0, 0);
      } else {
        codes = nonfinite ? nonfinite_bytes_16<FMT>(v[j]) : enc_bytes_16<FMT>(scale_slice(v[j], b1));
      }
      emit_slice<OP, FMT, MBS>(a, c, lane, codes, nonfinite ? 255 : b1, k, nonfinite);
    }
    if (OP == kOpQuant && MBS != kMbsNone && valid && (lane & 7) == 0)
      a.macro[c >> 3] = static_cast<uint8_t>(k);
    if (need && (lane & 1) == 0)
      list[atomicAdd(&count, 1)] = static_cast<uint32_t>(c - tile0) | (static_cast<uint32_t>(k) << 16);
  }
  __syncthreads();

  // phase 2: 16 listed blocks per warp step
  const int n = count;
  for (int base = w * 16; base < n; base += kWarps * 16) {
    const int idx = base + (lane >> 1);
    const bool has = idx < n;
    const uint32_t entry = has ? list[idx] : 0u;
    const int64_t c = tile0 + (entry & 0xFFFFu) + (lane & 1);
    const int k = static_cast<int>(entry >> 16);
    V16 x;
#pragma unroll
    for (int i = 0; i < 8; ++i) x.w[i] = 0;
    if (has) x = ld_stream32(a.x + 32 * c);
    const uint32_t pa = pair_max(amax_bits16(x));
    const int b1 = MBS == kMbsNone ? rule_byte<FMT, kFloor>(pa) : mbs_byte(pa, k, 0);
    uint4 codes;
    bool up;
    if constexpr (FMT == kFmtE2M1) {
      const OasEval e = MBS == kMbsNone ? oas_eval16(x, b1) : oas_eval_mbs16(x, b1, k);
      up = e.delta + __shfl_xor_sync(kFull, e.delta, 1) > 0;
      const uint2 c2 = up ? e.c2 : e.c1;
      codes = make_uint4(c2.x, c2.y, 0, 0);
    } else {
      const OasEvalBytes e = oas_eval_bytes16<FMT>(x, b1);
      up = pair_sum_i128(e.delta) > 0;
      codes = up ? e.c2 : e.c1;
    }
    if (has) emit_slice<OP, FMT, MBS>(a, c, lane, codes, up ? b1 + 1 : b1, k, false);
  }
}

// ------------------------------------------------------- MBS-Dynamic path --

// Sum of squared errors of one 128-element macro block under factor k, in
// double, in element order: each d is exact in float, d*d exact in double, so
// the running sum rounds exactly as a sequential double sum does.
// xs: the 128 magnitudes |x| as floats; amax[128 / BS]: sub-block amax bits
// (sub-blocks of BS = 32 elements, or 16 for MXFP4 at block 16).
// Rounding under f uses the bracket of enc_mbs_cvt_16, 8 elements at a time.
template <int RULE, int BS>
__device__ __forceinline__ double macro_sse_k(const float* xs, const uint32_t* amax, int k) {
  const FactorBracket fb = factor_bracket(k);
  double sse = 0.0;
#pragma unroll 1
  for (int b = 0; b < 128 / BS; ++b) {
    int byte = mbs_byte(amax[b], k, 0);
    if (RULE == kOas) {
      const int b2 = mbs_byte(amax[b], k, 1);
      if (b2 != byte && mbs_oas_band(amax[b], byte, k)) {
        // exact SSE difference of the two candidates (see oas_eval_mbs16)
        const float inv1 = inv_scale_from_byte(byte);
        const float f2 = fb.f * 2.0f;
        int acc = 0;
#pragma unroll 1
        for (int i = 0; i < BS; i += 8) {
          float s[8], h[8], q1[8], q2[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            s[j] = xs[BS * b + i + j] * inv1;
            h[j] = s[j] * 0.5f;
          }
          e2m1x8_values(mbs_codes8(s, fb.L, fb.H), q1);
          e2m1x8_values(mbs_codes8(h, fb.L, fb.H), q2);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int D1 = small_int(fmaf(-q1[j], fb.f, s[j]) * 512.0f);
            const int D2 = small_int(fmaf(-q2[j], f2, s[j]) * 512.0f);
            acc += D1 * D1 - D2 * D2;
          }
        }
        if (acc > 0) byte = b2;
      }
    }
    const float m = inv_scale_from_byte(byte);                          // 2^-E
    const double p = __longlong_as_double(static_cast<long long>(byte - 127 + 1023) << 52);
#pragma unroll 1
    for (int i = 0; i < BS; i += 8) {
      float s[8], q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) s[j] = xs[BS * b + i + j] * m;
      e2m1x8_values(mbs_codes8(s, fb.L, fb.H), q);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // s - q f is exact (both are multiples of 2^-9 below 2^5, or q = 0)
        const double d = static_cast<double>(fmaf(-q[j], fb.f, s[j])) * p;   // exact
        sse = fma(d, d, sse);
      }
    }
  }
  return sse;
}

// ----------------------------------------------------- MBS-Dynamic sweep --
//
// The definition evaluates all 256 factors element by element (macro_sse_k
// above does exactly that for one k). The same argmin follows from an exact
// sweep over k:
//
// For sub-block i with amax exponent field ex and mantissa m7, the byte is
// B0 = max(ex - 2, 0) while k <= 2 m7 (regime 0) and B1 = max(ex - 3, 0)
// above (regime 1). Within a regime the scale 2^E is fixed, and with
// t = |x| 2^-E, F = 256 + k and the code value q = Q / 2 (Q in
// {0,1,2,3,4,6,8,12}), the error is d = (T - Q F) 2^(E-9) with T = 512 t. T is
// an integer whenever t > 1/4 ("big"; t has 8 significant bits). Smaller
// elements round to 0 for every k and contribute x^2.
//
// The code of a big element is the number of midpoints mu it lies above:
// t / f > mu, or t / f == mu with the even neighbour above. With M = 4 mu in
// {1,3,5,7,10,14,20} that is an integer test of 2T against M F. So the code
// drops by one at the integer breakpoint F_m of each midpoint m, at most twice
// over F in [256, 511]. Per sub-block and regime,
//   SSE(k) = 2^(2E-18) (C - 2 F A(k) + F^2 B(k)) + X,
// with C = sum of T^2, A = sum of T Q, B = sum of Q^2 over the big elements,
// and X = sum of x^2 over the others. A and B are step functions of k, built
// from per-k event deltas in shared memory and a prefix scan. Every term of
// the bracket is an integer below 2^34, exact in double.
//
// Under OAS each sub-block takes, for every k, the smaller SSE of its byte
// and the coarser candidate max(ex - 1 - r, 0) (an exact comparison in the
// definition, the finer one on a tie): a second level of the same sums.
//
// The argmin must match the element-order double sums of the definition.
// These sums are within 127 u of the exact SSE, and the sweep's doubles
// within about 16 u (u = 2^-53). So any k whose swept value exceeds the
// minimum by more than a factor 1 + 2^-40 cannot be the argmin or tie with
// it. The remaining candidates (usually one) are re-evaluated in element
// order by macro_sse_k. A minimum of exactly 0 means the exact SSE is 0 for
// those k, so their double sums are 0 too and the smallest wins.

constexpr int kSweepThreads = 128;
constexpr int kSweepWarps = kSweepThreads / 32;

// Rows of per-k deltas are padded by 4 words every 32 entries, so that the
// scan's 16-byte loads (8 consecutive k per lane) hit distinct banks.
constexpr int kSweepRow = 256 + 32;
__device__ __forceinline__ int sweep_slot(int k) { return k + ((k >> 5) << 2); }

// Levels of sub-block scale per regime: FLOOR has one (B_r); OAS two
// (B_r and the coarser max(ex - 1 - r, 0)), of which the smaller SSE counts.
template <int RULE>
struct SweepShared {
  static constexpr int kLevels = RULE == kOas ? 2 : 1;
  float xs[4][128 + 1];                  // magnitudes of the warp's 4 macro blocks
  int d[2 * 2 * kLevels][kSweepRow];     // per-k deltas of A and B for each (regime, level)
  uint8_t cand[256];                     // candidate k for the element-order re-evaluation
};

// Q = 2 x the E2M1 magnitude of code c (0..7).
__device__ __forceinline__ int code_q2(int c) {
  return c <= 4 ? c : (c == 5 ? 6 : (c == 6 ? 8 : 12));
}

// Prefix sums of row[0..255] at this lane's 8 consecutive k (8 lane + j),
// then the lane's entries cleared for the next use.
__device__ __forceinline__ void scan_row8(int* row, int lane, int out[8]) {
  int4* p = reinterpret_cast<int4*>(row + sweep_slot(8 * lane));
  const int4 u = p[0], w = p[1];
  out[0] = u.x;
  out[1] = out[0] + u.y;
  out[2] = out[1] + u.z;
  out[3] = out[2] + u.w;
  out[4] = out[3] + w.x;
  out[5] = out[4] + w.y;
  out[6] = out[5] + w.z;
  out[7] = out[6] + w.w;
  int incl = out[7];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += t;
  }
  const int excl = incl - out[7];
#pragma unroll
  for (int j = 0; j < 8; ++j) out[j] += excl;
  p[0] = make_int4(0, 0, 0, 0);
  p[1] = make_int4(0, 0, 0, 0);
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// The MBS-Dynamic factor of macro block g of this warp (warp-collective).
// am: the 4 sub-block amax bits (0 for a macro block holding NaN/Inf, whose
// staged magnitudes are zeros).
template <int RULE, int BS>
__device__ __forceinline__ int sweep_macro(SweepShared<RULE>& sh, int g, const uint32_t* am,
                                           int lane) {
  constexpr int NL = SweepShared<RULE>::kLevels;
  double tot[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) tot[j] = 0.0;
  const float* xs = sh.xs[g];
#pragma unroll 1
  for (int i = 0; i < 128 / BS; ++i) {
    const int ex = static_cast<int>(am[i] >> 7);
    const int K = 2 * static_cast<int>(am[i] & 0x7F);   // regime 0 for k <= K
    // one element per lane (16-element sub-blocks: lanes 16..31 add nothing)
    const float xf = (BS == 32 || lane < 16) ? xs[BS * i + lane] : 0.0f;
    const uint32_t xb = __float_as_uint(xf) >> 16;       // |x| as bf16 bits
    const int exx = static_cast<int>(xb >> 7);
    const int sig = exx ? static_cast<int>(128 | (xb & 0x7F)) : static_cast<int>(xb & 0x7F);
    const double x2 = static_cast<double>(xf) * static_cast<double>(xf);   // exact
    // per (regime r, level u), index q = 2 r + u ... flattened as r * NL + u
    int a0[2 * NL], b0[2 * NL];
    unsigned cc[2 * NL];
    double xt[2 * NL], scl[2 * NL];
#pragma unroll
    for (int q = 0; q < 2 * NL; ++q) {
      const int r = q / NL, u = q % NL;
      const int Bl = max(ex - 2 + u - r, 0);   // the sub-block byte (MBS rule, OAS candidate u)
      // T = 512 |x| 2^(127 - Bl) = sig 2^sh (sh <= 5 whenever T > 128)
      const int sh_ = (exx ? exx : 1) + 2 - Bl;
      const bool big = sh_ > 0 || (sh_ == 0 && sig > 128);
      const int T = big ? (sig << sh_) : 0;
      const int T2 = 2 * T;
      // F_m: the first F at which the element is no longer above midpoint m
      int Fm[7];
      Fm[0] = T2;                 // 1/4, even below: above iff 2T > F
      Fm[1] = T2 / 3 + 1;         // 3/4, even above: above iff 2T >= 3F
      Fm[2] = (T2 + 4) / 5;       // 5/4
      Fm[3] = T2 / 7 + 1;         // 7/4
      Fm[4] = (T2 + 9) / 10;      // 5/2
      Fm[5] = T2 / 14 + 1;        // 7/2
      Fm[6] = (T2 + 19) / 20;     // 5
      int c0 = 0;
#pragma unroll
      for (int m = 0; m < 7; ++m) c0 += Fm[m] > 256 ? 1 : 0;
      // Q[m] - Q[m+1] and Q[m]^2 - Q[m+1]^2 when the code drops from m+1 to m
      constexpr int kDq[7] = {-1, -1, -1, -1, -2, -2, -4};
      constexpr int kDq2[7] = {-1, -3, -5, -7, -20, -28, -80};
#pragma unroll
      for (int m = 0; m < 7; ++m) {
        const int km = Fm[m] - 256;
        if (km >= 1 && km <= 255) {
          atomicAdd(&sh.d[2 * q][sweep_slot(km)], T * kDq[m]);
          atomicAdd(&sh.d[2 * q + 1][sweep_slot(km)], kDq2[m]);
        }
      }
      const int q0 = code_q2(c0);
      a0[q] = __reduce_add_sync(kFull, T * q0);
      b0[q] = __reduce_add_sync(kFull, q0 * q0);
      cc[q] = __reduce_add_sync(kFull, static_cast<unsigned>(T * T));
      xt[q] = warp_sum_f64(big ? 0.0 : x2);
      scl[q] = __longlong_as_double(static_cast<long long>(2 * (Bl - 127) - 18 + 1023) << 52);
    }
    __syncwarp();
    // A(k), B(k) per level, of the regime each of this lane's k falls in
    int sa[NL][8], sb[NL][8];
#pragma unroll
    for (int u = 0; u < NL; ++u) {
      int pa[8], pb[8];
      scan_row8(sh.d[2 * u], lane, pa);
      scan_row8(sh.d[2 * u + 1], lane, pb);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sa[u][j] = a0[u] + pa[j];
        sb[u][j] = b0[u] + pb[j];
      }
      scan_row8(sh.d[2 * (NL + u)], lane, pa);
      scan_row8(sh.d[2 * (NL + u) + 1], lane, pb);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (8 * lane + j > K) {
          sa[u][j] = a0[NL + u] + pa[j];
          sb[u][j] = b0[NL + u] + pb[j];
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int k = 8 * lane + j;
      const int r0 = k > K ? NL : 0;
      const int F = 256 + k;
      double best = 0.0;
#pragma unroll
      for (int u = 0; u < NL; ++u) {
        // S = C - 2 F A + F^2 B = C + F (F B - 2 A): F B - 2 A fits in 25
        // bits, the product and the (non-negative) sum in 34
        const int inner = F * sb[u][j] - 2 * sa[u][j];
        const long long S = static_cast<long long>(r0 ? cc[NL + u] : cc[u]) +
                            static_cast<long long>(F) * inner;
        const double v = fma(static_cast<double>(S), r0 ? scl[NL + u] : scl[u],
                             r0 ? xt[NL + u] : xt[u]);
        best = u == 0 ? v : fmin(best, v);   // OAS: the smaller of the two scales
      }
      tot[j] += best;
    }
    __syncwarp();   // every lane cleared its entries before the next scatter
  }

  double mn = tot[0];
#pragma unroll
  for (int j = 1; j < 8; ++j) mn = fmin(mn, tot[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mn = fmin(mn, __shfl_xor_sync(kFull, mn, o));
  const double thr = mn * (1.0 + 0x1p-40);
  unsigned m8 = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) m8 |= (tot[j] <= thr ? 1u : 0u) << j;
  const int cnt = static_cast<int>(__reduce_add_sync(kFull, static_cast<unsigned>(__popc(m8))));
  if (cnt == 1 || mn == 0.0) {
    const unsigned mine = m8 ? 8u * lane + __ffs(m8) - 1 : 256u;
    return static_cast<int>(__reduce_min_sync(kFull, mine));
  }
  // near-ties: the element-order double sums decide
  int pos = __popc(m8);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(kFull, pos, o);
    if (lane >= o) pos += t;
  }
  pos -= __popc(m8);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if ((m8 >> j) & 1u) sh.cand[pos++] = static_cast<uint8_t>(8 * lane + j);
  __syncwarp();
  double best = 0.0;
  int bk = 256;
#pragma unroll 1
  for (int o = 0; o < cnt; o += 32) {
    const int idx = o + lane;
    if (idx < cnt) {
      const int kc = sh.cand[idx];
      const double s = macro_sse_k<RULE, BS>(xs, am, kc);
      if (bk == 256 || s < best || (s == best && kc < bk)) {
        best = s;
        bk = kc;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ob = __shfl_xor_sync(kFull, best, o);
    const int ok = __shfl_xor_sync(kFull, bk, o);
    if (ok != 256 && (bk == 256 || ob < best || (ob == best && ok < bk))) {
      best = ob;
      bk = ok;
    }
  }
  __syncwarp();   // cand is free again
  return bk;
}

template <int OP, int RULE, int FMT>
__global__ void __launch_bounds__(kSweepThreads, 4) mbs_sweep_kernel(StreamArgs a) {
  constexpr int BS = FMT == kFmtE2M1B16 ? 16 : 32;   // sub-block size
  __shared__ __align__(16) SweepShared<RULE> shared[kSweepWarps];
  SweepShared<RULE>& sh = shared[threadIdx.x >> 5];
  const int lane = threadIdx.x & 31;
  const int grp = lane >> 3;
  const int l8 = lane & 7;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  double sd = 0.0, sx = 0.0;
#pragma unroll
  for (int q = 0; q < 4 * SweepShared<RULE>::kLevels; ++q) {
    int4* p = reinterpret_cast<int4*>(&sh.d[q][sweep_slot(8 * lane)]);
    p[0] = make_int4(0, 0, 0, 0);
    p[1] = make_int4(0, 0, 0, 0);
  }
  for (int64_t tile = warp; tile * 32 < a.nslices; tile += nwarps) {
    const int64_t c = tile * 32 + lane;
    const bool valid = c < a.nslices;
    uint32_t a16, pa, A;
    bool finite;
    {
      V16 v;
#pragma unroll
      for (int i = 0; i < 8; ++i) v.w[i] = 0;
      if (valid) v = ld_stream32(a.x + 32 * c);
      a16 = amax_bits16(v);
      pa = pair_max(a16);
      A = oct_max(pa);
      finite = A < 0x7F80u;
      __syncwarp();   // the previous tile's reads of xs are done
#pragma unroll
      for (int i = 0; i < 16; ++i) sh.xs[grp][16 * l8 + i] = finite ? fabsf(elem(v, i)) : 0.0f;
      __syncwarp();
    }
    int k = 0;
#pragma unroll 1
    for (int gg = 0; gg < 4; ++gg) {
      const bool fin_g = __shfl_sync(kFull, A, gg << 3) < 0x7F80u;
      uint32_t am[128 / BS];
#pragma unroll
      for (int b = 0; b < 128 / BS; ++b) {
        const uint32_t ab = BS == 32 ? __shfl_sync(kFull, pa, (gg << 3) + 2 * b)
                                     : __shfl_sync(kFull, a16, (gg << 3) + b);
        am[b] = fin_g ? ab : 0u;
      }
      const int kg = sweep_macro<RULE, BS>(sh, gg, am, lane);
      if (gg == grp) k = kg;
    }
    if (!finite) k = 0;
    // the slice again (from L2) rather than held in registers through the sweep
    V16 v, g;
#pragma unroll
    for (int i = 0; i < 8; ++i) v.w[i] = g.w[i] = 0;
    if (valid) {
      v = ld_stream32(a.x + 32 * c);
      if (OP == kOpFakeBwd) g = ld_stream32(a.gy + 32 * c);
    }
    if constexpr (BS == 32)
      process_slice<OP, kFmtE2M1, RULE, kMbsDynamic>(a, v, g, c, valid, lane, pa, k, sd, sx);
    else
      process_slice16<OP, kFmtE2M1B16, RULE, kMbsDynamic>(a, v, g, c, valid, lane, k, sd, sx);
  }
  if (OP == kOpError) reduce_totals<kSweepWarps>(sd, sx, a.totals);
}

// ------------------------------------------------------------- dequantize --

struct DequantArgs {
  const uint8_t* codes;
  const uint8_t* scales;
  const uint8_t* macro;   // may be null
  int64_t nslices;
  uint8_t* out;           // bf16 (32 bytes per slice) or float (64 bytes per slice)
  ScaleMap smap;
};

template <int FMT, int OUT32, int U>
__global__ void __launch_bounds__(kThreads) dequant_kernel(DequantArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  // E2M1 elements (two per byte), and blocks of 16 (one scale per slice)
  constexpr bool kPacked = FMT == kFmtE2M1 || FMT == kFmtE2M1B16 || FMT == kFmtNvfp4;
  constexpr int kSliceShift = (FMT == kFmtE2M1B16 || FMT == kFmtNvfp4) ? 0 : 1;
  for (int64_t tile = warp; tile * 32 * U < a.nslices; tile += nwarps) {
    const int64_t base = tile * 32 * U + lane;
    uint2 c4[U];
    uint4 c8[U];
    int sb[U], kk[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t c = base + 32 * j;
      const bool valid = c < a.nslices;
      if (kPacked) c4[j] = valid ? ld_stream8(a.codes + 8 * c) : make_uint2(0, 0);
      else c8[j] = valid ? ld_stream16(a.codes + 16 * c) : make_uint4(0, 0, 0, 0);
      sb[j] = valid ? a.scales[scale_offset(a.smap, c >> kSliceShift)] : 0;
      kk[j] = (valid && a.macro) ? a.macro[c >> 3] : 0;
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t c = base + 32 * j;
      if (c >= a.nslices) continue;
      const int E = sb[j] - 127;
      if ((FMT == kFmtE2M1 || FMT == kFmtE2M1B16) && kk[j] == 0 && e2m1_table_scale_ok(sb[j])) {
        // common case: the products are normal bf16 values, read straight off
        // a table of the 8 magnitudes scaled by 2^E (exact)
        const V16 b = e2m1x16_to_bf16(c4[j], e2m1_table(E));
        if (OUT32) {
          V16 o0, o1;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            o0.w[2 * i] = b.w[i] << 16;
            o0.w[2 * i + 1] = b.w[i] & 0xFFFF0000u;
            o1.w[2 * i] = b.w[4 + i] << 16;
            o1.w[2 * i + 1] = b.w[4 + i] & 0xFFFF0000u;
          }
          st_stream32(a.out + 64 * c, o0);
          st_stream32(a.out + 64 * c + 32, o1);
        } else {
          st_stream32(a.out + 32 * c, b);
        }
        continue;
      }
      // value * (256 + k) 2^(E-8), or value * s for an NVFP4 scale s (exact);
      // a NaN scale makes every output NaN
      float p;
      bool nan_scale;
      if constexpr (FMT == kFmtNvfp4) {
        p = e4m3_value(sb[j]);
        nan_scale = isnan(p);
      } else {
        p = kk[j] ? static_cast<float>(256 + kk[j]) * pow2f(E - 8) : pow2f(E);
        nan_scale = sb[j] == 255;
      }
      F16 y;
      if constexpr (kPacked) y = dec_e2m1_16(c4[j], p);
      else y = dec_bytes_16<FMT>(c8[j], p);
      if (OUT32) {
        V16 o0, o1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o0.w[i] = (nan_scale || isnan(y.v[i])) ? kNaNf32 : __float_as_uint(y.v[i]);
          o1.w[i] = (nan_scale || isnan(y.v[8 + i])) ? kNaNf32 : __float_as_uint(y.v[8 + i]);
        }
        st_stream32(a.out + 64 * c, o0);
        st_stream32(a.out + 64 * c + 32, o1);
      } else {
        V16 o;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint32_t p2 = pack_bf16x2(y.v[2 * i], y.v[2 * i + 1]);
          if (nan_scale || isnan(y.v[2 * i])) p2 = (p2 & 0xFFFF0000u) | kNaNbf16;
          if (nan_scale || isnan(y.v[2 * i + 1]))
            p2 = (p2 & 0xFFFFu) | (static_cast<uint32_t>(kNaNbf16) << 16);
          o.w[i] = p2;
        }
        st_stream32(a.out + 32 * c, o);
      }
    }
  }
}

// ------------------------------------------------------------- launching --

namespace {

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

// Grid size: one warp per tile when waves == 0, else at most `waves` times the
// resident capacity (SMs x blocks per SM); never more blocks than tiles need.
template <typename K>
int grid_for(K kernel, int64_t tiles, int waves = MX_GRID_WAVES) {
  const int64_t need = (tiles + (kThreads / 32) - 1) / (kThreads / 32);
  if (waves == 0) return static_cast<int>(need > 0 ? need : 1);
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0);
  if (per_sm < 1) per_sm = 1;
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm * waves;
  return static_cast<int>(need < cap ? (need > 0 ? need : 1) : cap);
}

// Slices per lane in flight in the plain streaming kernels (32 bytes each).
#ifndef MX_STREAM_UNROLL
#define MX_STREAM_UNROLL 2
#endif
constexpr int kUnroll = MX_STREAM_UNROLL;
// Slices per lane in flight in the dequantize kernel.
#ifndef MX_DEQUANT_UNROLL
#define MX_DEQUANT_UNROLL 4
#endif

template <int OP, int FMT, int RULE, int MBS>
cudaError_t launch_stream(const StreamArgs& a, cudaStream_t st) {
  // the error kernel ends with one double atomic per CTA: keep its grid small
  const int waves = OP == kOpError ? 1 : MX_GRID_WAVES;
  if constexpr (MBS == kMbsDynamic) {
    auto kern = mbs_sweep_kernel<OP, RULE, FMT>;
    const int64_t tiles = (a.nslices + 31) / 32;
    int64_t grid = (tiles + kSweepWarps - 1) / kSweepWarps;
    if (OP == kOpError) {
      int per_sm = 0;
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kSweepThreads, 0);
      const int64_t cap = static_cast<int64_t>(sm_count()) * (per_sm > 0 ? per_sm : 1);
      if (grid > cap) grid = cap;
    }
    kern<<<static_cast<int>(grid > 0 ? grid : 1), kSweepThreads, 0, st>>>(a);
  } else if constexpr ((OP == kOpQuant || OP == kOpFakeFwd) && RULE == kOas && FMT != kFmtE2M1B16) {
    constexpr int kTile = (kThreads / 32) * 32 * kUnroll;   // slices per CTA
    const int64_t grid = (a.nslices + kTile - 1) / kTile;
    oas_kernel<OP, FMT, MBS, kUnroll><<<static_cast<int>(grid), kThreads, 0, st>>>(a);
  } else {
    constexpr int U = (MBS == kMbsNone) ? kUnroll : 1;
    auto kern = stream_kernel<OP, FMT, RULE, MBS, U>;
    const int grid = grid_for(kern, (a.nslices + 32 * U - 1) / (32 * U), waves);
    kern<<<grid, kThreads, 0, st>>>(a);
  }
  return cudaGetLastError();
}

// One-byte formats: FLOOR, CEIL and (float elements) OAS; no macro factor.
template <int OP, int FMT>
cudaError_t dispatch_bytes(const StreamArgs& a, int rule, cudaStream_t st) {
  if (rule == kFloor) return launch_stream<OP, FMT, kFloor, kMbsNone>(a, st);
  if constexpr (FMT != kFmtInt8) {
    if (rule == kOas) return launch_stream<OP, FMT, kOas, kMbsNone>(a, st);
  }
  return launch_stream<OP, FMT, kCeil, kMbsNone>(a, st);
}

template <int OP>
cudaError_t dispatch_stream(const StreamArgs& a, int fmt, int scaling, cudaStream_t st) {
  const int rule = scaling & 0xF;
  const int mbs = scaling >> 4;
  if (fmt == kFmtNvfp4) return launch_stream<OP, kFmtNvfp4, kFloor, kMbsNone>(a, st);
  if (fmt == kFmtE2M1B16) {
    const int mbs = scaling >> 4;
    if (mbs == kMbsStatic) {
      if (rule == kFloor) return launch_stream<OP, kFmtE2M1B16, kFloor, kMbsStatic>(a, st);
      return launch_stream<OP, kFmtE2M1B16, kOas, kMbsStatic>(a, st);
    }
    if (mbs == kMbsDynamic) {
      if (rule == kFloor) return launch_stream<OP, kFmtE2M1B16, kFloor, kMbsDynamic>(a, st);
      return launch_stream<OP, kFmtE2M1B16, kOas, kMbsDynamic>(a, st);
    }
    switch (rule) {
      case kFloor: return launch_stream<OP, kFmtE2M1B16, kFloor, kMbsNone>(a, st);
      case kCeil: return launch_stream<OP, kFmtE2M1B16, kCeil, kMbsNone>(a, st);
      case kOasRule: return launch_stream<OP, kFmtE2M1B16, kOasRule, kMbsNone>(a, st);
      default: return launch_stream<OP, kFmtE2M1B16, kOas, kMbsNone>(a, st);
    }
  }
  switch (fmt) {
    case kFmtE4M3: return dispatch_bytes<OP, kFmtE4M3>(a, rule, st);
    case kFmtE5M2: return dispatch_bytes<OP, kFmtE5M2>(a, rule, st);
    case kFmtE3M2: return dispatch_bytes<OP, kFmtE3M2>(a, rule, st);
    case kFmtE2M3: return dispatch_bytes<OP, kFmtE2M3>(a, rule, st);
    case kFmtInt8: return dispatch_bytes<OP, kFmtInt8>(a, rule, st);
    default: break;
  }
  if (mbs == kMbsNone) {
    switch (rule) {
      case kFloor: return launch_stream<OP, kFmtE2M1, kFloor, kMbsNone>(a, st);
      case kCeil: return launch_stream<OP, kFmtE2M1, kCeil, kMbsNone>(a, st);
      case kOasRule: return launch_stream<OP, kFmtE2M1, kOasRule, kMbsNone>(a, st);
      default: return launch_stream<OP, kFmtE2M1, kOas, kMbsNone>(a, st);
    }
  }
  if (mbs == kMbsStatic) {
    if (rule == kFloor) return launch_stream<OP, kFmtE2M1, kFloor, kMbsStatic>(a, st);
    return launch_stream<OP, kFmtE2M1, kOas, kMbsStatic>(a, st);
  }
  if (rule == kFloor) return launch_stream<OP, kFmtE2M1, kFloor, kMbsDynamic>(a, st);
  return launch_stream<OP, kFmtE2M1, kOas, kMbsDynamic>(a, st);
}

StreamArgs stream_args(const void* x, int64_t n) {
  StreamArgs a{};
  a.x = static_cast<const uint8_t*>(x);
  a.nslices = n / 16;
  return a;
}

}  // namespace

cudaError_t launch_quantize(const void* x, int64_t n, int fmt, int scaling, void* codes,
                            uint8_t* scales, uint8_t* macro, ScaleMap sm, cudaStream_t st) {
  StreamArgs a = stream_args(x, n);
  a.smap = sm;
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = scales;
  a.macro = macro;
  return dispatch_stream<kOpQuant>(a, fmt, scaling, st);
}

cudaError_t launch_fake_fwd(const void* x, int64_t n, int fmt, int scaling, void* y,
                            uint8_t* scales_out, ScaleMap sm, cudaStream_t st) {
  StreamArgs a = stream_args(x, n);
  a.smap = sm;
  a.out = static_cast<uint8_t*>(y);
  a.scales = scales_out;
  return dispatch_stream<kOpFakeFwd>(a, fmt, scaling, st);
}

cudaError_t launch_fake_bwd(const void* x, const void* gy, int64_t n, int fmt, int scaling,
                            void* gx, cudaStream_t st) {
  StreamArgs a = stream_args(x, n);
  a.gy = static_cast<const uint8_t*>(gy);
  a.out = static_cast<uint8_t*>(gx);
  return dispatch_stream<kOpFakeBwd>(a, fmt, scaling, st);
}

cudaError_t launch_block_error(const void* x, int64_t n, int fmt, int scaling, float* block_sse,
                               double* totals, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(totals, 0, 2 * sizeof(double), st);
  if (e != cudaSuccess) return e;
  if (n == 0) return cudaSuccess;
  StreamArgs a = stream_args(x, n);
  a.block_sse = block_sse;
  a.totals = totals;
  return dispatch_stream<kOpError>(a, fmt, scaling, st);
}

template <int FMT, int U>
void launch_dequant_bytes(const DequantArgs& a, int64_t tiles, int out_fp32, cudaStream_t st) {
  if (out_fp32) {
    auto k = dequant_kernel<FMT, 1, U>;
    k<<<grid_for(k, tiles), kThreads, 0, st>>>(a);
  } else {
    auto k = dequant_kernel<FMT, 0, U>;
    k<<<grid_for(k, tiles), kThreads, 0, st>>>(a);
  }
}

cudaError_t launch_dequantize(const void* codes, const uint8_t* scales, const uint8_t* macro,
                              int64_t n, int fmt, int out_fp32, void* out, ScaleMap sm,
                              cudaStream_t st) {
  DequantArgs a{};
  a.smap = sm;
  a.codes = static_cast<const uint8_t*>(codes);
  a.scales = scales;
  a.macro = macro;
  a.nslices = n / 16;
  a.out = static_cast<uint8_t*>(out);
  constexpr int U = MX_DEQUANT_UNROLL;
  const int64_t tiles = (a.nslices + 32 * U - 1) / (32 * U);
  if (fmt == kFmtE2M1) {
    if (out_fp32) {
      auto k = dequant_kernel<kFmtE2M1, 1, U>;
      k<<<grid_for(k, tiles), kThreads, 0, st>>>(a);
    } else {
      auto k = dequant_kernel<kFmtE2M1, 0, U>;
      k<<<grid_for(k, tiles), kThreads, 0, st>>>(a);
    }
  } else {
    switch (fmt) {
      case kFmtE2M1B16: launch_dequant_bytes<kFmtE2M1B16, U>(a, tiles, out_fp32, st); break;
      case kFmtNvfp4: launch_dequant_bytes<kFmtNvfp4, U>(a, tiles, out_fp32, st); break;
      case kFmtE4M3: launch_dequant_bytes<kFmtE4M3, U>(a, tiles, out_fp32, st); break;
      case kFmtE5M2: launch_dequant_bytes<kFmtE5M2, U>(a, tiles, out_fp32, st); break;
      case kFmtE3M2: launch_dequant_bytes<kFmtE3M2, U>(a, tiles, out_fp32, st); break;
      case kFmtE2M3: launch_dequant_bytes<kFmtE2M3, U>(a, tiles, out_fp32, st); break;
      default: launch_dequant_bytes<kFmtInt8, U>(a, tiles, out_fp32, st); break;
    }
  }
  return cudaGetLastError();
}

}  // namespace mxk
