// MX block-32 kernels for sm_100a: quantize, fake-quant forward/backward,
// block error (one streaming template), and dequantize.
//
// Every kernel is a persistent grid-stride loop over "warp tiles" of 32*U
// consecutive 16-byte chunks (U chunks per lane, all loads of a tile issued
// before any arithmetic so that each lane keeps U x 16 bytes in flight).
// Nothing is staged through shared memory except the 128 values of a macro
// block during the MBS-Dynamic search; no kernel waits on a flag.
//
// Sources restated: "[vLLM] MXFP8/MXFP4: microscaling format quantization"
// (MX format table; MXFP8 block-32 scaling; MXFP4 packing), "[Axolotl] MXFP4
// quantization support" (2-3: block 32, fake-quant of activations and
// weights), "Unveiling the Potential of Quantization with MXFP4" (2.A OAS,
// 2.B MBS, 3-4 QSNR).

#include "mx_device.cuh"
#include "mx_launch.h"

namespace mxk {

struct StreamArgs {
  const uint4* x;     // bf16 input, 8 per chunk
  const uint4* gy;    // bf16 upstream gradient (backward only)
  int64_t nchunks;
  void* codes;        // FP4: 4 bytes per chunk; FP8: 8 bytes per chunk
  uint8_t* scales;    // one byte per block (chunk >> 2)
  uint8_t* macro;     // one byte per macro block (chunk >> 4)
  uint4* out;         // bf16 y (forward) or grad_x (backward)
  float* block_sse;   // one float per block (error)
  double* totals;     // {sum d^2, sum x^2} (error)
};

constexpr int kOpQuant = 0, kOpFakeFwd = 1, kOpFakeBwd = 2, kOpError = 3;
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kThreads = 256;

// Per-block scale state as every lane of the block's quad sees it.
struct BlockScale {
  int byte;       // E8M0 byte (255 for a non-finite block)
  int k;          // macro factor index (0 without MBS)
  bool nonfinite;
};

// Scale decision for the quad holding `v` (all 32 lanes must call it).
template <int FMT, int RULE, int MBS>
__device__ __forceinline__ BlockScale decide_scale(const uint4& v, uint32_t qa, int k) {
  BlockScale s;
  s.nonfinite = qa >= 0x7F80u;
  s.k = k;
  if (MBS == kMbsNone) {
    s.byte = rule_byte<FMT, RULE>(qa);
    if (RULE == kOas) {
      const int b2 = max(static_cast<int>(qa >> 7) - 1, 0);
      const bool need = !s.nonfinite && (qa & 0x7F) > 96 && b2 != s.byte;
      if (__any_sync(kFull, need)) {
        int d = oas_delta8(v, inv_scale_from_byte(s.byte));
        d += __shfl_xor_sync(kFull, d, 1);
        d += __shfl_xor_sync(kFull, d, 2);
        if (need && d > 0) s.byte = b2;
      }
    }
  } else {
    s.byte = mbs_floor_byte(qa, k);
    if (RULE == kOas) {
      const int ex = static_cast<int>(qa >> 7);
      const int m7 = static_cast<int>(qa & 0x7F);
      const int b2 = ex == 0 ? 0 : max(ex - 1 - ((2 * m7 < k) ? 1 : 0), 0);
      const bool need = !s.nonfinite && b2 != s.byte;
      if (__any_sync(kFull, need)) {
        const Thresholds T = mbs_thresholds(k);
        int d = oas_delta_mbs8(v, s.byte, T, k);
        d += __shfl_xor_sync(kFull, d, 1);
        d += __shfl_xor_sync(kFull, d, 2);
        if (need && d > 0) s.byte = b2;
      }
    }
  }
  if (s.nonfinite) s.byte = 255;
  return s;
}

// Dequantized values (exact floats, signed) of one lane's 8 elements.
template <int FMT, int MBS>
__device__ __forceinline__ F8 block_values(const uint4& v, const BlockScale& s, uint32_t& codes4,
                                           uint2& codes8) {
  F8 y;
  const int E = s.byte - 127;
  if (FMT == kFmtE2M1) {
    if (MBS == kMbsNone) {
      codes4 = enc_e2m1_8(scaled8(v, inv_scale_from_byte(s.byte)));
      y = dec_e2m1_8(codes4);
      const float p = pow2f(E);
#pragma unroll
      for (int i = 0; i < 8; ++i) y.v[i] *= p;
    } else {
      const Thresholds T = mbs_thresholds(s.k);
      codes4 = enc_mbs_8(v, s.byte, T);
      y = dec_e2m1_8(codes4);
      // value * (256 + k) is exact (at most 12 bits); so is the power of two.
      const float fk = static_cast<float>(256 + s.k);
      const float p8 = pow2f(E - 8);
#pragma unroll
      for (int i = 0; i < 8; ++i) y.v[i] = (y.v[i] * fk) * p8;
    }
  } else {
    codes8 = enc_e4m3_8(scaled8(v, inv_scale_from_byte(s.byte)));
    y = dec_e4m3_8(codes8);
    const float p = pow2f(E);
#pragma unroll
    for (int i = 0; i < 8; ++i) y.v[i] *= p;
  }
  return y;
}

template <int OP, int FMT, int RULE, int MBS>
__device__ __forceinline__ void process_chunk(const StreamArgs& a, const uint4& v, const uint4& g,
                                              int64_t c, bool valid, int lane, uint32_t qa, int k,
                                              double& sd, double& sx) {
  const BlockScale s = decide_scale<FMT, RULE, MBS>(v, qa, k);

  if (OP == kOpQuant) {
    if (FMT == kFmtE2M1) {
      uint32_t codes;
      if (s.nonfinite) codes = nonfinite_e2m1_8(v);
      else if (MBS == kMbsNone) codes = enc_e2m1_8(scaled8(v, inv_scale_from_byte(s.byte)));
      else codes = enc_mbs_8(v, s.byte, mbs_thresholds(s.k));
      if (valid) st_stream4(static_cast<uint32_t*>(a.codes) + c, codes);
    } else {
      const uint2 codes = s.nonfinite ? nonfinite_e4m3_8(v)
                                      : enc_e4m3_8(scaled8(v, inv_scale_from_byte(s.byte)));
      if (valid) st_stream8(static_cast<uint2*>(a.codes) + c, codes);
    }
    if (valid && (lane & 3) == 0) a.scales[c >> 2] = static_cast<uint8_t>(s.byte);
    if (MBS != kMbsNone && valid && (lane & 15) == 0) a.macro[c >> 4] = static_cast<uint8_t>(s.k);
    return;
  }

  if (OP == kOpFakeFwd) {
    uint4 o;
    if (s.nonfinite) {
      const uint32_t nn = (static_cast<uint32_t>(kNaNbf16) << 16) | kNaNbf16;
      o = make_uint4(nn, nn, nn, nn);
    } else {
      uint32_t c4 = 0;
      uint2 c8 = make_uint2(0, 0);
      const F8 y = block_values<FMT, MBS>(v, s, c4, c8);   // signed, exact
      o.x = pack_bf16x2(y.v[0], y.v[1]);
      o.y = pack_bf16x2(y.v[2], y.v[3]);
      o.z = pack_bf16x2(y.v[4], y.v[5]);
      o.w = pack_bf16x2(y.v[6], y.v[7]);
    }
    if (valid) st_stream16(a.out + c, o);
    if (a.scales && valid && (lane & 3) == 0) a.scales[c >> 2] = static_cast<uint8_t>(s.byte);
    return;
  }

  if (OP == kOpFakeBwd) {
    uint4 o = make_uint4(0, 0, 0, 0);
    if (!s.nonfinite) {
      const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
      const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
      uint32_t ow[4];
      if (MBS == kMbsNone) {
        const float inv = inv_scale_from_byte(s.byte);
        const float lim = Elem<FMT>::maxv;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const bool plo = fabsf(bf_lo(xw[j])) * inv <= lim;
          const bool phi = fabsf(bf_hi(xw[j])) * inv <= lim;
          ow[j] = (plo ? (gw[j] & 0xFFFFu) : 0u) | (phi ? (gw[j] & 0xFFFF0000u) : 0u);
        }
      } else {
        const float m = inv_scale_from_byte(s.byte);
        const float lim = 6.0f * static_cast<float>(256 + s.k) * 0.00390625f;   // 6 f, exact
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const bool plo = fabsf(bf_lo(xw[j])) * m <= lim;
          const bool phi = fabsf(bf_hi(xw[j])) * m <= lim;
          ow[j] = (plo ? (gw[j] & 0xFFFFu) : 0u) | (phi ? (gw[j] & 0xFFFF0000u) : 0u);
        }
      }
      o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
    }
    if (valid) st_stream16(a.out + c, o);
    return;
  }

  if (OP == kOpError) {
    double bd = 0.0, bx = 0.0;
    const float xs[8] = {bf_lo(v.x), bf_hi(v.x), bf_lo(v.y), bf_hi(v.y),
                         bf_lo(v.z), bf_hi(v.z), bf_lo(v.w), bf_hi(v.w)};
    if (s.nonfinite) {
      bd = __int_as_float(0x7FC00000);
#pragma unroll
      for (int i = 0; i < 8; ++i) bx = fma(static_cast<double>(xs[i]), static_cast<double>(xs[i]), bx);
    } else {
      uint32_t c4 = 0;
      uint2 c8 = make_uint2(0, 0);
      const F8 y = block_values<FMT, MBS>(v, s, c4, c8);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const double d = static_cast<double>(xs[i] - y.v[i]);   // exact in float
        bd = fma(d, d, bd);
        bx = fma(static_cast<double>(xs[i]), static_cast<double>(xs[i]), bx);
      }
    }
    double q = bd;
    q += __shfl_xor_sync(kFull, q, 1);
    q += __shfl_xor_sync(kFull, q, 2);
    if (valid) {
      if (a.block_sse && (lane & 3) == 0) a.block_sse[c >> 2] = static_cast<float>(q);
      sd += bd;
      sx += bx;
    }
  }
}

// Warp-wide (within each 16-lane half) maximum of the quad amaxes.
__device__ __forceinline__ uint32_t half_max(uint32_t qa) {
  uint32_t A = max(qa, __shfl_xor_sync(kFull, qa, 4));
  return max(A, __shfl_xor_sync(kFull, A, 8));
}

template <int OP, int FMT, int RULE, int MBS, int U>
__global__ void __launch_bounds__(kThreads) stream_kernel(StreamArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  double sd = 0.0, sx = 0.0;
  for (int64_t tile = warp; tile * 32 * U < a.nchunks; tile += nwarps) {
    const int64_t base = tile * 32 * U + lane;
    uint4 v[U], g[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t c = base + 32 * j;
      v[j] = c < a.nchunks ? ld_stream16(a.x + c) : make_uint4(0, 0, 0, 0);
      if (OP == kOpFakeBwd) g[j] = c < a.nchunks ? ld_stream16(a.gy + c) : make_uint4(0, 0, 0, 0);
      else g[j] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t c = base + 32 * j;
      const uint32_t qa = quad_max(amax_bits8(v[j]));
      int k = 0;
      if (MBS == kMbsStatic) k = mbs_static_k(half_max(qa));
      process_chunk<OP, FMT, RULE, MBS>(a, v[j], g[j], c, c < a.nchunks, lane, qa, k, sd, sx);
    }
  }
  if (OP == kOpError) {
    __shared__ double red[2][kThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sd += __shfl_xor_sync(kFull, sd, o);
      sx += __shfl_xor_sync(kFull, sx, o);
    }
    const int w = threadIdx.x >> 5;
    if (lane == 0) {
      red[0][w] = sd;
      red[1][w] = sx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double td = 0.0, tx = 0.0;
      for (int i = 0; i < kThreads / 32; ++i) {
        td += red[0][i];
        tx += red[1][i];
      }
      atomicAdd(a.totals, td);
      atomicAdd(a.totals + 1, tx);
    }
  }
}

// ------------------------------------------------------- MBS-Dynamic path --

// Sum of squared errors of one 128-element macro block under factor k, in
// double, in element order (each d is exact in float and d*d exact in double,
// so the running sum rounds exactly as a sequential double sum does).
// xs: the 128 magnitudes |x| as floats; amax[4]: sub-block amax bits.
template <int RULE>
__device__ __forceinline__ double macro_sse_k(const float* xs, const uint32_t amax[4], int k) {
  const Thresholds T = mbs_thresholds(k);
  const float fk = static_cast<float>(256 + k);
  double sse = 0.0;
#pragma unroll 1
  for (int b = 0; b < 4; ++b) {
    int byte = mbs_floor_byte(amax[b], k);
    if (RULE == kOas) {
      const int ex = static_cast<int>(amax[b] >> 7);
      const int m7 = static_cast<int>(amax[b] & 0x7F);
      const int b2 = ex == 0 ? 0 : max(ex - 1 - ((2 * m7 < k) ? 1 : 0), 0);
      if (b2 != byte) {
        const float inv1 = inv_scale_from_byte(byte);
        int acc = 0;
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
          const float s = xs[32 * b + i] * inv1;
          const int c1 = mbs_round(s, T);
          const int c2 = mbs_round(s * 0.5f, T);
          const int i1 = __float2int_rn(s * 512.0f - static_cast<float>(e2m1_halves(c1)) * fk);
          const int i2 = __float2int_rn(s * 512.0f - static_cast<float>(2 * e2m1_halves(c2)) * fk);
          acc += i1 * i1 - i2 * i2;
        }
        if (acc > 0) byte = b2;
      }
    }
    const float m = inv_scale_from_byte(byte);                          // 2^-E
    const double p = __longlong_as_double(static_cast<long long>(byte - 127 + 1023) << 52);
#pragma unroll 8
    for (int i = 0; i < 32; ++i) {
      const float s = xs[32 * b + i] * m;
      const int c = mbs_round(s, T);
      // s - h (256 + k) / 512 is exact (both sides are multiples of 2^-9 below 2^5)
      const float ds = s - static_cast<float>(e2m1_halves(c)) * fk * 0.001953125f;
      const double d = static_cast<double>(ds) * p;                             // exact
      sse = fma(d, d, sse);
    }
  }
  return sse;
}

template <int OP, int RULE>
__global__ void __launch_bounds__(kThreads) mbs_dynamic_kernel(StreamArgs a) {
  // two macro blocks per warp step, 16 lanes each; +1 float pads the second
  // half so the two broadcast reads of a step fall in different banks
  __shared__ float stage[kThreads / 32][2][128 + 1];
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int l16 = lane & 15;
  const int w = threadIdx.x >> 5;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  double sd = 0.0, sx = 0.0;
  float* xs = stage[w][half];
  for (int64_t tile = warp; tile * 32 < a.nchunks; tile += nwarps) {
    const int64_t c = tile * 32 + lane;
    const bool valid = c < a.nchunks;
    const uint4 v = valid ? ld_stream16(a.x + c) : make_uint4(0, 0, 0, 0);
    const uint4 g = (OP == kOpFakeBwd && valid) ? ld_stream16(a.gy + c) : make_uint4(0, 0, 0, 0);
    const uint32_t qa = quad_max(amax_bits8(v));
    const uint32_t A = half_max(qa);
    uint32_t amax[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) amax[b] = __shfl_sync(kFull, qa, (half << 4) + 4 * b);
    if (A >= 0x7F80u) {
#pragma unroll
      for (int b = 0; b < 4; ++b) amax[b] = 0;
    }
    // Every lane runs the same search so the shuffles stay converged; a macro
    // block holding NaN/Inf searches zeros and then uses k = 0.
    const bool finite = A < 0x7F80u;
    __syncwarp();
    const float f8[8] = {bf_lo(v.x), bf_hi(v.x), bf_lo(v.y), bf_hi(v.y),
                         bf_lo(v.z), bf_hi(v.z), bf_lo(v.w), bf_hi(v.w)};
#pragma unroll
    for (int i = 0; i < 8; ++i) xs[8 * l16 + i] = finite ? fabsf(f8[i]) : 0.0f;
    __syncwarp();
    double best = 0.0;
    int best_k = -1;
#pragma unroll 1
    for (int j = 0; j < 16; ++j) {
      const int kk = l16 + 16 * j;
      const double s = macro_sse_k<RULE>(xs, amax, kk);
      if (best_k < 0 || s < best) {
        best = s;
        best_k = kk;
      }
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const double ob = __shfl_xor_sync(kFull, best, o);
      const int ok = __shfl_xor_sync(kFull, best_k, o);
      if (ob < best || (ob == best && ok < best_k)) {
        best = ob;
        best_k = ok;
      }
    }
    const int k = finite ? best_k : 0;
    process_chunk<OP, kFmtE2M1, RULE, kMbsDynamic>(a, v, g, c, valid, lane, qa, k, sd, sx);
  }
  if (OP == kOpError) {
    __shared__ double red[2][kThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sd += __shfl_xor_sync(kFull, sd, o);
      sx += __shfl_xor_sync(kFull, sx, o);
    }
    if (lane == 0) {
      red[0][w] = sd;
      red[1][w] = sx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double td = 0.0, tx = 0.0;
      for (int i = 0; i < kThreads / 32; ++i) {
        td += red[0][i];
        tx += red[1][i];
      }
      atomicAdd(a.totals, td);
      atomicAdd(a.totals + 1, tx);
    }
  }
}

// ------------------------------------------------------------- dequantize --

struct DequantArgs {
  const void* codes;
  const uint8_t* scales;
  const uint8_t* macro;   // may be null
  int64_t nchunks;
  void* out;              // bf16 (16 bytes per chunk) or float (32 bytes per chunk)
};

template <int FMT, int OUT32, int U>
__global__ void __launch_bounds__(kThreads) dequant_kernel(DequantArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t tile = warp; tile * 32 * U < a.nchunks; tile += nwarps) {
    const int64_t base = tile * 32 * U + lane;
    uint32_t c4[U];
    uint2 c8[U];
    int sb[U], kk[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t c = base + 32 * j;
      const bool valid = c < a.nchunks;
      if (FMT == kFmtE2M1) c4[j] = valid ? ld_stream4(static_cast<const uint32_t*>(a.codes) + c) : 0u;
      else c8[j] = valid ? ld_stream8(static_cast<const uint2*>(a.codes) + c) : make_uint2(0, 0);
      sb[j] = valid ? a.scales[c >> 2] : 0;
      kk[j] = (valid && a.macro) ? a.macro[c >> 4] : 0;
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t c = base + 32 * j;
      if (c >= a.nchunks) continue;
      F8 y = FMT == kFmtE2M1 ? dec_e2m1_8(c4[j]) : dec_e4m3_8(c8[j]);
      const int E = sb[j] - 127;
      if (kk[j] != 0) {
        const float fk = static_cast<float>(256 + kk[j]);
        const float p8 = pow2f(E - 8);
#pragma unroll
        for (int i = 0; i < 8; ++i) y.v[i] = (y.v[i] * fk) * p8;
      } else {
        const float p = pow2f(E);
#pragma unroll
        for (int i = 0; i < 8; ++i) y.v[i] *= p;
      }
      const bool nan_scale = sb[j] == 255;
      if (OUT32) {
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          o[i] = (nan_scale || isnan(y.v[i])) ? kNaNf32 : __float_as_uint(y.v[i]);
        uint4* dst = static_cast<uint4*>(a.out) + 2 * c;
        st_stream16(dst, make_uint4(o[0], o[1], o[2], o[3]));
        st_stream16(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
      } else {
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t p = pack_bf16x2(y.v[2 * i], y.v[2 * i + 1]);
          if (nan_scale || isnan(y.v[2 * i])) p = (p & 0xFFFF0000u) | kNaNbf16;
          if (nan_scale || isnan(y.v[2 * i + 1])) p = (p & 0xFFFFu) | (static_cast<uint32_t>(kNaNbf16) << 16);
          o[i] = p;
        }
        st_stream16(static_cast<uint4*>(a.out) + c, make_uint4(o[0], o[1], o[2], o[3]));
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

template <typename K>
int grid_for(K kernel, int64_t tiles) {
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0);
  if (per_sm < 1) per_sm = 1;
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
  const int64_t need = (tiles + (kThreads / 32) - 1) / (kThreads / 32);
  return static_cast<int>(need < cap ? (need > 0 ? need : 1) : cap);
}

constexpr int kUnroll = 4;

template <int OP, int FMT, int RULE, int MBS>
cudaError_t launch_stream(const StreamArgs& a, cudaStream_t st) {
  if (MBS == kMbsDynamic) {
    auto kern = mbs_dynamic_kernel<OP, RULE>;
    const int grid = grid_for(kern, (a.nchunks + 31) / 32);
    kern<<<grid, kThreads, 0, st>>>(a);
  } else {
    constexpr int U = (MBS == kMbsNone) ? kUnroll : 2;
    auto kern = stream_kernel<OP, FMT, RULE, MBS, U>;
    const int grid = grid_for(kern, (a.nchunks + 32 * U - 1) / (32 * U));
    kern<<<grid, kThreads, 0, st>>>(a);
  }
  return cudaGetLastError();
}

template <int OP>
cudaError_t dispatch_stream(const StreamArgs& a, int fmt, int scaling, cudaStream_t st) {
  const int rule = scaling & 0xF;
  const int mbs = scaling >> 4;
  if (fmt == kFmtE4M3) {
    if (rule == kFloor) return launch_stream<OP, kFmtE4M3, kFloor, kMbsNone>(a, st);
    return launch_stream<OP, kFmtE4M3, kCeil, kMbsNone>(a, st);
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

}  // namespace

cudaError_t launch_quantize(const void* x, int64_t n, int fmt, int scaling, void* codes,
                            uint8_t* scales, uint8_t* macro, cudaStream_t st) {
  StreamArgs a{};
  a.x = static_cast<const uint4*>(x);
  a.nchunks = n / 8;
  a.codes = codes;
  a.scales = scales;
  a.macro = macro;
  return dispatch_stream<kOpQuant>(a, fmt, scaling, st);
}

cudaError_t launch_fake_fwd(const void* x, int64_t n, int fmt, int scaling, void* y,
                            uint8_t* scales_out, cudaStream_t st) {
  StreamArgs a{};
  a.x = static_cast<const uint4*>(x);
  a.nchunks = n / 8;
  a.out = static_cast<uint4*>(y);
  a.scales = scales_out;
  return dispatch_stream<kOpFakeFwd>(a, fmt, scaling, st);
}

cudaError_t launch_fake_bwd(const void* x, const void* gy, int64_t n, int fmt, int scaling,
                            void* gx, cudaStream_t st) {
  StreamArgs a{};
  a.x = static_cast<const uint4*>(x);
  a.gy = static_cast<const uint4*>(gy);
  a.nchunks = n / 8;
  a.out = static_cast<uint4*>(gx);
  return dispatch_stream<kOpFakeBwd>(a, fmt, scaling, st);
}

cudaError_t launch_block_error(const void* x, int64_t n, int fmt, int scaling, float* block_sse,
                               double* totals, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(totals, 0, 2 * sizeof(double), st);
  if (e != cudaSuccess) return e;
  if (n == 0) return cudaSuccess;
  StreamArgs a{};
  a.x = static_cast<const uint4*>(x);
  a.nchunks = n / 8;
  a.block_sse = block_sse;
  a.totals = totals;
  return dispatch_stream<kOpError>(a, fmt, scaling, st);
}

cudaError_t launch_dequantize(const void* codes, const uint8_t* scales, const uint8_t* macro,
                              int64_t n, int fmt, int out_fp32, void* out, cudaStream_t st) {
  DequantArgs a{};
  a.codes = codes;
  a.scales = scales;
  a.macro = macro;
  a.nchunks = n / 8;
  a.out = out;
  constexpr int U = 4;
  const int64_t tiles = (a.nchunks + 32 * U - 1) / (32 * U);
  if (fmt == kFmtE2M1) {
    if (out_fp32) {
      auto k = dequant_kernel<kFmtE2M1, 1, U>;
      k<<<grid_for(k, tiles), kThreads, 0, st>>>(a);
    } else {
      auto k = dequant_kernel<kFmtE2M1, 0, U>;
      k<<<grid_for(k, tiles), kThreads, 0, st>>>(a);
    }
  } else {
    if (out_fp32) {
      auto k = dequant_kernel<kFmtE4M3, 1, U>;
      k<<<grid_for(k, tiles), kThreads, 0, st>>>(a);
    } else {
      auto k = dequant_kernel<kFmtE4M3, 0, U>;
      k<<<grid_for(k, tiles), kThreads, 0, st>>>(a);
    }
  }
  return cudaGetLastError();
}

}  // namespace mxk
