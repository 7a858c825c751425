// BATQuant apply step, alone or fused with the MX quantizer, for sm_100a.
//
// "BATQuant: Outlier-resilient MXFP4 Quantization via Learnable Block-wise
// Optimization", technical summary section 2: every 32-element MX block j of
// a row is multiplied by its own matrix P_j = B_j (x) A (A is a x a and
// shared by all blocks, B_j is b x b and private, a b = 32), clipped to
// [beta^min_j min y, beta^max_j max y] of the block, and quantized. With the
// element index i = p a + q the Kronecker structure gives
//   y[r a + s] = sum_p B_j[p][r] Z[p][s],   Z[p][s] = sum_q x[p a + q] A[q][s],
// two small contractions (a + b multiply-adds per element instead of 32).
//
// Lane layout: the streaming quantizer's, a lane pair per block and 16
// elements per lane. For a <= 16 a lane holds b/2 whole rows of X and
// computes their Z rows; stage 2 needs all b rows, so each lane sums its own
// rows' terms into all 32 outputs and the pair swaps the partial sums of each
// other's outputs (16 shuffles). For a = 32 the swap happens in stage 1. The
// arithmetic order is therefore fixed as: fp32 fma chains in index order from
// -0, and where an index runs over both halves of the block, the chain of the
// lower half plus the chain of the upper half (fp32 addition commutes, so
// both lanes get the same bits). The clip uses exact comparisons; a block
// whose transformed values are not all finite is not clipped. One round to
// bf16 (NaN canonical), then the per-slice quantizer, unchanged.
//
// All of it is CUDA-core work: a contraction of 32-element vectors with
// 4 x 4 ... 32 x 32 factors whose rounding must be reproducible does not fit
// the tensor cores (whose accumulation order is not specified), and the
// kernel stays close to its issue-rate bound rather than to HBM.
//
// A CTA owns one 512-column chunk of many rows, so each lane's block column
// and parameters are fixed. A is staged once per CTA in shared memory, and
// copied into registers for a <= 4. A lane's terms of B_j sit in registers
// (a >= 4) or in shared memory (a <= 2), and its thresholds in registers.
// Rows stream through a per-thread cp.async ring in shared memory. Both
// stages issue packed fp32 fmas (two outputs per instruction).

#include "mx_stream.cuh"

namespace mxk {

constexpr int kOpBatApply = 4;   // write the transformed bf16 rows

struct BatParams {
  const float* A;      // [a, a] row-major
  const float* B;      // [cols / 32, b, b] row-major
  const float* bmin;   // [cols / 32] or null (then bmax is null too: no clip)
  const float* bmax;
  int64_t rows;
  int64_t spr;         // 16-element slices per row (cols / 16, even)
  int nchunks;         // 32-slice column chunks per row, ceil(spr / 32)
};

// Row tiles in flight per thread (cp.async ring in shared memory).
#ifndef MX_BAT_STAGES
#define MX_BAT_STAGES 6
#endif
constexpr int kBatStages = MX_BAT_STAGES;
constexpr int kBatRing = kBatStages * 32 * kThreads;   // ring bytes

// A is copied into registers for a <= MX_BAT_REG_A (else read from shared
// memory, two pairs per 16-byte load, shared by the lane's rows).
#ifndef MX_BAT_REG_A
#define MX_BAT_REG_A 4
#endif

// Shared-memory layout of B for a <= 2 (where a lane's rows of B_j do not fit
// in registers): the 16 blocks of the CTA's column chunk, rows of b floats,
// the rows of the block's second half (p >= b/2) 16 bytes further on, blocks
// `stride` floats apart. A lane reads 16 bytes at a time; with stride / 4 = 2 (mod 8) and the
// half offset, the 8 lanes of each quarter-warp phase (4 blocks x 2 halves)
// hit 8 distinct 16-byte bank groups, for its own columns and the partner's.
template <int AD> struct BatSmemB {
  static constexpr int BD = 32 / AD;
  static constexpr int RH = BD / 2;
  static constexpr int pitch = BD;
  static constexpr int half_off = 4;
  static constexpr int stride = AD == 1 ? 1032 : 264;
  static constexpr int floats = AD <= 2 ? 16 * stride : 0;
  __host__ __device__ static constexpr int offset(int p, int r) { return p * pitch + (p >= RH ? half_off : 0) + r; }
};

// A's shared-memory slot, rounded up to 16 bytes so that B stays aligned.
template <int AD> __host__ __device__ constexpr int bat_a_floats() { return (AD * AD + 3) / 4 * 4; }

template <int AD>
constexpr size_t bat_smem_bytes() {
  return kBatRing + sizeof(float) * (bat_a_floats<AD>() + BatSmemB<AD>::floats);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
__device__ __forceinline__ float min_nan(float a, float b) {
  float d;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Per-half clamp of packed bf16: min(max(v, lo), hi) (a NaN bound is ignored).
__device__ __forceinline__ uint32_t clamp_bf16x2(uint32_t v, uint32_t lo, uint32_t hi) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(v), "r"(lo));
  asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(d), "r"(hi));
  return d;
}

// The parameters one lane needs, for its fixed block column j and half h.
template <int AD>
struct LaneParams {
  static constexpr int BD = 32 / AD;
  static constexpr int RH = BD >= 2 ? BD / 2 : 1;   // rows of X (and Y) per lane
  static constexpr bool kRegB = AD >= 4;             // B_j's terms in registers
  static constexpr bool kRegA = AD <= MX_BAT_REG_A;  // A in registers
  float A[kRegA ? AD * AD : 1];
  float bo[kRegB ? RH * RH : 1];   // B_j[h RH + pp][h RH + rl]: own outputs (a = 32: B_j[0][0])
  float bt[kRegB ? RH * RH : 1];   // B_j[h RH + pp][(1 - h) RH + rl]: the partner's outputs
  const float* Bl;                 // a <= 2: row h RH of B_j in shared memory
  float bmin, bmax;
};

template <int AD>
__device__ __forceinline__ V16 bat_finish(float (&y)[16], const LaneParams<AD>& L, bool clip);

// The transformed, clipped 16 values of this lane (elements 16 h .. 16 h + 15
// of its block) as packed bf16.
template <int AD>
__device__ __forceinline__ V16 bat_slice(const V16& v, int h, const LaneParams<AD>& L,
                                         const float* As, bool clip) {
  constexpr int RH = LaneParams<AD>::RH;
  float xf[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) xf[i] = elem(v, i);

  float y[16];
  if constexpr (AD == 32) {
    // stage 1 over this lane's half of q, for its own 16 outputs and the
    // partner's (pairs of adjacent outputs per instruction); the partner's
    // partial sums complete this lane's outputs
    float2 zo[8], zt[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) zo[m] = zt[m] = make_float2(-0.0f, -0.0f);
    const float* Ah = As + (16 * h) * 32;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const float2 xq = make_float2(xf[q], xf[q]);
      const float4* ro = reinterpret_cast<const float4*>(Ah + q * 32 + 16 * h);
      const float4* rt = reinterpret_cast<const float4*>(Ah + q * 32 + 16 * (1 - h));
#pragma unroll
      for (int m4 = 0; m4 < 4; ++m4) {
        const float4 ao = ro[m4], at = rt[m4];
        zo[2 * m4] = ffma2(xq, make_float2(ao.x, ao.y), zo[2 * m4]);
        zo[2 * m4 + 1] = ffma2(xq, make_float2(ao.z, ao.w), zo[2 * m4 + 1]);
        zt[2 * m4] = ffma2(xq, make_float2(at.x, at.y), zt[2 * m4]);
        zt[2 * m4 + 1] = ffma2(xq, make_float2(at.z, at.w), zt[2 * m4 + 1]);
      }
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const float z0 = __fadd_rn(zo[m].x, __shfl_xor_sync(kFull, zt[m].x, 1));
      const float z1 = __fadd_rn(zo[m].y, __shfl_xor_sync(kFull, zt[m].y, 1));
      y[2 * m] = fmaf(L.bo[0], z0, -0.0f);
      y[2 * m + 1] = fmaf(L.bo[0], z1, -0.0f);
    }
  } else if constexpr (AD == 1) {
    // Z = x A[0][0]; stage 2 is the full 32 x 32 B_j (no decomposition), in
    // pairs of adjacent output rows: B_j's row pairs come 4 floats per load
    float z[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) z[i] = fmaf(xf[i], L.A[0], -0.0f);
    float2 yo[8], yt[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) yo[i] = yt[i] = make_float2(-0.0f, -0.0f);
    const float* Bo = L.Bl + h * RH;
    const float* Bt = L.Bl + (1 - h) * RH;
#pragma unroll
    for (int pp = 0; pp < RH; ++pp) {
      const float2 zd = make_float2(z[pp], z[pp]);
#pragma unroll
      for (int q4 = 0; q4 < RH / 4; ++q4) {
        const float4 bo = reinterpret_cast<const float4*>(Bo + pp * BatSmemB<AD>::pitch)[q4];
        const float4 bt = reinterpret_cast<const float4*>(Bt + pp * BatSmemB<AD>::pitch)[q4];
        yo[2 * q4] = ffma2(make_float2(bo.x, bo.y), zd, yo[2 * q4]);
        yo[2 * q4 + 1] = ffma2(make_float2(bo.z, bo.w), zd, yo[2 * q4 + 1]);
        yt[2 * q4] = ffma2(make_float2(bt.x, bt.y), zd, yt[2 * q4]);
        yt[2 * q4 + 1] = ffma2(make_float2(bt.z, bt.w), zd, yt[2 * q4 + 1]);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      y[2 * j] = __fadd_rn(yo[j].x, __shfl_xor_sync(kFull, yt[j].x, 1));
      y[2 * j + 1] = __fadd_rn(yo[j].y, __shfl_xor_sync(kFull, yt[j].y, 1));
    }
  } else if constexpr (AD == 2) {
    // stage 1 in pairs (Z[p][0], Z[p][1]); stage 2 in pairs of adjacent
    // output rows (Y[r][s], Y[r+1][s]) from 16-byte loads of B_j's rows
    float2 z2[8];
#pragma unroll
    for (int pp = 0; pp < RH; ++pp) {
      float2 acc = make_float2(-0.0f, -0.0f);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float xv = xf[pp * 2 + q];
        acc = ffma2(make_float2(xv, xv), make_float2(L.A[q * 2], L.A[q * 2 + 1]), acc);
      }
      z2[pp] = acc;
    }
    float2 yo[2][4], yt[2][4];   // [s][row pair]
#pragma unroll
    for (int i = 0; i < 4; ++i) yo[0][i] = yo[1][i] = yt[0][i] = yt[1][i] = make_float2(-0.0f, -0.0f);
    const float* Bo = L.Bl + h * RH;
    const float* Bt = L.Bl + (1 - h) * RH;
#pragma unroll
    for (int pp = 0; pp < RH; ++pp) {
      const float2 zd0 = make_float2(z2[pp].x, z2[pp].x);
      const float2 zd1 = make_float2(z2[pp].y, z2[pp].y);
#pragma unroll
      for (int q4 = 0; q4 < RH / 4; ++q4) {
        const float4 bo = reinterpret_cast<const float4*>(Bo + pp * BatSmemB<AD>::pitch)[q4];
        const float4 bt = reinterpret_cast<const float4*>(Bt + pp * BatSmemB<AD>::pitch)[q4];
        yo[0][2 * q4] = ffma2(make_float2(bo.x, bo.y), zd0, yo[0][2 * q4]);
        yo[0][2 * q4 + 1] = ffma2(make_float2(bo.z, bo.w), zd0, yo[0][2 * q4 + 1]);
        yo[1][2 * q4] = ffma2(make_float2(bo.x, bo.y), zd1, yo[1][2 * q4]);
        yo[1][2 * q4 + 1] = ffma2(make_float2(bo.z, bo.w), zd1, yo[1][2 * q4 + 1]);
        yt[0][2 * q4] = ffma2(make_float2(bt.x, bt.y), zd0, yt[0][2 * q4]);
        yt[0][2 * q4 + 1] = ffma2(make_float2(bt.z, bt.w), zd0, yt[0][2 * q4 + 1]);
        yt[1][2 * q4] = ffma2(make_float2(bt.x, bt.y), zd1, yt[1][2 * q4]);
        yt[1][2 * q4 + 1] = ffma2(make_float2(bt.z, bt.w), zd1, yt[1][2 * q4 + 1]);
      }
    }
    // element r * 2 + s of this lane's half
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int sc = 0; sc < 2; ++sc) {
        y[(2 * j) * 2 + sc] = __fadd_rn(yo[sc][j].x, __shfl_xor_sync(kFull, yt[sc][j].x, 1));
        y[(2 * j + 1) * 2 + sc] = __fadd_rn(yo[sc][j].y, __shfl_xor_sync(kFull, yt[sc][j].y, 1));
      }
    }
  } else {
    // pairs (s, s + 1) of adjacent outputs per instruction in both stages;
    // each A pair serves the lane's RH rows (the chains stay in q order)
    constexpr int AH = AD / 2;
    float2 z2[8];   // Z rows h RH .. h RH + RH - 1, column pairs
#pragma unroll
    for (int i = 0; i < 8; ++i) z2[i] = make_float2(-0.0f, -0.0f);
#pragma unroll
    for (int q = 0; q < AD; ++q) {
      float2 aq[AH];
      if constexpr (LaneParams<AD>::kRegA) {
#pragma unroll
        for (int m = 0; m < AH; ++m) aq[m] = make_float2(L.A[q * AD + 2 * m], L.A[q * AD + 2 * m + 1]);
      } else if constexpr (AD >= 4) {
#pragma unroll
        for (int m4 = 0; m4 < AD / 4; ++m4) {
          const float4 a4 = reinterpret_cast<const float4*>(As + q * AD)[m4];
          aq[2 * m4] = make_float2(a4.x, a4.y);
          aq[2 * m4 + 1] = make_float2(a4.z, a4.w);
        }
      } else {
        aq[0] = *reinterpret_cast<const float2*>(As + q * AD);
      }
#pragma unroll
      for (int pp = 0; pp < RH; ++pp) {
        const float xv = xf[pp * AD + q];
#pragma unroll
        for (int m = 0; m < AH; ++m) z2[pp * AH + m] = ffma2(make_float2(xv, xv), aq[m], z2[pp * AH + m]);
      }
    }
    // stage 2: this lane's rows' terms of its own outputs (rows h RH ..)
    // and of the partner's outputs (rows (1 - h) RH ..)
    float2 yo[8], yt[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) yo[i] = yt[i] = make_float2(-0.0f, -0.0f);
#pragma unroll
    for (int pp = 0; pp < RH; ++pp) {
#pragma unroll
      for (int rl = 0; rl < RH; ++rl) {
        static_assert(LaneParams<AD>::kRegB, "a >= 4 keeps B_j's terms in registers");
        const float bo = L.bo[pp * RH + rl];
        const float bt = L.bt[pp * RH + rl];
#pragma unroll
        for (int m = 0; m < AH; ++m) {
          yo[rl * AH + m] = ffma2(make_float2(bo, bo), z2[pp * AH + m], yo[rl * AH + m]);
          yt[rl * AH + m] = ffma2(make_float2(bt, bt), z2[pp * AH + m], yt[rl * AH + m]);
        }
      }
    }
    // __fadd_rn: a one-term chain (b = 2) is a rounded product, which must
    // not be contracted with this addition into one fma
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      y[2 * i] = __fadd_rn(yo[i].x, __shfl_xor_sync(kFull, yt[i].x, 1));
      y[2 * i + 1] = __fadd_rn(yo[i].y, __shfl_xor_sync(kFull, yt[i].y, 1));
    }
  }

  return bat_finish<AD>(y, L, clip);
}

// a = 2 (b = 16) for two rows u, w of the same column chunk (so the same B_j)
// at once: the transform of bat_slice, each 16-byte load of B_j's rows
// serving both rows, every output's fma chain in the same order (so the
// results are bat_slice's bit for bit). Stage 2 runs in two passes, this
// lane's own outputs and then the partner's, to bound the live registers.
__device__ __forceinline__ void bat_transform2_a2(const V16& vu, const V16& vw, int h,
                                                  const LaneParams<2>& L, float (&yu)[16],
                                                  float (&yw)[16]) {
  constexpr int RH = LaneParams<2>::RH;   // 8
  float2 zu[8], zw[8];
#pragma unroll
  for (int pp = 0; pp < RH; ++pp) {
    float2 au = make_float2(-0.0f, -0.0f), aw = make_float2(-0.0f, -0.0f);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float2 aq = make_float2(L.A[q * 2], L.A[q * 2 + 1]);
      const float xu = elem(vu, pp * 2 + q), xw = elem(vw, pp * 2 + q);
      au = ffma2(make_float2(xu, xu), aq, au);
      aw = ffma2(make_float2(xw, xw), aq, aw);
    }
    zu[pp] = au;
    zw[pp] = aw;
  }
  // pass 1: own outputs (rows h RH .. of Y), pass 2: the partner's
  float2 ou[2][4], ow[2][4];   // [s][row pair]
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    float2 cu[2][4], cw[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) cu[0][i] = cu[1][i] = cw[0][i] = cw[1][i] = make_float2(-0.0f, -0.0f);
    const float* Bc = L.Bl + (pass == 0 ? h : 1 - h) * RH;
#pragma unroll
    for (int pp = 0; pp < RH; ++pp) {
      const float2 u0 = make_float2(zu[pp].x, zu[pp].x), u1 = make_float2(zu[pp].y, zu[pp].y);
      const float2 w0 = make_float2(zw[pp].x, zw[pp].x), w1 = make_float2(zw[pp].y, zw[pp].y);
#pragma unroll
      for (int q4 = 0; q4 < RH / 4; ++q4) {
        const float4 b = reinterpret_cast<const float4*>(Bc + pp * BatSmemB<2>::pitch)[q4];
        const float2 b01 = make_float2(b.x, b.y), b23 = make_float2(b.z, b.w);
        cu[0][2 * q4] = ffma2(b01, u0, cu[0][2 * q4]);
        cu[0][2 * q4 + 1] = ffma2(b23, u0, cu[0][2 * q4 + 1]);
        cu[1][2 * q4] = ffma2(b01, u1, cu[1][2 * q4]);
        cu[1][2 * q4 + 1] = ffma2(b23, u1, cu[1][2 * q4 + 1]);
        cw[0][2 * q4] = ffma2(b01, w0, cw[0][2 * q4]);
        cw[0][2 * q4 + 1] = ffma2(b23, w0, cw[0][2 * q4 + 1]);
        cw[1][2 * q4] = ffma2(b01, w1, cw[1][2 * q4]);
        cw[1][2 * q4 + 1] = ffma2(b23, w1, cw[1][2 * q4 + 1]);
      }
    }
    if (pass == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ou[0][i] = cu[0][i];
        ou[1][i] = cu[1][i];
        ow[0][i] = cw[0][i];
        ow[1][i] = cw[1][i];
      }
    } else {
      // element r * 2 + s of this lane's half: own chain + the partner's
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int sc = 0; sc < 2; ++sc) {
          yu[(2 * j) * 2 + sc] = __fadd_rn(ou[sc][j].x, __shfl_xor_sync(kFull, cu[sc][j].x, 1));
          yu[(2 * j + 1) * 2 + sc] = __fadd_rn(ou[sc][j].y, __shfl_xor_sync(kFull, cu[sc][j].y, 1));
          yw[(2 * j) * 2 + sc] = __fadd_rn(ow[sc][j].x, __shfl_xor_sync(kFull, cw[sc][j].x, 1));
          yw[(2 * j + 1) * 2 + sc] = __fadd_rn(ow[sc][j].y, __shfl_xor_sync(kFull, cw[sc][j].y, 1));
        }
      }
    }
  }
}

// The clip of the lane's 16 transformed values and their rounding to bf16.
template <int AD>
__device__ __forceinline__ V16 bat_finish(float (&y)[16], const LaneParams<AD>& L, bool clip) {
  uint32_t lo2 = 0, hi2 = 0;
  bool packed_clip = false;
  if (clip) {
    float mx = y[0], mn = y[0];
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      mx = max_nan(mx, y[i]);
      mn = min_nan(mn, y[i]);
    }
    mx = max_nan(mx, __shfl_xor_sync(kFull, mx, 1));
    mn = min_nan(mn, __shfl_xor_sync(kFull, mn, 1));
    if (isfinite(mx) && isfinite(mn)) {
      const float lo = __fmul_rn(L.bmin, mn);
      const float hi = __fmul_rn(L.bmax, mx);
      lo2 = pack_bf16x2(lo, lo);
      hi2 = pack_bf16x2(hi, hi);
      if ((lo2 & 0x7FFFu) != 0 && (hi2 & 0x7FFFu) != 0) {
        // Rounding to bf16 is monotone, so it commutes with min and max:
        // clamping the rounded values to the rounded bounds gives the
        // rounded clamp. With both rounded bounds nonzero a tie is between
        // identical values, so the bits agree too (a NaN bound is ignored
        // by both forms).
        packed_clip = true;
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float t = y[i] < lo ? lo : y[i];
          y[i] = t > hi ? hi : t;
        }
      }
    }
  }
  V16 o;
#pragma unroll
  for (int i = 0; i < 8; ++i) o.w[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
  if (packed_clip) {
#pragma unroll
    for (int i = 0; i < 8; ++i) o.w[i] = clamp_bf16x2(o.w[i], lo2, hi2);
  }
  return o;
}

// NaN halves of a slice -> the canonical quiet NaN 0x7FC0 (only called for
// blocks whose max magnitude is NaN or Inf).
__device__ __forceinline__ void canonical_nan(V16& v) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t w = v.w[i];
    if ((w & 0x7FFFu) > 0x7F80u) w = (w & 0xFFFF0000u) | kNaNbf16;
    if (((w >> 16) & 0x7FFFu) > 0x7F80u) w = (w & 0xFFFFu) | (static_cast<uint32_t>(kNaNbf16) << 16);
    v.w[i] = w;
  }
}

// One CTA owns one 32-slice column chunk (16 blocks, 512 columns) of the rows
// g * 8 + w + t * G * 8 (warp w, CTA group g of G): each lane's block column,
// and so its parameters, never changes, and a warp reads 1 KB of one row per
// step. Each thread streams its 32 bytes of successive rows through a ring of
// kBatStages slots (cp.async, waited per thread: no block-wide barrier after
// the parameters are staged).
// Resident CTAs per SM the register budget is cut for: 3 (80 registers) where
// that costs no or few spills, else 2.
#ifndef MX_BAT_MINB_WIDE
#define MX_BAT_MINB_WIDE 3
#endif
// a = 2 carries two rows per step (twice the live values): 2 CTAs per SM.
#ifndef MX_BAT_MINB_A2
#define MX_BAT_MINB_A2 2
#endif
__host__ __device__ constexpr int bat_min_blocks(int ad) {
  return (ad == 8 || ad == 16) ? 3 : (ad == 32 ? MX_BAT_MINB_WIDE : (ad == 2 ? MX_BAT_MINB_A2 : 2));
}

template <int AD, int OP, int FMT, int RULE, int MBS>
__global__ void __launch_bounds__(kThreads, bat_min_blocks(AD)) bat_kernel(StreamArgs a, BatParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  float* As = reinterpret_cast<float*>(smem + kBatRing);
  float* Bs = As + bat_a_floats<AD>();
  const int cc = blockIdx.x % p.nchunks;
  const int64_t g = blockIdx.x / p.nchunks;
  const int64_t G = gridDim.x / p.nchunks;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int64_t cs = static_cast<int64_t>(cc) * 32 + lane;   // slice within the row
  const bool col_ok = cs < p.spr;
  const int h = lane & 1;
  const int64_t nb = p.spr >> 1;
  const int64_t j = col_ok ? (cs >> 1) : 0;

  for (int i = tid; i < AD * AD; i += kThreads) As[i] = p.A[i];
  if constexpr (AD <= 2) {
    using SB = BatSmemB<AD>;
    for (int i = tid; i < 16 * SB::BD * SB::BD; i += kThreads) {
      const int jl = i / (SB::BD * SB::BD), e = i % (SB::BD * SB::BD);
      const int64_t jj = static_cast<int64_t>(cc) * 16 + jl;
      Bs[jl * SB::stride + SB::offset(e / SB::BD, e % SB::BD)] =
          jj < nb ? p.B[jj * SB::BD * SB::BD + e] : 0.0f;
    }
  }
  __syncthreads();

  LaneParams<AD> L;
  constexpr int BD = LaneParams<AD>::BD, RH = LaneParams<AD>::RH;
  if constexpr (LaneParams<AD>::kRegA) {
#pragma unroll
    for (int i = 0; i < AD * AD; ++i) L.A[i] = As[i];
  } else {
    L.A[0] = As[0];
  }
  if constexpr (AD == 32) {
    L.bo[0] = p.B[j];
    L.bt[0] = 0.0f;
  } else if constexpr (LaneParams<AD>::kRegB) {
    const float* Bj = p.B + j * (BD * BD) + (h * RH) * BD;
#pragma unroll
    for (int pp = 0; pp < RH; ++pp) {
#pragma unroll
      for (int rl = 0; rl < RH; ++rl) {
        L.bo[pp * RH + rl] = Bj[pp * BD + h * RH + rl];
        L.bt[pp * RH + rl] = Bj[pp * BD + (1 - h) * RH + rl];
      }
    }
  } else {
    L.bo[0] = L.bt[0] = 0.0f;
  }
  // a <= 2: this lane's rows h RH .. of B_j in shared memory
  L.Bl = Bs + (lane >> 1) * BatSmemB<AD>::stride + BatSmemB<AD>::offset(h * RH, 0);
  const bool clip = p.bmin != nullptr;
  L.bmin = clip ? p.bmin[j] : 0.0f;
  L.bmax = clip ? p.bmax[j] : 0.0f;

  uint8_t* slot0 = smem + tid * 16;   // slot s, half k at slot0 + (2 s + k) * kThreads * 16
  const int64_t rstride = G * (kThreads / 32);
  auto issue = [&](int64_t r, int st) {
    const bool ok = col_ok && r < p.rows;
    const uint8_t* src = ok ? a.x + ((r * p.spr + cs) << 5) : a.x;
    const int n = ok ? 16 : 0;
    cp_async16(slot0 + (2 * st) * kThreads * 16, src, n);
    cp_async16(slot0 + (2 * st + 1) * kThreads * 16, ok ? src + 16 : src, n);
    cp_async_commit();
  };
  const int64_t r0 = g * (kThreads / 32) + w;
#pragma unroll
  for (int d = 0; d < kBatStages - 1; ++d) issue(r0 + d * rstride, d);

  double sd = 0.0, sx = 0.0;
  int st = 0;
  auto read_slot = [&](int sl) {
    V16 v;
    const uint4 lo = *reinterpret_cast<const uint4*>(slot0 + (2 * sl) * kThreads * 16);
    const uint4 hi = *reinterpret_cast<const uint4*>(slot0 + (2 * sl + 1) * kThreads * 16);
    v.w[0] = lo.x; v.w[1] = lo.y; v.w[2] = lo.z; v.w[3] = lo.w;
    v.w[4] = hi.x; v.w[5] = hi.y; v.w[6] = hi.z; v.w[7] = hi.w;
    return v;
  };
  auto emit = [&](int64_t r, V16& yv) {
    const int64_t c = r * p.spr + cs;
    const uint32_t pa = pair_max(amax_bits16(yv));
    if (pa >= 0x7F80u) canonical_nan(yv);
    if constexpr (OP == kOpBatApply) {
      if (col_ok) st_stream32(a.out + 32 * c, yv);
    } else {
      int k = 0;
      if (MBS == kMbsStatic) k = mbs_static_k(oct_max(pa));
      process_slice<kOpQuant, FMT, RULE, MBS>(a, yv, yv, c, col_ok, lane, pa, k, sd, sx);
    }
  };
  if constexpr (AD == 2) {
    // two rows (r, r + rstride) per step: the ring's two oldest slots are
    // read, refilled with the rows kBatStages - 1 and kBatStages strides on,
    // and both rows go through the transform together
    static_assert(kBatStages >= 3, "two rows per step need three slots or more");
    for (int64_t r = r0; r < p.rows; r += 2 * rstride) {
      cp_async_wait<kBatStages - 3>();
      const V16 vu = read_slot(st);
      const V16 vw = read_slot(st + 1 == kBatStages ? 0 : st + 1);
      issue(r + (kBatStages - 1) * rstride, st == 0 ? kBatStages - 1 : st - 1);
      issue(r + kBatStages * rstride, st);
      st = st + 2 >= kBatStages ? st + 2 - kBatStages : st + 2;
      float yu[16], yw[16];
      bat_transform2_a2(vu, vw, h, L, yu, yw);
      V16 ou = bat_finish<AD>(yu, L, clip);
      emit(r, ou);
      if (r + rstride < p.rows) {   // warp-uniform: rows are per warp
        V16 ow = bat_finish<AD>(yw, L, clip);
        emit(r + rstride, ow);
      }
    }
  } else {
    for (int64_t r = r0; r < p.rows; r += rstride) {
      issue(r + (kBatStages - 1) * rstride, st == 0 ? kBatStages - 1 : st - 1);
      cp_async_wait<kBatStages - 1>();
      const V16 v = read_slot(st);
      st = st == kBatStages - 1 ? 0 : st + 1;
      V16 yv = bat_slice<AD>(v, h, L, As, clip);
      emit(r, yv);
    }
  }
  cp_async_wait<0>();
}

namespace {

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

template <int AD, int OP, int FMT, int RULE, int MBS>
cudaError_t launch_bat_kernel(const StreamArgs& a, const BatParams& p, cudaStream_t st) {
  auto kern = bat_kernel<AD, OP, FMT, RULE, MBS>;
  constexpr size_t smem = bat_smem_bytes<AD>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (per_sm < 1) per_sm = 1;
  // G CTA groups per column chunk: fill the resident capacity, but no group
  // without rows
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
  const int64_t row_groups = (p.rows + kThreads / 32 - 1) / (kThreads / 32);
  int64_t G = cap / p.nchunks;
  if (G < 1) G = 1;
  if (G > row_groups) G = row_groups;
  const int64_t grid = G * p.nchunks;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<int>(grid), kThreads, smem, st>>>(a, p);
  return cudaGetLastError();
}

// The quantizer configurations of the single-pass streaming kernel.
template <int AD>
cudaError_t dispatch_bat(const StreamArgs& a, const BatParams& p, int op, int fmt, int scaling,
                         cudaStream_t st) {
  if (op == kOpBatApply) return launch_bat_kernel<AD, kOpBatApply, kFmtE2M1, kFloor, kMbsNone>(a, p, st);
  const int rule = scaling & 0xF;
  const bool mbs = (scaling >> 4) != 0;
  switch (fmt) {
    case kFmtE2M1:
      if (mbs) {
        if (rule == kOas) return launch_bat_kernel<AD, kOpQuant, kFmtE2M1, kOas, kMbsStatic>(a, p, st);
        return launch_bat_kernel<AD, kOpQuant, kFmtE2M1, kFloor, kMbsStatic>(a, p, st);
      }
      switch (rule) {
        case kCeil: return launch_bat_kernel<AD, kOpQuant, kFmtE2M1, kCeil, kMbsNone>(a, p, st);
        case kOasRule: return launch_bat_kernel<AD, kOpQuant, kFmtE2M1, kOasRule, kMbsNone>(a, p, st);
        case kOas: return launch_bat_kernel<AD, kOpQuant, kFmtE2M1, kOas, kMbsNone>(a, p, st);
        default: return launch_bat_kernel<AD, kOpQuant, kFmtE2M1, kFloor, kMbsNone>(a, p, st);
      }
#define MXK_BAT_BYTES(F)                                                                     \
  case F:                                                                                   \
    if (rule == kCeil) return launch_bat_kernel<AD, kOpQuant, F, kCeil, kMbsNone>(a, p, st); \
    if (rule == kOas) return launch_bat_kernel<AD, kOpQuant, F, kOas, kMbsNone>(a, p, st);   \
    return launch_bat_kernel<AD, kOpQuant, F, kFloor, kMbsNone>(a, p, st);
      MXK_BAT_BYTES(kFmtE4M3)
      MXK_BAT_BYTES(kFmtE5M2)
      MXK_BAT_BYTES(kFmtE3M2)
      MXK_BAT_BYTES(kFmtE2M3)
#undef MXK_BAT_BYTES
    case kFmtInt8:
      if (rule == kCeil) return launch_bat_kernel<AD, kOpQuant, kFmtInt8, kCeil, kMbsNone>(a, p, st);
      return launch_bat_kernel<AD, kOpQuant, kFmtInt8, kFloor, kMbsNone>(a, p, st);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_bat(const void* x, int64_t rows, int64_t cols, int a_dim, const float* A,
                       const float* B, const float* beta_min, const float* beta_max, int fmt,
                       int scaling, void* codes, uint8_t* scales, uint8_t* macro, void* y,
                       ScaleMap sm, cudaStream_t st) {
  StreamArgs a{};
  a.x = static_cast<const uint8_t*>(x);
  a.nslices = rows * cols / 16;
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = scales;
  a.macro = macro;
  a.out = static_cast<uint8_t*>(y);
  a.smap = sm;
  const int64_t spr = cols / 16;
  if ((spr + 31) / 32 > 0x7FFFFFFF) return cudaErrorInvalidValue;
  BatParams p{A, B, beta_min, beta_max, rows, spr, static_cast<int>((spr + 31) / 32)};
  const int op = y ? kOpBatApply : kOpQuant;
  switch (a_dim) {
    case 1: return dispatch_bat<1>(a, p, op, fmt, scaling, st);
    case 2: return dispatch_bat<2>(a, p, op, fmt, scaling, st);
    case 4: return dispatch_bat<4>(a, p, op, fmt, scaling, st);
    case 8: return dispatch_bat<8>(a, p, op, fmt, scaling, st);
    case 16: return dispatch_bat<16>(a, p, op, fmt, scaling, st);
    case 32: return dispatch_bat<32>(a, p, op, fmt, scaling, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mxk
