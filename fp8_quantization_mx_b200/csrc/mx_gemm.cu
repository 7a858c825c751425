// Block-scaled MXFP4 GEMM on the sm_100 tensor cores, with the MX
// quantization of the bf16 activations fused into its prologue.
//
//   D[M, N] = A[M, K] . B[N, K]^T,   A and B MXFP4 (E2M1 elements, one E8M0
//   scale per 32 elements along K), fp32 accumulation in tensor memory.
//
// This is the consumer the sources place the MX scale work beside: "Unveiling
// the Potential of Quantization with MXFP4", section 2.B (the scale work runs
// on the vector cores next to the tensor-core GEMM) and section 4 (its
// overhead measured against the GEMM); "[vLLM] MXFP8/MXFP4", MXFP4 MoE section
// (the SM100 MoE kernels consume MXFP4 weights with their E8M0 scales).
//
// One CTA computes a 128 x BN tile of D (BN = 128 or 256) with one
// tcgen05.mma.kind::mxf4.block_scale (M = 128, N = BN, K = 64) at a time,
// over K-blocks of 256 elements (128 code bytes per row: one 128-byte
// swizzle atom), in an S-stage shared-memory ring:
//   warp 0     TMA: B's code tile (2-D tensor map, 128-byte swizzle) and B's
//              scale tiles (bulk copies of the tiled layout MX_SCALES_MMA
//              writes); A's as well when A comes pre-quantized
//   warp 1     TMEM allocation; one thread copies the stage's scale tiles
//              into TMEM (tcgen05.cp) and issues the four MMAs of the
//              K-block, then commits to the stage's "empty" barrier
//   warps 2-9  (fused) quantize A's 128 x 256 bf16 tile of the K-block with
//              the streaming kernels' per-slice quantizer straight from
//              global memory into the swizzled operand tile and the scale
//              tile in shared memory: the quantized activations never reach
//              HBM; then the epilogue
//   warps 2-5  (pre-quantized A) the epilogue
// Epilogue: TMEM -> registers (tcgen05.ld, one row per thread), fp32 -> bf16
// (or fp32) -> global.
//
// Every wait is bounded in time (mbar_wait): a wait that runs out sets the
// caller's status word and the CTA drains its in-flight copies and MMAs,
// frees its TMEM and returns.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mx_stream.cuh"
#include "mx_tc.cuh"

namespace mxk {

namespace {

constexpr int kGemmBM = 128;       // rows of A per tile: the MMA's M
constexpr int kGemmBK = 256;       // elements of K per stage
constexpr uint32_t kRowBytes = 128;  // code bytes per row per stage
constexpr uint32_t kTileA = kGemmBM * kRowBytes;
constexpr uint32_t kSfTile = 512;  // 128 rows x 4 scales

// Status codes a timed-out wait leaves in *status (which role gave up).
constexpr int kStatusProducer = 1, kStatusMmaB = 2, kStatusMmaA = 3, kStatusQuant = 4,
              kStatusEpilogue = 5, kStatusDrain = 6;

struct GemmArgs {
  const uint8_t* a_bf16;    // fused: bf16 A [M, K]
  const uint8_t* a_scales;  // pre-quantized: A's scales, tiled layout
  const uint8_t* b_scales;  // B's scales, tiled layout
  uint8_t* d;               // D [M, N], bf16 or float
  uint8_t* a_codes_out;     // fused, nullable: A's codes [M, K/2]
  uint8_t* a_scales_out;    // fused, nullable: A's scales, tiled layout
  int* status;              // nullable
  int64_t M, N, K;
  int out_fp32;
};

template <int BN, int S, bool FUSED>
struct GemmCfg {
  static constexpr int kQuantWarps = FUSED ? 8 : 4;   // warps after the two control warps
  static constexpr int kThreads = (2 + kQuantWarps) * 32;
  static constexpr uint32_t kTileB = BN * kRowBytes;
  static constexpr uint32_t kSfA = 2 * kSfTile;                   // one band, two K-tiles
  static constexpr uint32_t kSfB = (BN / 128) * 2 * kSfTile;      // BN/128 bands
  static constexpr uint32_t kStage = kTileA + kTileB + kSfA + kSfB;
  static constexpr uint32_t kBarBytes = 8 * (3 * S + 1) + 8;
  static constexpr uint32_t kSmem = S * kStage + kBarBytes + 1024;   // + alignment slack
  // TMEM: BN accumulator columns, then per stage 8 columns of A scales and
  // BN/16 of B scales (two K-tiles x bands x 4 columns)
  static constexpr uint32_t kSfCols = 8 + BN / 16;
  static constexpr uint32_t kColsUsed = BN + S * kSfCols;
  static constexpr uint32_t kTmemCols = kColsUsed <= 256 ? 256 : 512;
  static_assert(kColsUsed <= 512, "TMEM columns");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

template <int BN, int S, bool FUSED, int RULE>
__global__ void __launch_bounds__(GemmCfg<BN, S, FUSED>::kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs g) {
  using C = GemmCfg<BN, S, FUSED>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;   // 128-byte swizzle atoms need 1024 alignment
  uint8_t* const gbase = smem_raw + (base - raw);
  const uint32_t sA = base;
  const uint32_t sB = sA + S * kTileA;
  const uint32_t sSFA = sB + S * C::kTileB;
  const uint32_t sSFB = sSFA + S * C::kSfA;
  const uint32_t sBar = sSFB + S * C::kSfB;
  auto fullB = [&](int s) { return sBar + 8u * s; };
  auto fullA = [&](int s) { return sBar + 8u * (S + s); };
  auto empty = [&](int s) { return sBar + 8u * (2 * S + s); };
  const uint32_t tfull = sBar + 8u * (3 * S);
  uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(gbase + (sBar + 8u * (3 * S + 1) - base));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kGemmBM;
  const int nk = static_cast<int>(g.K / kGemmBK);
  const int64_t T = g.K / 128;   // scale tiles per 128-row band

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(fullB(s), 1);
      tc::mbar_init(fullA(s), FUSED ? C::kQuantWarps : 1);
      tc::mbar_init(empty(s), 1);
    }
    tc::mbar_init(tfull, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tc::smem_addr(tmem_holder), C::kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      tc::prefetch_tmap(&tmB);
      if (!FUSED) tc::prefetch_tmap(&tmA);
      // B's scale bands present in the tiled buffer (rows padded to 128)
      const int64_t nb0 = n0 / 128;
      const int64_t bands_total = (g.N + 127) / 128;
      const int64_t left = bands_total - nb0;
      const int nbands = static_cast<int>(left < BN / 128 ? left : BN / 128);
      const uint32_t tx = C::kTileB + nbands * 2 * kSfTile + (FUSED ? 0u : kTileA + 2 * kSfTile);
      int armed = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (kb / S) & 1;
        if (!tc::mbar_wait(empty(s), ph ^ 1, abort_flag, g.status, kStatusProducer)) break;
        tc::mbar_arrive_expect_tx(fullB(s), tx);
        tc::tma_load_2d(sB + s * C::kTileB, &tmB, kb * static_cast<int>(kRowBytes),
                        static_cast<int>(n0), fullB(s));
        for (int band = 0; band < nbands; ++band)
          tc::bulk_load(sSFB + s * C::kSfB + band * 2 * kSfTile,
                        g.b_scales + ((nb0 + band) * T + 2 * kb) * kSfTile, 2 * kSfTile, fullB(s));
        if (!FUSED) {
          tc::tma_load_2d(sA + s * kTileA, &tmA, kb * static_cast<int>(kRowBytes),
                          static_cast<int>(m0), fullB(s));
          tc::bulk_load(sSFA + s * C::kSfA, g.a_scales + ((m0 / 128) * T + 2 * kb) * kSfTile,
                        2 * kSfTile, fullB(s));
        }
        armed = kb + 1;
      }
      // every copy this thread issued has landed before the CTA can exit
      for (int kb = max(0, armed - S); kb < armed; ++kb)
        tc::mbar_wait(fullB(kb % S), (kb / S) & 1, abort_flag, g.status, kStatusDrain, false);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (kb / S) & 1;
        if (!tc::mbar_wait(fullB(s), ph, abort_flag, g.status, kStatusMmaB)) break;
        if (FUSED && !tc::mbar_wait(fullA(s), ph, abort_flag, g.status, kStatusMmaA)) break;
        tc::tc_fence_after();
        const uint32_t sfa = tmem + BN + s * C::kSfCols;
        const uint32_t sfb = sfa + 8;
        tc::tmem_cp_sf(sfa, tc::sf_desc(sSFA + s * C::kSfA));
        tc::tmem_cp_sf(sfa + 4, tc::sf_desc(sSFA + s * C::kSfA + kSfTile));
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int band = 0; band < BN / 128; ++band)
            tc::tmem_cp_sf(sfb + t * (BN / 32) + band * 4,
                           tc::sf_desc(sSFB + s * C::kSfB + band * 2 * kSfTile + t * kSfTile));
        const uint64_t adesc = tc::kmajor_sw128_desc(sA + s * kTileA);
        const uint64_t bdesc = tc::kmajor_sw128_desc(sB + s * C::kTileB);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // K = 64 per MMA: 32 code bytes further along the swizzled rows;
          // scales: K-tile kk / 2, byte (kk % 2) * 2 of the 32-bit word
          const int t = kk >> 1;
          tc::mma_mxf4(tmem, adesc + 2 * kk, bdesc + 2 * kk,
                       tc::idesc_mxf4(kGemmBM, BN, (kk & 1) * 2), sfa + t * 4, sfb + t * (BN / 32),
                       (kb | kk) != 0);
        }
        tc::tc_commit(empty(s));
      }
      // arrives once every MMA issued above has completed (also after a
      // break, so that TMEM is never freed under a running MMA)
      tc::tc_commit(tfull);
    }
    __syncwarp();
  } else {
    const int qw = warp - 2;
    if constexpr (FUSED) {
      // ------------------------------------------- prologue: quantize A
      // warp qw owns rows 16 qw .. 16 qw + 15 of the tile; per pass p, lanes
      // 0-15 take row 16 qw + 2p and lanes 16-31 the next; lane j16 = lane &
      // 15 takes elements 16 j16 .. 16 j16 + 15 of the K-block (a lane pair
      // is one 32-element block)
      const int j16 = lane & 15;
      const int64_t K2 = g.K * 2;   // bf16 row pitch in bytes
      const bool write_a = (blockIdx.x == 0);
      V16 v[8], nv[8];
      auto load = [&](int kb, V16 (&dst)[8]) {
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const int r = 16 * qw + 2 * p + (lane >> 4);
          const int64_t m = m0 + r;
          if (m < g.M) {
            dst[p] = ld_stream32(g.a_bf16 + m * K2 + (static_cast<int64_t>(kb) * kGemmBK + 16 * j16) * 2);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[p].w[i] = 0;
          }
        }
      };
      if (nk > 0) load(0, v);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (kb / S) & 1;
        if (kb + 1 < nk) load(kb + 1, nv);
        // every lane waits (acquire), and the warp leaves together: the
        // quantizer below uses warp collectives
        const bool ok = tc::mbar_wait(empty(s), ph ^ 1, abort_flag, g.status, kStatusQuant);
        if (!__all_sync(kFull, ok)) break;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const int r = 16 * qw + 2 * p + (lane >> 4);
          const uint32_t pa = pair_max(amax_bits16(v[p]));
          const BlockScale bs = decide_scale<kFmtE2M1, RULE, kMbsNone>(v[p], pa, 0);
          const uint2 c = codes_fp4<kMbsNone>(v[p], bs);
          const uint32_t dst = sA + s * kTileA + r * kRowBytes +
                               ((((j16 >> 1) ^ (r & 7)) & 7) << 4) + ((j16 & 1) << 3);
          asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(dst), "r"(c.x), "r"(c.y) : "memory");
          const int j = j16 >> 1;   // block column within the K-block, 0..7
          if ((lane & 1) == 0) {
            const uint32_t sdst = sSFA + s * C::kSfA + (j >> 2) * kSfTile + (r & 31) * 16 +
                                  ((r >> 5) & 3) * 4 + (j & 3);
            asm volatile("st.shared.u8 [%0], %1;" ::"r"(sdst), "r"(bs.byte) : "memory");
          }
          if (write_a) {
            const int64_t m = m0 + r;
            if (g.a_codes_out && m < g.M)
              st_stream8(g.a_codes_out + m * (g.K / 2) + static_cast<int64_t>(kb) * kRowBytes + 8 * j16, c);
            if (g.a_scales_out && (lane & 1) == 0)
              g.a_scales_out[((m0 / 128) * T + 2 * kb + (j >> 2)) * kSfTile + (r & 31) * 16 +
                             ((r >> 5) & 3) * 4 + (j & 3)] = static_cast<uint8_t>(bs.byte);
          }
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(fullA(s));
        if (kb + 1 < nk) {
#pragma unroll
          for (int p = 0; p < 8; ++p) v[p] = nv[p];
        }
      }
    }
    // ------------------------------------------------------------ epilogue
    // warp w reads TMEM lanes 32 (w % 4) .. + 31 (its quarter); with eight
    // warps the two sets of four split the columns
    constexpr int kGroups = C::kQuantWarps / 4;
    const int q = warp & 3;
    const int grp = qw / 4;
    const bool got = tc::mbar_wait(tfull, 0, abort_flag, g.status, kStatusEpilogue, false);
    tc::tc_fence_after();
    // warp-uniform: tcgen05.ld is a whole-warp instruction
    const bool done = __all_sync(kFull, got && !*abort_flag);
    if (done) {
      const int row = q * 32 + lane;
      const int64_t m = m0 + row;
      for (int c0 = grp * (BN / kGroups); c0 < (grp + 1) * (BN / kGroups); c0 += 32) {
        uint32_t r[32];
        tc::tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0, r);
        if (m < g.M) {
#pragma unroll
          for (int gq = 0; gq < 4; ++gq) {
            const int64_t n = n0 + c0 + 8 * gq;
            if (n < g.N) {
              if (g.out_fp32) {
                uint4* o = reinterpret_cast<uint4*>(g.d + (m * g.N + n) * 4);
                o[0] = make_uint4(r[8 * gq], r[8 * gq + 1], r[8 * gq + 2], r[8 * gq + 3]);
                o[1] = make_uint4(r[8 * gq + 4], r[8 * gq + 5], r[8 * gq + 6], r[8 * gq + 7]);
              } else {
                uint32_t h[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const __nv_bfloat162 b2 = __floats2bfloat162_rn(
                      __uint_as_float(r[8 * gq + 2 * i]), __uint_as_float(r[8 * gq + 2 * i + 1]));
                  h[i] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                *reinterpret_cast<uint4*>(g.d + (m * g.N + n) * 2) = make_uint4(h[0], h[1], h[2], h[3]);
              }
            }
          }
        }
      }
    }
    tc::tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------- host side --

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (the
// library links no driver library).
EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Tensor map of a [rows, K/2] uint8 code matrix read in 128-byte x box_rows
// boxes with the 128-byte swizzle (rows past the end read as zero).
bool code_tmap(CUtensorMap* tm, const void* codes, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  const cuuint32_t box[2] = {kRowBytes, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int S, bool FUSED, int RULE>
cudaError_t launch_gemm_cfg(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g,
                            cudaStream_t st) {
  using C = GemmCfg<BN, S, FUSED>;
  auto kern = gemm_kernel<BN, S, FUSED, RULE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((g.N + BN - 1) / BN),
                  static_cast<unsigned>((g.M + kGemmBM - 1) / kGemmBM));
  kern<<<grid, C::kThreads, C::kSmem, st>>>(tmA, tmB, g);
  return cudaGetLastError();
}

template <bool FUSED, int RULE>
cudaError_t launch_gemm_bn(bool wide, const CUtensorMap& tmA, const CUtensorMap& tmB,
                           const GemmArgs& g, cudaStream_t st) {
  if (wide) return launch_gemm_cfg<256, 4, FUSED, RULE>(tmA, tmB, g, st);
  return launch_gemm_cfg<128, 6, FUSED, RULE>(tmA, tmB, g, st);
}

}  // namespace

cudaError_t launch_gemm(const void* a, const uint8_t* a_scales, int a_rule, const void* b_codes,
                        const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, int out_fp32,
                        void* d, void* a_codes_out, uint8_t* a_scales_out, int* status,
                        cudaStream_t st) {
  const bool fused = a_scales == nullptr;
  // 256-wide tiles unless that leaves SMs idle on a small problem
  const bool wide = N > 128 && ((M + kGemmBM - 1) / kGemmBM) * ((N + 255) / 256) >= 148;
  CUtensorMap tmA{}, tmB{};
  if (!code_tmap(&tmB, b_codes, N, K, wide ? 256 : 128)) return cudaErrorInvalidValue;
  if (!fused && !code_tmap(&tmA, a, M, K, kGemmBM)) return cudaErrorInvalidValue;
  GemmArgs g{};
  g.a_bf16 = fused ? static_cast<const uint8_t*>(a) : nullptr;
  g.a_scales = a_scales;
  g.b_scales = b_scales;
  g.d = static_cast<uint8_t*>(d);
  g.a_codes_out = static_cast<uint8_t*>(a_codes_out);
  g.a_scales_out = a_scales_out;
  g.status = status;
  g.M = M;
  g.N = N;
  g.K = K;
  g.out_fp32 = out_fp32;
  if (!fused) return launch_gemm_bn<false, kFloor>(wide, tmA, tmB, g, st);
  switch (a_rule) {
    case kCeil: return launch_gemm_bn<true, kCeil>(wide, tmA, tmB, g, st);
    case kOasRule: return launch_gemm_bn<true, kOasRule>(wide, tmA, tmB, g, st);
    case kOas: return launch_gemm_bn<true, kOas>(wide, tmA, tmB, g, st);
    default: return launch_gemm_bn<true, kFloor>(wide, tmA, tmB, g, st);
  }
}

}  // namespace mxk
