// Block-scaled MXFP4 GEMM on the sm_100 tensor cores, and the MX
// quantization of its bf16 activations in the same launch.
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
//              writes); A's as well when A is in memory quantized
//   warp 1     TMEM allocation; one thread copies the stage's scale tiles
//              into TMEM (tcgen05.cp) and issues the four MMAs of the
//              K-block, then commits to the stage's "empty" barrier
//   warps 2-9  the epilogue: TMEM -> registers (tcgen05.ld, one row per
//              thread, two warps per 32-lane quarter splitting the columns),
//              the accumulator released to the next tile, then fp32 -> bf16
//              (or fp32) -> global
// The kernels are persistent (one CTA per SM looping over tiles), so the next
// tile's loads overlap the previous tile's epilogue. Four kernels share this
// body:
//   gemm_kernel              A pre-quantized
//   gemm_staged_kernel       bf16 A: six more warps per CTA quantize A into
//                            global codes and scales while the GEMM runs on
//                            the 128-row bands already counted complete
//   gemm_staged_sync_kernel  bf16 A, one wave of tiles: every warp quantizes,
//                            a grid barrier, then the GEMM
//   gemm_fused_kernel        bf16 A quantized on chip in the prologue by the
//                            work warps, shared across a thread-block cluster
//
// Every wait is bounded in time (mbar_wait, counter_wait): a wait that runs
// out sets the caller's status word and the CTA drains its in-flight copies
// and MMAs, frees its TMEM and returns.

#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "mx.h"
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
              kStatusEpilogue = 5, kStatusDrain = 6, kStatusStaging = 7, kStatusReady = 8;

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

// Shared-memory plan common to both kernels: S stages of (A codes, B codes,
// A scale tiles, B scale tiles), then (fused) one bf16 staging tile of A,
// then the barriers.
template <int BN, int S, bool FUSED>
struct GemmCfg {
  static constexpr int kWorkWarps = 8;   // quantizer (fused) and epilogue warps
  static constexpr int kThreads = (2 + kWorkWarps) * 32;
  static constexpr uint32_t kTileB = BN * kRowBytes;
  static constexpr uint32_t kSfA = 2 * kSfTile;                   // one band, two K-tiles
  static constexpr uint32_t kSfB = (BN / 128) * 2 * kSfTile;      // BN/128 bands
  static constexpr uint32_t kStage = kTileA + kTileB + kSfA + kSfB;
  static constexpr uint32_t kStaging = FUSED ? kGemmBM * kGemmBK * 2 : 0;   // bf16 A tile
  static constexpr uint32_t kBarBytes = 8 * (4 * S + 3) + 8;
  static constexpr uint32_t kSmem = S * kStage + kStaging + kBarBytes + 1024;   // + alignment
  // TMEM: BN accumulator columns, then per stage 8 columns of A scales and
  // BN/16 of B scales (two K-tiles x bands x 4 columns)
  static constexpr uint32_t kSfCols = 8 + BN / 16;
  static constexpr uint32_t kColsUsed = BN + S * kSfCols;
  static constexpr uint32_t kTmemCols = kColsUsed <= 256 ? 256 : 512;
  static_assert(kColsUsed <= 512, "TMEM columns");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// Addresses of one CTA's shared-memory plan.
template <int BN, int S, bool FUSED>
struct Smem {
  using C = GemmCfg<BN, S, FUSED>;
  uint32_t base, sA, sB, sSFA, sSFB, sStg, sBar;
  uint32_t* tmem_holder;
  volatile int* abort_flag;
  __device__ explicit Smem(uint8_t* raw_ptr) {
    const uint32_t raw = tc::smem_addr(raw_ptr);
    base = (raw + 1023u) & ~1023u;   // 128-byte swizzle atoms need 1024-byte alignment
    sA = base;
    sB = sA + S * kTileA;
    sSFA = sB + S * C::kTileB;
    sSFB = sSFA + S * C::kSfA;
    sStg = sSFB + S * C::kSfB;
    sBar = sStg + C::kStaging;
    tmem_holder = reinterpret_cast<uint32_t*>(raw_ptr + (sBar + 8u * (4 * S + 3) - raw));
    abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  }
  __device__ uint32_t fullB(int s) const { return sBar + 8u * s; }
  __device__ uint32_t fullA(int s) const { return sBar + 8u * (S + s); }
  __device__ uint32_t empty(int s) const { return sBar + 8u * (2 * S + s); }
  __device__ uint32_t tfull() const { return sBar + 8u * (3 * S); }
  __device__ uint32_t tempty() const { return sBar + 8u * (3 * S + 1); }
  __device__ uint32_t stg_full() const { return sBar + 8u * (3 * S + 2); }
  __device__ uint32_t qfree(int s) const { return sBar + 8u * (3 * S + 3 + s); }
};

// One K-block on the tensor cores (one thread): the stage's scale tiles into
// TMEM, then four MMAs of K = 64.
template <int BN, int S, bool FUSED>
__device__ __forceinline__ void issue_kblock(const Smem<BN, S, FUSED>& sm, uint32_t tmem, int s,
                                             bool first) {
  using C = GemmCfg<BN, S, FUSED>;
  const uint32_t sfa = tmem + BN + s * C::kSfCols;
  const uint32_t sfb = sfa + 8;
  tc::tmem_cp_sf(sfa, tc::sf_desc(sm.sSFA + s * C::kSfA));
  tc::tmem_cp_sf(sfa + 4, tc::sf_desc(sm.sSFA + s * C::kSfA + kSfTile));
#pragma unroll
  for (int tt = 0; tt < 2; ++tt)
#pragma unroll
    for (int band = 0; band < BN / 128; ++band)
      tc::tmem_cp_sf(sfb + tt * (BN / 32) + band * 4,
                     tc::sf_desc(sm.sSFB + s * C::kSfB + band * 2 * kSfTile + tt * kSfTile));
  const uint64_t adesc = tc::kmajor_sw128_desc(sm.sA + s * kTileA);
  const uint64_t bdesc = tc::kmajor_sw128_desc(sm.sB + s * C::kTileB);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    // K = 64 per MMA: 32 code bytes further along the swizzled rows; scales:
    // K-tile kk / 2, byte (kk % 2) * 2 of the 32-bit word
    const int tt = kk >> 1;
    tc::mma_mxf4(tmem, adesc + 2 * kk, bdesc + 2 * kk, tc::idesc_mxf4(kGemmBM, BN, (kk & 1) * 2),
                 sfa + tt * 4, sfb + tt * (BN / 32), !(first && kk == 0));
  }
}

// Epilogue of one tile by the eight work warps: warp w reads TMEM lanes
// 32 (w % 4) .. + 31 (its quarter), warps 2-5 the first half of the columns
// and warps 6-9 the second. bf16 out: the values are rounded into registers,
// the accumulator released (tmem_empty), then stored; float out: stored from
// each load, then released. Returns false when the kernel is aborting.
template <int BN, int S, bool FUSED>
__device__ __forceinline__ bool epilogue_tile(const Smem<BN, S, FUSED>& sm, const GemmArgs& g,
                                              uint32_t tmem, uint32_t tile_par, int64_t m0,
                                              int64_t n0, int warp, int lane) {
  const int q = warp & 3;
  const int c_begin = ((warp - 2) / 4) * (BN / 2);
  const bool got =
      tc::mbar_wait(sm.tfull(), tile_par, sm.abort_flag, g.status, kStatusEpilogue, false);
  tc::tc_fence_after();
  // one decision for all eight warps (tcgen05.ld is a whole-warp instruction,
  // and the fused kernel's work warps meet at named barriers afterwards)
  if (!tc::named_all(3, GemmCfg<BN, S, FUSED>::kWorkWarps * 32, got && !*sm.abort_flag))
    return false;
  const int64_t m = m0 + q * 32 + lane;
  constexpr int kCols = BN / 2;
  const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + c_begin;
  if (g.out_fp32) {
    // float out: straight from each TMEM load to global, then the release
#pragma unroll 1
    for (int c0 = 0; c0 < kCols; c0 += 32) {
      uint32_t r[32];
      tc::tmem_ld32(taddr + c0, r);
      if (m < g.M) {
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
          const int64_t n = n0 + c_begin + c0 + 8 * gq;
          if (n < g.N) {
            uint4* o = reinterpret_cast<uint4*>(g.d + (m * g.N + n) * 4);
            o[0] = make_uint4(r[8 * gq], r[8 * gq + 1], r[8 * gq + 2], r[8 * gq + 3]);
            o[1] = make_uint4(r[8 * gq + 4], r[8 * gq + 5], r[8 * gq + 6], r[8 * gq + 7]);
          }
        }
      }
    }
    tc::tc_fence_before();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(sm.tempty());
    return true;
  }
  // bf16 out: the whole row share as packed bf16 pairs in registers, the
  // accumulator released, then the stores
  uint32_t h[kCols / 2];
#pragma unroll
  for (int c0 = 0; c0 < kCols; c0 += 32) {
    uint32_t r[32];
    tc::tmem_ld32(taddr + c0, r);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const __nv_bfloat162 b2 =
          __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
      h[c0 / 2 + i] = *reinterpret_cast<const uint32_t*>(&b2);
    }
  }
  tc::tc_fence_before();
  __syncwarp();
  if (lane == 0) tc::mbar_arrive(sm.tempty());
  if (m < g.M) {
#pragma unroll
    for (int gq = 0; gq < kCols / 8; ++gq) {
      const int64_t n = n0 + c_begin + 8 * gq;
      if (n < g.N)
        *reinterpret_cast<uint4*>(g.d + (m * g.N + n) * 2) =
            make_uint4(h[4 * gq], h[4 * gq + 1], h[4 * gq + 2], h[4 * gq + 3]);
    }
  }
  return true;
}

// What the persistent GEMM body runs beside the GEMM. NoPrologue: nothing,
// A arrives quantized. QuantPrologue: kWarps more warps per CTA (after the
// epilogue warps) quantize A (bf16) into the codes and tiled scales the GEMM
// reads, warp tiles of 32 U slices dealt over the grid in slice order, and
// count the slices done per 128-row m-tile in `ready` (relaxed adds after a
// proxy fence and a release fence: the GEMM reads them with TMA); the producer
// waits (acquire, bounded) until an m-tile is complete before its first load
// of that m-tile's A. The GEMM of the first m-tiles thus starts while the
// rest of A is being quantized, and the epilogue warps never wait on it.
struct NoPrologue {
  static constexpr bool kActive = false;
  __device__ bool wait_mtile(int64_t, volatile int*, int*) const { return true; }
};

template <int RULE>
struct QuantPrologue {
  static constexpr bool kActive = true;
  static constexpr int kWarps = 6;
  static constexpr int U = 4;   // slices per lane per warp tile (32 U slices), two tiles in flight
  // Warps per CTA in the first round: the quantizer warps and the epilogue
  // warps, which are idle until the first accumulator is complete; the
  // first-round tiles are the first m-tiles, which the first wave needs.
  static constexpr int kFirstRound = 8 + kWarps;
  StreamArgs q;                 // the quantizer's view of A (slices of 16 elements)
  unsigned long long* ready;    // [ceil(M / 128)], zero at launch
  int64_t mtile_slices;         // slices per m-tile: 128 K / 16 (a multiple of 32 U)

  __device__ bool wait_mtile(int64_t mt, volatile int* abort, int* status) const {
    const int64_t left = q.nslices - mt * mtile_slices;
    const unsigned long long target =
        static_cast<unsigned long long>(left < mtile_slices ? left : mtile_slices);
    if (!tc::counter_wait(ready + mt, target, abort, status, kStatusReady)) return false;
    // acquired through the generic proxy; the loads that follow are TMA's
    tc::fence_proxy_async_global();
    return true;
  }

  __device__ void load_tile(int64_t tile, int lane, V16 (&v)[U]) const {
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t c = tile * 32 * U + lane + 32 * j;
#pragma unroll
      for (int i = 0; i < 8; ++i) v[j].w[i] = 0;
      if (c < q.nslices) v[j] = ld_stream32(q.x + 32 * c);
    }
  }

  // The slices of a finished warp tile counted to its m-tile (lane 0).
  __device__ void count(int64_t tile) const {
    const int64_t first = tile * 32 * U;
    const int64_t n = q.nslices - first < 32 * U ? q.nslices - first : 32 * U;
    tc::red_relaxed_add(ready + first / mtile_slices, static_cast<unsigned long long>(n));
  }

  // Quantizes warp tiles t0, then t1, t1 + step, t1 + 2 step, ... (t1 > t0;
  // t1 = INT64_MAX, step 0: t0 alone) with the next tile's loads in flight
  // while one is quantized. t0 is published on its own, the rest two at a
  // time (one release fence, which waits for the stores, for two tiles).
  __device__ void run(int64_t t0, int64_t t1, int64_t step, int lane) const {
    const int64_t ntiles = (q.nslices + 32 * U - 1) / (32 * U);
    double sd = 0.0, sx = 0.0;
    V16 v[U], nv[U];
    load_tile(t0, lane, v);
    int64_t held = -1;   // a finished tile not yet published
    bool first = true;
    for (int64_t tile = t0, next = t1; tile < ntiles; tile = next, next += step) {
      if (next < ntiles) load_tile(next, lane, nv);
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int64_t c = tile * 32 * U + lane + 32 * j;
        const uint32_t pa = pair_max(amax_bits16(v[j]));
        process_slice<kOpQuant, kFmtE2M1, RULE, kMbsNone>(q, v[j], v[j], c, c < q.nslices, lane,
                                                           pa, 0, sd, sx);
      }
      if (!first && held < 0 && next < ntiles) {
        held = tile;
      } else {
        // the codes and scales of the held tile and this one (generic-proxy
        // stores of all 32 lanes) are published to their m-tiles
        tc::fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) {
          tc::fence_release_gpu();
          if (held >= 0) count(held);
          count(tile);
        }
        held = -1;
      }
      first = false;
#pragma unroll
      for (int j = 0; j < U; ++j) v[j] = nv[j];
    }
  }
};

// ------------------------------------------- pre-quantized A: persistent --
// CTA b takes tiles b, b + gridDim.x, ... (tile t: m-tile t / tiles_n, n-tile
// t % tiles_n). The stage ring runs on across tiles; the accumulator is
// handed between the MMA issuer and the epilogue by the tmem_full /
// tmem_empty barriers, so the next tile's loads proceed while the epilogue
// drains the accumulator.
template <int BN, int S, class Pro>
__device__ __forceinline__ void gemm_pre_body(const CUtensorMap* tmA, const CUtensorMap* tmB,
                                              const GemmArgs& g, uint8_t* smem_raw,
                                              const Pro& pro) {
  using C = GemmCfg<BN, S, false>;
  const Smem<BN, S, false> sm(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk = static_cast<int>(g.K / kGemmBK);
  const int64_t T = g.K / 128;   // scale tiles per 128-row band
  const int64_t tiles_n = (g.N + BN - 1) / BN;
  const int64_t ntiles = ((g.M + kGemmBM - 1) / kGemmBM) * tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(sm.fullB(s), 1);
      tc::mbar_init(sm.empty(s), 1);
    }
    tc::mbar_init(sm.tfull(), 1);
    tc::mbar_init(sm.tempty(), C::kWorkWarps);
    *sm.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tc::smem_addr(sm.tmem_holder), C::kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *sm.tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      tc::prefetch_tmap(tmB);
      tc::prefetch_tmap(tmA);
      const int64_t bands_total = (g.N + 127) / 128;
      int64_t it = 0;   // K-blocks issued so far (the ring position)
      int64_t ready_mt = -1;   // the last m-tile known to be quantized
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
        const int64_t mt = t / tiles_n;
        const int64_t m0 = mt * kGemmBM;
        const int64_t n0 = (t % tiles_n) * BN;
        // B's scale bands present in the tiled buffer (rows padded to 128)
        const int64_t nb0 = n0 / 128;
        const int64_t left = bands_total - nb0;
        const int nbands = static_cast<int>(left < BN / 128 ? left : BN / 128);
        const uint32_t tx = C::kTileB + nbands * 2 * kSfTile + kTileA + 2 * kSfTile;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = static_cast<int>(it % S);
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1;
          if (!tc::mbar_wait(sm.empty(s), ph ^ 1, sm.abort_flag, g.status, kStatusProducer)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(sm.fullB(s), tx);
          tc::tma_load_2d(sm.sB + s * C::kTileB, tmB, kb * static_cast<int>(kRowBytes),
                          static_cast<int>(n0), sm.fullB(s));
          for (int band = 0; band < nbands; ++band)
            tc::bulk_load(sm.sSFB + s * C::kSfB + band * 2 * kSfTile,
                          g.b_scales + ((nb0 + band) * T + 2 * kb) * kSfTile, 2 * kSfTile,
                          sm.fullB(s));
          // (the stage's B is on its way while this waits for A's m-tile)
          bool got = true;
          if (Pro::kActive && mt != ready_mt) {
            got = pro.wait_mtile(mt, sm.abort_flag, g.status);
            ready_mt = mt;
          }
          // loaded even after a failed wait (in bounds; the result is then
          // undefined and the status set), so that the stage completes and
          // the drain below stays exact
          tc::tma_load_2d(sm.sA + s * kTileA, tmA, kb * static_cast<int>(kRowBytes),
                          static_cast<int>(m0), sm.fullB(s));
          tc::bulk_load(sm.sSFA + s * C::kSfA, g.a_scales + ((m0 / 128) * T + 2 * kb) * kSfTile,
                        2 * kSfTile, sm.fullB(s));
          if (!got) {
            ok = false;
            ++it;
            break;
          }
        }
      }
      // every copy this thread issued has landed before the CTA can exit
      for (int64_t j = (it > S ? it - S : 0); j < it; ++j)
        tc::mbar_wait(sm.fullB(static_cast<int>(j % S)), static_cast<uint32_t>(j / S) & 1,
                      sm.abort_flag, g.status, kStatusDrain, false);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int64_t it = 0;
      uint32_t tile_par = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x, tile_par ^= 1) {
        // the epilogue has read the previous tile's accumulator
        ok = tc::mbar_wait(sm.tempty(), tile_par ^ 1, sm.abort_flag, g.status, kStatusMmaB);
        if (ok) tc::tc_fence_after();
        for (int kb = 0; ok && kb < nk; ++kb, ++it) {
          const int s = static_cast<int>(it % S);
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1;
          if (!tc::mbar_wait(sm.fullB(s), ph, sm.abort_flag, g.status, kStatusMmaB)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          issue_kblock(sm, tmem, s, kb == 0);
          tc::tc_commit(sm.empty(s));
        }
        // committed on every exit, so that the epilogue never waits for a
        // commit that will not come and TMEM is never freed under an MMA
        tc::tc_commit(sm.tfull());
      }
    }
    __syncwarp();
  } else if (warp >= 2 + C::kWorkWarps) {
    // --------------------------------------------- quantizer (QuantPrologue)
    if constexpr (Pro::kActive) {
      const int64_t first_round = static_cast<int64_t>(gridDim.x) * Pro::kFirstRound;
      pro.run(static_cast<int64_t>(blockIdx.x) * Pro::kFirstRound + (warp - 2),
              first_round + static_cast<int64_t>(blockIdx.x) * Pro::kWarps +
                  (warp - 2 - C::kWorkWarps),
              static_cast<int64_t>(gridDim.x) * Pro::kWarps, lane);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    if constexpr (Pro::kActive) {
      // one first-round tile each (the epilogue waits for an MMA that waits
      // for the first m-tiles)
      pro.run(static_cast<int64_t>(blockIdx.x) * Pro::kFirstRound + (warp - 2), INT64_MAX, 0,
              lane);
    }
    uint32_t tile_par = 0;
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, tile_par ^= 1) {
      if (!epilogue_tile(sm, g, tmem, tile_par, (t / tiles_n) * kGemmBM, (t % tiles_n) * BN,
                         warp, lane))
        break;
    }
    tc::tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, int S>
__global__ void __launch_bounds__(GemmCfg<BN, S, false>::kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  gemm_pre_body<BN, S>(&tmA, &tmB, g, smem_raw, NoPrologue{});
}

// ------------------------------------ bf16 A staged through L2, one launch --
// Cooperative (every CTA resident, so that a producer's wait on another CTA's
// quantizer warps always ends): the quantizer warps of the whole grid
// quantize A into the caller's code and scale buffers (which stay in L2 at
// GEMM sizes) while the GEMM runs on the m-tiles already complete.
template <int BN, int S, int RULE>
__global__ void __launch_bounds__(GemmCfg<BN, S, false>::kThreads + 32 * QuantPrologue<RULE>::kWarps,
                                  1)
    gemm_staged_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, const GemmArgs g,
                       const QuantPrologue<RULE> pro) {
  extern __shared__ uint8_t smem_raw[];
  gemm_pre_body<BN, S>(&tmA, &tmB, g, smem_raw, pro);
}

// The same when the GEMM's tiles fit in one wave: every tile needs all of A
// before its first MMA, so nothing overlaps; every warp of the grid
// quantizes A, a grid-wide barrier, then the GEMM (no counters to clear).
template <int BN, int S, int RULE>
__global__ void __launch_bounds__(GemmCfg<BN, S, false>::kThreads, 1)
    gemm_staged_sync_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmB, const GemmArgs g,
                            const StreamArgs q) {
  extern __shared__ uint8_t smem_raw[];
  {
    constexpr int U = 2;   // slices per lane in flight (8 measured no faster)
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    double sd = 0.0, sx = 0.0;
    for (int64_t tile = warp; tile * 32 * U < q.nslices; tile += nwarps) {
      const int64_t base = tile * 32 * U + lane;
      V16 v[U];
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int64_t c = base + 32 * j;
#pragma unroll
        for (int i = 0; i < 8; ++i) v[j].w[i] = 0;
        if (c < q.nslices) v[j] = ld_stream32(q.x + 32 * c);
      }
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int64_t c = base + 32 * j;
        const uint32_t pa = pair_max(amax_bits16(v[j]));
        process_slice<kOpQuant, kFmtE2M1, RULE, kMbsNone>(q, v[j], v[j], c, c < q.nslices, lane, pa,
                                                           0, sd, sx);
      }
    }
    // the codes were written through the generic proxy; TMA (the async
    // proxy) reads them after the barrier
    tc::fence_proxy_async_global();
  }
  cooperative_groups::this_grid().sync();
  gemm_pre_body<BN, S>(&tmA, &tmB, g, smem_raw, NoPrologue{});
}

// ---------------------------------------- bf16 A quantized in the prologue --
// A cluster of CL CTAs works on one m-tile and CL adjacent n-tiles at a time
// (a "unit"; units are taken persistently, the cluster's CTAs in step). The
// K-blocks of the unit are dealt round-robin over the cluster (K-block `it`
// of the ring, counted across units, belongs to CTA it % CL): its owner
// TMA-loads the 128 x 256 bf16 tile of A into a staging buffer, quantizes it
// with the streaming kernels' per-slice quantizer into its own operand stage
// (codes in the swizzled layout, scales in the MMA tile layout), and pushes
// the 16 KB code tile and 1 KB scale tile into every other CTA's stage with
// shared-to-shared bulk copies that complete on that CTA's mbarrier. Every
// CTA's MMA commit arrives on the "empty" barrier of every CTA, so no stage is
// refilled (locally or by a push) before all CTAs are done with it. Each CTA
// thus quantizes 1/CL of A's tiles, and the quantized A stays on chip.
template <int BN, int S, int CL, int RULE>
__global__ void __launch_bounds__(GemmCfg<BN, S, true>::kThreads, 1)
    gemm_fused_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                      const GemmArgs g) {
  using C = GemmCfg<BN, S, true>;
  extern __shared__ uint8_t smem_raw[];
  const Smem<BN, S, true> sm(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = CL > 1 ? tc::cluster_rank() : 0;
  const int64_t cluster = blockIdx.x / CL;
  const int64_t nclusters = gridDim.x / CL;
  const int nk = static_cast<int>(g.K / kGemmBK);
  const int64_t T = g.K / 128;   // scale tiles per 128-row band
  const int64_t tiles_n = (g.N + BN - 1) / BN;
  const int64_t groups_n = (tiles_n + CL - 1) / CL;
  const int64_t units = ((g.M + kGemmBM - 1) / kGemmBM) * groups_n;
  // ring position `it` -> (unit, K-block); this CTA's units are cluster,
  // cluster + nclusters, ...
  auto unit_of = [&](int64_t it) { return cluster + (it / nk) * nclusters; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(sm.fullB(s), 1);
      tc::mbar_init(sm.fullA(s), 1);
      tc::mbar_init(sm.empty(s), CL);
      tc::mbar_init(sm.qfree(s), 1);
    }
    tc::mbar_init(sm.tfull(), 1);
    tc::mbar_init(sm.tempty(), C::kWorkWarps);
    tc::mbar_init(sm.stg_full(), 1);
    *sm.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tc::smem_addr(sm.tmem_holder), C::kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (CL > 1) tc::cluster_sync();   // peers' barriers exist before any push
  const uint32_t tmem = *sm.tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      tc::prefetch_tmap(&tmB);
      const int64_t bands_total = (g.N + 127) / 128;
      int64_t it = 0;
      bool ok = true;
      for (int64_t u = cluster; ok && u < units; u += nclusters) {
        const int64_t n0 = ((u % groups_n) * CL + rank) * BN;   // may lie past N: zero B
        const int64_t nb0 = n0 / 128;
        const int64_t left = bands_total - nb0;
        const int nbands = static_cast<int>(left <= 0 ? 0 : (left < BN / 128 ? left : BN / 128));
        const uint32_t tx = C::kTileB + nbands * 2 * kSfTile;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = static_cast<int>(it % S);
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1;
          if (!tc::mbar_wait(sm.empty(s), ph ^ 1, sm.abort_flag, g.status, kStatusProducer)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(sm.fullB(s), tx);
          tc::tma_load_2d(sm.sB + s * C::kTileB, &tmB, kb * static_cast<int>(kRowBytes),
                          static_cast<int>(n0), sm.fullB(s));
          for (int band = 0; band < nbands; ++band)
            tc::bulk_load(sm.sSFB + s * C::kSfB + band * 2 * kSfTile,
                          g.b_scales + ((nb0 + band) * T + 2 * kb) * kSfTile, 2 * kSfTile,
                          sm.fullB(s));
          // a K-block another CTA quantizes arrives by its push; for one of
          // this CTA's own, the stage is handed to the quantizer. (The
          // quantizer visits only its own K-blocks, so it cannot wait on the
          // "empty" barrier itself: an mbarrier answers only for the parity
          // of its last phase, and the quantizer may be several phases
          // away. This thread waits on every phase in order.)
          if (it % CL != rank)
            tc::mbar_arrive_expect_tx(sm.fullA(s), kTileA + 2 * kSfTile);
          else
            tc::mbar_arrive(sm.qfree(s));
        }
      }
      for (int64_t j = (it > S ? it - S : 0); j < it; ++j) {
        const int s = static_cast<int>(j % S);
        const uint32_t ph = static_cast<uint32_t>(j / S) & 1;
        // this thread's copies have landed, and every CTA's MMA is done with
        // the last stages: no push into this CTA's memory, and none out of
        // it, is still in flight when the CTA exits
        tc::mbar_wait(sm.fullB(s), ph, sm.abort_flag, g.status, kStatusDrain, false);
        tc::mbar_wait(sm.empty(s), ph, sm.abort_flag, g.status, kStatusDrain, false);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int64_t it = 0;
      uint32_t tile_par = 0;
      bool ok = true;
      for (int64_t u = cluster; ok && u < units; u += nclusters, tile_par ^= 1) {
        ok = tc::mbar_wait(sm.tempty(), tile_par ^ 1, sm.abort_flag, g.status, kStatusMmaB);
        if (ok) tc::tc_fence_after();
        for (int kb = 0; ok && kb < nk; ++kb, ++it) {
          const int s = static_cast<int>(it % S);
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1;
          if (!tc::mbar_wait(sm.fullB(s), ph, sm.abort_flag, g.status, kStatusMmaB) ||
              !tc::mbar_wait(sm.fullA(s), ph, sm.abort_flag, g.status, kStatusMmaA)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          issue_kblock(sm, tmem, s, kb == 0);
          if (CL > 1)
            tc::tc_commit_multicast(sm.empty(s), static_cast<uint16_t>((1u << CL) - 1));
          else
            tc::tc_commit(sm.empty(s));
        }
        tc::tc_commit(sm.tfull());
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------ quantizer (own K-blocks), epilogue
    // lane j16 = lane & 15 takes elements 16 j16 .. 16 j16 + 15 of the
    // K-block (a lane pair is one 32-element block); the rows are below
    const int ew = warp - 2;
    const int j16 = lane & 15;
    const int j = j16 >> 1;   // block column within the K-block, 0..7
    const bool leader = (ew == 0 && lane == 0);
    const int64_t total = static_cast<int64_t>(nk) *
                          ((units - cluster + nclusters - 1) / nclusters);   // this CTA's ring length
    // staging loads: issued by the leader for this CTA's K-blocks in ring order
    auto stage_in = [&](int64_t it) {
      const int64_t u = unit_of(it);
      const int kb = static_cast<int>(it % nk);
      tc::mbar_arrive_expect_tx(sm.stg_full(), C::kStaging);
      tc::tma_load_2d(sm.sStg, &tmX, kb * kGemmBK, static_cast<int>((u / groups_n) * kGemmBM),
                      sm.stg_full());
    };
    bool stg_pending = false;   // (leader) a staging load is in flight
    if (leader && rank < total) {
      tc::prefetch_tmap(&tmX);
      stage_in(rank);
      stg_pending = true;
    }
    int64_t it = 0;
    uint32_t tile_par = 0, stg_par = 0;
    uint32_t qpar = 0;   // bit s: parity of the next qfree phase of stage s
    bool ok = true;
    for (int64_t u = cluster; ok && u < units; u += nclusters, tile_par ^= 1) {
      const int64_t m0 = (u / groups_n) * kGemmBM;
      const int64_t n0 = ((u % groups_n) * CL + rank) * BN;
      const bool write_a = (u % groups_n) == 0;   // the first n-group writes A's codes out
      for (int kb = 0; kb < nk; ++kb, ++it) {
        if (it % CL != rank) continue;
        const int s = static_cast<int>(it % S);
        // every thread waits (acquire); the eight warps then take one
        // decision, since they meet at a named barrier below
        const bool got_stg =
            tc::mbar_wait(sm.stg_full(), stg_par, sm.abort_flag, g.status, kStatusStaging);
        const bool got = got_stg && tc::mbar_wait(sm.qfree(s), (qpar >> s) & 1, sm.abort_flag,
                                                  g.status, kStatusQuant);
        if (got) qpar ^= 1u << s;
        if (got_stg) {
          stg_par ^= 1;
          stg_pending = false;
        }
        if (!tc::named_all(2, C::kWorkWarps * 32, got)) {
          ok = false;
          break;
        }
        // pass p: rows 16 p + 2 ew (lanes 0-15) and 16 p + 2 ew + 1 (lanes
        // 16-31); passes wholly past M are skipped (their rows of D are never
        // stored, so what the stage holds there does not matter)
        const int64_t valid = g.M - m0;
        const int npass = valid >= 128 ? 8 : static_cast<int>((valid + 15) / 16);
        // the warp's slices are read four at a time before any is
        // processed, so that four independent blocks' dependency chains
        // interleave; a lane reads the two 16-byte halves of its 32 bytes in
        // an order that spreads each quarter-warp over all 32 banks
        const uint32_t hsw = ((lane >> 2) & 1) * 16;
#pragma unroll
        for (int p0 = 0; p0 < 8; p0 += 4) {
          V16 v[4];
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            const int p = p0 + i4;
            if (p < npass) {
              const int r = 16 * p + 2 * ew + (lane >> 4);
              const uint32_t src = sm.sStg + r * (kGemmBK * 2) + j16 * 32;
              uint32_t a[4], b[4];
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                           : "r"(src + hsw));
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
                           : "r"(src + (hsw ^ 16)));
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                v[i4].w[i] = hsw ? b[i] : a[i];
                v[i4].w[4 + i] = hsw ? a[i] : b[i];
              }
            }
          }
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            const int p = p0 + i4;
            const int r = 16 * p + 2 * ew + (lane >> 4);
            if (p >= npass) {
              // the tiled scale buffer's padding rows hold zeros
              if (write_a && g.a_scales_out && (lane & 1) == 0)
                g.a_scales_out[((m0 / 128) * T + 2 * kb + (j >> 2)) * kSfTile + (r & 31) * 16 +
                               ((r >> 5) & 3) * 4 + (j & 3)] = 0;
              continue;
            }
            const uint32_t pa = pair_max(amax_bits16(v[i4]));
            const BlockScale bs = decide_scale<kFmtE2M1, RULE, kMbsNone>(v[i4], pa, 0);
            const uint2 c = codes_fp4<kMbsNone>(v[i4], bs);
            const uint32_t dst = sm.sA + s * kTileA + r * kRowBytes +
                                 ((((j16 >> 1) ^ (r & 7)) & 7) << 4) + ((j16 & 1) << 3);
            asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(dst), "r"(c.x), "r"(c.y) : "memory");
            const uint32_t sdst = sm.sSFA + s * C::kSfA + (j >> 2) * kSfTile + (r & 31) * 16 +
                                  ((r >> 5) & 3) * 4 + (j & 3);
            if ((lane & 1) == 0)
              asm volatile("st.shared.u8 [%0], %1;" ::"r"(sdst), "r"(bs.byte) : "memory");
            if (write_a) {
              const int64_t m = m0 + r;
              if (g.a_codes_out && m < g.M)
                st_stream8(g.a_codes_out + m * (g.K / 2) + static_cast<int64_t>(kb) * kRowBytes + 8 * j16, c);
              if (g.a_scales_out && (lane & 1) == 0)
                g.a_scales_out[((m0 / 128) * T + 2 * kb + (j >> 2)) * kSfTile + (r & 31) * 16 +
                               ((r >> 5) & 3) * 4 + (j & 3)] = static_cast<uint8_t>(bs.byte);
            }
          }
        }
        tc::fence_proxy_async_smem();
        tc::named_sync(1, C::kWorkWarps * 32);   // the stage is written, the staging tile read
        if (leader) {
          if (it + CL < total) {
            stage_in(it + CL);
            stg_pending = true;
          }
#pragma unroll
          for (uint32_t p = 1; p < CL; ++p) {
            const uint32_t peer = (rank + p) % CL;
            const uint32_t bar = tc::mapa(sm.fullA(s), peer);
            tc::bulk_push(tc::mapa(sm.sA + s * kTileA, peer), sm.sA + s * kTileA, kTileA, bar);
            tc::bulk_push(tc::mapa(sm.sSFA + s * C::kSfA, peer), sm.sSFA + s * C::kSfA,
                          2 * kSfTile, bar);
          }
          tc::mbar_arrive(sm.fullA(s));
        }
      }
      if (!ok) break;
      if (!epilogue_tile(sm, g, tmem, tile_par, m0, n0, warp, lane)) break;
    }
    // a staging load issued but never consumed (abort) lands before the exit
    if (leader && stg_pending)
      tc::mbar_wait(sm.stg_full(), stg_par, sm.abort_flag, g.status, kStatusDrain, false);
    tc::tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, C::kTmemCols);
  }
  if (CL > 1) tc::cluster_sync();   // no CTA leaves while a peer may still address it
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

// Tensor map of bf16 A [M, K] read in 256-element x 128-row boxes, row-major
// in shared memory without swizzle (rows past M read as zero).
bool bf16_tmap(CUtensorMap* tm, const void* a, int64_t M, int64_t K) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K * 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kGemmBK), static_cast<cuuint32_t>(kGemmBM)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stream-ordered scratch comes from a memory pool this library creates once
// per device and never trims (release threshold: all), so that after the
// first call an allocation maps no memory and costs the host microseconds;
// the default pool gives its memory back at every synchronisation and maps it
// again on the next call. The pools live as long as the process.
cudaError_t scratch_pool(cudaMemPool_t* out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static cudaMemPool_t pools[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    e = cudaMemPoolCreate(&p, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = ~0ull;
    e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) {
      cudaMemPoolDestroy(p);
      return e;
    }
    pools[dev] = p;
  }
  *out = pools[dev];
  return cudaSuccess;
}

int sm_count_of_current_device(cudaError_t* e) {
  int dev = 0, sms = 0;
  *e = cudaGetDevice(&dev);
  if (*e == cudaSuccess) *e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int BN, int S>
cudaError_t launch_prequant(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g,
                            cudaStream_t st) {
  using C = GemmCfg<BN, S, false>;
  auto kern = gemm_kernel<BN, S>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (the shared memory allows no second), never
  // more CTAs than tiles
  const int64_t tiles = ((g.M + kGemmBM - 1) / kGemmBM) * ((g.N + BN - 1) / BN);
  const int sms = sm_count_of_current_device(&e);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
  kern<<<grid, C::kThreads, C::kSmem, st>>>(tmA, tmB, g);
  return cudaGetLastError();
}

template <int BN, int S, int RULE>
cudaError_t launch_staged(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g,
                          const StreamArgs& q, unsigned long long* ready, cudaStream_t st) {
  using C = GemmCfg<BN, S, false>;
  auto kern = gemm_staged_kernel<BN, S, RULE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  const int sms = sm_count_of_current_device(&e);
  if (e != cudaSuccess) return e;
  // one CTA per SM, all resident at once (the producers wait on other CTAs'
  // quantizer warps); CTAs beyond the tile count only quantize
  CUtensorMap a_map = tmA, b_map = tmB;
  GemmArgs ga = g;
  QuantPrologue<RULE> pro{};
  pro.q = q;
  pro.ready = ready;
  pro.mtile_slices = static_cast<int64_t>(kGemmBM) * g.K / 16;
  void* args[] = {&a_map, &b_map, &ga, &pro};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(sms),
                                  dim3(C::kThreads + 32 * QuantPrologue<RULE>::kWarps), args,
                                  C::kSmem, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int BN, int S, int RULE>
cudaError_t launch_staged_sync(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g,
                               const StreamArgs& q, cudaStream_t st) {
  using C = GemmCfg<BN, S, false>;
  auto kern = gemm_staged_sync_kernel<BN, S, RULE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((g.M + kGemmBM - 1) / kGemmBM) * ((g.N + BN - 1) / BN);
  const int sms = sm_count_of_current_device(&e);
  if (e != cudaSuccess) return e;
  // every CTA resident at once (one per SM): the grid barrier needs it
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
  CUtensorMap a_map = tmA, b_map = tmB;
  GemmArgs ga = g;
  StreamArgs qa = q;
  void* args[] = {&a_map, &b_map, &ga, &qa};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(C::kThreads),
                                  args, C::kSmem, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The staged form for one rounding rule: the grid-barrier kernel when the
// GEMM's tiles fit in one wave, else the overlapped kernel with its per-m-tile
// ready counts at `ready` (zero on the stream before the launch).
template <int RULE>
cudaError_t launch_staged_rule(bool wide, bool one_wave, const CUtensorMap& tmA,
                               const CUtensorMap& tmB, const GemmArgs& g, const StreamArgs& q,
                               unsigned long long* ready, cudaStream_t st) {
  if (one_wave)
    return wide ? launch_staged_sync<256, 4, RULE>(tmA, tmB, g, q, st)
                : launch_staged_sync<128, 6, RULE>(tmA, tmB, g, q, st);
  return wide ? launch_staged<256, 4, RULE>(tmA, tmB, g, q, ready, st)
              : launch_staged<128, 6, RULE>(tmA, tmB, g, q, ready, st);
}

// Where a staged launch keeps A's quantized form and its band counters:
// codes [M, K/2], then (256-byte aligned) the tiled scales, then the counters
// (one per 128-row band), each part present only where needed.
struct StagedScratch {
  size_t scales, ready, end;
};

StagedScratch staged_scratch(int64_t M, int64_t K, bool codes, bool scales, bool ready) {
  const auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  const size_t mtiles = static_cast<size_t>((M + kGemmBM - 1) / kGemmBM);
  StagedScratch l{};
  l.scales = codes ? up(static_cast<size_t>(M) * static_cast<size_t>(K / 2)) : 0;
  l.ready = l.scales + (scales ? up(mtiles * static_cast<size_t>(K / 128) * kSfTile) : 0);
  l.end = l.ready + (ready ? mtiles * 8 : 0);
  return l;
}

// Zeroes, on the stream, what a staged launch reads before writing: the
// padding rows of the last band of `scales` (when M is not a multiple of
// 128) and the band counters at `ready`; a NULL pointer skips its part.
cudaError_t clear_staged(uint8_t* scales, unsigned long long* ready, int64_t M, int64_t K,
                         cudaStream_t st) {
  const int64_t mtiles = (M + kGemmBM - 1) / kGemmBM;
  if (scales && M % kGemmBM != 0) {
    const size_t band = static_cast<size_t>(K / 128) * kSfTile;
    const cudaError_t e = cudaMemsetAsync(scales + (mtiles - 1) * band, 0, band, st);
    if (e != cudaSuccess) return e;
  }
  if (ready) return cudaMemsetAsync(ready, 0, static_cast<size_t>(mtiles) * 8, st);
  return cudaSuccess;
}

template <int BN, int S, int CL, int RULE>
cudaError_t launch_fused(const CUtensorMap& tmX, const CUtensorMap& tmB, const GemmArgs& g,
                         cudaStream_t st) {
  using C = GemmCfg<BN, S, true>;
  auto kern = gemm_fused_kernel<BN, S, CL, RULE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  const int64_t tiles_n = (g.N + BN - 1) / BN;
  const int64_t units = ((g.M + kGemmBM - 1) / kGemmBM) * ((tiles_n + CL - 1) / CL);
  const int sms = sm_count_of_current_device(&e);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // persistent clusters: as many as can be resident at once, never more than
  // there are units
  cfg.gridDim = dim3(static_cast<unsigned>((sms / CL) * CL));
  int max_clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
  if (e != cudaSuccess) return e;
  if (max_clusters < 1) return cudaErrorInvalidConfiguration;
  const int64_t nclusters = units < max_clusters ? units : max_clusters;
  cfg.gridDim = dim3(static_cast<unsigned>(nclusters * CL));
  e = cudaLaunchKernelEx(&cfg, kern, tmX, tmB, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The cluster width of the fused kernel: up to MX_GEMM_MAX_CLUSTER (a
// build-time knob, default 4) CTAs share each A tile, no wider than the row
// of N tiles.
#ifndef MX_GEMM_MAX_CLUSTER
#define MX_GEMM_MAX_CLUSTER 4
#endif
template <int BN, int S, int RULE>
cudaError_t launch_fused_cl(const CUtensorMap& tmX, const CUtensorMap& tmB, const GemmArgs& g,
                            cudaStream_t st) {
  const int64_t tiles_n = (g.N + BN - 1) / BN;
  if (MX_GEMM_MAX_CLUSTER >= 4 && tiles_n >= 4) return launch_fused<BN, S, 4, RULE>(tmX, tmB, g, st);
  if (MX_GEMM_MAX_CLUSTER >= 2 && tiles_n >= 2) return launch_fused<BN, S, 2, RULE>(tmX, tmB, g, st);
  return launch_fused<BN, S, 1, RULE>(tmX, tmB, g, st);
}

template <int RULE>
cudaError_t launch_fused_bn(bool wide, const CUtensorMap& tmX, const CUtensorMap& tmB,
                            const GemmArgs& g, cudaStream_t st) {
  if (wide) return launch_fused_cl<256, 3, RULE>(tmX, tmB, g, st);
  return launch_fused_cl<128, 4, RULE>(tmX, tmB, g, st);
}

}  // namespace

cudaError_t launch_gemm(const void* a, const uint8_t* a_scales, int a_rule, bool a_on_chip,
                        const void* b_codes, const uint8_t* b_scales, int64_t M, int64_t N,
                        int64_t K, int out_fp32, void* d, void* a_codes_out,
                        uint8_t* a_scales_out, int* status, cudaStream_t st) {
  const bool fused = a_scales == nullptr;
  // 256-wide tiles unless that leaves SMs idle on a small problem
  const bool wide = N > 128 && ((M + kGemmBM - 1) / kGemmBM) * ((N + 255) / 256) >= 148;
  CUtensorMap tmA{}, tmB{};
  if (!code_tmap(&tmB, b_codes, N, K, wide ? 256 : 128)) return cudaErrorInvalidValue;
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
  if (!fused) {
    if (!code_tmap(&tmA, a, M, K, kGemmBM)) return cudaErrorInvalidValue;
    return wide ? launch_prequant<256, 4>(tmA, tmB, g, st) : launch_prequant<128, 6>(tmA, tmB, g, st);
  }
  if (a_on_chip) {
    if (!bf16_tmap(&tmA, a, M, K)) return cudaErrorInvalidValue;
    switch (a_rule) {
      case kCeil: return launch_fused_bn<kCeil>(wide, tmA, tmB, g, st);
      case kOasRule: return launch_fused_bn<kOasRule>(wide, tmA, tmB, g, st);
      case kOas: return launch_fused_bn<kOas>(wide, tmA, tmB, g, st);
      default: return launch_fused_bn<kFloor>(wide, tmA, tmB, g, st);
    }
  }
  // Staged: A is quantized into the caller's buffers, or (where the caller
  // gives none) into stream-ordered scratch, and the GEMM runs on them in the
  // same cooperative launch; one scratch allocation holds what the caller
  // does not give and the band counters.
  cudaError_t e = cudaSuccess;
  const int sms = sm_count_of_current_device(&e);
  if (e != cudaSuccess) return e;
  const int64_t bn = wide ? 256 : 128;
  const bool one_wave = ((M + kGemmBM - 1) / kGemmBM) * ((N + bn - 1) / bn) <= sms;
  uint8_t* codes = static_cast<uint8_t*>(a_codes_out);
  uint8_t* scales = a_scales_out;
  const StagedScratch l = staged_scratch(M, K, !codes, !scales, !one_wave);
  uint8_t* scratch = nullptr;
  if (l.end > 0) {
    cudaMemPool_t pool = nullptr;
    e = scratch_pool(&pool);
    if (e != cudaSuccess) return e;
    e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&scratch), l.end, pool, st);
    if (e != cudaSuccess) return e;
    if (!codes) codes = scratch;
  }
  // (the caller's scales had their padding cleared by the API layer)
  const bool own_scales = !scales;
  if (own_scales) scales = scratch + l.scales;
  auto* ready = one_wave ? nullptr : reinterpret_cast<unsigned long long*>(scratch + l.ready);
  e = clear_staged(own_scales ? scales : nullptr, ready, M, K, st);
  if (e == cudaSuccess && !code_tmap(&tmA, codes, M, K, kGemmBM)) e = cudaErrorInvalidValue;
  if (e == cudaSuccess) {
    StreamArgs q{};
    q.x = static_cast<const uint8_t*>(a);
    q.nslices = M * K / 16;
    q.codes = codes;
    q.scales = scales;
    q.smap.bpr = K / 32;
    q.smap.nct = (K / 32 + 3) / 4;
    q.smap.inv = 1.0 / static_cast<double>(K / 32);
    g.a_scales = scales;
    switch (a_rule) {
      case kCeil: e = launch_staged_rule<kCeil>(wide, one_wave, tmA, tmB, g, q, ready, st); break;
      case kOasRule:
        e = launch_staged_rule<kOasRule>(wide, one_wave, tmA, tmB, g, q, ready, st);
        break;
      case kOas: e = launch_staged_rule<kOas>(wide, one_wave, tmA, tmB, g, q, ready, st); break;
      default: e = launch_staged_rule<kFloor>(wide, one_wave, tmA, tmB, g, q, ready, st);
    }
  }
  if (scratch) {
    const cudaError_t ef = cudaFreeAsync(scratch, st);
    if (e == cudaSuccess) e = ef;
  }
  return e;
}

// ------------------------------------ quantize + GEMM without allocation --
// Callers that may not allocate device memory while they run (a serving
// process that reserves its memory once at start-up and keeps it fixed, or a
// runtime whose memory pools are unavailable) cannot use the default staged
// form, which takes A's quantized form and the band counters from a
// stream-ordered pool. This variant takes them from one array in the
// library's device memory, of fixed size; every call shares it.

}  // namespace mxk

// The array (file scope). Host code cannot use its name as an address: the
// device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t mx_noalloc_scratch[MX_NOALLOC_SCRATCH_BYTES];

namespace mxk {

// codes [M, K/2], then (256-byte aligned) the tiled scales, then the band
// counters; the total must fit the array.
bool noalloc_fits(int64_t M, int64_t K) {
  return staged_scratch(M, K, true, true, true).end <=
         static_cast<size_t>(MX_NOALLOC_SCRATCH_BYTES);
}

namespace {

// The array's device address on the current device, looked up on the first
// call on that device.
cudaError_t noalloc_scratch(uint8_t** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static uint8_t* ptrs[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, mx_noalloc_scratch);
    if (e != cudaSuccess) return e;
    ptrs[dev] = static_cast<uint8_t*>(p);
  }
  *out = ptrs[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_quant_gemm_noalloc(const void* a, int a_rule, const void* b_codes,
                                      const uint8_t* b_scales, int64_t M, int64_t N, int64_t K,
                                      int out_fp32, void* d, int* status, cudaStream_t st) {
  if (!noalloc_fits(M, K)) return cudaErrorInvalidValue;
  uint8_t* base = nullptr;
  cudaError_t e = noalloc_scratch(&base);
  if (e != cudaSuccess) return e;
  const StagedScratch l = staged_scratch(M, K, true, true, true);
  uint8_t* codes = base;
  uint8_t* scales = base + l.scales;
  const bool wide = N > 128 && ((M + kGemmBM - 1) / kGemmBM) * ((N + 255) / 256) >= 148;
  const int64_t bn = wide ? 256 : 128;
  const int sms = sm_count_of_current_device(&e);
  if (e != cudaSuccess) return e;
  const bool one_wave = ((M + kGemmBM - 1) / kGemmBM) * ((N + bn - 1) / bn) <= sms;
  auto* ready = one_wave ? nullptr : reinterpret_cast<unsigned long long*>(base + l.ready);
  // the array keeps the previous call's bytes: zero what is read before it
  // is written (the padding rows of the last band of scales, the counters)
  e = clear_staged(scales, ready, M, K, st);
  if (e != cudaSuccess) return e;
  CUtensorMap tmA{}, tmB{};
  if (!code_tmap(&tmB, b_codes, N, K, wide ? 256 : 128)) return cudaErrorInvalidValue;
  if (!code_tmap(&tmA, codes, M, K, kGemmBM)) return cudaErrorInvalidValue;
  GemmArgs g{};
  g.a_bf16 = static_cast<const uint8_t*>(a);
  g.a_scales = scales;
  g.b_scales = b_scales;
  g.d = static_cast<uint8_t*>(d);
  g.status = status;
  g.M = M;
  g.N = N;
  g.K = K;
  g.out_fp32 = out_fp32;
  StreamArgs q{};
  q.x = static_cast<const uint8_t*>(a);
  q.nslices = M * K / 16;
  q.codes = codes;
  q.scales = scales;
  q.smap.bpr = K / 32;
  q.smap.nct = (K / 32 + 3) / 4;
  q.smap.inv = 1.0 / static_cast<double>(K / 32);
  switch (a_rule) {
    case kCeil: return launch_staged_rule<kCeil>(wide, one_wave, tmA, tmB, g, q, ready, st);
    case kOasRule: return launch_staged_rule<kOasRule>(wide, one_wave, tmA, tmB, g, q, ready, st);
    case kOas: return launch_staged_rule<kOas>(wide, one_wave, tmA, tmB, g, q, ready, st);
    default: return launch_staged_rule<kFloor>(wide, one_wave, tmA, tmB, g, q, ready, st);
  }
}

}  // namespace mxk
