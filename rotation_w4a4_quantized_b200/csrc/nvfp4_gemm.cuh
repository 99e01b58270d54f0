// nvfp4_gemm.cuh -- block-scaled FP4 GEMM with fused dequantisation on tcgen05 (sm_100a): the
// floating-point variant of the rotated 4-bit layer.
//
// What it computes (ComfyUI issue #14735, ConvRot author's comment: ConvRot also suits
// floating-point quantisation; here in NVFP4, e2m1 elements with an unsigned-e4m3 scale per 16
// consecutive K and an fp32 scale per row):
//   acc[m,n] = sum_k (ex[m,k] * sx_blk[m, k/16]) * (ew[n,k] * sw_blk[n, k/16])   (fp32 on the
//              tensor cores; every product is exact, the sum is accumulated in fp32)
//   Y[m,n]   = bf16_rne((acc * gx[m]) * gw[n] + float(bias[n]))
//
// How (B200 design): e2m1 is a native operand type of tcgen05.mma kind::mxf4nvf4, read packed
// (two per byte) from shared memory, so the codes go from HBM to the tensor cores by TMA with no
// conversion stage. Persistent CTA pairs walk 256 x 192 output tiles. Per K stage (256 elements
// = 128 bytes per row) each CTA loads its 128 A rows and its 96 B rows (completing on the even
// CTA's barrier) and the stage's distinct block-scale bytes (completing on its own barrier):
// A's 512-byte atoms as the activation quantisation writes them, and the first lane quadrant
// (1 KB) of each of B's 4096-byte weight images, 6 KB in all. The MMA reads a 64-K chunk's
// scales (4 per row) from 4 tensor-memory columns of 32 lanes, the same in every lane quadrant
// (A: row r at lane r % 32, column r / 32; B: two such groups of 4 columns, one per 128-row half
// of the tile). Four scale warps per CTA, one per lane quadrant, put them there with
// tcgen05.st, so the tensor pipe runs no tcgen05.cp (the copies run in order with the MMAs and
// cost it about 30 ns each). Tensor memory holds two 192-column accumulators and two
// 48-column scale buffers: the warps fill buffer g % 2 with stage g's scales once the MMAs of
// stage g - 2 have completed (that stage's own commit on `empty`), while the MMAs of stage
// g - 1 run. The even CTA's MMA thread waits for a stage's codes and scales and issues its 4
// block-scaled MMAs (K = 64 each). Epilogue as in the integer GEMMs (fp32 accumulator), one
// staging block per warp. Every wait is bounded.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "gemm_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace convrot {

namespace fp4_detail {

using gemm_common::kEpiWarps;

constexpr int BM = 256;          // tile rows per CTA pair
constexpr int BMC = BM / 2;      // A rows per CTA (TMEM lanes)
constexpr int BN = 192;          // tile columns (accumulator columns)
constexpr int BNC = BN / 2;      // B rows per CTA
constexpr int BKB = 128;         // bytes of packed e2m1 per row per stage (256 K)
constexpr int kChunks = 4;       // MMAs (64 K each) per stage
#ifndef CONVROT_FP4_STAGES
#define CONVROT_FP4_STAGES 6
#endif
constexpr int SU = CONVROT_FP4_STAGES;
constexpr int kSfWarps = 4;      // scale warps (one per TMEM lane quadrant)
constexpr int kThreads = 32 * (2 + kEpiWarps + kSfWarps);
constexpr int kAccCols = BN;
constexpr int kTmemCols = 512;
// two scale buffers (stage g in buffer g % 2), each A (4 columns per chunk) then B (8 columns
// per chunk)
constexpr int kSfCol = 2 * kAccCols;                   // 384
constexpr int kSfBufCols = 12 * kChunks;               // 48
constexpr int kSfbOff = 4 * kChunks;                   // 16
static_assert(kSfCol % 8 == 0 && kSfBufCols % 8 == 0 && kSfbOff % 8 == 0 &&
                  kSfCol + 2 * kSfBufCols <= kTmemCols,
              "TMEM budget");

// tile rows of the block-scale layouts (activations: 128-row tiles of atoms; weights: 192-row
// tiles of images)
constexpr int kSfTileA = BMC;
constexpr int kSfTileB = BN;
constexpr int kEpiBufs = 1;
constexpr int kEpiSmem = kEpiWarps * kEpiBufs * gemm_common::kStageBytes;

constexpr int kTA = BMC * BKB;               // 16 KB
constexpr int kTB = BNC * BKB;               // 12 KB
// Scale chunks hold 4 scales per row and cover 64 K: 4 per stage.
constexpr int kSfK = 64;
constexpr int kSfChunks = BKB * 2 / kSfK;                // per stage
constexpr int kSA = kSfChunks * 512;                     // 2 KB: A's atoms of a stage
constexpr int kSB = kSfChunks * 1024;                    // 4 KB: B images' first quadrants
constexpr uint32_t kStageTx = 2u * (kTA + kTB);          // code tiles of the pair
constexpr uint32_t kSfTx = kSA + kSB;                    // this CTA's scales

struct Smem {
  static constexpr int uA = 0;
  static constexpr int uB = uA + SU * kTA;
  static constexpr int sA = uB + SU * kTB;
  static constexpr int sB = sA + SU * kSA;
  static constexpr int stg = sB + SU * kSB;
  static constexpr int bars = stg + kEpiSmem;
  static constexpr int n_bars = 3 * SU + 4 + 1 + 2;
  static constexpr int misc = bars + n_bars * 8;
  static constexpr int total = misc + 16;
};
static_assert(Smem::uB % 1024 == 0 && Smem::sA % 1024 == 0, "1024-byte aligned tiles");
constexpr size_t kSmemBytes = Smem::total + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

using TileGrid = gemm_common::TileGrid<BM, BN>;

template <GemmOut kMode>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                  const __grid_constant__ CUtensorMap tmY, const float* __restrict__ gx,
                  const float* __restrict__ gw, const uint16_t* __restrict__ bias,
                  void* __restrict__ out, int64_t ldo, int M, int N, int K4, int tma_out) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + Smem::bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + SU;
  uint64_t* acc_full = bars + 2 * SU;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint64_t* sf_full = mma_done + 1;          // this CTA's scales of a stage have landed
  uint64_t* sf_ready = sf_full + SU;         // (even CTA) a scale buffer is written in both CTAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + Smem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + Smem::misc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const TileGrid grid{(M + BM - 1) / BM, (N + BN - 1) / BN};
  const int num_tiles = grid.count();
  const int kc_total = K4 / 64;                          // 64-K chunks per row
  const int num_k = (kc_total + kChunks - 1) / kChunks;  // stages per tile
  const int sf_total = (K4 + kSfK - 1) / kSfK;           // scale chunks per row

  if (threadIdx.x == 0) {
    for (int i = 0; i < SU; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
      mbar_init(sf_full + i, 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(sf_ready + i, 2 * kSfWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 2 * kEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSA);
    tma_prefetch_desc(&tmSB);
    if (tma_out) tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dependency_wait();   // set-up above overlapped the previous kernel's tail
  launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t full_even = mapa_shared(smem_u32(full), 0);
      uint32_t g = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += num_pairs) {
        int m0, n0;
        grid.coords(t, m0, n0);
        const int a_tile = (m0 + static_cast<int>(rank) * BMC) / kSfTileA;
        const int b_tile = n0 / kSfTileB;
        for (int s = 0; s < num_k; ++s, ++g) {
          const uint32_t slot = g % SU;
          if (g >= SU && !mbar_wait(empty + slot, ((g / SU) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full + slot, kStageTx);
          const uint32_t bar = full_even + slot * 8;
          tma_load_2d_pair(base + Smem::uA + slot * kTA, &tmA, bar, s * BKB,
                           m0 + static_cast<int>(rank) * BMC);
          tma_load_2d_pair(base + Smem::uB + slot * kTB, &tmB, bar, s * BKB,
                           n0 + static_cast<int>(rank) * BNC);
          // this CTA's scales: A's atoms of the stage (rows of 128 bytes, 4 per atom; atoms
          // past the tile's end read zeros) and the first 8 of each B image's 32 rows
          mbar_arrive_expect_tx(sf_full + slot, kSfTx);
          tma_load_3d(base + Smem::sA + slot * kSA, &tmSA, sf_full + slot, 0,
                      s * kSfChunks * 4, a_tile);
          tma_load_3d(base + Smem::sB + slot * kSB, &tmSB, sf_full + slot, 0, 0,
                      b_tile * sf_total + s * kSfChunks);
        }
      }
      if (rank == 0) {
        for (uint32_t s = (g > SU ? g - SU : 0); s < g; ++s) {
          uint32_t polls = 0;
          while (!mbar_try_wait_cluster(full + (s % SU), (s / SU) & 1) && ++polls < kMaxPolls) {
          }
        }
      }
      // this CTA's scale loads complete on its own barrier; on a normal exit the scale warps
      // have consumed every phase, after a wait that gave up some may still be landing: let
      // them land before the CTA's shared memory goes away
      for (uint32_t s = (g > SU ? g - SU : 0); s < g; ++s) {
        uint32_t polls = 0;
        while (!mbar_try_wait(sf_full + (s % SU), (s / SU) & 1) && ++polls < kMaxPolls) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_fp4_bs(BM, BN);
      uint32_t g = 0;
      int ti = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += num_pairs, ++ti) {
        const int b = ti & 1;
        if (ti >= 2 && !mbar_wait_cluster(acc_empty + b, ((ti >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * kAccCols;
        for (int s = 0; s < num_k && ok; ++s, ++g) {
          const uint32_t slot = g % SU;
          if (!mbar_wait_cluster(full + slot, (g / SU) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nck = (kc_total - s * kChunks) < kChunks ? (kc_total - s * kChunks) : kChunks;
          const uint32_t a0 = smem_u32(base + Smem::uA + slot * kTA);
          const uint32_t b0 = smem_u32(base + Smem::uB + slot * kTB);
          // CTA-scope acquire: the writers' tcgen05.wait::st completed their stores before
          // they arrived
          if (!mbar_wait(sf_ready + (g & 1), (g >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa = tmem_base + kSfCol + (g & 1) * kSfBufCols;
          const uint32_t sfb = sfa + kSfbOff;
          for (int q = 0; q < nck; ++q) {
            const uint32_t acc = (s > 0 || q > 0) ? 1u : 0u;
            mma_fp4_bs_pair(d_tmem, smem_desc_k128(a0 + q * 32), smem_desc_k128(b0 + q * 32),
                            idesc, sfa + 4 * q, sfb + 8 * q, acc);
          }
          mma_commit_pair(empty + slot, 0x3);
        }
        if (ok) mma_commit_pair(acc_full + b, 0x3);
      }
      mma_commit_pair(mma_done, 0x3);
    }
    if (lane == 0) {
      uint32_t polls = 0;
      while (!mbar_try_wait_cluster(mma_done, 0) && ++polls < kMaxPolls) {
      }
    }
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    const uint32_t acc_empty_even = mapa_shared(smem_u32(acc_empty), 0);
    unsigned char* stg = base + Smem::stg + (warp - 2) * kEpiBufs * gemm_common::kStageBytes;
    int ti = 0;
    uint32_t nstore = 0;
    for (int t = pair; t < num_tiles; t += num_pairs, ++ti) {
      const int b = ti & 1;
      if (!mbar_wait_cluster(acc_full + b, (ti >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      int m0, n0;
      grid.coords(t, m0, n0);
      const int row0 = m0 + static_cast<int>(rank) * BMC + q * 32;
      const uint32_t acc_tmem = tmem_base + b * kAccCols + (static_cast<uint32_t>(q * 32) << 16);
      gemm_common::epilogue_tile<kMode, BN, 0, true, kEpiBufs, true>(
          acc_tmem, row0, n0, M, N, gx, gw, bias, out, ldo, tma_out, &tmY, stg, nstore,
          acc_empty_even + b * 8);
    }
    if (lane == 0) bulk_wait_group<0>();
  } else {
    // ------------------------------------------------------------------ scale warps (6..9)
    // Warp w writes TMEM lanes 32 (w % 4) .. + 31; each lane L holds row L of every scale
    // group: A's atom bytes 16 L .. 16 L + 15 (4 columns), B's half h at 256 (L / 8) + 128 h +
    // 16 (L % 8) of the image's first quadrant (4 columns per half).
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t ready_even = mapa_shared(smem_u32(sf_ready), 0);
    const uint32_t b_off = 256u * static_cast<uint32_t>(lane >> 3) + 16u * (lane & 7);
    uint32_t g = 0;
    bool ok = true;
    for (int t = pair; t < num_tiles && ok; t += num_pairs) {
      for (int s = 0; s < num_k; ++s, ++g) {
        const uint32_t slot = g % SU;
        ok = __all_sync(0xffffffffu, mbar_wait(sf_full + slot, (g / SU) & 1, abort_flag));
        if (!ok) break;
        // the stage's scales into registers (whole staging area; chunks past the tile's end
        // land in columns no MMA reads), then into buffer g % 2 with one store per operand
        constexpr int kC = kSfChunks;
        const unsigned char* sa = base + Smem::sA + slot * kSA + 16 * lane;
        const unsigned char* sb = base + Smem::sB + slot * kSB + b_off;
        uint32_t ra[4 * kC], rb[8 * kC];
#pragma unroll
        for (int k = 0; k < kC; ++k) {
          const uint4 va = *reinterpret_cast<const uint4*>(sa + 512 * k);
          const uint4 vb0 = *reinterpret_cast<const uint4*>(sb + 1024 * k);
          const uint4 vb1 = *reinterpret_cast<const uint4*>(sb + 1024 * k + 128);
          ra[4 * k] = va.x; ra[4 * k + 1] = va.y; ra[4 * k + 2] = va.z; ra[4 * k + 3] = va.w;
          rb[8 * k] = vb0.x; rb[8 * k + 1] = vb0.y; rb[8 * k + 2] = vb0.z; rb[8 * k + 3] = vb0.w;
          rb[8 * k + 4] = vb1.x; rb[8 * k + 5] = vb1.y; rb[8 * k + 6] = vb1.z;
          rb[8 * k + 7] = vb1.w;
        }
        // buffer g % 2 was last read by the MMAs of stage g - 2 (their commit on `empty`)
        if (g >= 2) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(empty + (g - 2) % SU, ((g - 2) / SU) & 1, abort_flag));
          if (!ok) break;
        }
        tc_fence_after();
        const uint32_t sfa = lane_base + kSfCol + (g & 1) * kSfBufCols;
        tmem_st_32x32b_x16(sfa, ra);
        tmem_st_32x32b_x32(sfa + kSfbOff, rb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(ready_even + 8 * (g & 1));
      }
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <GemmOut kMode>
cudaError_t launch_mode(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmSA,
                        const CUtensorMap& tmSB, const CUtensorMap& tmY, const float* gx,
                        const float* gw, const uint16_t* bias, void* out, int64_t ldo, int64_t M,
                        int64_t N, int64_t K4, int tma_out, cudaStream_t stream) {
  auto k = nvfp4_gemm_kernel<kMode>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int64_t pairs_max = gemm_common::num_sms() / 2;
  const int64_t pairs = tiles < pairs_max ? tiles : pairs_max;
  return launch_overlapped(k, dim3(static_cast<unsigned>(2 * pairs)), dim3(kThreads), kSmemBytes,
                           stream, tmA, tmB, tmSA, tmSB, tmY, gx, gw, bias, out, ldo,
                           static_cast<int>(M), static_cast<int>(N), static_cast<int>(K4),
                           tma_out);
}

// The activation scale atoms as a 3-D tensor {128 bytes, 128-byte row (4 per atom, chunk-major),
// 128-row tile}: a {128, 4 x chunks per stage, 1} box is one stage's atoms. A chunk holds 4
// scales per row (64 columns of K).
inline bool make_act_scale_map(CUtensorMap* map, const uint8_t* sfx, int64_t M, int64_t K4) {
  constexpr int sf_k = kSfK, chunks_per_stage = kSfChunks;
  auto enc = gemm_common::get_encode_fn();
  if (!enc) return false;
  const int64_t kc_even = ((K4 + sf_k - 1) / sf_k + 1) & ~int64_t(1);
  const int64_t tiles = (M + kSfTileA - 1) / kSfTileA;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(4 * kc_even),
                        static_cast<cuuint64_t>(tiles)};
  cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(kc_even * 512)};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(4 * chunks_per_stage), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(sfx), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The weight scale images as a 3-D tensor {128 bytes, 128-byte row (32 per image), image}: a
// {128, 8, chunks per stage} box is the first lane quadrant of one stage's images.
inline bool make_weight_scale_map(CUtensorMap* map, const uint8_t* sfw, int64_t images) {
  constexpr int chunks_per_stage = kSfChunks;
  auto enc = gemm_common::get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, 32, static_cast<cuuint64_t>(images)};
  cuuint64_t strides[2] = {128, 4096};
  cuuint32_t box[3] = {128, 8, static_cast<cuuint32_t>(chunks_per_stage)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(sfw), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace fp4_detail

// Bytes of the block scales for `rows` rows and K4 columns (tiles of tile_rows): one 4096-byte
// image per tile and chunk (weights), or one 512-byte atom per tile and chunk with the chunk
// count rounded up to even (activations); a chunk is sf_k = 64 (NVFP4) or 128 (MXFP4) columns.
inline int64_t nvfp4_sf_bytes(int64_t rows, int64_t K4, int tile_rows, int layout,
                              int sf_k = 64) {
  const int64_t tiles = (rows + tile_rows - 1) / tile_rows;
  const int64_t kc = (K4 + sf_k - 1) / sf_k;
  return layout == kSfActAtoms ? tiles * ((kc + 1) & ~int64_t(1)) * 512 : tiles * kc * 4096;
}

inline cudaError_t launch_nvfp4_gemm(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx,
                                     const float* gx, const uint8_t* qw, int64_t ldqw,
                                     const uint8_t* sfw, const float* gw, const uint16_t* bias,
                                     void* out, int64_t ldo, int64_t M, int64_t N, int64_t K4,
                                     GemmOut mode, cudaStream_t stream) {
  using namespace fp4_detail;
  CUtensorMap tmA, tmB, tmSA, tmSB, tmY;
  std::memset(&tmY, 0, sizeof(tmY));
  if (!gemm_common::make_u8_map(&tmA, qx, M, K4 / 2, ldqx, BKB, BMC, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!gemm_common::make_u8_map(&tmB, qw, N, K4 / 2, ldqw, BKB, BNC, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int64_t images = nvfp4_sf_bytes(N, K4, kSfTileB, kSfWeightImage) / 4096;
  if (!make_act_scale_map(&tmSA, sfx, M, K4)) return cudaErrorInvalidValue;
  if (!make_weight_scale_map(&tmSB, sfw, images)) return cudaErrorInvalidValue;
  const int tma_out = gemm_common::setup_out_map(&tmY, mode, out, M, N, ldo);
  if (mode == GemmOut::kDequantBf16)
    return launch_mode<GemmOut::kDequantBf16>(tmA, tmB, tmSA, tmSB, tmY, gx, gw, bias, out, ldo,
                                              M, N, K4, tma_out, stream);
  return launch_mode<GemmOut::kRawS32>(tmA, tmB, tmSA, tmSB, tmY, gx, gw, bias, out, ldo, M, N,
                                       K4, 0, stream);
}

}  // namespace convrot
