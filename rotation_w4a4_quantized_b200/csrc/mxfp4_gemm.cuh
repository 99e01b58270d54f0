// mxfp4_gemm.cuh -- block-scaled MXFP4 GEMM with fused bias on tcgen05 (sm_100a): the
// floating-point variant of the rotated 4-bit layer in the OCP microscaling format.
//
// What it computes (ComfyUI issue #14735, ConvRot author's comment: ConvRot also suits
// floating-point quantisation; here in MXFP4, e2m1 elements with a power-of-two (e8m0) scale per
// 32 consecutive K and no row scale):
//   acc[m,n] = sum_k (ex[m,k] * 2^sx[m, k/32]) * (ew[n,k] * 2^sw[n, k/32])   (fp32 on the
//              tensor cores; every product is exact, the sum is accumulated in fp32)
//   Y[m,n]   = bf16_rne(acc + float(bias[n]))
//
// How (B200 design): e2m1 is a native operand type of tcgen05.mma kind::mxf4nvf4, read packed
// (two per byte) from shared memory, so the codes go from HBM to the tensor cores by TMA with no
// conversion stage; the block scales ride along. Persistent CTA pairs walk 256 x 224 output
// tiles (224 accumulator columns x 2 buffers + one stage of scale factors fit the 512 TMEM
// columns). Per K stage (256 elements = 128 bytes per row) each CTA loads its 128 A rows, its
// 112 B rows and the stage's block scales (A: its 128 rows; B: all 224 rows of the tile, the
// same in both CTAs), pre-tiled in global memory in the order tcgen05.cp wants them; all copies
// complete on the even CTA's barrier. The even CTA's MMA thread copies the scales into tensor
// memory and issues 4 block-scaled MMAs (K = 64 each, two per 128-K scale chunk, selecting the
// chunk's scale bytes by the descriptor's scale-factor ids) per stage. One tcgen05.cp 128x256b
// (128 lanes x 8 columns) places the scales of A's two chunks, or both 128-row halves of one of
// B's, from a 4-fold replicated 4096-byte image: 1 + 2 copies per stage. B's images come from
// the weight prepack; A's are assembled by the loads themselves: the activation quantisation
// writes plain 512-byte atoms, and four 1 KB tensor copies (one per lane quadrant, a 5-D view
// of the atoms whose box interleaves the two chunks' 128-byte pieces) build the image in shared
// memory. The copies run in the tensor pipe in issue order with the MMAs; with 3 per stage
// this is faster than writing the scales from warps (the NVFP4 GEMM's way, whose 256 x 192
// tiles this format does not need). Epilogue as in the integer GEMMs (fp32 accumulator), one
// staging block per warp. Every wait is bounded.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "gemm_common.cuh"
#include "internal.h"
#include "nvfp4_gemm.cuh"
#include "ptx.cuh"

namespace convrot {

namespace mx_detail {

using gemm_common::kEpiWarps;

constexpr int BM = 256;          // tile rows per CTA pair
constexpr int BMC = BM / 2;      // A rows per CTA (TMEM lanes)
constexpr int BN = 224;          // tile columns (accumulator columns)
constexpr int BNC = BN / 2;      // B rows per CTA
constexpr int BKB = 128;         // bytes of packed e2m1 per row per stage (256 K)
constexpr int kChunks = 4;       // MMAs (64 K each) per stage
constexpr int SU = 5;            // ring stages
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kAccCols = BN;
constexpr int kTmemCols = 512;
constexpr int kSfaCol = 2 * kAccCols;                  // 448: 4 columns per chunk
constexpr int kSfbCol = kSfaCol + 4 * kChunks;         // 464: 8 columns per chunk
static_assert(kSfbCol + 8 * kChunks <= kTmemCols, "TMEM budget");

// tile rows of the block-scale layouts (activations: 128-row tiles of atoms; weights: 224-row
// tiles of images)
constexpr int kSfTileA = BMC;
constexpr int kSfTileB = BN;
constexpr int kEpiBufs = 1;
constexpr int kEpiSmem = kEpiWarps * kEpiBufs * gemm_common::kStageBytes;

constexpr int kTA = BMC * BKB;               // 16 KB
constexpr int kTB = BNC * BKB;               // 14 KB
// Scale chunks hold 4 scales per row and cover 128 K: 2 per stage.
constexpr int kSfK = 128;
constexpr int kSfChunks = BKB * 2 / kSfK;                // per stage
constexpr int kSA = kSfChunks / 2 * 4096;                // 4 KB: A's pair image
constexpr int kSB = kSfChunks * 4096;                    // 8 KB: B's images (128 lanes x 32 B)
constexpr uint32_t kStageTx = 2u * (kTA + kTB + kSA + kSB);

struct Smem {
  static constexpr int uA = 0;
  static constexpr int uB = uA + SU * kTA;
  static constexpr int sA = uB + SU * kTB;
  static constexpr int sB = sA + SU * kSA;
  static constexpr int stg = sB + SU * kSB;
  static constexpr int bars = stg + kEpiSmem;
  static constexpr int n_bars = 2 * SU + 4 + 1;
  static constexpr int misc = bars + n_bars * 8;
  static constexpr int total = misc + 16;
};
static_assert(Smem::uB % 1024 == 0 && Smem::sA % 1024 == 0, "1024-byte aligned tiles");
constexpr size_t kSmemBytes = Smem::total + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

using TileGrid = gemm_common::TileGrid<BM, BN>;

template <GemmOut kMode>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mxfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                  const __grid_constant__ CUtensorMap tmY, const uint16_t* __restrict__ bias,
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
  constexpr int kMmaPerSf = kSfK / 64;                   // MMAs per scale chunk
  const int sf_total = (K4 + kSfK - 1) / kSfK;           // scale chunks per row

  if (threadIdx.x == 0) {
    for (int i = 0; i < SU; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
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
          // A: per pair of chunks, one 1 KB copy of the two atoms into each lane quadrant
          // of the pair's image (box {128 B, 2 chunks, 4 pieces}); pairs past the tile's
          // end read zeros
          for (int p = 0; p < kSfChunks / 2; ++p)
            for (int q = 0; q < 4; ++q)
              tma_load_5d_pair(base + Smem::sA + slot * kSA + p * 4096 + q * 1024, &tmSA, bar,
                               0, 0, 0, s * (kSfChunks / 2) + p, a_tile);
          // B: images viewed as rows of 128 bytes (32 per image), one per scale chunk
          tma_load_2d_pair(base + Smem::sB + slot * kSB, &tmSB, bar, 0,
                           (b_tile * sf_total + s * kSfChunks) * 32);
        }
      }
      if (rank == 0) {
        for (uint32_t s = (g > SU ? g - SU : 0); s < g; ++s) {
          uint32_t polls = 0;
          while (!mbar_try_wait_cluster(full + (s % SU), (s / SU) & 1) && ++polls < kMaxPolls) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_fp4_bs(BM, BN, true);
      const uint32_t sfa = tmem_base + kSfaCol;
      const uint32_t sfb = tmem_base + kSfbCol;
      uint32_t g = 0;
      int ti = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += num_pairs, ++ti) {
        const int b = ti & 1;
        if (ti >= 2 && !mbar_wait_cluster(acc_empty + b, ((ti >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * kAccCols;
        for (int s = 0; s < num_k; ++s, ++g) {
          const uint32_t slot = g % SU;
          if (!mbar_wait_cluster(full + slot, (g / SU) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nck = (kc_total - s * kChunks) < kChunks ? (kc_total - s * kChunks) : kChunks;
          const uint32_t a0 = smem_u32(base + Smem::uA + slot * kTA);
          const uint32_t b0 = smem_u32(base + Smem::uB + slot * kTB);
          const uint32_t sa0 = smem_u32(base + Smem::sA + slot * kSA);
          const uint32_t sb0 = smem_u32(base + Smem::sB + slot * kSB);
          const int nsf = (nck + kMmaPerSf - 1) / kMmaPerSf;   // scale chunks in this stage
          for (int p = 0; 2 * p < nsf; ++p)
            tmem_cp_128x256b_pair(sfa + 8 * p, smem_desc_rows32(sa0 + 4096 * p));
          for (int q = 0; q < nsf; ++q)
            tmem_cp_128x256b_pair(sfb + 8 * q, smem_desc_rows32(sb0 + 4096 * q));
          for (int q = 0; q < nck; ++q) {
            const int sc = q / kMmaPerSf;                     // this MMA's scale chunk
            const uint32_t acc = (s > 0 || q > 0) ? 1u : 0u;
            mma_mxf4_bs_pair(d_tmem, smem_desc_k128(a0 + q * 32), smem_desc_k128(b0 + q * 32),
                             idesc_sf_ids(idesc, 2u * (q & 1)), sfa + 4 * sc, sfb + 8 * sc, acc);
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
  } else {
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
      gemm_common::epilogue_tile<kMode, BN, 0, true, kEpiBufs, false>(
          acc_tmem, row0, n0, M, N, nullptr, nullptr, bias, out, ldo, tma_out, &tmY, stg, nstore,
          acc_empty_even + b * 8);
    }
    if (lane == 0) bulk_wait_group<0>();
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
                        const CUtensorMap& tmSB, const CUtensorMap& tmY, const uint16_t* bias,
                        void* out, int64_t ldo, int64_t M, int64_t N, int64_t K4, int tma_out,
                        cudaStream_t stream) {
  auto k = mxfp4_gemm_kernel<kMode>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int64_t pairs_max = gemm_common::num_sms() / 2;
  const int64_t pairs = tiles < pairs_max ? tiles : pairs_max;
  return launch_overlapped(k, dim3(static_cast<unsigned>(2 * pairs)), dim3(kThreads), kSmemBytes,
                           stream, tmA, tmB, tmSA, tmSB, tmY, bias, out, ldo,
                           static_cast<int>(M), static_cast<int>(N), static_cast<int>(K4),
                           tma_out);
}

// The activation scale atoms as a 5-D tensor {128 bytes, chunk parity (2), 128-byte piece (4),
// chunk pair, 128-row tile}: a {128, 2, 4, 1, 1} box lands in shared memory as one lane
// quadrant of the pair's 4096-byte image (piece p of chunk 2k + h at 256 p + 128 h). A chunk
// holds 4 scales per row: sf_k = 64 (NVFP4) or 128 (MXFP4) columns of K.
inline bool make_act_scale_map(CUtensorMap* map, const uint8_t* sfx, int64_t M, int64_t K4,
                               int sf_k) {
  auto enc = gemm_common::get_encode_fn();
  if (!enc) return false;
  const int64_t kc_even = ((K4 + sf_k - 1) / sf_k + 1) & ~int64_t(1);
  const int64_t tiles = (M + kSfTileA - 1) / kSfTileA;
  cuuint64_t dims[5] = {128, 2, 4, static_cast<cuuint64_t>(kc_even / 2),
                        static_cast<cuuint64_t>(tiles)};
  cuuint64_t strides[4] = {512, 128, 1024, static_cast<cuuint64_t>(kc_even * 512)};
  cuuint32_t box[5] = {128, 2, 4, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<uint8_t*>(sfx), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace mx_detail

inline cudaError_t launch_mxfp4_gemm(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx,
                                     const uint8_t* qw, int64_t ldqw, const uint8_t* sfw,
                                     const uint16_t* bias, void* out, int64_t ldo, int64_t M,
                                     int64_t N, int64_t K4, GemmOut mode, cudaStream_t stream) {
  using namespace mx_detail;
  CUtensorMap tmA, tmB, tmSA, tmSB, tmY;
  std::memset(&tmY, 0, sizeof(tmY));
  if (!gemm_common::make_u8_map(&tmA, qx, M, K4 / 2, ldqx, BKB, BMC, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!gemm_common::make_u8_map(&tmB, qw, N, K4 / 2, ldqw, BKB, BNC, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // scale buffers viewed as rows of 128 bytes
  const int64_t sb_rows = nvfp4_sf_bytes(N, K4, kSfTileB, kSfWeightImage, kSfK) / 128;
  if (!make_act_scale_map(&tmSA, sfx, M, K4, kSfK)) return cudaErrorInvalidValue;
  if (!gemm_common::make_u8_map(&tmSB, sfw, sb_rows, 128, 128, 128, kSB / 128,
                                CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int tma_out = gemm_common::setup_out_map(&tmY, mode, out, M, N, ldo);
  if (mode == GemmOut::kDequantBf16)
    return launch_mode<GemmOut::kDequantBf16>(tmA, tmB, tmSA, tmSB, tmY, bias, out, ldo, M, N, K4,
                                              tma_out, stream);
  return launch_mode<GemmOut::kRawS32>(tmA, tmB, tmSA, tmSB, tmY, bias, out, ldo, M, N, K4, 0,
                                       stream);
}

}  // namespace convrot
