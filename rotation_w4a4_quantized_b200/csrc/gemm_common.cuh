// gemm_common.cuh -- pieces shared by the W4A4 and W8A8 tcgen05 GEMMs: the tile walk, the
// dequantising TMA-store epilogue, and tensor-map construction.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace convrot {
namespace gemm_common {

constexpr int kEpiWarps = 4;                       // one warp per TMEM lane quadrant
constexpr int kEpiCols = 32;                       // accumulator columns per epilogue chunk
constexpr int kStageBytes = 32 * kEpiCols * 2;     // one 32 x 32 bf16 staging block (2 KB)
constexpr int kEpiSmem = 2 * kEpiWarps * kStageBytes;   // double-buffered per epilogue warp

// Byte offset of 16-byte chunk `chunk` of row `row` in a K-major, 128-byte-swizzled tile
// (rows of 128 bytes, 8-row atoms of 1024 bytes): the layout the MMA descriptors describe.
__device__ __forceinline__ uint32_t swz128(int row, int chunk) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int BM, int BN>
struct TileGrid {
  int tiles_m, tiles_n;
  __device__ __forceinline__ int count() const { return tiles_m * tiles_n; }
  // Consecutive tiles share the B (weight) tile and walk down M.
  __device__ __forceinline__ void coords(int t, int& m0, int& n0) const {
    m0 = (t % tiles_m) * BM;
    n0 = (t / tiles_m) * BN;
  }
};

// Dequantise one finished accumulator block -- this warp's 32 TMEM lanes (rows row0..row0+31)
// x BN columns starting at n0 -- and store it:
//   Y[m,n] = bf16_rne((float(acc >> kShift) * sx[m]) * sw[n] + float(bias[n]))
// (kShift = 8 when the accumulator holds 256 * acc: the arithmetic shift of the integer
// accumulator is exact, so the formula runs on the exact acc whatever the row scale's
// magnitude). As soon as the last columns are in registers the warp arrives on
// `acc_empty_addr` (a shared::cluster barrier address) so the MMA can reuse the accumulator.
// bf16 blocks of 32 x 32 are staged in shared memory with the 64-byte swizzle and written by
// TMA stores when `tma_out`; otherwise element stores are used. kRawS32 stores acc >> kShift.
// With kF32Acc the accumulator holds fp32 values (block-scaled FP4 MMA): the formula is the same
// with float(acc) = acc, and the raw mode stores the fp32 accumulator.
// kStageBufs staging blocks per warp (2: a block is refilled while the previous store reads the
// other; 1 when shared memory is short: each refill waits for the warp's previous store).
// kScaled = false: no row and column scales (y = acc + bias; sx and sw are not read).
template <GemmOut kMode, int BN, int kShift, bool kF32Acc = false, int kStageBufs = 2,
          bool kScaled = true>
__device__ __forceinline__ void epilogue_tile(uint32_t acc_tmem, int row0, int n0, int M, int N,
                                              const float* __restrict__ sx,
                                              const float* __restrict__ sw,
                                              const uint16_t* __restrict__ bias,
                                              void* __restrict__ out, int64_t ldo, int tma_out,
                                              const CUtensorMap* tmY, unsigned char* stg,
                                              uint32_t& nstore, uint32_t acc_empty_addr) {
  // the hand-back below fires on the last chunk: the tile must be whole chunks wide
  static_assert(BN % kEpiCols == 0, "tile width must be a multiple of the epilogue chunk");
  const int lane = threadIdx.x & 31;
  const int m = row0 + lane;
  const bool row_ok = m < M;
  const float sxm = !kScaled ? 1.f : ((row_ok && sx) ? sx[m] : 0.f);
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += kEpiCols) {
    uint32_t acc[kEpiCols];
    tmem_ld_32x32b_x32(acc_tmem + c0, acc);
    tmem_ld_wait();
    if (c0 + kEpiCols == BN) {
      // the whole accumulator is in registers: hand it back to the MMA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_addr);
    }
    const int nb = n0 + c0;
    if (nb >= N) continue;
    if constexpr (kMode == GemmOut::kRawS32) {
      if (!row_ok) continue;
      uint32_t* dst = reinterpret_cast<uint32_t*>(out) + static_cast<int64_t>(m) * ldo + nb;
#pragma unroll
      for (int i = 0; i < kEpiCols; ++i)
        if (nb + i < N)
          dst[i] = kF32Acc ? acc[i] : static_cast<uint32_t>(static_cast<int32_t>(acc[i]) >> kShift);
    } else {
      // per-column weight scale and bias: lane i fetches column nb + i, then broadcast
      const int nl = nb + lane < N ? nb + lane : N - 1;
      const float sw_l = kScaled ? __ldg(sw + nl) : 1.f;
      const float b_l =
          bias ? __uint_as_float(static_cast<uint32_t>(__ldg(bias + nl)) << 16) : 0.f;
      uint32_t pkd[kEpiCols / 2];
#pragma unroll
      for (int i = 0; i < kEpiCols; i += 2) {
        const float a0 = kF32Acc ? __uint_as_float(acc[i])
                                 : static_cast<float>(static_cast<int32_t>(acc[i]) >> kShift);
        const float a1 = kF32Acc ? __uint_as_float(acc[i + 1])
                                 : static_cast<float>(static_cast<int32_t>(acc[i + 1]) >> kShift);
        float v0 = a0 * sxm;
        float v1 = a1 * sxm;
        v0 = v0 * __shfl_sync(0xffffffffu, sw_l, i);
        v1 = v1 * __shfl_sync(0xffffffffu, sw_l, i + 1);
        if (bias) {
          v0 = v0 + __shfl_sync(0xffffffffu, b_l, i);
          v1 = v1 + __shfl_sync(0xffffffffu, b_l, i + 1);
        }
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(pkd[i / 2]) : "f"(v1), "f"(v0));
      }
      if (tma_out && row0 < M) {
        // stage the warp's 32 x 32 bf16 block (64-byte rows, 64B swizzle) and TMA-store it
        static_assert(kStageBufs == 1 || kStageBufs == 2, "one or two staging blocks");
        unsigned char* buf = stg + (nstore % kStageBufs) * kStageBytes;
        if (nstore >= kStageBufs) {
          if (lane == 0) bulk_wait_group_read<kStageBufs - 1>();
          __syncwarp();
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(pkd[4 * c], pkd[4 * c + 1], pkd[4 * c + 2], pkd[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tmY, buf, nb, row0);
          bulk_commit_group();
        }
        ++nstore;
      } else if (!tma_out && row_ok) {
        uint16_t* dst = reinterpret_cast<uint16_t*>(out) + static_cast<int64_t>(m) * ldo + nb;
#pragma unroll
        for (int i = 0; i < kEpiCols; ++i)
          if (nb + i < N) dst[i] = static_cast<uint16_t>((pkd[i / 2] >> ((i & 1) * 16)) & 0xFFFFu);
      }
    }
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D uint8 tensor map over a byte matrix [rows, width] with row stride ld bytes, boxes of
// box_rows x box_bytes.
inline bool make_u8_map(CUtensorMap* map, const uint8_t* ptr, int64_t rows, int64_t width,
                        int64_t ld, int box_bytes, int box_rows, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D bf16 tensor map over the output [M, N] (row stride ld elements), 32 x 32 boxes with the
// 64-byte swizzle used by the epilogue staging buffers.
inline bool make_out_map(CUtensorMap* map, const void* ptr, int64_t M, int64_t N, int64_t ld) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kEpiCols), 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 output goes through TMA stores when the base and row stride are 16-byte aligned.
inline int setup_out_map(CUtensorMap* map, GemmOut mode, const void* out, int64_t M, int64_t N,
                         int64_t ld) {
  if (mode != GemmOut::kDequantBf16 || (reinterpret_cast<uintptr_t>(out) & 15) != 0 ||
      ((ld * 2) & 15) != 0)
    return 0;
  return make_out_map(map, out, M, N, ld) ? 1 : 0;
}

inline int num_sms() {
  static int sms[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (sms[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    sms[dev] = v;
  }
  return sms[dev];
}

}  // namespace gemm_common
}  // namespace convrot
