// internal.h -- limits and enums shared by the C ABI layer and the kernel sources.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

namespace convrot {

// Epilogue selector for the W4A4 GEMM.
enum class GemmOut { kDequantBf16, kRawS32 };

// Largest K_pad the quant kernel accepts (one CTA holds a whole row).
constexpr int64_t kMaxQuantKPad = 32768;
// Largest K_pad the GEMM accepts (|acc| * 256 must fit in int32).
constexpr int64_t kMaxGemmKPad = 131072;

// NVFP4 block-scale layouts written by the quantisation and read by the block-scaled GEMM:
// weights as 4096-byte images that one 128-lane tensor-memory copy reads (one per N tile of the
// GEMM, 192 rows for NVFP4 and 224 for MXFP4, and chunk); activations as 512-byte atoms (one per
// 128-row tile and chunk, the chunk count per tile rounded up to even). The MXFP4 GEMM's tensor
// copies expand the atoms into such images; the NVFP4 GEMM reads the atoms and the first
// quadrant of each weight image and writes the scales into tensor memory from its warps.
enum Fp4SfLayout : int { kSfWeightImage = 0, kSfActAtoms = 1 };

// Programmatic dependent launch: the hot kernels are launched with programmatic stream
// serialisation, so a kernel's launch and set-up (barrier init, tensor memory allocation,
// tensor-map prefetch) may overlap the tail of the kernel before it in the stream. Each of them
// executes grid_dependency_wait() before its first access to global memory, which waits for
// the preceding grid to complete and its writes to become visible (an immediate return when
// there is no such grid), and lets its own successor launch early with launch_dependents().
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KParams, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(KParams...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace convrot
