// capi.cu -- the C ABI of the ConvLinear4bit hot path (declared in include/convrot.h).
//
// This is the library's single translation unit: it pulls in the kernel sources, defines the
// device status word, checks every argument on the host before anything is enqueued, and
// launches on the caller's stream. It allocates no memory.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "../../include/convrot.h"
#include "internal.h"
#include "ptx.cuh"
#include "rht_quant.cuh"
#include "rht_quant_ring.cuh"
#include "w4a4_gemm.cuh"
#include "w8a8_gemm.cuh"
#include "mxfp4_gemm.cuh"
#include "nvfp4_gemm.cuh"

// Scratch of convrot_w4a4_linear_fused_noalloc (the packed activation codes and row scales of
// one call): a fixed device array, so that the call allocates nothing. Every GPU that loads the
// library holds it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CONVROT_NOALLOC_SCRATCH_BYTES];

namespace convrot {
namespace {

constexpr int kMaxDevices = 64;

bool valid_group(int g) { return g == 16 || g == 64 || g == 256 || g == 1024; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Per device: whether it was queried, and whether it is an sm_100 part.
int g_dev_ok[kMaxDevices] = {};
bool g_dev_checked[kMaxDevices] = {};

int check_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return CONVROT_ERR_DEVICE;
  }
  if (dev < kMaxDevices && g_dev_checked[dev]) return g_dev_ok[dev] ? CONVROT_OK : CONVROT_ERR_DEVICE;
  // the library is built for sm_100a alone: arch-specific code does not load on other
  // compute capability 10.x parts
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return CONVROT_ERR_DEVICE;
  }
  const bool ok = (major == 10 && minor == 0);
  if (dev < kMaxDevices) {
    g_dev_ok[dev] = ok ? 1 : 0;
    g_dev_checked[dev] = true;
  }
  return ok ? CONVROT_OK : CONVROT_ERR_DEVICE;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA; }

// Shared checks of the rotate+quantise calls (activations and weights); a code row holds
// K_pad / 2 bytes (packed int4) or K_pad bytes (int8).
int check_quant_args(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group,
                     const uint8_t* q, int64_t ldq, const float* s, bool int8_codes) {
  if (!valid_group(group)) return CONVROT_ERR_INVALID_GROUP;
  if (M < 0 || K < 0) return CONVROT_ERR_SHAPE;
  if (M == 0) return CONVROT_OK;
  const int64_t K_pad = (K + group - 1) / group * group;
  if (M >= (int64_t(1) << 31) || K_pad > kMaxQuantKPad) return CONVROT_ERR_SHAPE;
  if (ldx < K || ldq < (int8_codes ? K_pad : K_pad / 2)) return CONVROT_ERR_SHAPE;
  if (s == nullptr) return CONVROT_ERR_NULL;
  if (K > 0 && (X == nullptr || q == nullptr)) return CONVROT_ERR_NULL;
  if (!aligned(s, 4)) return CONVROT_ERR_ALIGN;
  if (K > 0 && (!aligned(X, 16) || !aligned(q, 16) || (ldx % 8) != 0 || (ldq % 16) != 0))
    return CONVROT_ERR_ALIGN;
  return CONVROT_OK;
}

// qmax = 7: packed int4 codes; qmax = 127: int8 codes.
int rotate_quant(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group, uint8_t* q,
                 int64_t ldq, float* s, convrot_stream_t stream, int qmax) {
  int st = check_quant_args(X, M, K, ldx, group, q, ldq, s, qmax == 127);
  if (st != CONVROT_OK || M == 0) return st;
  if ((st = check_device()) != CONVROT_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return from_cuda(cudaMemsetAsync(s, 0, static_cast<size_t>(M) * sizeof(float), cs));
  return from_cuda(launch_rht_quant(X, M, K, ldx, group, q, ldq, s, cs, qmax));
}

// Shared checks of the GEMM calls; a code row holds K_pad / 2 bytes (packed int4) or K_pad
// bytes (int8).
int gemm_args(const uint8_t* qx, int64_t ldqx, const uint8_t* qw, int64_t ldqw, const void* out,
              int64_t ldo, int64_t M, int64_t N, int64_t K_pad, bool int8_codes) {
  if (M < 0 || N < 0 || K_pad < 0) return CONVROT_ERR_SHAPE;
  if (M == 0 || N == 0) return CONVROT_OK;
  if (K_pad == 0 || (K_pad % 16) != 0 || K_pad > kMaxGemmKPad) return CONVROT_ERR_SHAPE;
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return CONVROT_ERR_SHAPE;
  const int64_t row_bytes = int8_codes ? K_pad : K_pad / 2;
  if (ldqx < row_bytes || ldqw < row_bytes || ldo < N) return CONVROT_ERR_SHAPE;
  if (qx == nullptr || qw == nullptr || out == nullptr) return CONVROT_ERR_NULL;
  if (!aligned(qx, 16) || !aligned(qw, 16)) return CONVROT_ERR_ALIGN;
  if ((ldqx % 16) != 0 || (ldqw % 16) != 0) return CONVROT_ERR_ALIGN;
  return CONVROT_OK;
}

// One warp waits on an mbarrier that nothing arrives on, at most `polls` times, then records
// a timeout in the status word and returns: the failure path of every bounded wait, without a
// fault or a hang.
__global__ void selftest_wait_kernel(uint32_t polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    uint32_t i = 0;
    while (!mbar_try_wait(&bar, 0) && ++i < polls) {
    }
    if (i >= polls) atomicExch(&g_device_status, kStatusTimeout);
  }
}

int64_t nvfp4_k(int64_t K, int group) {
  const int64_t K_pad = (K + group - 1) / group * group;
  return (K_pad + 63) / 64 * 64;
}

// NVFP4 rotate+quantise: codes K4 / 2 bytes per row, block scales as images of `layout` for
// tiles of `tile_rows`.
int rotate_quant_fp4(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group, uint8_t* q,
                     int64_t ldq, uint8_t* sf, float* g, int tile_rows, int layout,
                     convrot_stream_t stream) {
  if (!valid_group(group)) return CONVROT_ERR_INVALID_GROUP;
  if (M < 0 || K < 0) return CONVROT_ERR_SHAPE;
  if (M == 0) return CONVROT_OK;
  const int64_t K4 = nvfp4_k(K, group);
  if (M >= (int64_t(1) << 31) || K4 > kMaxQuantKPad) return CONVROT_ERR_SHAPE;
  if (ldx < K || ldq < K4 / 2) return CONVROT_ERR_SHAPE;
  if (g == nullptr) return CONVROT_ERR_NULL;
  if (K > 0 && (X == nullptr || q == nullptr || sf == nullptr)) return CONVROT_ERR_NULL;
  if (!aligned(g, 4)) return CONVROT_ERR_ALIGN;
  if (K > 0 && (!aligned(X, 16) || !aligned(q, 16) || !aligned(sf, 16) || (ldx % 8) != 0 ||
                (ldq % 16) != 0))
    return CONVROT_ERR_ALIGN;
  int st = check_device();
  if (st != CONVROT_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) return from_cuda(cudaMemsetAsync(g, 0, static_cast<size_t>(M) * sizeof(float), cs));
  return from_cuda(launch_rht_quant_fp4(X, M, K, ldx, group, q, ldq, g, sf, tile_rows, layout, cs));
}

int fp4_gemm_args(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx, const uint8_t* qw,
                  int64_t ldqw, const uint8_t* sfw, const void* out, int64_t ldo, int64_t M,
                  int64_t N, int64_t K4) {
  if (M < 0 || N < 0 || K4 < 0) return CONVROT_ERR_SHAPE;
  if (M == 0 || N == 0) return CONVROT_OK;
  if (K4 == 0 || (K4 % 64) != 0 || K4 > kMaxGemmKPad) return CONVROT_ERR_SHAPE;
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return CONVROT_ERR_SHAPE;
  if (ldqx < K4 / 2 || ldqw < K4 / 2 || ldo < N) return CONVROT_ERR_SHAPE;
  if (!qx || !qw || !sfx || !sfw || !out) return CONVROT_ERR_NULL;
  if (!aligned(qx, 16) || !aligned(qw, 16) || !aligned(sfx, 16) || !aligned(sfw, 16))
    return CONVROT_ERR_ALIGN;
  if ((ldqx % 16) != 0 || (ldqw % 16) != 0) return CONVROT_ERR_ALIGN;
  return CONVROT_OK;
}

// MXFP4 rotate+quantise (same argument rules as NVFP4, without row scales).
int rotate_quant_mx(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group, uint8_t* q,
                    int64_t ldq, uint8_t* sf, int tile_rows, int layout,
                    convrot_stream_t stream) {
  if (!valid_group(group)) return CONVROT_ERR_INVALID_GROUP;
  if (M < 0 || K < 0) return CONVROT_ERR_SHAPE;
  if (M == 0 || K == 0) return CONVROT_OK;
  const int64_t K4 = nvfp4_k(K, group);
  if (M >= (int64_t(1) << 31) || K4 > kMaxQuantKPad) return CONVROT_ERR_SHAPE;
  if (ldx < K || ldq < K4 / 2) return CONVROT_ERR_SHAPE;
  if (X == nullptr || q == nullptr || sf == nullptr) return CONVROT_ERR_NULL;
  if (!aligned(X, 16) || !aligned(q, 16) || !aligned(sf, 16) || (ldx % 8) != 0 ||
      (ldq % 16) != 0)
    return CONVROT_ERR_ALIGN;
  int st = check_device();
  if (st != CONVROT_OK) return st;
  return from_cuda(launch_rht_quant_mx(X, M, K, ldx, group, q, ldq, sf, tile_rows, layout,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

// The fused layer's workspace: packed activation codes [M, round_up(K_pad / 2, 16)], then the
// row scales at the next 256-byte boundary.
int64_t fused_codes_ld(int64_t K_pad) { return (K_pad / 2 + 15) / 16 * 16; }
int64_t fused_scales_offset(int64_t M, int64_t K_pad) {
  return (M * fused_codes_ld(K_pad) + 255) / 256 * 256;
}
int64_t fused_workspace_bytes(int64_t M, int64_t K_pad) {
  return fused_scales_offset(M, K_pad) + (M * 4 + 255) / 256 * 256;
}

// The device address of the no-alloc scratch array (below), looked up once per device: in host
// code the array's name is only a host-side stand-in, never a device address.
constexpr int64_t kNoAllocScratchBytes = CONVROT_NOALLOC_SCRATCH_BYTES;
std::atomic<void*> g_noalloc_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device (looked up on first use).
int noalloc_scratch(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return CONVROT_ERR_DEVICE;
  }
  void* p = g_noalloc_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return CONVROT_ERR_CUDA;
    }
    g_noalloc_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *addr = p;
  return CONVROT_OK;
}

}  // namespace
}  // namespace convrot

using namespace convrot;

extern "C" {

const char* convrot_status_string(int status) {
  switch (status) {
    case CONVROT_OK: return "CONVROT_OK";
    case CONVROT_ERR_INVALID_GROUP: return "CONVROT_ERR_INVALID_GROUP: group must be 16, 64, 256 or 1024";
    case CONVROT_ERR_SHAPE: return "CONVROT_ERR_SHAPE: invalid size, stride or size limit";
    case CONVROT_ERR_NULL: return "CONVROT_ERR_NULL: required pointer is NULL";
    case CONVROT_ERR_ALIGN: return "CONVROT_ERR_ALIGN: pointer or stride misaligned";
    case CONVROT_ERR_DEVICE: return "CONVROT_ERR_DEVICE: no sm_100 (B200-class) device current";
    case CONVROT_ERR_CUDA: return "CONVROT_ERR_CUDA: CUDA runtime call or launch failed";
    case CONVROT_ERR_TIMEOUT: return "CONVROT_ERR_TIMEOUT: a kernel gave up a bounded wait";
    default: return "CONVROT_ERR_UNKNOWN";
  }
}

int64_t convrot_padded_k(int64_t K, int group) {
  if (!valid_group(group) || K < 0) return -1;
  return (K + group - 1) / group * group;
}

int convrot_make_rht(int group, float* R_dev, convrot_stream_t stream) {
  if (!valid_group(group)) return CONVROT_ERR_INVALID_GROUP;
  if (R_dev == nullptr) return CONVROT_ERR_NULL;
  if (!aligned(R_dev, 4)) return CONVROT_ERR_ALIGN;
  int st = check_device();
  if (st != CONVROT_OK) return st;
  return from_cuda(launch_make_rht(group, R_dev, reinterpret_cast<cudaStream_t>(stream)));
}

int convrot_rotate_quant_act(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group,
                             uint8_t* qx, int64_t ldq, float* sx, convrot_stream_t stream) {
  return rotate_quant(X, M, K, ldx, group, qx, ldq, sx, stream, 7);
}

int convrot_prepack_weight(const uint16_t* W, int64_t N, int64_t K, int64_t ldw, int group,
                           uint8_t* qw, int64_t ldqw, float* sw, convrot_stream_t stream) {
  return rotate_quant(W, N, K, ldw, group, qw, ldqw, sw, stream, 7);
}

int convrot_w4a4_linear(const uint8_t* qx, int64_t ldqx, const float* sx, const uint8_t* qw,
                        int64_t ldqw, const float* sw, const uint16_t* bias, uint16_t* Y,
                        int64_t ldy, int64_t M, int64_t N, int64_t K_pad,
                        convrot_stream_t stream) {
  int st = gemm_args(qx, ldqx, qw, ldqw, Y, ldy, M, N, K_pad, false);
  if (st != CONVROT_OK || M == 0 || N == 0) return st;
  if (sx == nullptr || sw == nullptr) return CONVROT_ERR_NULL;
  if (!aligned(sx, 4) || !aligned(sw, 4) || !aligned(bias, 2) || !aligned(Y, 2))
    return CONVROT_ERR_ALIGN;
  if ((st = check_device()) != CONVROT_OK) return st;
  return from_cuda(launch_w4a4_gemm(qx, ldqx, sx, qw, ldqw, sw, bias, Y, ldy, M, N, K_pad,
                                    GemmOut::kDequantBf16, reinterpret_cast<cudaStream_t>(stream)));
}

int convrot_w4a4_gemm_s32(const uint8_t* qx, int64_t ldqx, const uint8_t* qw, int64_t ldqw,
                          int32_t* acc, int64_t ldacc, int64_t M, int64_t N, int64_t K_pad,
                          convrot_stream_t stream) {
  int st = gemm_args(qx, ldqx, qw, ldqw, acc, ldacc, M, N, K_pad, false);
  if (st != CONVROT_OK || M == 0 || N == 0) return st;
  if (!aligned(acc, 4)) return CONVROT_ERR_ALIGN;
  if ((st = check_device()) != CONVROT_OK) return st;
  return from_cuda(launch_w4a4_gemm(qx, ldqx, nullptr, qw, ldqw, nullptr, nullptr, acc, ldacc, M,
                                    N, K_pad, GemmOut::kRawS32,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

int convrot_rotate_quant_i8(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group,
                            uint8_t* q, int64_t ldq, float* s, convrot_stream_t stream) {
  return rotate_quant(X, M, K, ldx, group, q, ldq, s, stream, 127);
}

int convrot_w8a8_linear(const uint8_t* qx, int64_t ldqx, const float* sx, const uint8_t* qw,
                        int64_t ldqw, const float* sw, const uint16_t* bias, uint16_t* Y,
                        int64_t ldy, int64_t M, int64_t N, int64_t K_pad,
                        convrot_stream_t stream) {
  int st = gemm_args(qx, ldqx, qw, ldqw, Y, ldy, M, N, K_pad, true);
  if (st != CONVROT_OK || M == 0 || N == 0) return st;
  if (sx == nullptr || sw == nullptr) return CONVROT_ERR_NULL;
  if (!aligned(sx, 4) || !aligned(sw, 4) || !aligned(bias, 2) || !aligned(Y, 2))
    return CONVROT_ERR_ALIGN;
  if ((st = check_device()) != CONVROT_OK) return st;
  return from_cuda(launch_w8a8_gemm(qx, ldqx, sx, qw, ldqw, sw, bias, Y, ldy, M, N, K_pad,
                                    GemmOut::kDequantBf16, reinterpret_cast<cudaStream_t>(stream)));
}

int convrot_w8a8_gemm_s32(const uint8_t* qx, int64_t ldqx, const uint8_t* qw, int64_t ldqw,
                          int32_t* acc, int64_t ldacc, int64_t M, int64_t N, int64_t K_pad,
                          convrot_stream_t stream) {
  int st = gemm_args(qx, ldqx, qw, ldqw, acc, ldacc, M, N, K_pad, true);
  if (st != CONVROT_OK || M == 0 || N == 0) return st;
  if (!aligned(acc, 4)) return CONVROT_ERR_ALIGN;
  if ((st = check_device()) != CONVROT_OK) return st;
  return from_cuda(launch_w8a8_gemm(qx, ldqx, nullptr, qw, ldqw, nullptr, nullptr, acc, ldacc, M,
                                    N, K_pad, GemmOut::kRawS32,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

int64_t convrot_nvfp4_k(int64_t K, int group) {
  if (!valid_group(group) || K < 0) return -1;
  return nvfp4_k(K, group);
}

int64_t convrot_nvfp4_scale_bytes(int64_t rows, int64_t K, int group, int operand) {
  if (!valid_group(group) || K < 0 || rows < 0 || (operand != 0 && operand != 1)) return -1;
  return operand == 0 ? nvfp4_sf_bytes(rows, nvfp4_k(K, group), fp4_detail::kSfTileA,
                                       kSfActAtoms)
                      : nvfp4_sf_bytes(rows, nvfp4_k(K, group), fp4_detail::kSfTileB,
                                       kSfWeightImage);
}

int convrot_rotate_quant_act_nvfp4(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                                   int group, uint8_t* qx, int64_t ldq, uint8_t* sfx, float* gx,
                                   convrot_stream_t stream) {
  return rotate_quant_fp4(X, M, K, ldx, group, qx, ldq, sfx, gx, fp4_detail::kSfTileA,
                          kSfActAtoms, stream);
}

int convrot_prepack_weight_nvfp4(const uint16_t* W, int64_t N, int64_t K, int64_t ldw, int group,
                                 uint8_t* qw, int64_t ldqw, uint8_t* sfw, float* gw,
                                 convrot_stream_t stream) {
  return rotate_quant_fp4(W, N, K, ldw, group, qw, ldqw, sfw, gw, fp4_detail::kSfTileB,
                          kSfWeightImage, stream);
}

int convrot_nvfp4_linear(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx, const float* gx,
                         const uint8_t* qw, int64_t ldqw, const uint8_t* sfw, const float* gw,
                         const uint16_t* bias, uint16_t* Y, int64_t ldy, int64_t M, int64_t N,
                         int64_t K4, convrot_stream_t stream) {
  int st = fp4_gemm_args(qx, ldqx, sfx, qw, ldqw, sfw, Y, ldy, M, N, K4);
  if (st != CONVROT_OK || M == 0 || N == 0) return st;
  if (gx == nullptr || gw == nullptr) return CONVROT_ERR_NULL;
  if (!aligned(gx, 4) || !aligned(gw, 4) || !aligned(bias, 2) || !aligned(Y, 2))
    return CONVROT_ERR_ALIGN;
  if ((st = check_device()) != CONVROT_OK) return st;
  return from_cuda(launch_nvfp4_gemm(qx, ldqx, sfx, gx, qw, ldqw, sfw, gw, bias, Y, ldy, M, N, K4,
                                     GemmOut::kDequantBf16,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

int convrot_nvfp4_gemm_f32(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx, const uint8_t* qw,
                           int64_t ldqw, const uint8_t* sfw, float* acc, int64_t ldacc, int64_t M,
                           int64_t N, int64_t K4, convrot_stream_t stream) {
  int st = fp4_gemm_args(qx, ldqx, sfx, qw, ldqw, sfw, acc, ldacc, M, N, K4);
  if (st != CONVROT_OK || M == 0 || N == 0) return st;
  if (!aligned(acc, 4)) return CONVROT_ERR_ALIGN;
  if ((st = check_device()) != CONVROT_OK) return st;
  return from_cuda(launch_nvfp4_gemm(qx, ldqx, sfx, nullptr, qw, ldqw, sfw, nullptr, nullptr, acc,
                                     ldacc, M, N, K4, GemmOut::kRawS32,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

int64_t convrot_mxfp4_scale_bytes(int64_t rows, int64_t K, int group, int operand) {
  if (!valid_group(group) || K < 0 || rows < 0 || (operand != 0 && operand != 1)) return -1;
  constexpr int kSfK = mx_detail::kSfK;
  return operand == 0 ? nvfp4_sf_bytes(rows, nvfp4_k(K, group), mx_detail::kSfTileA,
                                       kSfActAtoms, kSfK)
                      : nvfp4_sf_bytes(rows, nvfp4_k(K, group), mx_detail::kSfTileB,
                                       kSfWeightImage, kSfK);
}

int convrot_rotate_quant_act_mxfp4(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                                   int group, uint8_t* qx, int64_t ldq, uint8_t* sfx,
                                   convrot_stream_t stream) {
  return rotate_quant_mx(X, M, K, ldx, group, qx, ldq, sfx, mx_detail::kSfTileA, kSfActAtoms,
                         stream);
}

int convrot_prepack_weight_mxfp4(const uint16_t* W, int64_t N, int64_t K, int64_t ldw, int group,
                                 uint8_t* qw, int64_t ldqw, uint8_t* sfw,
                                 convrot_stream_t stream) {
  return rotate_quant_mx(W, N, K, ldw, group, qw, ldqw, sfw, mx_detail::kSfTileB, kSfWeightImage,
                         stream);
}

int convrot_mxfp4_linear(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx, const uint8_t* qw,
                         int64_t ldqw, const uint8_t* sfw, const uint16_t* bias, uint16_t* Y,
                         int64_t ldy, int64_t M, int64_t N, int64_t K4,
                         convrot_stream_t stream) {
  int st = fp4_gemm_args(qx, ldqx, sfx, qw, ldqw, sfw, Y, ldy, M, N, K4);
  if (st != CONVROT_OK || M == 0 || N == 0) return st;
  if (!aligned(bias, 2) || !aligned(Y, 2)) return CONVROT_ERR_ALIGN;
  if ((st = check_device()) != CONVROT_OK) return st;
  return from_cuda(launch_mxfp4_gemm(qx, ldqx, sfx, qw, ldqw, sfw, bias, Y, ldy, M, N, K4,
                                     GemmOut::kDequantBf16,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

int convrot_mxfp4_gemm_f32(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx, const uint8_t* qw,
                           int64_t ldqw, const uint8_t* sfw, float* acc, int64_t ldacc, int64_t M,
                           int64_t N, int64_t K4, convrot_stream_t stream) {
  int st = fp4_gemm_args(qx, ldqx, sfx, qw, ldqw, sfw, acc, ldacc, M, N, K4);
  if (st != CONVROT_OK || M == 0 || N == 0) return st;
  if (!aligned(acc, 4)) return CONVROT_ERR_ALIGN;
  if ((st = check_device()) != CONVROT_OK) return st;
  return from_cuda(launch_mxfp4_gemm(qx, ldqx, sfx, qw, ldqw, sfw, nullptr, acc, ldacc, M, N, K4,
                                     GemmOut::kRawS32, reinterpret_cast<cudaStream_t>(stream)));
}

int64_t convrot_w4a4_fused_workspace_bytes(int64_t M, int64_t K, int group) {
  if (!valid_group(group) || K < 0 || M < 0) return -1;
  return fused_workspace_bytes(M, (K + group - 1) / group * group);
}

int convrot_w4a4_linear_fused(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group,
                              const uint8_t* qw, int64_t ldqw, const float* sw,
                              const uint16_t* bias, uint16_t* Y, int64_t ldy, int64_t N,
                              void* workspace, int64_t workspace_bytes, convrot_stream_t stream) {
  if (!valid_group(group)) return CONVROT_ERR_INVALID_GROUP;
  if (M < 0 || N < 0 || K < 0) return CONVROT_ERR_SHAPE;
  if (M == 0 || N == 0) return CONVROT_OK;
  if (K == 0) return CONVROT_ERR_SHAPE;
  if (workspace == nullptr) return CONVROT_ERR_NULL;
  const int64_t K_pad = (K + group - 1) / group * group;
  const int64_t ldq = fused_codes_ld(K_pad);
  uint8_t* qx = static_cast<uint8_t*>(workspace);
  float* sx = reinterpret_cast<float*>(qx + fused_scales_offset(M, K_pad));
  int st = check_quant_args(X, M, K, ldx, group, qx, ldq, sx, false);
  if (st != CONVROT_OK) return st;
  if ((st = gemm_args(qx, ldq, qw, ldqw, Y, ldy, M, N, K_pad, false)) != CONVROT_OK) return st;
  if (workspace_bytes < fused_workspace_bytes(M, K_pad)) return CONVROT_ERR_SHAPE;
  if (!aligned(workspace, 256)) return CONVROT_ERR_ALIGN;
  if (sw == nullptr) return CONVROT_ERR_NULL;
  if (!aligned(sw, 4) || !aligned(bias, 2) || !aligned(Y, 2)) return CONVROT_ERR_ALIGN;
  if ((st = check_device()) != CONVROT_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (launch_rht_quant(X, M, K, ldx, group, qx, ldq, sx, cs, 7) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  return from_cuda(launch_w4a4_gemm(qx, ldq, sx, qw, ldqw, sw, bias, Y, ldy, M, N, K_pad,
                                    GemmOut::kDequantBf16, cs));
}

int convrot_w4a4_linear_fused_noalloc(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                                      int group, const uint8_t* qw, int64_t ldqw, const float* sw,
                                      const uint16_t* bias, uint16_t* Y, int64_t ldy, int64_t N,
                                      convrot_stream_t stream) {
  if (!valid_group(group)) return CONVROT_ERR_INVALID_GROUP;
  if (M < 0 || N < 0 || K < 0) return CONVROT_ERR_SHAPE;
  if (M == 0 || N == 0) return CONVROT_OK;
  // larger than the built-in scratch array: rejected before anything is looked up or launched
  if (fused_workspace_bytes(M, (K + group - 1) / group * group) > kNoAllocScratchBytes)
    return CONVROT_ERR_SHAPE;
  int st = check_device();
  if (st != CONVROT_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != CONVROT_OK) return st;
  return convrot_w4a4_linear_fused(X, M, K, ldx, group, qw, ldqw, sw, bias, Y, ldy, N, scratch,
                                   kNoAllocScratchBytes, stream);
}

int convrot_selftest_bounded_wait(int polls, convrot_stream_t stream) {
  if (polls < 1 || static_cast<uint32_t>(polls) > kMaxPolls) return CONVROT_ERR_SHAPE;
  int st = check_device();
  if (st != CONVROT_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint32_t>(polls));
  return from_cuda(cudaGetLastError());
}

int convrot_device_status(int* status, int clear) {
  if (status == nullptr) return CONVROT_ERR_NULL;
  int st = check_device();
  if (st != CONVROT_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return CONVROT_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
      return CONVROT_ERR_CUDA;
  }
  *status = v;
  return CONVROT_OK;
}

}  // extern "C"
