/*
 * convrot.h -- C ABI of the ConvLinear4bit (ConvRot W4A4) hot path for NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources cited by page title and section):
 *
 *  - "ConvRot: Rotation-Based Plug-and-Play 4-bit Quantization for Diffusion Transformers",
 *    Abstract and Fig. 3: ConvLinear4bit replaces a linear layer by rotation, quantisation,
 *    GEMM and dequantisation; the rotation is a regular Hadamard transform (RHT) applied to
 *    non-overlapping windows ("groups") of each activation row. Def. 2.3 / Thm. 2.3: the
 *    regular Hadamard matrix is built as a Kronecker power.
 *  - ComfyUI issue #14735, ConvRot author's comment: group sizes are powers of 4
 *    (16, 64, 256, 1024); K is zero-padded to a multiple of the group inside the algorithm.
 *  - "v2.3.4: Krea2 ConvRot INT8 Quantization Release", "Mathematical Formulation": weights
 *    are rotated the same way and get one scale per output channel, scale = row absmax / qmax.
 *  - comfy-kitchen PR #65 "Basic convrot int4 support": int4 codes packed two per byte along K;
 *    int4_linear scales the integer product by x_scale (per token) and weight_scale (per
 *    output channel), adds bias, in fp32, casting to the output dtype last.
 *
 * Fixed readings (where the pages are silent):
 *  - H4 = J4 - 2*I4; H_g = H4 (x) ... (x) H4 (log4 g factors); R = H_g / sqrt(g) (symmetric,
 *    orthogonal). Row x (padded to K_pad = ceil(K/g)*g with zeros) maps to x * blockdiag(R).
 *  - Symmetric int4: scale s = fp32(max|x_rot| / 7), code = round-half-even(x_rot / s) in
 *    [-7, 7]. A row with max|x_rot| = 0 gets s = 0 and all codes 0.
 *  - Packing: byte b of a row holds code k = 2b in bits 0..3 and k = 2b+1 in bits 4..7
 *    (two's complement nibbles).
 *  - Output: y[m,n] = bf16_rne( (float(acc[m,n]) * sx[m]) * sw[n] + float(bias[n]) ),
 *    acc = sum over k < K_pad of qx[m,k] * qw[n,k] (exact integer).
 *
 * Conventions shared by every entry point:
 *  - All buffers are DEVICE pointers allocated and owned by the caller; the library never
 *    allocates or frees memory and keeps no pointer after the call returns.
 *  - All work is enqueued asynchronously on `stream` (NULL = legacy default stream). The
 *    functions return before the GPU finishes. The rotate/quantise and GEMM kernels are
 *    launched with programmatic stream serialisation: their launch and set-up may overlap the
 *    end of the previous kernel on the stream, but none of them reads or writes a caller
 *    buffer before that kernel has completed, so stream order holds as for plain launches
 *    (also inside CUDA-graph capture).
 *  - Arguments are checked on the host before anything is enqueued; on a non-zero return
 *    nothing was enqueued (except CONVROT_ERR_CUDA, which reports a failed launch).
 *  - Sizes are element counts unless named *_bytes. Row strides (ld*) are in elements of the
 *    buffer's own type (bf16 elements for X/W/Y, bytes for the packed code buffers).
 *  - bf16 buffers are passed as uint16_t bit patterns.
 *  - No CPU fallback exists: the kernels need an sm_100 device (CONVROT_ERR_DEVICE otherwise).
 *  - Inputs containing NaN or Inf give unspecified codes and scales (not checked).
 */
#ifndef CONVROT_H_
#define CONVROT_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without pulling in the CUDA headers. */
typedef struct CUstream_st* convrot_stream_t;

typedef enum {
  CONVROT_OK = 0,
  CONVROT_ERR_INVALID_GROUP = 1, /* group not in {16, 64, 256, 1024} */
  CONVROT_ERR_SHAPE = 2,         /* negative size, ld < width, or size limit exceeded */
  CONVROT_ERR_NULL = 3,          /* required pointer is NULL while its size is non-zero */
  CONVROT_ERR_ALIGN = 4,         /* pointer or stride violates the alignment rule of the call */
  CONVROT_ERR_DEVICE = 5,        /* current device is not sm_100 (B200 class) or no device */
  CONVROT_ERR_CUDA = 6,          /* a CUDA runtime call or kernel launch failed */
  CONVROT_ERR_TIMEOUT = 7        /* a kernel gave up a bounded wait (see convrot_device_status) */
} convrot_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* convrot_status_string(int status);

/* ceil(K / group) * group, or -1 if group is not a valid group size or K < 0.
 * Pure host function (no CUDA call). ComfyUI issue #14735: "padding inside the algorithm". */
int64_t convrot_padded_k(int64_t K, int group);

/* Writes the normalised regular Hadamard rotation R (fp32, [group, group], row-major, dense)
 * to R_dev: R[i][j] = (-1)^(number of equal base-4 digits of i and j) / sqrt(group), which is
 * H4 (x) ... (x) H4 / sqrt(group) with H4 = J4 - 2*I4 ("ConvRot" paper, Def. 2.3 and
 * Thm. 2.3). Every entry is +-2^-k, exact in fp32. R_dev: device, 4-byte aligned, group*group
 * floats, caller-owned. Errors: INVALID_GROUP, NULL, DEVICE, CUDA. */
int convrot_make_rht(int group, float* R_dev, convrot_stream_t stream);

/* Online activation path ("ConvRot" paper, Fig. 3; comfy-kitchen PR #65 packing):
 *   for each row m < M of X (bf16 [M, K], row stride ldx elements):
 *     x_rot = pad(X[m, :K], K_pad) * blockdiag(R_group)
 *     sx[m] = fp32(max|x_rot| / 7)
 *     qx[m, 0 .. K_pad/2) = packed int4 codes round_half_even(x_rot / sx[m])
 *   qx: uint8 [M, ldq] (row stride ldq BYTES >= K_pad/2); only the first K_pad/2 bytes of
 *       each row are written.
 *   sx: float [M].
 * Alignment: X and qx 16-byte aligned; ldx a multiple of 8 elements; ldq a multiple of 16
 * bytes; sx 4-byte aligned. M == 0 or K == 0 is a no-op for codes (K == 0 writes sx = 0 when
 * M > 0). Limits: M < 2^31, K_pad <= 32768 (one CTA holds a whole row).
 * Errors: INVALID_GROUP, SHAPE, NULL, ALIGN, DEVICE, CUDA. */
int convrot_rotate_quant_act(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group,
                             uint8_t* qx, int64_t ldq, float* sx, convrot_stream_t stream);

/* Offline weight prepack: the same rotation and per-row quantisation applied to the rows of
 * W (bf16 [N, K]), i.e. one scale per output channel ("v2.3.4: Krea2 ConvRot INT8
 * Quantization Release", "Mathematical Formulation": W_rot = W H^T, scale_i over j of row i;
 * weight_scale float32 [out_features, 1]). Same layout, alignment and error rules as
 * convrot_rotate_quant_act with (X, M, ldx, qx, ldq, sx) -> (W, N, ldw, qw, ldqw, sw). */
int convrot_prepack_weight(const uint16_t* W, int64_t N, int64_t K, int64_t ldw, int group,
                           uint8_t* qw, int64_t ldqw, float* sw, convrot_stream_t stream);

/* W4A4 GEMM with fused dequantisation (comfy-kitchen PR #65, int4_linear with the fp32
 * accumulation fix; "ConvRot" paper, Abstract: GEMM + dequantisation):
 *   acc[m,n] = sum_{k < K_pad} qx[m,k] * qw[n,k]       (exact integer, tcgen05 kind::i8)
 *   Y[m,n]   = bf16_rne((float(acc) * sx[m]) * sw[n] + float(bias[n]))   (bias may be NULL)
 *   qx: uint8 [M, ldqx]  (packed codes as written by convrot_rotate_quant_act)
 *   qw: uint8 [N, ldqw]  (packed codes as written by convrot_prepack_weight)
 *   sx: float [M], sw: float [N], bias: bf16 [N] or NULL, Y: bf16 [M, ldy] (ldy >= N).
 * K_pad must be a positive multiple of 16 (it is a multiple of the group size).
 * Alignment: qx, qw 16-byte aligned; ldqx, ldqw multiples of 16 bytes (tensor-memory-access
 * rule); Y, bias 2-byte aligned, sx, sw 4-byte aligned, any ldy >= N (16-byte vector stores
 * are used when Y is 16-byte aligned and ldy is a multiple of 8, element stores otherwise).
 * Limits: M, N < 2^31, K_pad <= 131072 (|256 * acc| must fit in int32). M == 0 or N == 0 is a
 * no-op.
 * Errors: SHAPE, NULL, ALIGN, DEVICE, CUDA. */
int convrot_w4a4_linear(const uint8_t* qx, int64_t ldqx, const float* sx,
                        const uint8_t* qw, int64_t ldqw, const float* sw,
                        const uint16_t* bias, uint16_t* Y, int64_t ldy,
                        int64_t M, int64_t N, int64_t K_pad, convrot_stream_t stream);

/* Test export of the same GEMM without dequantisation: acc (int32 [M, ldacc]) receives the
 * exact integer sums acc[m,n] = sum_{k < K_pad} qx[m,k] * qw[n,k] (|acc| <= 49 * K_pad).
 * Same rules as convrot_w4a4_linear (acc 4-byte aligned, any ldacc >= N). */
int convrot_w4a4_gemm_s32(const uint8_t* qx, int64_t ldqx, const uint8_t* qw, int64_t ldqw,
                          int32_t* acc, int64_t ldacc, int64_t M, int64_t N, int64_t K_pad,
                          convrot_stream_t stream);

/* ---- W8A8 variant ------------------------------------------------------------------------
 * "v2.3.4: Krea2 ConvRot INT8 Quantization Release", "Mathematical Formulation": the same
 * group-wise rotation, then symmetric per-row int8 quantisation with scale = absmax / 127 for
 * the weight; ComfyUI issue #14735, author's comment: ConvRot W8A8 is integrated in Comfy.
 * Activations get the same per-token treatment (the reading the W4A4 path uses). */

/* Rotate + quantise to int8 (activations per token, or weights per output channel; the
 * operation is the same):
 *   for each row m < M of X (bf16 [M, K], row stride ldx elements):
 *     x_rot = pad(X[m, :K], K_pad) * blockdiag(R_group)
 *     s[m]  = fp32(max|x_rot| / 127)
 *     q[m, 0 .. K_pad) = int8 codes round_half_even(x_rot / s[m]), one per byte
 *   q: uint8 [M, ldq] (row stride ldq BYTES >= K_pad, two's-complement int8 codes); only the
 *      first K_pad bytes of each row are written. s: float [M].
 * Alignment, limits, no-op cases and errors as convrot_rotate_quant_act. */
int convrot_rotate_quant_i8(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group,
                            uint8_t* q, int64_t ldq, float* s, convrot_stream_t stream);

/* W8A8 GEMM with fused dequantisation (same epilogue as convrot_w4a4_linear):
 *   acc[m,n] = sum_{k < K_pad} qx[m,k] * qw[n,k]       (exact integer, tcgen05 kind::i8)
 *   Y[m,n]   = bf16_rne((float(acc) * sx[m]) * sw[n] + float(bias[n]))   (bias may be NULL)
 *   qx: uint8 [M, ldqx], qw: uint8 [N, ldqw] (int8 codes as written by
 *   convrot_rotate_quant_i8; ldqx, ldqw >= K_pad BYTES). Other arguments, alignment and errors
 *   as convrot_w4a4_linear. Limits: M, N < 2^31, K_pad a positive multiple of 16 and
 *   <= 131072 (127 * 127 * K_pad must fit in int32). */
int convrot_w8a8_linear(const uint8_t* qx, int64_t ldqx, const float* sx,
                        const uint8_t* qw, int64_t ldqw, const float* sw,
                        const uint16_t* bias, uint16_t* Y, int64_t ldy,
                        int64_t M, int64_t N, int64_t K_pad, convrot_stream_t stream);

/* Test export of the W8A8 GEMM without dequantisation: acc (int32 [M, ldacc]) receives
 * acc[m,n] = sum_{k < K_pad} qx[m,k] * qw[n,k] exactly (|acc| <= 16129 * K_pad). Same rules
 * as convrot_w8a8_linear (acc 4-byte aligned, any ldacc >= N). */
int convrot_w8a8_gemm_s32(const uint8_t* qx, int64_t ldqx, const uint8_t* qw, int64_t ldqw,
                          int32_t* acc, int64_t ldacc, int64_t M, int64_t N, int64_t K_pad,
                          convrot_stream_t stream);

/* ---- NVFP4 variant -----------------------------------------------------------------------
 * ComfyUI issue #14735, ConvRot author's comment: ConvRot also suits floating-point
 * quantisation. The pages define no format; this library uses NVFP4 at per-token granularity:
 *   x_rot = the same group RHT of the row, padded with zero groups to K4 = round_up(K_pad, 64)
 *   g[m]  = fp32(max|x_rot[m,:]| / (6 * 448))                           (row scale)
 *   s[m,b] = e4m3_rne_sat(max over block b of |x_rot| / (6 * g[m]))     (16 K per block b)
 *   e[m,k] = e2m1_rne_sat(x_rot[m,k] / (s[m,k/16] * g[m]))              (elements)
 * e2m1: +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}; e4m3: unsigned, 3 mantissa bits, largest 448. Elements
 * are packed two per byte along K (k = 2b in the low nibble); row stride ldq BYTES >= K4 / 2.
 * Block scales are stored in the order the GEMM moves them into tensor memory. Within a 128-row
 * group and 64-K chunk, the scale of row r and block b (of the 4 in the chunk) belongs at byte
 * 16 (r % 32) + 4 ((r % 128) / 32) + b of a 512-byte atom. Activations: rows in tiles of 128,
 * one atom per tile and chunk, the chunk count per tile rounded up to even (the padding atom is
 * not written). Weights: rows in tiles of 192 (the NVFP4 GEMM's N tile), one 4096-byte image
 * per tile and chunk: 128 lanes L x 32 bytes, lane L byte j at 256 (L / 8) + 128 (j / 16) + 16 (L % 8) +
 * j % 16, row r's scales in the four lanes L = r % 32 + 32 q (q = 0..3) at byte
 * 4 ((r % 128) / 32) + b of the half j / 16 = r / 128.
 * Buffer sizes come from convrot_nvfp4_scale_bytes. */

/* K4 = round_up(round_up(K, group), 64), the K the NVFP4 calls run over; -1 on bad arguments. */
int64_t convrot_nvfp4_k(int64_t K, int group);

/* Bytes of the tiled block-scale buffer for `rows` rows: operand 0 = activations (A),
 * 1 = weights (B). -1 on bad arguments. Pure host function. */
int64_t convrot_nvfp4_scale_bytes(int64_t rows, int64_t K, int group, int operand);

/* Rotate + quantise activations (X bf16 [M, K]) to NVFP4: qx uint8 [M, ldq] (K4 / 2 bytes per
 * row written), sfx (convrot_nvfp4_scale_bytes(M, K, group, 0) bytes, 16-byte aligned), gx float
 * [M]. Alignment, limits (K4 <= 32768) and errors as convrot_rotate_quant_act. */
int convrot_rotate_quant_act_nvfp4(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                                   int group, uint8_t* qx, int64_t ldq, uint8_t* sfx, float* gx,
                                   convrot_stream_t stream);

/* The same for weights W bf16 [N, K] (scales tiled for the B operand, operand 1). */
int convrot_prepack_weight_nvfp4(const uint16_t* W, int64_t N, int64_t K, int64_t ldw, int group,
                                 uint8_t* qw, int64_t ldqw, uint8_t* sfw, float* gw,
                                 convrot_stream_t stream);

/* Block-scaled FP4 GEMM with fused dequantisation (tcgen05 kind::mxf4nvf4, fp32 accumulation):
 *   acc[m,n] = sum_{k < K4} (e_x[m,k] s_x[m,k/16]) (e_w[n,k] s_w[n,k/16])
 *   Y[m,n]   = bf16_rne((acc * gx[m]) * gw[n] + float(bias[n]))          (bias may be NULL)
 * K4 a positive multiple of 64, <= 131072. Alignment: qx, qw, sfx, sfw 16-byte aligned; ldqx,
 * ldqw multiples of 16 bytes and >= K4 / 2; gx, gw 4-byte; Y, bias 2-byte; any ldy >= N.
 * Errors: SHAPE, NULL, ALIGN, DEVICE, CUDA. */
int convrot_nvfp4_linear(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx, const float* gx,
                         const uint8_t* qw, int64_t ldqw, const uint8_t* sfw, const float* gw,
                         const uint16_t* bias, uint16_t* Y, int64_t ldy, int64_t M, int64_t N,
                         int64_t K4, convrot_stream_t stream);

/* Test export of the same GEMM without the row/column scales: acc (float [M, ldacc]) receives
 * the fp32 block-scaled accumulator. Same rules (acc 4-byte aligned). */
int convrot_nvfp4_gemm_f32(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx, const uint8_t* qw,
                           int64_t ldqw, const uint8_t* sfw, float* acc, int64_t ldacc, int64_t M,
                           int64_t N, int64_t K4, convrot_stream_t stream);

/* ---- MXFP4 variant -----------------------------------------------------------------------
 * The same floating-point reading as the NVFP4 variant with the OCP Microscaling MXFP4 format:
 *   x_rot = the group RHT of the row, padded with zero groups to K4 = round_up(K_pad, 64)
 *   X[m,b] = clamp(floor(log2(max over block b of |x_rot|)) - 2, -127, 127)   (32 K per block b;
 *            -127 for an all-zero block), stored as the e8m0 byte X + 127
 *   e[m,k] = e2m1_rne_sat(x_rot[m,k] / 2^X[m,k/32])                             (elements)
 * There is no per-row scale. Elements are packed as for NVFP4. Scale bytes use the NVFP4
 * layouts with 128-K chunks of 4 scales in place of 64-K chunks: within a 128-row group and
 * 128-K chunk, the scale of row r and block b (of the 4 in the chunk) belongs at byte
 * 16 (r % 32) + 4 ((r % 128) / 32) + b of a 512-byte atom; activations store the atoms (128-row
 * tiles, chunk count per tile rounded up to even), weights the 4-fold replicated 4096-byte
 * images of 224-row tiles (the MXFP4 GEMM's N tile). Buffer sizes come from
 * convrot_mxfp4_scale_bytes; K4 from convrot_nvfp4_k. */

/* Bytes of the scale buffer for `rows` rows: operand 0 = activations, 1 = weights; -1 on bad
 * arguments. Pure host function. */
int64_t convrot_mxfp4_scale_bytes(int64_t rows, int64_t K, int group, int operand);

/* Rotate + quantise activations (X bf16 [M, K]) to MXFP4: qx uint8 [M, ldq] (K4 / 2 bytes per
 * row written), sfx (convrot_mxfp4_scale_bytes(M, K, group, 0) bytes, 16-byte aligned).
 * Alignment, limits (K4 <= 32768) and errors as convrot_rotate_quant_act_nvfp4. */
int convrot_rotate_quant_act_mxfp4(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                                   int group, uint8_t* qx, int64_t ldq, uint8_t* sfx,
                                   convrot_stream_t stream);

/* The same for weights W bf16 [N, K] (operand 1 layout). */
int convrot_prepack_weight_mxfp4(const uint16_t* W, int64_t N, int64_t K, int64_t ldw, int group,
                                 uint8_t* qw, int64_t ldqw, uint8_t* sfw,
                                 convrot_stream_t stream);

/* Block-scaled FP4 GEMM (tcgen05 kind::mxf4nvf4, 32-element blocks, e8m0 scales, fp32
 * accumulation):
 *   acc[m,n] = sum_{k < K4} (e_x[m,k] 2^X_x[m,k/32]) (e_w[n,k] 2^X_w[n,k/32])
 *   Y[m,n]   = bf16_rne(acc + float(bias[n]))                            (bias may be NULL)
 * Rules and errors as convrot_nvfp4_linear. */
int convrot_mxfp4_linear(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx, const uint8_t* qw,
                         int64_t ldqw, const uint8_t* sfw, const uint16_t* bias, uint16_t* Y,
                         int64_t ldy, int64_t M, int64_t N, int64_t K4, convrot_stream_t stream);

/* Test export: the fp32 accumulator of the same GEMM into acc (float [M, ldacc]). */
int convrot_mxfp4_gemm_f32(const uint8_t* qx, int64_t ldqx, const uint8_t* sfx, const uint8_t* qw,
                           int64_t ldqw, const uint8_t* sfw, float* acc, int64_t ldacc, int64_t M,
                           int64_t N, int64_t K4, convrot_stream_t stream);

/* ---- The whole layer in one call ---------------------------------------------------------
 * "ConvRot" paper, Abstract and Fig. 3: ConvLinear4bit is a plug-and-play module that
 * integrates rotation, quantisation, GEMM and dequantisation. One call computes, from the bf16
 * activations, exactly what convrot_rotate_quant_act followed by convrot_w4a4_linear computes
 * (the same codes, scales and output formula):
 *   Y[m,n] = bf16_rne((float(acc[m,n]) * sx[m]) * sw[n] + float(bias[n]))
 * The packed activation codes and their scales live in the caller's workspace for the
 * duration of the call (contents undefined afterwards; nothing else may use it while the call
 * runs on the GPU).
 *   X: bf16 [M, ldx]; qw, sw, bias: as for convrot_w4a4_linear (qw from
 *   convrot_prepack_weight with the same group); Y: bf16 [M, ldy], ldy >= N.
 *   workspace: device, 256-byte aligned, at least convrot_w4a4_fused_workspace_bytes(M, K,
 *   group) bytes (packed codes [M, round_up(K_pad / 2, 16)], then the row scales).
 * Limits: 0 < K, K_pad <= 32768, M, N < 2^31. Alignment: X 16-byte aligned with ldx a multiple
 * of 8; qw, Y, bias, sw as for convrot_w4a4_linear. M == 0 or N == 0 is a no-op.
 * Errors: INVALID_GROUP, SHAPE, NULL, ALIGN, DEVICE, CUDA. */
int64_t convrot_w4a4_fused_workspace_bytes(int64_t M, int64_t K, int group);

int convrot_w4a4_linear_fused(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group,
                              const uint8_t* qw, int64_t ldqw, const float* sw,
                              const uint16_t* bias, uint16_t* Y, int64_t ldy, int64_t N,
                              void* workspace, int64_t workspace_bytes, convrot_stream_t stream);

/* Size of the library's built-in scratch array used by convrot_w4a4_linear_fused_noalloc. */
#define CONVROT_NOALLOC_SCRATCH_BYTES (8 * 1024 * 1024)

/* The one-call layer for callers that cannot allocate device memory. Nothing in the paper
 * corresponds to this entry point: it exists for callers that are handed streams and tensors
 * but cannot obtain memory of their own at call time -- for example code that runs while a
 * stream is being captured into a CUDA graph (cudaMalloc is not a stream operation and is not
 * allowed during such a capture), or a plugin inside another runtime that owns the allocator and
 * gives the plugin no workspace. It computes exactly what convrot_w4a4_linear_fused computes,
 * with the same arguments except the workspace: the packed codes and scales go to a fixed
 * scratch array of CONVROT_NOALLOC_SCRATCH_BYTES (8 MiB) that the library holds in device
 * memory on every GPU where it is loaded, until the process exits. The call allocates nothing.
 *  - The first call on a device looks up the array's device address (cudaGetSymbolAddress),
 *    with that device current; make that first call before any stream capture begins.
 *  - Every call on a device uses the same array. Calls whose work overlaps on the GPU (on two
 *    streams, or from two host threads) race on it and give undefined results; calls that follow
 *    each other in one stream are safe. The array keeps the last call's contents; nothing in it
 *    needs to start at zero (each call writes every byte it reads).
 *  - Shapes whose workspace (convrot_w4a4_fused_workspace_bytes(M, K, group)) exceeds the array
 *    are rejected with CONVROT_ERR_SHAPE before anything runs; e.g. M = 4608 tokens fit for
 *    K_pad <= 3584 (FLUX's QKV and MLP-up activations, K = 3072), any M <= 512 for
 *    K_pad <= 16384.
 * Other limits, alignment rules and errors as convrot_w4a4_linear_fused; CONVROT_ERR_CUDA also
 * reports a failed address lookup. */
int convrot_w4a4_linear_fused_noalloc(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                                      int group, const uint8_t* qw, int64_t ldqw, const float* sw,
                                      const uint16_t* bias, uint16_t* Y, int64_t ldy, int64_t N,
                                      convrot_stream_t stream);

/* Test export of the failure path: launches one warp that waits on a barrier nothing arrives
 * on, gives up after `polls` polls (1 .. 2^24; each poll suspends for a hardware-chosen time
 * window) and records CONVROT_ERR_TIMEOUT in the device status word, exactly as a kernel's
 * bounded wait does. Nothing faults or hangs; the context stays usable. Errors: SHAPE (polls out
 * of range), DEVICE, CUDA. */
int convrot_selftest_bounded_wait(int polls, convrot_stream_t stream);

/* Reads (and if `clear` != 0 resets) the device-side status word of the current device that
 * kernels set when a bounded wait gives up (CONVROT_ERR_TIMEOUT) -- a hang turned into an
 * error. Synchronises the current device. *status receives CONVROT_OK or the recorded code. */
int convrot_device_status(int* status, int clear);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H_ */
