// rht_quant.cuh -- fused group-wise regular Hadamard transform + symmetric per-row int4
// quantisation + nibble packing, for sm_100a.
//
// What it computes ("ConvRot: Rotation-Based Plug-and-Play 4-bit Quantization for Diffusion
// Transformers", Fig. 3 and Thm. 2.3; ComfyUI issue #14735, author's comment; "v2.3.4: Krea2
// ConvRot INT8 Quantization Release", "Mathematical Formulation"; comfy-kitchen PR #65
// packing): for every row, pad K with zeros to K_pad, multiply each group of G columns by
// R = H4^(x)k / 2^k (H4 = J4 - 2 I4, 4^k = G), take the row absmax, scale = absmax / 7,
// codes = round-half-even(x_rot / scale), two codes per byte (even k in the low nibble).
//
// How (B200 design):
//  * One thread owns 64 consecutive elements of a row ("chunk") in registers. H_G is applied
//    as radix-4 butterfly stages, one per base-4 digit of the in-group index: for the 4
//    elements that differ only in that digit, y_i = S - 2 x_i with S their sum (this is
//    H4 = J4 - 2 I4 applied along the digit), in packed fp32x2 arithmetic. Scaling by 2^-k is
//    exact and folded into the quantisation multiplier.
//  * Digits 0..2 (strides 1, 4, 16) live inside a chunk. For G = 256 digit 3 spans the 4
//    chunks of a group (4 lanes of one warp): they swap 16-value blocks with three shuffle
//    rounds (see the slot layout below). For G = 1024 (digits 3, 4 over 16 lanes) the lanes
//    exchange their values once through an XOR-swizzled shared-memory tile.
//  * The persistent register-resident kernel here (direct 128-bit loads, the next row group's
//    data prefetched into registers while the current one is transformed) serves the shapes
//    the row-streaming kernel of rht_quant_ring.cuh does not take (K not a multiple of 8, rows
//    longer than 16384 columns) and the floating-point (NVFP4, MXFP4) modes.
//  * The row absmax is combined across the row's threads with one shared-memory atomicMax
//    (non-negative floats order like their bit patterns).
//  * Rounding uses fma(v, inv, 1.5 * 2^23): the fp32 sum rounds v * inv to the nearest
//    integer (ties to even) in one step, and the integer is read back from the low mantissa
//    bits: the low nibble (int4) or byte (int8) of the bit pattern is already the code in two's
//    complement, so byte permutes gather the codes (int4: one masked merge of even and odd
//    codes per 32-bit word).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <numeric>

#include "internal.h"
#include "ptx.cuh"

namespace convrot {

namespace quant_detail {

constexpr int kChunk = 64;          // elements per thread

// Radix-4 stage along the base-4 digit whose stride is S (in chunk-local element index):
// H4 = J4 - 2 I4 applied to every 4-tuple {b, b+S, b+2S, b+3S}: y_i = S_sum - 2 x_i.
// Values are handled as pairs (v[2j], v[2j+1]) with Blackwell's packed fp32 instructions:
// for S >= 4 the two elements of a pair sit in two different 4-tuples with the same structure,
// so one packed add/fma serves both; for S == 1 a 4-tuple is two pairs.
template <int S>
__device__ __forceinline__ void radix4_stage(float (&v)[kChunk]) {
  const float2 m2 = make_float2(-2.f, -2.f);
  if constexpr (S == 1) {
#pragma unroll
    for (int b = 0; b < kChunk; b += 4) {
      float2 pa = make_float2(v[b], v[b + 1]);
      float2 pb = make_float2(v[b + 2], v[b + 3]);
      const float2 t = __fadd2_rn(pa, pb);            // (x0 + x2, x1 + x3)
      const float sum = t.x + t.y;
      const float2 sv = make_float2(sum, sum);
      pa = __ffma2_rn(pa, m2, sv);
      pb = __ffma2_rn(pb, m2, sv);
      v[b] = pa.x;
      v[b + 1] = pa.y;
      v[b + 2] = pb.x;
      v[b + 3] = pb.y;
    }
  } else {
#pragma unroll
    for (int b = 0; b < kChunk; b += 2) {
      if ((b / S) % 4 == 0) {
        float2 x0 = make_float2(v[b], v[b + 1]);
        float2 x1 = make_float2(v[b + S], v[b + S + 1]);
        float2 x2 = make_float2(v[b + 2 * S], v[b + 2 * S + 1]);
        float2 x3 = make_float2(v[b + 3 * S], v[b + 3 * S + 1]);
        const float2 sv = __fadd2_rn(__fadd2_rn(x0, x1), __fadd2_rn(x2, x3));
        x0 = __ffma2_rn(x0, m2, sv);
        x1 = __ffma2_rn(x1, m2, sv);
        x2 = __ffma2_rn(x2, m2, sv);
        x3 = __ffma2_rn(x3, m2, sv);
        v[b] = x0.x;
        v[b + 1] = x0.y;
        v[b + S] = x1.x;
        v[b + S + 1] = x1.y;
        v[b + 2 * S] = x2.x;
        v[b + 2 * S + 1] = x2.y;
        v[b + 3 * S] = x3.x;
        v[b + 3 * S + 1] = x3.y;
      }
    }
  }
}

__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xFFFF0000u);
}

// Four int8 codes of v[0..3] * inv -> one 32-bit word, code 0 in byte 0. The rounded sum's bit
// pattern is 0x4B400000 + q, so its low byte is already q in two's complement (|q| <= 127:
// |v| <= absmax and absmax * inv exceeds 127 by a few ulp at most, so no code saturates).
__device__ __forceinline__ uint32_t code_bytes4(float v0, float v1, float v2, float v3,
                                                float inv) {
  const float2 m = make_float2(12582912.0f, 12582912.0f);
  const float2 ii = make_float2(inv, inv);
  const float2 r01 = __ffma2_rn(make_float2(v0, v1), ii, m);
  const float2 r23 = __ffma2_rn(make_float2(v2, v3), ii, m);
  const uint32_t lo = __byte_perm(__float_as_uint(r01.x), __float_as_uint(r01.y), 0x0040);
  const uint32_t hi = __byte_perm(__float_as_uint(r23.x), __float_as_uint(r23.y), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// Eight codes of v[0..7] * inv (rounded half-to-even) -> one word, code i in bits 4i .. 4i+3.
// The low nibble of the rounded sum's bit pattern (0x4B400000 + q) is q in 4-bit two's
// complement (|q| <= 7), so the codes are gathered with byte permutes and one masked merge.
__device__ __forceinline__ uint32_t code_nibbles8(const float* v, float inv) {
  const float2 m = make_float2(12582912.0f, 12582912.0f);
  const float2 ii = make_float2(inv, inv);
  const float2 r01 = __ffma2_rn(make_float2(v[0], v[1]), ii, m);
  const float2 r23 = __ffma2_rn(make_float2(v[2], v[3]), ii, m);
  const float2 r45 = __ffma2_rn(make_float2(v[4], v[5]), ii, m);
  const float2 r67 = __ffma2_rn(make_float2(v[6], v[7]), ii, m);
  const uint32_t e = __byte_perm(__byte_perm(__float_as_uint(r01.x), __float_as_uint(r23.x), 0x0040),
                                 __byte_perm(__float_as_uint(r45.x), __float_as_uint(r67.x), 0x0040),
                                 0x5410);
  const uint32_t o = __byte_perm(__byte_perm(__float_as_uint(r01.y), __float_as_uint(r23.y), 0x0040),
                                 __byte_perm(__float_as_uint(r45.y), __float_as_uint(r67.y), 0x0040),
                                 0x5410);
  return (e & 0x0F0F0F0Fu) | ((o << 4) & 0xF0F0F0F0u);
}

template <int G>
__host__ __device__ constexpr int log4_of() {
  return (G == 16) ? 2 : (G == 64) ? 3 : (G == 256) ? 4 : 5;
}

// H_1024 on the 64 values this thread owns, in place (unnormalised: entries +-1). Digits 0..2
// run in registers; then the 16 threads of a group exchange their values once through xbuf (one
// 256-byte row per thread, 16-byte chunk index XOR (row & 7)) and run digits 3 and 4. On entry
// v[4 ch .. 4 ch + 3] holds the chunk's 4-column piece ch ^ perm (perm = 0: natural order; a
// digit-wise permutation of the pieces leaves digits 0..2 unchanged); on return v[] holds the
// values in the layout documented at store_codes().
template <int G>
__device__ __forceinline__ void transform_chunk(float (&v)[kChunk], float4* __restrict__ xbuf,
                                                int tid, int perm = 0) {
  static_assert(G == 1024, "G <= 256 use the slot layout (transform_slots)");
  radix4_stage<1>(v);
  radix4_stage<4>(v);
  radix4_stage<16>(v);
  float4* mine = xbuf + tid * 16;
  const int wx = perm ^ (tid & 7);
#pragma unroll
  for (int ch = 0; ch < 16; ++ch)
    mine[ch ^ wx] = make_float4(v[4 * ch], v[4 * ch + 1], v[4 * ch + 2], v[4 * ch + 3]);
  __syncwarp();
  // group = 16 threads; thread j takes column chunk j (4 columns) of all 16 rows.
  const int j = tid & 15;
  const int t0 = tid & ~15;
#pragma unroll
  for (int a = 0; a < 16; ++a) {
    const int rr = t0 + a;
    const float4 w = xbuf[rr * 16 + (j ^ (rr & 7))];
    v[a * 4 + 0] = w.x;
    v[a * 4 + 1] = w.y;
    v[a * 4 + 2] = w.z;
    v[a * 4 + 3] = w.w;
  }
  radix4_stage<4>(v);   // digit 3 = a bits 0..1
  radix4_stage<16>(v);  // digit 4 = a bits 2..3
}

// max |v| as a tree (8 independent chains, then a short tree) rather than one serial chain
__device__ __forceinline__ float chunk_absmax(const float (&v)[kChunk]) {
  float m[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) m[j] = fabsf(v[j]);
#pragma unroll
  for (int i = 8; i < kChunk; i += 8)
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = fmaxf(m[j], fabsf(v[i + j]));
  return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

// Quantise and store the codes of chunk c of one row (qr = row start in the code buffer).
// Layout of v[]:
//   G <= 64 : v[i] is column 64c + i.
//   G == 1024 (after transform_chunk): thread j = c & 15 of group c >> 4; v[a*4 + e] is column
//             1024 (c >> 4) + 64a + 4j + e.
// (G = 256 uses the slot layout and store_slots.)
template <int G>
__device__ __forceinline__ void store_codes(const float (&v)[kChunk], float inv,
                                            uint8_t* __restrict__ qr, int c, int K_pad) {
  if constexpr (G <= 64) {
    uint32_t wd[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) wd[w] = code_nibbles8(v + 8 * w, inv);
    const int byte0 = c * (kChunk / 2);
    if (c * kChunk + kChunk <= K_pad) {
      uint4* dst = reinterpret_cast<uint4*>(qr + byte0);
      dst[0] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      dst[1] = make_uint4(wd[4], wd[5], wd[6], wd[7]);
    } else {
      // ragged last chunk (G = 16 only): store the 16-column groups below K_pad.
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        if (c * kChunk + gi * 16 < K_pad)
          *reinterpret_cast<uint2*>(qr + byte0 + gi * 8) = make_uint2(wd[2 * gi], wd[2 * gi + 1]);
      }
    }
  } else {
    // 4 consecutive codes per a (16 bits at byte 32 a + 2 j of the group's 512 bytes): the low
    // nibbles of the rounded sums' bit patterns, gathered by byte permutes as in code_nibbles8
    const int j = c & 15;
    uint8_t* qg = qr + (c >> 4) * 512 + 2 * j;
    const float2 m = make_float2(12582912.0f, 12582912.0f);
    const float2 ii = make_float2(inv, inv);
#pragma unroll
    for (int a = 0; a < 16; ++a) {
      const float2 r01 = __ffma2_rn(make_float2(v[a * 4 + 0], v[a * 4 + 1]), ii, m);
      const float2 r23 = __ffma2_rn(make_float2(v[a * 4 + 2], v[a * 4 + 3]), ii, m);
      const uint32_t e = __byte_perm(__float_as_uint(r01.x), __float_as_uint(r23.x), 0x0040);
      const uint32_t o = __byte_perm(__float_as_uint(r01.y), __float_as_uint(r23.y), 0x0040);
      *reinterpret_cast<uint16_t*>(qg + a * 32) =
          static_cast<uint16_t>((e & 0x0F0Fu) | ((o << 4) & 0xF0F0u));
    }
  }
}

// int8 variant of store_codes (one code per byte, row of K_pad bytes); same v[] layouts.
template <int G>
__device__ __forceinline__ void store_codes_i8(const float (&v)[kChunk], float inv,
                                               uint8_t* __restrict__ qr, int c, int K_pad) {
  if constexpr (G <= 64) {
    uint32_t wd[16];
#pragma unroll
    for (int w = 0; w < 16; ++w)
      wd[w] = code_bytes4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3], inv);
    uint4* dst = reinterpret_cast<uint4*>(qr + c * kChunk);
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      // a ragged last chunk (G = 16 only) stores the 16-column groups below K_pad
      if (c * kChunk + gi * 16 < K_pad)
        dst[gi] = make_uint4(wd[4 * gi], wd[4 * gi + 1], wd[4 * gi + 2], wd[4 * gi + 3]);
    }
  } else {
    const int j = c & 15;
    const int q_grp = c >> 4;
#pragma unroll
    for (int a = 0; a < 16; ++a)
      *reinterpret_cast<uint32_t*>(qr + q_grp * 1024 + a * 64 + 4 * j) =
          code_bytes4(v[a * 4], v[a * 4 + 1], v[a * 4 + 2], v[a * 4 + 3], inv);
  }
}

// scale = fp32(absmax / QM) of the normalised row; inv multiplies unnormalised values.
template <int G, int QM>
__device__ __forceinline__ void row_scale(unsigned int amax_bits, float& scale, float& inv) {
  constexpr float kNorm = 1.0f / static_cast<float>(1 << log4_of<G>());
  const float amax = __uint_as_float(amax_bits) * kNorm;
  scale = __fdiv_rn(amax, static_cast<float>(QM));
  inv = (scale > 0.f) ? __frcp_rn(scale) * kNorm : 0.f;
}

// QM = 7: packed int4 codes; QM = 127: int8 codes, one per byte.
template <int G, int QM>
__device__ __forceinline__ void store_row_codes(const float (&v)[kChunk], float inv,
                                                uint8_t* __restrict__ qr, int c, int K_pad) {
  static_assert(QM == 7 || QM == 127, "int4 or int8 codes");
  if constexpr (QM == 7)
    store_codes<G>(v, inv, qr, c, K_pad);
  else
    store_codes_i8<G>(v, inv, qr, c, K_pad);
}

// ---------------------------------------------------------------------------------------------
// NVFP4 codes (QM == kQmFp4): e2m1 elements, one unsigned e4m3 scale per 16 consecutive K, an
// fp32 scale per row g = amax / (6 * 448). Elements are packed two per byte (k = 2b in the low
// nibble). Block scales are written in the order the block-scaled GEMM moves them into tensor
// memory. Within a 128-row group and 64-K chunk the scale of row r and block b (of the 4 in
// the chunk) belongs at byte 16 (r % 32) + 4 ((r % 128) / 32) + b of a 512-byte atom.
//  * activations (tiles of 128 rows): the atoms themselves, one per tile and chunk, the chunk
//    count per tile rounded up to even (the padding atom is never written);
//  * weights (tiles of the GEMM's N tile: 192 rows for NVFP4, 224 for MXFP4): one 4096-byte
//    image per tile and chunk, the layout one 128-lane copy reads: 128 lanes L of 32 bytes,
//    lane L byte j at 256 (L / 8) + 128 (j / 16) + 16 (L % 8) + j % 16; row r's scales are in
//    the four lanes L = r % 32 + 32 q (q = 0..3) at byte 4 ((r % 128) / 32) + b of the half
//    j / 16 = r / 128.
constexpr int kQmFp4 = 6;

struct Fp4Out {
  uint8_t* sf;        // block scales (as above)
  int tile_rows;      // 192 / 224 (NVFP4 / MXFP4 weights) or 128 (activations)
  int kc_per_row;     // chunks of 4 scales per row: K4 / 64 (NVFP4), ceil(K4 / 128) (MXFP4)
  int layout;         // Fp4SfLayout
};

// Byte offset of block scale (row, blk) (weights: replica 0; replica q sits q * 1024 bytes
// further on), split into a per-row part (computed once per row) and a per-block part.
struct Fp4SfRow {
  int64_t base;       // offset of (row, block 0)
  int64_t chunk;      // bytes from one 64-K chunk to the next
};

__device__ __forceinline__ Fp4SfRow fp4_sf_row(int64_t row, const Fp4Out& o) {
  const int rr = static_cast<int>(row);          // rows < 2^31
  const int tile = rr / o.tile_rows;
  const int r = rr - tile * o.tile_rows;
  const int lane = r & 31;
  if (o.layout == kSfActAtoms) {
    const int kc_even = (o.kc_per_row + 1) & ~1;
    return Fp4SfRow{static_cast<int64_t>(tile) * kc_even * 512 + 16 * lane + 4 * ((r >> 5) & 3),
                    512};
  }
  return Fp4SfRow{static_cast<int64_t>(tile) * o.kc_per_row * 4096 + (lane >> 3) * 256 +
                      16 * (lane & 7) + 4 * ((r >> 5) & 3) + 128 * (r >> 7),
                  4096};
}

// Store the 4 block scales of one 64-K chunk (block blk, a multiple of 4, and the next three)
// as one 32-bit word (weights: into all four replicas).
__device__ __forceinline__ void fp4_sf_store4(const Fp4Out& o, const Fp4SfRow& sr, int blk,
                                              uint32_t s4) {
  uint8_t* p = o.sf + sr.base + (blk >> 2) * sr.chunk;
  const int replicas = o.layout == kSfActAtoms ? 1 : 4;
  for (int q = 0; q < replicas; ++q) *reinterpret_cast<uint32_t*>(p + q * 1024) = s4;
}

// e4m3 byte of a non-negative value (round to nearest even, saturating at 448), and its value.
__device__ __forceinline__ uint32_t e4m3_byte(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

// The value of a byte < 0x80: its 4 exponent and 3 mantissa bits placed at the top of an fp32
// exponent and mantissa, scaled by 2^120 (the difference of the two exponent biases, 127 - 7).
// Exact for normal and subnormal e4m3 (the fp32 operand is then subnormal; no flush to zero).
__device__ __forceinline__ float e4m3_value(uint32_t byte) {
  return __uint_as_float(byte << 20) * 0x1p120f;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Eight values -> eight e2m1 nibbles (element 0 in bits 0..3), round to nearest even, saturating.
// The scaling multiplies run in packed fp32x2 form.
__device__ __forceinline__ uint32_t e2m1_pack8(const float* x, float s) {
  const float2 ss = make_float2(s, s);
  const float2 p0 = __fmul2_rn(make_float2(x[0], x[1]), ss);
  const float2 p1 = __fmul2_rn(make_float2(x[2], x[3]), ss);
  const float2 p2 = __fmul2_rn(make_float2(x[4], x[5]), ss);
  const float2 p3 = __fmul2_rn(make_float2(x[6], x[7]), ss);
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(p0.x), "f"(p0.y), "f"(p1.x), "f"(p1.y), "f"(p2.x), "f"(p2.y), "f"(p3.x), "f"(p3.y));
  return r;
}

__device__ __forceinline__ uint32_t e2m1_pack4(const float* x, float s) {
  uint16_t r;
  asm("{\n\t.reg .b8 b0, b1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "mov.b16 %0, {b0, b1};\n\t}"
      : "=h"(r)
      : "f"(x[0] * s), "f"(x[1] * s), "f"(x[2] * s), "f"(x[3] * s));
  return r;
}

// Per-row constants of the NVFP4 mode: r6 = kNorm / (6 g) turns an unnormalised block maximum
// into the e4m3 scale argument, kng = kNorm / g turns 1 / scale into the element multiplier.
struct Fp4Row {
  float g, r6, kng;
};

template <int G>
__device__ __forceinline__ Fp4Row fp4_row(float g) {
  constexpr float kNorm = 1.0f / static_cast<float>(1 << log4_of<G>());
  // kNorm is a power of two, so kNorm * rcp_rn(d) is the correctly rounded kNorm / d
  return g > 0.f ? Fp4Row{g, kNorm * __frcp_rn(6.0f * g), kNorm * __frcp_rn(g)}
                 : Fp4Row{0.f, 0.f, 0.f};
}

// Block scale byte from the block's (unnormalised) absmax; `mult` multiplies unnormalised
// values into element units (0 when the block scale is 0). The reciprocal of the scale is the
// hardware approximation (within one ulp; the scale is a normal fp32 >= 2^-9).
__device__ __forceinline__ uint32_t fp4_block(float bmax_unnorm, const Fp4Row& rw, float& mult) {
  const uint32_t s = (rw.g > 0.f) ? e4m3_byte(bmax_unnorm * rw.r6) : 0u;
  mult = (s != 0u) ? rw.kng * rcp_approx(e4m3_value(s)) : 0.f;
  return s;
}

__device__ __forceinline__ float absmax16(const float* x) {
  float m[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) m[j] = fmaxf(fmaxf(fabsf(x[j]), fabsf(x[4 + j])),
                                           fmaxf(fabsf(x[8 + j]), fabsf(x[12 + j])));
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// Quantise and store chunk c of one row in NVFP4 (layouts as store_codes for G <= 64, as
// store_slots for G = 256, as blocks_1024 leaves them for G = 1024: in every case v[16r ..
// 16r + 15] is one 16-column block, whose maximum |v| is bm[r]). Every lane of the warp calls
// this (G >= 256 trade scale bytes between lanes); `active` gates the stores.
//
// Block scales leave as one 32-bit word per thread (the 4 blocks of one 64-K chunk) instead of
// four scattered bytes. G = 256: thread j (of 4) holds the blocks of chunks 4 (c >> 2) + (j ^ r)
// at byte position j; it stores chunk 4 (c >> 2) + j, taking byte m of the word of thread
// j ^ m. G = 1024: thread 4t + u holds the blocks of chunks 16 (c >> 4) + 4u + r at byte
// position t; it stores chunk 16 (c >> 4) + 4u + t, taking byte t of the word of thread
// 4 (t ^ m) + u.
template <int G>
__device__ __forceinline__ void store_fp4(const float (&v)[kChunk], const float (&bm)[4], float g,
                                          uint8_t* __restrict__ qr, int64_t row, int c, int j,
                                          const Fp4Out& o, bool active) {
  const Fp4Row rw = fp4_row<G>(g);
  const Fp4SfRow sr = fp4_sf_row(row, o);
  uint32_t sbytes = 0, w[8];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float mult;
    sbytes |= fp4_block(bm[r], rw, mult) << (8 * r);
    w[2 * r] = e2m1_pack8(v + 16 * r, mult);
    w[2 * r + 1] = e2m1_pack8(v + 16 * r + 8, mult);
  }
  if constexpr (G <= 64) {
    if (!active) return;
    uint4* dst = reinterpret_cast<uint4*>(qr + 32 * c);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    fp4_sf_store4(o, sr, 4 * c, sbytes);
  } else {
    // idx: this thread's position among the 4 that share chunks; unit: lane distance between them
    constexpr int unit = (G == 256) ? 1 : 4;
    const int idx = (G == 256) ? j : ((c & 15) >> 2);
    uint32_t word = ((sbytes >> (8 * ((G == 256) ? 0 : idx))) & 0xFFu) << (8 * idx);
#pragma unroll
    for (int m = 1; m < 4; ++m) {
      const uint32_t other = __shfl_xor_sync(0xffffffffu, sbytes, m * unit);
      const int byte = (G == 256) ? m : idx;
      word |= ((other >> (8 * byte)) & 0xFFu) << (8 * (idx ^ m));
    }
    if (!active) return;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int col = (G == 256) ? 256 * (c >> 2) + 64 * (j ^ r) + 16 * j
                                 : 1024 * (c >> 4) + 64 * (4 * (c & 3) + r) + 16 * idx;
      *reinterpret_cast<uint2*>(qr + col / 2) = make_uint2(w[2 * r], w[2 * r + 1]);
    }
    const int chunk = (G == 256) ? 4 * (c >> 2) + j : 16 * (c >> 4) + 4 * (c & 3) + idx;
    fp4_sf_store4(o, sr, 4 * chunk, word);
  }
}

// MXFP4 codes (QM == kQmMx): e2m1 elements and one power-of-two scale 2^X per 32 consecutive K,
// X = floor(log2(max |x_rot| over the block)) - 2 clamped to [-127, 127] (-127 for an all-zero
// block), stored as the e8m0 byte X + 127; no per-row scale. Scale bytes use the NVFP4 layouts
// with 128-K chunks of 4 scales in place of 64-K chunks of 4 scales.
constexpr int kQmMx = 5;

// e8m0 byte of the block maximum of unnormalised values (x_rot = v * 2^-k, k = log4 G) and the
// multiplier that turns those values into element units (v * 2^-k / 2^X); 0 for a zero block.
template <int G>
__device__ __forceinline__ uint32_t mx_block(float bmax_unnorm, float& mult) {
  constexpr int k = log4_of<G>();
  constexpr float kNorm = 1.0f / static_cast<float>(1 << k);
  if (!(bmax_unnorm > 0.f)) {
    mult = 0.f;
    return 0u;
  }
  uint32_t b = __float_as_uint(bmax_unnorm);
  int ef = static_cast<int>((b >> 23) & 0xFFu);
  if (ef == 0) ef = static_cast<int>((__float_as_uint(bmax_unnorm * 0x1p64f) >> 23) & 0xFFu) - 64;
  int X = ef - 127 - k - 2;                        // floor(log2(bmax * 2^-k)) - 2
  X = X < -127 ? -127 : (X > 127 ? 127 : X);
  // 2^-X as fp32 (2^-127 is subnormal), then the exact 2^-k
  const float inv = X == 127 ? __uint_as_float(0x00400000u) : __uint_as_float((127 - X) << 23);
  mult = inv * kNorm;
  return static_cast<uint32_t>(X + 127);
}

// Store one scale byte (32-block blk of the row; weights: into all four replicas).
__device__ __forceinline__ void mx_sf_store1(const Fp4Out& o, const Fp4SfRow& sr, int blk,
                                             uint32_t s) {
  uint8_t* p = o.sf + sr.base + (blk >> 2) * sr.chunk + (blk & 3);
  const int replicas = o.layout == kSfActAtoms ? 1 : 4;
  for (int q = 0; q < replicas; ++q) p[q * 1024] = static_cast<uint8_t>(s);
}

// Quantise and store chunk c of one row in MXFP4 (layouts as store_fp4; bm[r] = max |v| of the
// 16-column block in slot r). A 32-column block is two of those: for G <= 64 the slots 2h, 2h + 1
// of one thread; for G = 256 this thread's slot r and slot r ^ 1 of lane j ^ 1; for G = 1024
// slot r of this thread and of lane ^ 4. Every lane calls this (the partners trade maxima).
//
// Scale bytes leave as one 32-bit word (the 4 scales of a 128-K chunk) from half the threads:
// G <= 64 (when `pairs`: chunks per row even, so chunks 2h and 2h + 1 of a row sit in lanes
// 2i, 2i + 1): the even chunk's thread stores blocks 2c .. 2c + 3, two of them its partner's.
// G = 256: blocks of thread j at 8 (c >> 2) + 2 (j ^ r) + j / 2 for slot r; threads j = 0 and
// j = 2 (lanes 2 apart) trade their bytes and store chunks 2 (c >> 2) and 2 (c >> 2) + 1.
// G = 1024: blocks at 32 (c >> 4) + 8 (c & 3) + 2r + idx / 2 for idx = (c & 15) >> 2 in {0, 2}
// (lanes 8 apart); idx 0 stores chunk 8 (c >> 4) + 2 (c & 3), idx 2 the next one. Otherwise
// (G <= 64, odd chunk count) each thread stores its two bytes alone.
template <int G>
__device__ __forceinline__ void store_mx(const float (&v)[kChunk], const float (&bm)[4],
                                         uint8_t* __restrict__ qr, int64_t row, int c, int j,
                                         const Fp4Out& o, bool active, bool pairs) {
  const Fp4SfRow sr = fp4_sf_row(row, o);
  float b32[4];
  if constexpr (G <= 64) {
    b32[0] = b32[1] = fmaxf(bm[0], bm[1]);
    b32[2] = b32[3] = fmaxf(bm[2], bm[3]);
  } else if constexpr (G == 256) {
    float other[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) other[r] = __shfl_xor_sync(0xffffffffu, bm[r], 1);
#pragma unroll
    for (int r = 0; r < 4; ++r) b32[r] = fmaxf(bm[r], other[r ^ 1]);
  } else {
#pragma unroll
    for (int r = 0; r < 4; ++r) b32[r] = fmaxf(bm[r], __shfl_xor_sync(0xffffffffu, bm[r], 4));
  }
  uint32_t w[8], sb[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float mult;
    sb[r] = mx_block<G>(b32[r], mult);
    w[2 * r] = e2m1_pack8(v + 16 * r, mult);
    w[2 * r + 1] = e2m1_pack8(v + 16 * r + 8, mult);
  }
  const uint32_t own = sb[0] | (sb[1] << 8) | (sb[2] << 16) | (sb[3] << 24);
  if constexpr (G <= 64) {
    // __byte_perm(x, y, s): byte i of the result is byte s_i of {y : x} (x bytes 0-3, y 4-7)
    const uint32_t other = pairs ? __shfl_xor_sync(0xffffffffu, own, 1) : 0u;
    if (!active) return;
    uint4* dst = reinterpret_cast<uint4*>(qr + 32 * c);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    if (!pairs) {
      mx_sf_store1(o, sr, 2 * c, sb[0]);
      mx_sf_store1(o, sr, 2 * c + 1, sb[2]);
    } else if ((c & 1) == 0) {
      fp4_sf_store4(o, sr, 2 * c, __byte_perm(own, other, 0x6420));
    }
  } else {
    constexpr int kPartner = (G == 256) ? 2 : 8;
    const uint32_t other = __shfl_xor_sync(0xffffffffu, own, kPartner);
    if (!active) return;
    const int idx = (G == 256) ? j : ((c & 15) >> 2);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int col = (G == 256) ? 256 * (c >> 2) + 64 * (j ^ r) + 16 * j
                                 : 1024 * (c >> 4) + 64 * (4 * (c & 3) + r) + 16 * idx;
      *reinterpret_cast<uint2*>(qr + col / 2) = make_uint2(w[2 * r], w[2 * r + 1]);
    }
    if (G == 256 && j == 0)
      fp4_sf_store4(o, sr, 8 * (c >> 2), __byte_perm(own, other, 0x7160));
    else if (G == 256 && j == 2)
      fp4_sf_store4(o, sr, 8 * (c >> 2) + 4, __byte_perm(own, other, 0x1706));
    else if (G == 1024 && idx == 0)
      fp4_sf_store4(o, sr, 32 * (c >> 4) + 8 * (c & 3), __byte_perm(own, other, 0x5140));
    else if (G == 1024 && idx == 2)
      fp4_sf_store4(o, sr, 32 * (c >> 4) + 8 * (c & 3) + 4, __byte_perm(own, other, 0x3726));
  }
}

// G = 1024, NVFP4 mode: regroup the transformed chunk so that every thread holds whole
// 16-column blocks. Before (transform_chunk<1024>): thread j of a 16-lane group holds
// v[4a + e] = column 64a + 4j + e of its 1024-group, a = 0..15. After: thread j = 4t + u holds
// v[16r + 4k + e] = column 64 (4u + r) + 16t + 4k + e, i.e. block t of the 64-column rows
// a = 4u .. 4u + 3. The exchange runs through the threads' own 256-byte shared rows; the float4
// of row a sits at slot a ^ sw(j) ^ 2 (a / 8) with sw(j) = (j % 4) ^ 5 ((j / 4) % 2), which puts
// both the stores (8 lanes, one a each) and the loads (8 lanes: 2 source threads x 4 rows) on 8
// distinct 16-byte bank groups.
__device__ __forceinline__ void blocks_1024(float (&v)[kChunk], float4* __restrict__ xbuf,
                                            int tid) {
  const int j = tid & 15;
  float4* mine = xbuf + tid * 16;
  __syncwarp();                     // the transform's loads from these rows are complete
  const int swm = (j & 3) ^ (((j >> 2) & 1) * 5);
#pragma unroll
  for (int a = 0; a < 16; ++a)
    mine[a ^ swm ^ ((a >> 3) << 1)] =
        make_float4(v[4 * a], v[4 * a + 1], v[4 * a + 2], v[4 * a + 3]);
  __syncwarp();
  const int t = j >> 2, u = j & 3;
  const float4* grp = xbuf + (tid - j) * 16;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int a = 4 * u + r;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int src = 4 * t + k;
      const int sw = k ^ ((t & 1) * 5);
      const float4 w = grp[src * 16 + (a ^ sw ^ ((a >> 3) << 1))];
      v[16 * r + 4 * k + 0] = w.x;
      v[16 * r + 4 * k + 1] = w.y;
      v[16 * r + 4 * k + 2] = w.z;
      v[16 * r + 4 * k + 3] = w.w;
    }
  }
  __syncwarp();                     // loads complete before the next round's stores
}

// ---------------------------------------------------------------------------------------------
// Register-resident kernel: direct loads with a one-group prefetch, cross-thread digits by
// warp shuffles (no shared-memory staging of the data).
//
// Slot layout (G = 256). A thread owns chunk c (64 consecutive columns) of its row, split into
// 4 blocks of 16 columns (one per value of base-4 digit 2); register slot s holds block s ^ j,
// where j = c mod 4 is the thread's position in its group. XOR acts digit by digit, so every
// radix-4 tuple is still a fixed set of slots, and in exchange round r (r = 1, 2, 3) each thread
// swaps slot r with thread j ^ r: its slot r holds the block that thread needs, and receives
// block j of that thread. Afterwards slot r holds block j of chunk c ^ r, i.e. digit 3 is
// indexed by slot. G <= 64 needs no exchange (natural order); G = 1024 loads in natural order
// and exchanges through shared memory (transform_chunk).

// 8 bf16 (one 16-byte unit) at column col of row xr; columns >= K read as 0.
template <int N>
__device__ __forceinline__ void load_bf16_unit(uint32_t* raw, const uint16_t* __restrict__ xr,
                                               int col, int K, bool active) {
  static_assert(N == 8, "unit of 8 bf16");
  if (active && col + N <= K) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(xr + col));
    raw[0] = u.x;
    raw[1] = u.y;
    raw[2] = u.z;
    raw[3] = u.w;
  } else {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const uint32_t lo = (active && col + 2 * i < K) ? xr[col + 2 * i] : 0u;
      const uint32_t hi = (active && col + 2 * i + 1 < K) ? xr[col + 2 * i + 1] : 0u;
      raw[i] = lo | (hi << 16);
    }
  }
}

// The 64 bf16 of chunk c of row xr, in slot layout, as 32 bf16 pairs.
template <int G>
__device__ __forceinline__ void load_chunk(uint32_t (&raw)[kChunk / 2],
                                           const uint16_t* __restrict__ xr, int c, int j, int K,
                                           bool active) {
  const int c0 = c * kChunk;
  if (__all_sync(0xffffffffu, active && c0 + kChunk <= K)) {
    // every lane's chunk lies inside its row (a warp-uniform test, so a ragged row end does
    // not split the warp): eight 16-byte loads in slot order, no per-unit checks
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = (G == 256) ? c0 + 16 * (s ^ j) + 8 * h : c0 + 16 * s + 8 * h;
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(xr + col));
        raw[8 * s + 4 * h + 0] = u.x;
        raw[8 * s + 4 * h + 1] = u.y;
        raw[8 * s + 4 * h + 2] = u.z;
        raw[8 * s + 4 * h + 3] = u.w;
      }
    return;
  }
  if ((K & 7) == 0) {
    // K a multiple of 8: each 16-byte unit lies wholly inside or wholly past the row end, so
    // a predicate per unit replaces the element-wise tail path
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = (G == 256) ? c0 + 16 * (s ^ j) + 8 * h : c0 + 16 * s + 8 * h;
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (active && col < K) u = __ldg(reinterpret_cast<const uint4*>(xr + col));
        raw[8 * s + 4 * h + 0] = u.x;
        raw[8 * s + 4 * h + 1] = u.y;
        raw[8 * s + 4 * h + 2] = u.z;
        raw[8 * s + 4 * h + 3] = u.w;
      }
    return;
  }
  if constexpr (G <= 64) {
#pragma unroll
    for (int l = 0; l < 8; ++l) load_bf16_unit<8>(raw + 4 * l, xr, c0 + 8 * l, K, active);
  } else {
    static_assert(G == 256, "slot layout for G = 256");
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        load_bf16_unit<8>(raw + 8 * s + 4 * h, xr, c0 + 16 * (s ^ j) + 8 * h, K, active);
  }
}

__device__ __forceinline__ void unpack_chunk(const uint32_t (&raw)[kChunk / 2],
                                             float (&v)[kChunk]) {
#pragma unroll
  for (int i = 0; i < kChunk / 2; ++i) bf16x2_to_f32(raw[i], v[2 * i], v[2 * i + 1]);
}

// H_G on the slot layout (unnormalised), G <= 256. The threads of one group are lanes that
// differ only in their two low bits; every lane of the warp takes part in the shuffles.
template <int G>
__device__ __forceinline__ void transform_slots(float (&v)[kChunk]) {
  static_assert(G <= 256, "G = 1024 uses transform_chunk");
  radix4_stage<1>(v);
  radix4_stage<4>(v);
  if constexpr (G >= 64) radix4_stage<16>(v);       // digit 2 (G = 256: across the 4 slots)
  if constexpr (G == 256) {
#pragma unroll
    for (int r = 1; r < 4; ++r)
#pragma unroll
      for (int e = 0; e < 16; ++e) v[16 * r + e] = __shfl_xor_sync(0xffffffffu, v[16 * r + e], r);
    radix4_stage<16>(v);                              // digit 3 = chunk index bits 0..1
  }
}

// Quantise and store chunk c after transform_slots. For G = 256 slot r then holds columns
// 256 (c >> 2) + 64 (j ^ r) + 16 j + e, e < 16; for G <= 64 the layout is natural (as
// store_codes).
template <int G, int QM>
__device__ __forceinline__ void store_slots(const float (&v)[kChunk], float inv,
                                            uint8_t* __restrict__ qr, int c, int j, int K_pad) {
  if constexpr (G <= 64) {
    store_row_codes<G, QM>(v, inv, qr, c, K_pad);
  } else {
    static_assert(G == 256, "slot layout for G = 256");
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float* b = v + 16 * r;
      const int col = 256 * (c >> 2) + 64 * (j ^ r) + 16 * j;
      if constexpr (QM == 7) {
        *reinterpret_cast<uint2*>(qr + col / 2) =
            make_uint2(code_nibbles8(b, inv), code_nibbles8(b + 8, inv));
      } else {
        *reinterpret_cast<uint4*>(qr + col) =
            make_uint4(code_bytes4(b[0], b[1], b[2], b[3], inv),
                       code_bytes4(b[4], b[5], b[6], b[7], inv),
                       code_bytes4(b[8], b[9], b[10], b[11], inv),
                       code_bytes4(b[12], b[13], b[14], b[15], inv));
      }
    }
  }
}

// Persistent: CTA b handles row groups b, b + gridDim.x, ... of R rows (R * P threads, P =
// ceil(K_pad / 64) chunks per row). While a group is transformed the next group's bf16 data is
// already loading into registers. The row absmax meets in shared memory (one atomicMax per
// thread, three rotating slots so one barrier per group suffices).
constexpr int kRegMaxRows = 256;

template <int G, int QM, int kMaxT, int kMinBlocks>
__global__ void __launch_bounds__(kMaxT, kMinBlocks)
rht_quant_reg_kernel(const uint16_t* __restrict__ X, int64_t M, int K, int64_t ldx, int K_pad,
                     uint8_t* __restrict__ Q, int64_t ldq, float* __restrict__ S, int R, int P,
                     int64_t num_groups, int team_rows, Fp4Out fp4) {
  __shared__ unsigned int amax_s[3 * kRegMaxRows];
  // G = 1024 exchanges through shared memory (one 256-byte row per thread): 15 shuffle rounds
  // of 4 values cost more than one XOR-swizzled store and load of the chunk
  extern __shared__ __align__(16) unsigned char smem_x[];
  float4* xbuf = reinterpret_cast<float4*>(smem_x);
  constexpr int kLoadG = (G == 1024) ? 64 : G;     // G = 1024 loads in natural order
  const int tid = threadIdx.x;
  const int r_local = tid / P;
  const int c = tid - r_local * P;
  const bool lane_ok = r_local < R;
  const int j = (G == 256) ? (c & 3) : 0;
  for (int i = tid; i < 3 * R; i += blockDim.x) amax_s[i] = 0u;
  __syncthreads();
  grid_dependency_wait();
  launch_dependents();

  uint32_t raw[kChunk / 2];
  int64_t rg = blockIdx.x;
  {
    const int64_t row = rg * R + r_local;
    const bool act = lane_ok && row < M;
    load_chunk<kLoadG>(raw, X + (act ? row : 0) * ldx, c, j, K, act);
  }
  for (int64_t i = 0; rg < num_groups; rg += gridDim.x, ++i) {
    const int64_t row = rg * R + r_local;
    const bool active = lane_ok && row < M;
    float v[kChunk];
    unpack_chunk(raw, v);
    const int64_t rg_next = rg + gridDim.x;
    if (rg_next < num_groups) {
      const int64_t row_n = rg_next * R + r_local;
      const bool act = lane_ok && row_n < M;
      load_chunk<kLoadG>(raw, X + (act ? row_n : 0) * ldx, c, j, K, act);
    }
    if constexpr (G == 1024)
      transform_chunk<G>(v, xbuf, tid);
    else
      transform_slots<G>(v);
    // NVFP4 / MXFP4: the maxima of the four 16-column blocks (NVFP4 also takes the row maximum
    // from them)
    float bm[4], m;
    if constexpr (QM == kQmFp4 || QM == kQmMx) {
      if constexpr (G == 1024) blocks_1024(v, xbuf, tid);
#pragma unroll
      for (int r = 0; r < 4; ++r) bm[r] = absmax16(v + 16 * r);
      m = fmaxf(fmaxf(bm[0], bm[1]), fmaxf(bm[2], bm[3]));
    } else {
      m = chunk_absmax(v);
    }
    if constexpr (QM == kQmMx) {
      // no row scale: no row maximum and no barrier
      store_mx<G>(v, bm, Q + (active ? row : 0) * ldq, row, c, j, fp4, active, (P & 1) == 0);
      continue;
    }
    unsigned int* am = amax_s + static_cast<int>(i % 3) * R;
    if (active) atomicMax(am + r_local, __float_as_uint(m));
    if (team_rows > 0) {
      // rows of this team fill whole warps: only the team's warps meet
      const int team = r_local / team_rows;
      named_barrier_sync(1 + team, team_rows * P);
      const int tt = tid - team * team_rows * P;
      if (tt < team_rows) amax_s[static_cast<int>((i + 2) % 3) * R + team * team_rows + tt] = 0u;
    } else {
      __syncthreads();
      if (tid < R) amax_s[static_cast<int>((i + 2) % 3) * R + tid] = 0u;
    }
    if constexpr (QM == kQmFp4) {
      float g = 0.f;
      if (active) {
        constexpr float kNorm = 1.0f / static_cast<float>(1 << log4_of<G>());
        g = __fdiv_rn(__uint_as_float(am[r_local]) * kNorm, 6.0f * 448.0f);
        if (c == 0) S[row] = g;
      }
      store_fp4<G>(v, bm, g, Q + (active ? row : 0) * ldq, row, c, j, fp4, active);
    } else if constexpr (QM == 7 || QM == 127) {
      if (active) {
        float scale, inv;
        row_scale<G, QM>(am[r_local], scale, inv);
        if (c == 0) S[row] = scale;
        if constexpr (G == 1024)
          store_row_codes<G, QM>(v, inv, Q + row * ldq, c, K_pad);
        else
          store_slots<G, QM>(v, inv, Q + row * ldq, c, j, K_pad);
      }
    }
  }
}

// R[i][j] = (-1)^(number of equal base-4 digits of i and j) / 2^k.
__global__ void make_rht_kernel(float* __restrict__ R, int G, int log4) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= G * G) return;
  const int i = idx / G, j = idx - (idx / G) * G;
  int eq = 0;
  for (int d = 0; d < log4; ++d) eq += (((i >> (2 * d)) & 3) == ((j >> (2 * d)) & 3)) ? 1 : 0;
  const float mag = 1.0f / static_cast<float>(1 << log4);
  R[idx] = (eq & 1) ? -mag : mag;
}

inline int sm_count() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    return 148;
  return v;
}

template <int G, int QM, int kMaxT, int kMinBlocks>
cudaError_t launch_reg_t(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int64_t K_pad,
                         uint8_t* Q, int64_t ldq, float* S, cudaStream_t stream,
                         Fp4Out fp4 = Fp4Out{nullptr, 0, 0, 0}) {
  const int P = static_cast<int>((K_pad + kChunk - 1) / kChunk);
  int r_max = kMaxT / P;
  if (r_max < 1) r_max = 1;
  if (r_max > kRegMaxRows) r_max = kRegMaxRows;
  auto kern = rht_quant_reg_kernel<G, QM, kMaxT, kMinBlocks>;
  auto smem_for = [](int threads) { return G == 1024 ? static_cast<size_t>(threads) * 256 : 0; };
  const int threads_max = ((r_max * P + 31) / 32) * 32;
  if (threads_max > kMaxT) return cudaErrorInvalidValue;
  if (smem_for(threads_max) > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_for(threads_max)));
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads_max,
                                                    smem_for(threads_max)) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t slots = static_cast<int64_t>(sm_count()) * per_sm;
  // Rows per group: the fewest that still finish in the same number of rounds, so that the
  // last round is (nearly) full instead of a short tail on a few CTAs.
  const int64_t rounds = (M + slots * r_max - 1) / (slots * r_max);
  int64_t R = (M + slots * rounds - 1) / (slots * rounds);
  if (R < 1) R = 1;
  if (R > r_max) R = r_max;
  // teams: the fewest rows whose threads fill whole warps; R a multiple of it, at most 15 teams
  int team_rows = 32 / std::gcd(P, 32);
  if (G == 1024 || team_rows > r_max) {
    team_rows = 0;
  } else {
    R = (R + team_rows - 1) / team_rows * team_rows;
    if (R > r_max) R = r_max / team_rows * team_rows;
    if (R / team_rows > 15) team_rows = 0;
  }
  const int threads = ((static_cast<int>(R) * P + 31) / 32) * 32;
  const int64_t groups = (M + R - 1) / R;
  const int64_t grid = groups < slots ? groups : slots;
  return launch_overlapped(kern, dim3(static_cast<unsigned>(grid)), dim3(threads),
                           smem_for(threads), stream, X, M, static_cast<int>(K), ldx,
                           static_cast<int>(K_pad), Q, ldq, S, static_cast<int>(R), P, groups,
                           team_rows, fp4);
}

// The row-streaming kernel (rht_quant_ring.cuh); cudaErrorNotSupported when the shape does not
// fit it.
template <int G, int QM>
cudaError_t launch_ring(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int64_t K_pad,
                        uint8_t* Q, int64_t ldq, float* S, cudaStream_t stream, Fp4Out fp4);

template <int G, int QM>
cudaError_t launch_g(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int64_t K_pad,
                     uint8_t* Q, int64_t ldq, float* S, cudaStream_t stream) {
  // K a multiple of 8 and rows of at most 16384 columns: whole rows stream into a shared ring
  {
    const cudaError_t e = launch_ring<G, QM>(X, M, K, ldx, K_pad, Q, ldq, S, stream,
                                             Fp4Out{nullptr, 0, 0, 0});
    if (e != cudaErrorNotSupported) return e;
  }
  // rows of up to 16384 columns: CTAs of at most 256 threads, two per SM; longer rows (at most
  // 32768 columns): one row per CTA of at most 512 threads
  if (K_pad <= 256 * kChunk)
    return launch_reg_t<G, QM, 256, 2>(X, M, K, ldx, K_pad, Q, ldq, S, stream);
  return launch_reg_t<G, QM, 512, 1>(X, M, K, ldx, K_pad, Q, ldq, S, stream);
}

}  // namespace quant_detail

// qmax = 7: packed int4 codes (K_pad / 2 bytes per row); qmax = 127: int8 codes (K_pad bytes).
inline cudaError_t launch_rht_quant(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int group,
                                    uint8_t* Q, int64_t ldq, float* S, cudaStream_t stream,
                                    int qmax = 7) {
  const int64_t K_pad = (K + group - 1) / group * group;
#define CONVROT_QUANT_CASE(G)                                                              \
  case G:                                                                                  \
    return qmax == 127 ? quant_detail::launch_g<G, 127>(X, M, K, ldx, K_pad, Q, ldq, S, stream) \
                       : quant_detail::launch_g<G, 7>(X, M, K, ldx, K_pad, Q, ldq, S, stream);
  if (qmax != 7 && qmax != 127) return cudaErrorInvalidValue;
  switch (group) {
    CONVROT_QUANT_CASE(16)
    CONVROT_QUANT_CASE(64)
    CONVROT_QUANT_CASE(256)
    CONVROT_QUANT_CASE(1024)
    default: return cudaErrorInvalidValue;
  }
#undef CONVROT_QUANT_CASE
}

// NVFP4: K4 = K_pad rounded up to 64 (whole zero groups past K_pad quantise to zero codes and
// zero block scales); codes K4 / 2 bytes per row, block scales as images of `layout`
// (Fp4SfLayout) for tiles of `tile_rows`.
inline cudaError_t launch_rht_quant_fp4(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                                        int group, uint8_t* Q, int64_t ldq, float* S, uint8_t* sf,
                                        int tile_rows, int layout, cudaStream_t stream) {
  using quant_detail::kQmFp4;
  const int64_t K_pad = (K + group - 1) / group * group;
  const int64_t K4 = (K_pad + 63) / 64 * 64;
  const quant_detail::Fp4Out o{sf, tile_rows, static_cast<int>(K4 / 64), layout};
#define CONVROT_FP4_CASE(G)                                                                   \
  case G:                                                                                     \
    if (G >= 256) {                                                                           \
      const cudaError_t e = quant_detail::launch_ring<G, kQmFp4>(X, M, K, ldx, K4, Q, ldq, S, \
                                                                 stream, o);                  \
      if (e != cudaErrorNotSupported) return e;                                               \
    }                                                                                         \
    return K4 <= 256 * quant_detail::kChunk                                                   \
               ? quant_detail::launch_reg_t<G, kQmFp4, 256, 2>(X, M, K, ldx, K4, Q, ldq, S,   \
                                                               stream, o)                     \
               : quant_detail::launch_reg_t<G, kQmFp4, 512, 1>(X, M, K, ldx, K4, Q, ldq, S,   \
                                                               stream, o);
  switch (group) {
    CONVROT_FP4_CASE(16)
    CONVROT_FP4_CASE(64)
    CONVROT_FP4_CASE(256)
    CONVROT_FP4_CASE(1024)
    default: return cudaErrorInvalidValue;
  }
#undef CONVROT_FP4_CASE
}

// MXFP4: K4 = K_pad rounded up to 64 as for NVFP4 (whole zero groups past K_pad quantise to
// zero codes and the smallest scale); codes K4 / 2 bytes per row, scale bytes in the layout
// `layout` for tiles of `tile_rows`, with 128-K chunks.
inline cudaError_t launch_rht_quant_mx(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                                       int group, uint8_t* Q, int64_t ldq, uint8_t* sf,
                                       int tile_rows, int layout, cudaStream_t stream) {
  using quant_detail::kQmMx;
  const int64_t K_pad = (K + group - 1) / group * group;
  const int64_t K4 = (K_pad + 63) / 64 * 64;
  const quant_detail::Fp4Out o{sf, tile_rows, static_cast<int>((K4 + 127) / 128), layout};
#define CONVROT_MX_CASE(G)                                                                    \
  case G:                                                                                     \
    return K4 <= 256 * quant_detail::kChunk                                                   \
               ? quant_detail::launch_reg_t<G, kQmMx, 256, 2>(X, M, K, ldx, K4, Q, ldq,       \
                                                              nullptr, stream, o)             \
               : quant_detail::launch_reg_t<G, kQmMx, 512, 1>(X, M, K, ldx, K4, Q, ldq,       \
                                                              nullptr, stream, o);
  switch (group) {
    CONVROT_MX_CASE(16)
    CONVROT_MX_CASE(64)
    CONVROT_MX_CASE(256)
    CONVROT_MX_CASE(1024)
    default: return cudaErrorInvalidValue;
  }
#undef CONVROT_MX_CASE
}

inline cudaError_t launch_make_rht(int group, float* R, cudaStream_t stream) {
  int log4 = 0;
  while ((1 << (2 * log4)) < group) ++log4;
  const int n = group * group;
  quant_detail::make_rht_kernel<<<(n + 255) / 256, 256, 0, stream>>>(R, group, log4);
  return cudaGetLastError();
}

}  // namespace convrot
