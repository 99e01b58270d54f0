// rht_quant_ring.cuh -- the row-streaming RHT + quantise kernel: whole token rows move from HBM
// into a deep shared-memory ring with one bulk copy each, and teams of warps rotate, quantise
// and pack them from there.
//
// What it computes is what rht_quant.cuh's kernels compute ("ConvRot" paper, Fig. 3 and
// Thm. 2.3: the group-wise regular Hadamard transform; "v2.3.4: Krea2 ConvRot INT8 Quantization
// Release", "Mathematical Formulation": per-row absmax scale; comfy-kitchen PR #65: two's
// complement nibbles, even k in the low nibble): per row, pad K with zeros to K_pad, multiply
// each group of G columns by H4^(x)k / 2^k, scale = absmax / QM, codes = round-half-even of
// x_rot / scale.
//
// Why a second kernel: the quantisation reads 2 bytes and writes half a byte per element, so it
// should stream at HBM speed, and a launch of it is short (a few microseconds on FLUX-sized
// activations). Register prefetch keeps one row group in flight per thread and caps the warps
// per SM; here the bytes in flight live in shared memory instead:
//  * One persistent CTA per SM owns a contiguous range of rows. Its producer thread issues one
//    cp.async.bulk per row (K * 2 bytes) into the next free slot of an S-deep ring (up to
//    ~200 KB), so at the start of a launch nearly all of a FLUX activation's rows for this SM
//    are requested at once and HBM is busy from the first microsecond.
//  * Compute warps form teams; a team takes TR rows per round (TR * P threads, P = K_pad / 64,
//    TR chosen so the team fills whole warps), one 64-column chunk per thread, exactly the
//    register work of the register-resident kernel (radix-4 butterflies, shuffles or an
//    XOR-swizzled shared exchange for the cross-thread digits, fma rounding, byte-permute
//    packing); the row absmax meets in a warp reduction per row, one shared atomicMax per row
//    and warp, and the team's own named barrier.
//  * A slot is released to the producer right after the team's warps have read it into
//    registers (one mbarrier arrive per warp), so the refill overlaps the transform.
//  * The ring needs no register prefetch, so a CTA runs up to 19 compute warps at <= 96
//    registers.
// Every wait is bounded; the per-round team barrier ORs the threads' "gave up" flags, so a team
// leaves together and no thread waits at a barrier its partners skipped.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "rht_quant.cuh"

namespace convrot {
namespace quant_detail {

constexpr int kRingMaxWarps = 19;            // compute warps per CTA (plus one producer warp)
constexpr int kRingMaxKPad = 16384;
constexpr int kRingMaxSmem = 227 * 1024;

struct RingPlan {
  int P;             // 64-column chunks (threads) per row, ceil(K_pad / 64)
  int TR;            // rows per team round
  int team_warps;    // warps per team (TR * P threads, rounded up to whole warps)
  int teams;         // teams per CTA
  int slots;         // ring depth (row groups of TR rows)
  int pitch;         // bytes per row in a slot: P * 128
  int slot_bytes;    // TR * pitch
  int64_t groups;    // row groups in all: ceil(M / TR)
};

// Bulk copy of `bytes` (a multiple of 16) from global memory into this CTA's shared memory,
// completion counted on `bar` (transaction bytes).
__device__ __forceinline__ void bulk_load_row(void* smem_dst, const void* gsrc, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void st_release_shared(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire_shared(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// Waits (bounded, like mbar_wait) until the producer has claimed ring slot `*seq` for row group
// k. A slot's "full" barrier is waited on by parity, and parity cannot tell phase n from phase
// n + 2: a team that reaches row group k while the slot still holds group k - slots (its copy
// not yet landed, or not yet read) would see the earlier phase's parity and pass. The producer
// publishes k only after group k - slots has been read and released, so once seq == k the
// barrier's current phase is group k's.
__device__ __forceinline__ bool wait_slot_claimed(const int* seq, int k, volatile int* abort) {
  if (ld_acquire_shared(seq) == k) return true;
  // not claimed yet: the producer is still issuing earlier copies; check every ~100 ns without
  // spending issue slots the working teams need
  for (uint32_t i = 0; i < kMaxPolls; ++i) {
    __nanosleep(100);
    if (ld_acquire_shared(seq) == k) return true;
    if (*abort) return false;
  }
  *abort = 1;
  atomicExch(&g_device_status, kStatusTimeout);
  return false;
}

// Bounded mbarrier wait for the teams and the producer. A failed try is followed by a
// nanosleep that doubles from 64 ns up to 512 ns: a team typically waits a few microseconds for
// its first rows, and retrying at once would spend the issue slots the working teams need on
// polling (an early version polled ~15 times per round, over 10 % of all instructions). Gives up
// after ~2^20 tries (> 0.5 s; the status word records the timeout).
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  uint32_t ns = 64;
  for (uint32_t i = 0; i < (1u << 20); ++i) {
    __nanosleep(ns);
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    ns = ns < 512 ? 2 * ns : 512;
  }
  *abort = 1;
  atomicExch(&g_device_status, kStatusTimeout);
  return false;
}

// scale = absmax / QM of the normalised row (absmax_bits: the unnormalised maximum) and the
// multiplier that turns unnormalised values into code units. The quotient is the product with
// the rounded reciprocal c = RN(1 / QM) plus one residual correction (Markstein's method: the
// residual a - q QM is exact in one fma), which rounds correctly or within one ulp; the
// multiplier uses the hardware reciprocal approximation (within one ulp), and rows whose scale is
// not a normal float take the correctly rounded reciprocal.
template <int G, int QM>
__device__ __forceinline__ void row_scale_fast(unsigned int amax_bits, float& scale, float& inv) {
  constexpr float kNorm = 1.0f / static_cast<float>(1 << log4_of<G>());
  constexpr float kRcpQ = 1.0f / static_cast<float>(QM);
  const float a = __uint_as_float(amax_bits) * kNorm;
  const float q0 = a * kRcpQ;
  const float r = __fmaf_rn(-q0, static_cast<float>(QM), a);
  scale = __fmaf_rn(r, kRcpQ, q0);
  if (scale >= 1.17549435e-38f)
    inv = rcp_approx(scale) * kNorm;
  else
    inv = (scale > 0.f) ? __frcp_rn(scale) * kNorm : 0.f;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max |v| over the chunk with three-input maxima (a tree of 32 instead of 63 two-input ones)
__device__ __forceinline__ float chunk_absmax3(const float (&v)[kChunk]) {
  float m[22];
#pragma unroll
  for (int j = 0; j < 21; ++j) m[j] = fmax3(fabsf(v[3 * j]), fabsf(v[3 * j + 1]), fabsf(v[3 * j + 2]));
  m[21] = fabsf(v[63]);
  float n[8];
#pragma unroll
  for (int j = 0; j < 7; ++j) n[j] = fmax3(m[3 * j], m[3 * j + 1], m[3 * j + 2]);
  n[7] = m[21];
  return fmax3(fmax3(n[0], n[1], n[2]), fmax3(n[3], n[4], n[5]), fmaxf(n[6], n[7]));
}

// Barrier over `count` threads (named barrier `id`) that returns the OR of every thread's `pred`.
__device__ __forceinline__ bool team_barrier_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// The 64 bf16 of one chunk from shared memory, for G <= 256 in the slot layout of the register
// kernel (register slot s holds the 16-column block s ^ j; j = team thread index mod 4), for
// G = 1024 in natural order with the 16-byte units permuted by perm (register unit i holds unit
// i ^ perm). Both keep a quarter-warp's loads on at most two threads per bank group.
template <int G>
__device__ __forceinline__ void lds_chunk(const unsigned char* __restrict__ src, int j, int perm,
                                          float (&v)[kChunk]) {
#pragma unroll
  for (int s = 0; s < 4; ++s)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int unit = (G == 1024) ? ((2 * s + h) ^ perm) : (2 * (s ^ j) + h);
      const uint4 u = *reinterpret_cast<const uint4*>(src + (unit << 4));
      float* d = v + 16 * s + 8 * h;
      bf16x2_to_f32(u.x, d[0], d[1]);
      bf16x2_to_f32(u.y, d[2], d[3]);
      bf16x2_to_f32(u.z, d[4], d[5]);
      bf16x2_to_f32(u.w, d[6], d[7]);
    }
}

// Shared-memory 16-byte loads and stores at explicit shared-window addresses. The ring and the
// exchange rows are laid out so that every address a thread needs is a per-round (or
// per-kernel) base XOR a compile-time constant, one logic instruction per access.
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(a)
               : "memory");
  return r;
}

__device__ __forceinline__ float4 lds128f(uint32_t a) {
  float4 r;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "r"(a)
               : "memory");
  return r;
}

__device__ __forceinline__ void sts128f(uint32_t a, float x, float y, float z, float w) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(x), "f"(y), "f"(z),
               "f"(w)
               : "memory");
}

// lds_chunk with the chunk at shared address src (128-byte aligned, so the unit index sits in
// address bits 4..6 and the permutations are XORs of the address).
template <int G>
__device__ __forceinline__ void lds_chunk_sa(uint32_t src, int j, int perm, float (&v)[kChunk]) {
  const uint32_t base = (G == 1024) ? (src | (static_cast<uint32_t>(perm) << 4))
                                    : (src | (static_cast<uint32_t>(j) << 5));
#pragma unroll
  for (int s = 0; s < 4; ++s)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      // G = 1024: unit (2 s + h) ^ perm; G <= 256: unit 2 (s ^ j) + h
      const uint32_t a = (G == 1024) ? (base ^ static_cast<uint32_t>((2 * s + h) << 4))
                                     : ((base ^ static_cast<uint32_t>(s << 5)) + 16 * h);
      const uint4 u = lds128(a);
      float* d = v + 16 * s + 8 * h;
      bf16x2_to_f32(u.x, d[0], d[1]);
      bf16x2_to_f32(u.y, d[2], d[3]);
      bf16x2_to_f32(u.z, d[4], d[5]);
      bf16x2_to_f32(u.w, d[6], d[7]);
    }
}

// transform_chunk<1024> with the exchange rows at shared address xb (this team's rows, 256-byte
// aligned; thread tt owns the 256 bytes at xb + 256 tt). Same arithmetic and layouts.
__device__ __forceinline__ void transform_chunk_1024_sa(float (&v)[kChunk], uint32_t xb, int tt,
                                                        int perm) {
  radix4_stage<1>(v);
  radix4_stage<4>(v);
  radix4_stage<16>(v);
  // row tt, 16-byte piece ch ^ perm ^ (tt & 7): base | (wx << 4), XOR (ch << 4)
  const uint32_t wbase = (xb + 256u * static_cast<uint32_t>(tt)) |
                         (static_cast<uint32_t>(perm ^ (tt & 7)) << 4);
#pragma unroll
  for (int ch = 0; ch < 16; ++ch)
    sts128f(wbase ^ static_cast<uint32_t>(ch << 4), v[4 * ch], v[4 * ch + 1], v[4 * ch + 2],
            v[4 * ch + 3]);
  __syncwarp();
  // thread j takes piece j of rows t0 + a (a = 0..15) at piece position j ^ (a & 7)
  const int j = tt & 15;
  const uint32_t rbase = xb + 256u * static_cast<uint32_t>(tt & ~15) + (static_cast<uint32_t>(j) << 4);
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const uint32_t ra = rbase ^ static_cast<uint32_t>(a << 4);
    const float4 w0 = lds128f(ra + 256u * a);
    const float4 w1 = lds128f(ra + 256u * (a + 8));
    v[a * 4 + 0] = w0.x;
    v[a * 4 + 1] = w0.y;
    v[a * 4 + 2] = w0.z;
    v[a * 4 + 3] = w0.w;
    v[(a + 8) * 4 + 0] = w1.x;
    v[(a + 8) * 4 + 1] = w1.y;
    v[(a + 8) * 4 + 2] = w1.z;
    v[(a + 8) * 4 + 3] = w1.w;
  }
  radix4_stage<4>(v);   // digit 3 = a bits 0..1
  radix4_stage<16>(v);  // digit 4 = a bits 2..3
}

// Codes of one chunk in the slot layout for G <= 64 (slot s holds columns 64 c + 16 (s ^ j) + e);
// blocks at or past K_pad (ragged last chunk, G = 16) are not stored.
template <int QM>
__device__ __forceinline__ void store_slots_small(const float (&v)[kChunk], float inv,
                                                  uint8_t* __restrict__ qr, int c, int j,
                                                  int K_pad) {
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const float* b = v + 16 * s;
    const int col = 64 * c + 16 * (s ^ j);
    if (col >= K_pad) continue;
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

// QM: 7 (packed int4), 127 (int8) or kQmFp4 (NVFP4, for G = 256 and 1024, whose register
// layouts match the register kernel's, with K_pad = K4). MXFP4 stays on the register kernel,
// which ran it faster (qkv 9.97 against 10.53 us here).
template <int G, int QM>
__global__ void __launch_bounds__(32 * (kRingMaxWarps + 1), 1)
rht_quant_ring_kernel(const uint16_t* __restrict__ X, int64_t M, int K, int64_t ldx, int K_pad,
                      uint8_t* __restrict__ Q, int64_t ldq, float* __restrict__ S, RingPlan pl,
                      Fp4Out fp4) {
  constexpr bool kFp = (QM == kQmFp4);
  static_assert(QM != kQmMx, "MXFP4 runs on the register kernel");
  static_assert(!kFp || G >= 256, "NVFP4: G = 256 or 1024 (slot layouts)");
  extern __shared__ __align__(1024) unsigned char smem_raw_rows[];
  // 1024-byte aligned base (the plan reserves the slack)
  unsigned char* smem_rows = smem_raw_rows + ((1024u - (smem_u32(smem_raw_rows) & 1023u)) & 1023u);
  const int team_threads = pl.team_warps * 32;
  const int ring_bytes = pl.slots * pl.slot_bytes;
  const int xbuf_bytes = (G == 1024) ? pl.teams * team_threads * 256 : 0;
  // exchange rows first (256-byte aligned rows), then the ring (128-byte aligned slots)
  unsigned char* ring = smem_rows + xbuf_bytes;
  unsigned int* amax = reinterpret_cast<unsigned int*>(ring + ring_bytes);
  const int amax_words = pl.teams * 3 * pl.TR;
  uint64_t* full = reinterpret_cast<uint64_t*>(amax + ((amax_words + 1) & ~1));
  uint64_t* empty = full + pl.slots;
  int* seq = reinterpret_cast<int*>(empty + pl.slots);     // row group each slot was claimed for
  volatile int* abort_flag = reinterpret_cast<volatile int*>(seq + pl.slots);

  const int tid = threadIdx.x;
  // this CTA's contiguous range of row groups
  const int64_t g_begin = static_cast<int64_t>(blockIdx.x) * pl.groups / gridDim.x;
  const int64_t g_end = static_cast<int64_t>(blockIdx.x + 1) * pl.groups / gridDim.x;
  const int n_local = static_cast<int>(g_end - g_begin);

  if (tid == 0) {
    for (int s = 0; s < pl.slots; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, pl.team_warps);
      seq[s] = -1;
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < amax_words; i += blockDim.x) amax[i] = 0u;
  // columns K .. P * 64 of every slot row read as zero: the copies never write them
  {
    const int tail_units = (pl.pitch - 2 * K) / 16;
    const int n = pl.slots * pl.TR * tail_units;
    for (int i = tid; i < n; i += blockDim.x) {
      const int r = i / tail_units;
      *reinterpret_cast<uint4*>(ring + r * pl.pitch + 2 * K + (i - r * tail_units) * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __syncthreads();
  grid_dependency_wait();
  launch_dependents();

  if (tid < 32) {
    // ------------------------------------------------------------------ producer
    if (tid == 0) {
      int issued = 0;
      int slot = 0;
      uint32_t phase = 0;
      for (int k = 0; k < n_local; ++k) {
        if (k >= pl.slots && !mbar_wait_backoff(empty + slot, phase ^ 1u, abort_flag)) break;
        const int64_t row0 = (g_begin + k) * pl.TR;
        const int rows = static_cast<int>(M - row0 < pl.TR ? M - row0 : pl.TR);
        unsigned char* dst = ring + slot * pl.slot_bytes;
        st_release_shared(seq + slot, k);
        mbar_arrive_expect_tx(full + slot, static_cast<uint32_t>(rows * 2 * K));
        for (int r = 0; r < rows; ++r)
          bulk_load_row(dst + r * pl.pitch, X + (row0 + r) * ldx, static_cast<uint32_t>(2 * K),
                        full + slot);
        issued = k + 1;
        if (++slot == pl.slots) {
          slot = 0;
          phase ^= 1u;
        }
      }
      // every issued copy lands before the CTA can exit (after an abort the consumers may
      // have left without waiting for them). The waits sleep between tries: this thread shares
      // a scheduler with compute warps for the rest of the launch.
      for (int k = issued > pl.slots ? issued - pl.slots : 0; k < issued; ++k) {
        uint64_t* bar = full + (k % pl.slots);
        const uint32_t parity = static_cast<uint32_t>(k / pl.slots) & 1u;
        for (uint32_t polls = 0; !mbar_try_wait(bar, parity) && polls < (1u << 20); ++polls)
          __nanosleep(512);
      }
    }
    return;
  }

  // ------------------------------------------------------------------ compute teams
  const int team = ((tid >> 5) - 1) / pl.team_warps;
  const int tt = tid - 32 - team * team_threads;          // thread index within the team
  const int r_local = tt / pl.P;
  const int c = tt - r_local * pl.P;
  const bool lane_ok = r_local < pl.TR;
  const int j = tt & 3;                                   // slot layout (G <= 256)
  const int perm = tt & 7;                                // unit permutation (G = 1024)
  unsigned int* am_team = amax + team * 3 * pl.TR;
  const uint32_t xbuf_sa = smem_u32(smem_rows) + 256u * static_cast<uint32_t>(team * team_threads);
  const uint32_t ring_sa = smem_u32(ring);
  const int bar_id = 1 + team;
  const int chunk_off = (lane_ok ? r_local * pl.pitch : 0) + c * 128;
  // the lanes of this warp that hold the same row (a warp holds parts of up to 32 rows): their
  // maximum is combined in registers and one lane per row enters it in shared memory
  const unsigned row_lanes = __match_any_sync(0xffffffffu, lane_ok ? r_local : -1);
  const bool row_leader = (tid & 31) == __ffs(row_lanes) - 1;

  int slot = team % pl.slots;
  uint32_t phase = static_cast<uint32_t>((team / pl.slots) & 1);
  int a3 = 0;                                             // rotating absmax slot
  for (int k = team; k < n_local; k += pl.teams) {
    const bool ok = wait_slot_claimed(seq + slot, k, abort_flag) &&
                    mbar_wait_backoff(full + slot, phase, abort_flag);
    float v[kChunk];
    lds_chunk_sa<G>(ring_sa + static_cast<uint32_t>(slot * pl.slot_bytes + chunk_off), j, perm,
                    v);
    // the slot may be refilled once every warp of the team has read it (generic reads ordered
    // before the asynchronous refill by the proxy fence)
    fence_proxy_async_smem();
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(empty + slot);

    if constexpr (G == 1024)
      transform_chunk_1024_sa(v, xbuf_sa, tt, perm << 1);
    else
      transform_slots<G>(v);
    // NVFP4: the maxima of the four 16-column blocks (G = 1024 first regroups whole blocks per
    // thread through the same exchange rows)
    float bm[4];
    float mx;
    if constexpr (kFp) {
      if constexpr (G == 1024)
        blocks_1024(v, reinterpret_cast<float4*>(smem_rows) + 16 * team * team_threads, tt);
#pragma unroll
      for (int r = 0; r < 4; ++r) bm[r] = absmax16(v + 16 * r);
      mx = fmaxf(fmaxf(bm[0], bm[1]), fmaxf(bm[2], bm[3]));
    } else {
      mx = chunk_absmax(v);
    }
    const unsigned m = __reduce_max_sync(row_lanes, __float_as_uint(mx));
    const int64_t row = (g_begin + k) * pl.TR + r_local;
    const bool active = lane_ok && row < M;
    unsigned int* am = am_team + a3 * pl.TR;
    if (active && row_leader) atomicMax(am + r_local, m);
    // the team meets once per round; a thread whose wait gave up makes the whole team leave
    if (team_barrier_or(bar_id, team_threads, !ok)) break;
    // the absmax slot of the previous round is no longer read by anyone: clear it for reuse
    if (tt < pl.TR) am_team[(a3 == 0 ? 2 : a3 - 1) * pl.TR + tt] = 0u;
    if constexpr (QM == kQmFp4) {
      float gr = 0.f;
      if (active) {
        constexpr float kNorm = 1.0f / static_cast<float>(1 << log4_of<G>());
        gr = __fdiv_rn(__uint_as_float(am[r_local]) * kNorm, 6.0f * 448.0f);
        if (c == 0) S[row] = gr;
      }
      store_fp4<G>(v, bm, gr, Q + (active ? row : 0) * ldq, row, c, j, fp4, active);
    } else if (active) {
      float scale, inv;
      row_scale_fast<G, QM>(am[r_local], scale, inv);
      if (c == 0) S[row] = scale;
      uint8_t* qr = Q + row * ldq;
      if constexpr (G == 1024)
        store_row_codes<G, QM>(v, inv, qr, c, K_pad);
      else if constexpr (G == 256)
        store_slots<G, QM>(v, inv, qr, c, j, K_pad);
      else
        store_slots_small<QM>(v, inv, qr, c, j, K_pad);
    }
    a3 = (a3 == 2) ? 0 : a3 + 1;
    slot += pl.teams;
    while (slot >= pl.slots) {
      slot -= pl.slots;
      phase ^= 1u;
    }
  }
}

// Plan of the ring kernel for one shape, or false when it does not apply (K not a multiple of 8,
// rows longer than kRingMaxKPad, or a ring slot larger than shared memory allows).
template <int G>
inline bool ring_plan(int64_t M, int64_t K, int64_t K_pad, RingPlan& pl, size_t& smem) {
  if (K <= 0 || (K % 8) != 0 || K_pad > kRingMaxKPad || M <= 0) return false;
  const int P = static_cast<int>((K_pad + 63) / 64);
  // rows per round: the fewest whose threads fill their warps to at least 15/16 (else the best
  // fill up to 16 warps)
  int TR = 0, best = 1;
  double best_fill = 0.0;
  for (int tr = 1; tr <= 32; ++tr) {
    const int th = tr * P;
    const int w = (th + 31) / 32;
    if (w > 16) break;
    const double fill = static_cast<double>(th) / (32.0 * w);
    if (fill >= 15.0 / 16.0) {
      TR = tr;
      break;
    }
    if (fill > best_fill) {
      best_fill = fill;
      best = tr;
    }
  }
  if (TR == 0) TR = best;
  pl.P = P;
  pl.TR = TR;
  pl.team_warps = (TR * P + 31) / 32;
  if (pl.team_warps > kRingMaxWarps) return false;
  pl.teams = kRingMaxWarps / pl.team_warps;
  if (pl.teams > 15) pl.teams = 15;                       // named barriers 1..15
  pl.pitch = P * 128;
  pl.slot_bytes = TR * pl.pitch;
  pl.groups = (M + TR - 1) / TR;
  const size_t xbuf = (G == 1024) ? static_cast<size_t>(pl.teams) * pl.team_warps * 32 * 256 : 0;
  const size_t amax = (static_cast<size_t>(pl.teams) * 3 * TR + 1) / 2 * 8;
  const size_t fixed = xbuf + amax + 16 + 1024;          // + alignment slack of the base
  if (fixed + pl.slot_bytes + 20 > static_cast<size_t>(kRingMaxSmem)) return false;
  // per slot: its bytes, two mbarriers and its claim word
  int slots = static_cast<int>((kRingMaxSmem - fixed) / (pl.slot_bytes + 20));
  if (slots > 64) slots = 64;
  pl.slots = slots;
  smem = static_cast<size_t>(slots) * (pl.slot_bytes + 20) + fixed;
  return true;
}

// Returns cudaErrorNotSupported when the shape does not fit the ring kernel.
template <int G, int QM>
cudaError_t launch_ring(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, int64_t K_pad,
                        uint8_t* Q, int64_t ldq, float* S, cudaStream_t stream,
                        Fp4Out fp4) {
  if constexpr (QM == kQmMx || (QM == kQmFp4 && G < 256)) {
    return cudaErrorNotSupported;   // MXFP4 and G <= 64 NVFP4: the register kernel
  } else {
    RingPlan pl;
    size_t smem = 0;
    if (!ring_plan<G>(M, K, K_pad, pl, smem)) return cudaErrorNotSupported;
    auto kern = rht_quant_ring_kernel<G, QM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t sms = sm_count();
    const int64_t grid = pl.groups < sms ? pl.groups : sms;
    const int threads = 32 * (1 + pl.teams * pl.team_warps);
    return launch_overlapped(kern, dim3(static_cast<unsigned>(grid)), dim3(threads), smem,
                             stream, X, M, static_cast<int>(K), ldx, static_cast<int>(K_pad), Q,
                             ldq, S, pl, fp4);
  }
}

}  // namespace quant_detail
}  // namespace convrot
