// common.cuh -- tile geometry, the in-register NVFP4 fake quantization of
// probability blocks, and small GEMM-issue helpers shared by the forward and
// backward attention kernels.
#pragma once

#include "device.cuh"

namespace attnqat {

constexpr int kBM = 128;                  // query rows per tile (TMEM lanes)
constexpr int kSoftWarps = 8;             // row warps: 2 per TMEM lane quarter, each owns 64 columns
// Warp roles: 0 TMA producer, 1 and kMmaB2 the two MMA-issuing threads (one
// thread issues a tcgen05.mma about every 58 cycles, barely faster than the
// tensor pipe retires a 128x128x16 f16 MMA, so its waits and commits would
// idle the pipe; two issuers split the MMA streams), 2..9 row warps, 11 idle
// (12 warps: the register budget per thread is that of 384 threads anyway).
constexpr int kMmaB2 = 2 + kSoftWarps;
constexpr int kThreads = 384;
constexpr int kBN = 128;                  // keys per tile
constexpr int kChunkBytes = 128 * 128;    // one 128-row x 128-byte swizzled chunk
constexpr float kLog2e = 1.4426950408889634f;

// Bytes of a 128-row x D tile of 16-bit elements (D/64 swizzled chunks).
template <int D>
struct Tile {
  static constexpr int kBytes = 128 * D * 2;
  static constexpr int kChunks = D / 64;
};

// fq of one block of 16 non-negative probabilities held in registers (one
// query row, 16 consecutive keys): s = E4M3(amax/6), each element rounded to
// the E2M1 grid of p/s (round to nearest even, saturating at 6).  Returns the
// 8 f16x2 words of r (the grid values, sign-free) and the block scale s as a
// float.  With s == 0 every r is 0.
//
// amax/6 is formed as amax * (1/6) and p/s as p * rcp.approx(s): for probabilities
// (exp of a float) exact ties have measure zero, so this selects the same
// codes as the exact quotients except within one float ulp of a rounding
// boundary.  Forward and backward use this same routine on the same bits, so
// they agree bit for bit.
__device__ __forceinline__ float fq16_probs(const float *p, uint32_t (&r)[8]) {
  const float amax = fmax3(fmax3(fmax3(p[0], p[1], p[2]), fmax3(p[3], p[4], p[5]), fmax3(p[6], p[7], p[8])),
                          fmax3(p[9], p[10], p[11]), fmax3(p[12], p[13], fmaxf(p[14], p[15])));
  const uint16_t code = cvt_e4m3x2(amax * (1.0f / 6.0f), 0.0f);
  const float s = unpack_f16x2(cvt_f16x2_from_e4m3x2(code)).x;
  const float inv = s > 0.0f ? rcp_approx(s) : 0.0f;
  const float2 inv2 = make_float2(inv, inv);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 x = mul2(make_float2(p[2 * i], p[2 * i + 1]), inv2);
    r[i] = e2m1_round_f16x2(x.x, x.y);
  }
  return s;
}

// The same fq of 16 probabilities as fq16_probs, step for step (same amax,
// same E4M3 scale, same p * rcp(s), same E2M1 rounding), returning the packed
// E2M1 codes (c[0]: elements 0..7, c[1]: 8..15) and the E4M3 scale byte:
// the operand of the block-scaled NVFP4 P V product.
__device__ __forceinline__ uint32_t fq4_probs(const float *p, uint32_t (&c)[2]) {
  const float amax = fmax3(fmax3(fmax3(p[0], p[1], p[2]), fmax3(p[3], p[4], p[5]), fmax3(p[6], p[7], p[8])),
                          fmax3(p[9], p[10], p[11]), fmax3(p[12], p[13], fmaxf(p[14], p[15])));
  const uint16_t code = cvt_e4m3x2(amax * (1.0f / 6.0f), 0.0f);
  const float s = unpack_f16x2(cvt_f16x2_from_e4m3x2(code)).x;
  const float inv = s > 0.0f ? rcp_approx(s) : 0.0f;
  const float2 inv2 = make_float2(inv, inv);
  float2 x[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = mul2(make_float2(p[2 * i], p[2 * i + 1]), inv2);
  c[0] = e2m1x8(x[0], x[1], x[2], x[3]);
  c[1] = e2m1x8(x[4], x[5], x[6], x[7]);
  return code & 0xFFu;
}

// f16x2 word with the f16 value of s (an E4M3 value, exact in f16) in both
// halves.
__device__ __forceinline__ uint32_t f16x2_broadcast(float s) {
  const uint32_t h = __half_as_ushort(__float2half_rn(s));
  return h | (h << 16);
}

// Power of two 2^e that maps a tensor's max magnitude `mx` into [2^13, 2^14):
// the scale of an fp16 copy of a bf16 tensor (dO, and Q, K or V when that
// operand is not quantized); 1 when mx is 0.  A bf16 value has 8 significant
// bits, so the copy is exact for every element within 2^27 of the largest,
// and an element below that moves by at most 2^-25 of the largest.
__device__ __forceinline__ float pow2_scale(float mx) {
  if (!(mx > 0.0f)) return 1.0f;
  int e = 13 - (static_cast<int>((__float_as_uint(mx) >> 23) & 0xFF) - 127);
  e = e < -120 ? -120 : (e > 120 ? 120 : e);
  return __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}

// Scale of the fp16 copy of dO (max |dO| is stats[3]).
__device__ __forceinline__ float do_scale(const float *stats) { return pow2_scale(stats[3]); }

// Scale of an operand's fp16 copy: pow2_scale of the max magnitude `amax`
// points at, or 1 for a quantized operand (null), whose fq values are exact
// in fp16 unscaled.
__device__ __forceinline__ float operand_scale(const float *amax) { return amax ? pow2_scale(*amax) : 1.0f; }

// The MMA helpers below take the descriptors of the operand tiles' base
// addresses and advance them by adding (byte offset >> 4) to the 14-bit
// address field (tiles sit below 256 KB of shared memory, so the field never
// carries): the issuing thread does no address arithmetic per instruction.
__device__ __forceinline__ uint64_t sdesc_add(uint64_t d, uint32_t byte_off) {
  return d + static_cast<uint64_t>(byte_off >> 4);
}

// Descriptors of 128-byte-swizzled 16-bit tiles: K-major, and MN-major with
// 64-element chunks kChunkBytes apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) { return sdesc_sw128(saddr, 16, 1024); }
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr) { return sdesc_sw128(saddr, kChunkBytes, 1024); }

// Issues D[tmem] (+)= A * B^T for two K-major 128-row tiles (128-byte swizzle,
// chunks of 64 K-elements kChunkBytes apart) over KSTEPS slices of K = 16.
// adesc/bdesc: sdesc_sw128(base, 16, 1024) of the two tiles.
template <int KSTEPS>
__device__ __forceinline__ void mma_kmajor(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk) {
    const uint32_t off = static_cast<uint32_t>(kk >> 2) * kChunkBytes + static_cast<uint32_t>(kk & 3) * 32u;
    umma_ss(d_tmem, sdesc_add(adesc, off), sdesc_add(bdesc, off), idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Issues D[tmem] (+)= A * B where A is a K-major 128-row tile and B an
// MN-major tile (K rows of 128 bytes, N in chunks of 64 elements kChunkBytes
// apart), K = 16 * KSTEPS.  adesc: sdesc_sw128(a, 16, 1024); bdesc:
// sdesc_sw128(b, kChunkBytes, 1024).
template <int KSTEPS>
__device__ __forceinline__ void mma_a_k_b_mn(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk) {
    const uint32_t aoff = static_cast<uint32_t>(kk >> 2) * kChunkBytes + static_cast<uint32_t>(kk & 3) * 32u;
    umma_ss(d_tmem, sdesc_add(adesc, aoff), sdesc_add(bdesc, static_cast<uint32_t>(kk) * 2048u), idesc,
            (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Issues D[tmem] (+)= A * B where both are MN-major tiles (K rows of 128
// bytes; M and N in chunks of 64 elements kChunkBytes apart).  Descriptors:
// sdesc_sw128(base, kChunkBytes, 1024).
template <int KSTEPS>
__device__ __forceinline__ void mma_mn_mn(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk) {
    const uint32_t off = static_cast<uint32_t>(kk) * 2048u;
    umma_ss(d_tmem, sdesc_add(adesc, off), sdesc_add(bdesc, off), idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Writes 64 16-bit values (32 packed words) as columns [64*half, 64*half+64)
// of row `row` of a 128 x 128 swizzled tile at `base` (exactly one chunk).
__device__ __forceinline__ void store_row_half(uint32_t base, uint32_t row, int half, const uint32_t *w) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const uint32_t addr = base + static_cast<uint32_t>(half) * kChunkBytes + sw128_offset(row, u);
    st_shared_v4(addr, w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
  }
}

// Writes NC 16-bit values (NC/2 packed words) as columns [col0, col0 + NC)
// of row `row` of a 128 x 128 swizzled tile at `base` (NC = 32 or 64, col0 a
// multiple of NC: within one 64-column chunk).
template <int NC>
__device__ __forceinline__ void store_row_cols(uint32_t base, uint32_t row, int col0, const uint32_t *w) {
#pragma unroll
  for (int u = 0; u < NC / 8; ++u) {
    const uint32_t addr = base + static_cast<uint32_t>(col0 >> 6) * kChunkBytes +
                          sw128_offset(row, static_cast<uint32_t>((col0 & 63) >> 3) + u);
    st_shared_v4(addr, w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
  }
}

// Role of a row warp (warps 2 .. 2 + 4 G - 1 with G row warps per TMEM lane
// quarter): the lane quarter it may access (warp id mod 4), its row in the
// 128-row tile and which of the G column groups of a 128-column tile it owns
// (`half`: 0 or 1 when G = 2).
struct RowRole {
  int wq;           // lane quarter
  uint32_t row;     // 0..127
  int half;         // 0 or 1
  uint32_t lane_addr;
  __device__ __forceinline__ RowRole(int warp, int lane) {
    wq = warp & 3;
    row = static_cast<uint32_t>(wq * 32 + lane);
    half = (warp - 2) >> 2;
    lane_addr = static_cast<uint32_t>(wq * 32) << 16;
  }
};

// Advances a dynamic shared-memory pointer to the next 1024-byte boundary of
// the shared window (the swizzle atoms and UMMA descriptors need it).
__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  const uint32_t pad = (1024u - (smem_u32(p) & 1023u)) & 1023u;
  return p + pad;
}

}  // namespace attnqat
