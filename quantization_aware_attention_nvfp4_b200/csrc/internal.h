// internal.h -- host-side interfaces between the C-ABI layer and the kernel
// translation units.  Not installed; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace attnqat {

struct FwdArgs {
  int Lq, Lk, nq_tiles, nk_tiles;
  float sm_scale;     // c
  float scale_log2;   // c * log2(e)
  const uint8_t *qsf;   // scale-factor tiles of fq(Q), fq(K) (NVFP4 S path)
  const uint8_t *ksf;
  const uint8_t *vsf;   // scale-factor tiles of fq(V) along tokens (NVFP4 P V path)
  // Every 16-bit operand of the MMAs is fp16: fq(X) unscaled (exact), or, for
  // an operand whose quantizer is off, X * 2^e with 2^e = pow2_scale(*amax_x).
  // amax_x points at that max magnitude, or is null for a quantized operand.
  const float *amax_q;
  const float *amax_k;
  const float *amax_v;
  __nv_bfloat16 *o;
  float *o32;   // float32 copy of O kept in the workspace for the backward's Delta
  float *lse;
  float *m;
  // block-sparse: key tiles of each query tile ([B*H][nq_tiles] rows of
  // stride nk_tiles, ascending) and their counts; null for dense attention
  const int32_t *kv_list;
  const int32_t *kv_count;
  // causal masking (Lq == Lk): the lists are the lower triangle of tiles and
  // each list's diagonal tile keeps keys <= the query row
  int causal;
  // 64-token block-sparse masks: list entries carry their quadrant bits
  int quad;
};

struct BwdArgs {
  int Lq, Lk, nq_tiles, nk_tiles;
  float sm_scale;
  float scale_log2;
  // stats[0] = max_i |dO_i|_1, stats[1] = max_i |Delta_i|, stats[2] = max |fq(V)|:
  // they bound |dS| and fix the power-of-two scale of the f16 dS operand;
  // stats[3] = max |dO| fixes the scale of the fp16 copy of dO.
  const float *stats;
  const float *amax_q;   // as FwdArgs: the scales of the fp16 operand copies
  const float *amax_k;
  const float *amax_v;
  const float *m;
  const float *lse;
  const float *delta;
  const uint8_t *qsf;   // scale-factor tiles of fq(Q), fq(K) (NVFP4 S in the dQ kernel)
  const uint8_t *ksf;
  __nv_bfloat16 *dq;
  __nv_bfloat16 *dk;
  __nv_bfloat16 *dv;
  // block-sparse (null for dense): key tiles per query tile (dQ kernel) and
  // query tiles per key tile ([B*H][nk_tiles] rows of stride nq_tiles, for
  // the dK/dV kernel), ascending, with their counts
  const int32_t *kv_list;
  const int32_t *kv_count;
  const int32_t *q_list;
  const int32_t *q_count;
  int causal;  // as FwdArgs::causal
  int quad;    // as FwdArgs::quad
};

// Forward.  Every 16-bit operand is fp16 (see FwdArgs::amax_q).  With fp4s
// (Q and K quantized) tq/tk map the packed NVFP4 codes {D/2 bytes, L, B*H}
// with (D/2) x 128 boxes and a D/2-byte swizzle, a.qsf/a.ksf point at their
// scale-factor tiles, and S runs as a block-scaled NVFP4 MMA; otherwise tq/tk
// map the fp16 copies of Q and K {D, L, B*H} with 64 x 128 boxes and 128-byte
// swizzle.  With pv4 (every quantizer on, Lk % 32 == 0) tv maps
// fq(V)'s packed codes {Lk/2 bytes, D, B*H} with 64-byte x D boxes and 64-byte
// swizzle, a.vsf their scale tiles, and P V is a block-scaled NVFP4 MMA;
// otherwise tv maps the fp16 copy of V (64 x 128 boxes, 128-byte swizzle) and
// P V is an fp16 MMA.
cudaError_t launch_fwd(int D, bool fp4s, bool pv4, bool quant_p, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const FwdArgs &a, int BH, cudaStream_t stream);

// dK/dV.  tq, tk, tv, tdo map the fp16 copies of Q, K, V and dO (64 x 128
// boxes, 128-byte swizzle); with fp4s tk maps K's packed NVFP4 codes instead
// and tq4 Q's codes (as for the forward), and S is block-scaled NVFP4.
cudaError_t launch_bwd_dkdv(int D, bool fp4s, bool quant_p, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, const CUtensorMap &tdo, const CUtensorMap &tq4,
                            const BwdArgs &a, int BH, cudaStream_t stream);
// dQ.  With fp4s, tq maps the packed NVFP4 Q codes (as for the forward), tk4
// the K codes, a.qsf/a.ksf their scale tiles, and tk the fp16 fq(K) that
// dQ = dS fq(K) reads; otherwise tq/tk map the fp16 copies and tk4 is unused.
// dsplit feeds dS as an fp16 hi + lo pair (always so without fp4s).
cudaError_t launch_bwd_dq(int D, bool fp4s, bool dsplit, const CUtensorMap &tq, const CUtensorMap &tk,
                          const CUtensorMap &tv, const CUtensorMap &tdo, const CUtensorMap &tk4, const BwdArgs &a,
                          int BH, cudaStream_t stream);

// NVFP4 fq of a strided bf16 view (see attnqat_quantize; cols need not be a
// multiple of 16 here: a ragged last block reads zeros); any of codes,
// scales, deq (bf16, same strides as x), deq_f16 and absmax (max |fq(x)|,
// folded in with an atomic max; must start at 0) may be null.  With
// sf_tile_rows = L > 0 (contiguous [heads*L, cols] rows), the scales go to
// the per-head, per-128-row-tile layout the block-scaled MMA reads from TMEM
// (padding rows of the last tile are not written); with sf_col_tiles (rows
// <= 128, e.g. V's D channels blocked along tokens) to the per-batch,
// per-128-column-tile layout of the same kind.
cudaError_t launch_quantize(const uint16_t *x, int64_t batch, int64_t rows, int64_t cols,
                            int64_t sb, int64_t sr, int64_t sc, uint8_t *codes, uint8_t *scales,
                            uint16_t *deq, uint16_t *deq_f16, float *absmax, cudaStream_t stream,
                            int64_t sf_tile_rows = 0, bool sf_col_tiles = false);

// NVFP4 with an FP32 global scale (see attnqat_quantize_gs): codes and
// scales as launch_quantize, deq (bf16 bits, may be null), and *gscale
// (also the scratch of the max-magnitude reduction).
cudaError_t launch_quantize_gs(const uint16_t *x, int64_t batch, int64_t rows, int64_t cols, int64_t sb,
                               int64_t sr, int64_t sc, uint8_t *codes, uint8_t *scales, uint16_t *deq,
                               float *gscale, cudaStream_t stream);

// delta[r] = sum_d dO[r][d] * O[r][d] over `rows` rows of D values (O float32,
// dO bf16); folds max_r |dO_r|_1 into stats[0], max_r |delta_r| into
// stats[1] and max |dO| into stats[3] (all must start at 0).
cudaError_t launch_delta(const float *o32, const __nv_bfloat16 *dO, float *delta, int64_t rows, int D,
                         float *stats, cudaStream_t stream);

// out = fp16(x * 2^e) over n bf16 elements (n % 8 == 0), 2^e =
// pow2_scale(*amax) (max |x| lands in [2^13, 2^14)).
cudaError_t launch_scale_f16(const __nv_bfloat16 *x, uint16_t *out, int64_t n, const float *amax,
                             cudaStream_t stream);

// Block-sparse tile lists from a tile mask [BH][nq][nk] (nonzero = the
// query tile attends the key tile): kv_list/kv_count per query tile and
// q_list/q_count per key tile, ascending (see sparse.cu).
cudaError_t launch_sparse_plan(const uint8_t *mask, int BH, int nq, int nk, int32_t *kv_list, int32_t *kv_count,
                               int32_t *q_list, int32_t *q_count, cudaStream_t stream);

// The same lists from a 64-token mask [BH][nq64][nk64] for the nq x nk
// 128-token tiles: entries tile | bits << 24, bit (qh * 2 + kh) set when the
// quadrant (query half qh, key half kh) is selected; tiles with no selected
// quadrant are left out.
cudaError_t launch_sparse64_plan(const uint8_t *mask, int BH, int nq64, int nk64, int nq, int nk, int32_t *kv_list,
                                 int32_t *kv_count, int32_t *q_list, int32_t *q_count, cudaStream_t stream);

// The same lists for causal masking with nt query and key tiles: key tiles
// 0..I for query tile I, query tiles J..nt-1 for key tile J.
cudaError_t launch_causal_plan(int BH, int nt, int32_t *kv_list, int32_t *kv_count, int32_t *q_list,
                               int32_t *q_count, cudaStream_t stream);

// VSA key-tile selection over T-token tiles (see sparse.cu): tile means into
// `means` (per head nq + nk rows of D floats: q's [nq][D], then k's stored
// transposed, [D][nk]), coarse scores into `scores`
// [BH][nq][nk], and the tile mask [BH][nq][nk] keeping the topk best key
// tiles per query tile (nq = ceil(Lq / T), nk = ceil(Lk / T)).
cudaError_t launch_vsa_select(const __nv_bfloat16 *q, const __nv_bfloat16 *k, int BH, int Lq, int Lk, int D, int T,
                              int topk, float *means, float *scores, uint8_t *mask, cudaStream_t stream);

// max |x| over n bf16 values folded into *out (must start at 0).
cudaError_t launch_absmax(const __nv_bfloat16 *x, int64_t n, float *out, cudaStream_t stream);

// Sets cudaFuncAttributeMaxDynamicSharedMemorySize for `kernel` once per
// device (thread-safe).
cudaError_t ensure_smem_attr(const void *kernel, int bytes);

}  // namespace attnqat
