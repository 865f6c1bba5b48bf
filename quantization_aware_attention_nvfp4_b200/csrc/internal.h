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
};

struct BwdArgs {
  int Lq, Lk, nq_tiles, nk_tiles;
  float sm_scale;
  float scale_log2;
  // stats[0] = max_i |dO_i|_1, stats[1] = max_i |Delta_i|, stats[2] = max |fq(V)|:
  // they bound |dS| and fix the power-of-two scale of the f16 dS operand;
  // stats[3] = max |dO| fixes the scale of the fp16 copy of dO.
  const float *stats;
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
};

// Forward.  tv: 3-D TMA map {D, L, B*H} with 64 x 128 boxes, 128-byte swizzle
// over fq(V) (pv_mode 1: fp16, 0: bf16); with pv_mode 2 (every quantizer on,
// Lk % 32 == 0) it maps fq(V)'s packed codes {Lk/2 bytes, D, B*H} with
// 64-byte x D boxes and 64-byte swizzle, a.vsf their scale tiles, and P V is
// a block-scaled NVFP4 MMA.  With qk_f16 (Q and K quantized) tq/tk map the
// packed NVFP4 codes {D/2 bytes, L, B*H} with (D/2) x 128 boxes and a
// D/2-byte swizzle, a.qsf/a.ksf point at their scale-factor tiles, and S runs
// as a block-scaled NVFP4 MMA; otherwise tq/tk map the bf16 Q and K.
cudaError_t launch_fwd(int D, bool qk_f16, int pv_mode, bool quant_p, const CUtensorMap &tq,
                       const CUtensorMap &tk, const CUtensorMap &tv, const FwdArgs &a, int BH,
                       cudaStream_t stream);

cudaError_t launch_bwd_dkdv(int D, bool qk_f16, bool quant_p, bool do_f16, const CUtensorMap &tq,
                            const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tdo,
                            const CUtensorMap &tq4, const BwdArgs &a, int BH, cudaStream_t stream);
// dQ.  With qk_f16, tq maps the packed NVFP4 Q codes (as for the forward),
// tk4 the K codes, a.qsf/a.ksf their scale tiles, and tk the fp16 fq(K) that
// dQ = dS fq(K) reads; otherwise tq/tk are bf16 and tk4 is unused.
cudaError_t launch_bwd_dq(int D, bool qk_f16, bool do_f16, const CUtensorMap &tq, const CUtensorMap &tk,
                          const CUtensorMap &tv, const CUtensorMap &tdo, const CUtensorMap &tk4,
                          const BwdArgs &a, int BH, cudaStream_t stream);

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

// out = fp16(dO * 2^e) over n elements (n % 8 == 0), 2^e = do_scale(stats).
cudaError_t launch_scale_do(const __nv_bfloat16 *dO, uint16_t *out, int64_t n, const float *stats,
                            cudaStream_t stream);

// Block-sparse tile lists from a tile mask [BH][nq][nk] (nonzero = the
// query tile attends the key tile): kv_list/kv_count per query tile and
// q_list/q_count per key tile, ascending (see sparse.cu).
cudaError_t launch_sparse_plan(const uint8_t *mask, int BH, int nq, int nk, int32_t *kv_list, int32_t *kv_count,
                               int32_t *q_list, int32_t *q_count, cudaStream_t stream);

// The same lists for causal masking with nt query and key tiles: key tiles
// 0..I for query tile I, query tiles J..nt-1 for key tile J.
cudaError_t launch_causal_plan(int BH, int nt, int32_t *kv_list, int32_t *kv_count, int32_t *q_list,
                               int32_t *q_count, cudaStream_t stream);

// VSA key-tile selection (see sparse.cu): tile means of q and k into
// `means` [BH][nq + nk][D], coarse scores into `scores` [BH][nq][nk], and the
// tile mask [BH][nq][nk] keeping the topk best key tiles per query tile.
cudaError_t launch_vsa_select(const __nv_bfloat16 *q, const __nv_bfloat16 *k, int BH, int Lq, int Lk, int D,
                              int topk, float *means, float *scores, uint8_t *mask, cudaStream_t stream);

// max |x| over n bf16 values folded into *out (must start at 0).
cudaError_t launch_absmax(const __nv_bfloat16 *x, int64_t n, float *out, cudaStream_t stream);

// Sets cudaFuncAttributeMaxDynamicSharedMemorySize for `kernel` once per
// device (thread-safe).
cudaError_t ensure_smem_attr(const void *kernel, int bytes);

}  // namespace attnqat
