// sparse.cu -- tile lists for block-sparse (VSA) fine attention.
//
// The caller selects, per (batch*head, 128-query tile), the 128-key tiles the
// tile attends to: a byte mask [B*H][nq][nk], nonzero = selected (the
// VSA_QAT_TRAIN_C128 backend of the vsqa-test-1.3b metadata attends each
// 128-token query cube to its top-k key cubes).  The attention kernels walk
// lists instead of a mask:
//   kv_list[bh][I][0..kv_count[bh][I])  ascending key tiles of query tile I
//                                        (forward and dQ kernels),
//   q_list[bh][J][0..q_count[bh][J])    ascending query tiles that selected
//                                        key tile J (dK/dV kernel),
// each row with stride nk (resp. nq).  One warp builds one list: it reads 32
// mask bytes per step and compacts the selected indices with a ballot, so the
// order is ascending and the build is deterministic.
#include "common.cuh"
#include "internal.h"

namespace attnqat {

__global__ void __launch_bounds__(256) sparse_plan_kernel(const uint8_t *__restrict__ mask, int BH, int nq, int nk,
                                                          int32_t *__restrict__ kv_list,
                                                          int32_t *__restrict__ kv_count,
                                                          int32_t *__restrict__ q_list,
                                                          int32_t *__restrict__ q_count) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(BH) * nq;
  if (w < rows) {
    // query tile I of head bh: scan its mask row
    const uint8_t *src = mask + w * nk;
    int32_t *dst = kv_list + w * nk;
    int cnt = 0;
    for (int j0 = 0; j0 < nk; j0 += 32) {
      const int j = j0 + lane;
      const bool sel = j < nk && src[j] != 0;
      const unsigned b = __ballot_sync(0xffffffffu, sel);
      if (sel) dst[cnt + __popc(b & ((1u << lane) - 1u))] = j;
      cnt += __popc(b);
    }
    if (lane == 0) kv_count[w] = cnt;
  } else if (w < rows + static_cast<int64_t>(BH) * nk) {
    // key tile J of head bh: scan its mask column
    const int64_t c = w - rows;
    const int64_t bh = c / nk;
    const int J = static_cast<int>(c - bh * nk);
    const uint8_t *src = mask + bh * nq * nk + J;
    int32_t *dst = q_list + c * nq;
    int cnt = 0;
    for (int i0 = 0; i0 < nq; i0 += 32) {
      const int i = i0 + lane;
      const bool sel = i < nq && src[static_cast<int64_t>(i) * nk] != 0;
      const unsigned b = __ballot_sync(0xffffffffu, sel);
      if (sel) dst[cnt + __popc(b & ((1u << lane) - 1u))] = i;
      cnt += __popc(b);
    }
    if (lane == 0) q_count[c] = cnt;
  }
}

cudaError_t launch_sparse_plan(const uint8_t *mask, int BH, int nq, int nk, int32_t *kv_list, int32_t *kv_count,
                               int32_t *q_list, int32_t *q_count, cudaStream_t stream) {
  const int64_t warps = static_cast<int64_t>(BH) * (nq + nk);
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  sparse_plan_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(mask, BH, nq, nk, kv_list, kv_count, q_list,
                                                                        q_count);
  return cudaGetLastError();
}

// 64-token block-sparse attention runs on the same 128 x 128 kernel tiles:
// the caller's mask has 64-token granularity [B*H][nq64][nk64], and a 128-
// token tile pair is listed when any of its four 64 x 64 quadrants is
// selected.  Each list entry carries those quadrants in its top byte,
// tile | bits << 24 with bit (qh * 2 + kh) for query half qh and key half kh,
// and the kernels mask the unselected quadrants (each row-warp thread owns
// one 64-key half of one query row, so a quadrant is whole threads).
__device__ __forceinline__ uint32_t quadrant_bits(const uint8_t *m, int nq64, int nk64, int I, int J) {
  uint32_t bits = 0;
#pragma unroll
  for (int qh = 0; qh < 2; ++qh) {
    const int i = 2 * I + qh;
    if (i >= nq64) break;
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      const int j = 2 * J + kh;
      if (j < nk64 && m[static_cast<int64_t>(i) * nk64 + j] != 0) bits |= 1u << (qh * 2 + kh);
    }
  }
  return bits;
}

__global__ void __launch_bounds__(256) sparse64_plan_kernel(const uint8_t *__restrict__ mask, int BH, int nq64,
                                                            int nk64, int nq, int nk, int32_t *__restrict__ kv_list,
                                                            int32_t *__restrict__ kv_count,
                                                            int32_t *__restrict__ q_list,
                                                            int32_t *__restrict__ q_count) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(BH) * nq;
  if (w < rows) {
    // query tile I of head bh: its key tiles with their quadrants
    const int64_t bh = w / nq;
    const int I = static_cast<int>(w - bh * nq);
    const uint8_t *m = mask + bh * nq64 * nk64;
    int32_t *dst = kv_list + w * nk;
    int cnt = 0;
    for (int j0 = 0; j0 < nk; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t bits = j < nk ? quadrant_bits(m, nq64, nk64, I, j) : 0u;
      const unsigned b = __ballot_sync(0xffffffffu, bits != 0);
      if (bits) dst[cnt + __popc(b & ((1u << lane) - 1u))] = static_cast<int32_t>(static_cast<uint32_t>(j) | (bits << 24));
      cnt += __popc(b);
    }
    if (lane == 0) kv_count[w] = cnt;
  } else if (w < rows + static_cast<int64_t>(BH) * nk) {
    // key tile J of head bh: the query tiles that selected part of it
    const int64_t c = w - rows;
    const int64_t bh = c / nk;
    const int J = static_cast<int>(c - bh * nk);
    const uint8_t *m = mask + bh * nq64 * nk64;
    int32_t *dst = q_list + c * nq;
    int cnt = 0;
    for (int i0 = 0; i0 < nq; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t bits = i < nq ? quadrant_bits(m, nq64, nk64, i, J) : 0u;
      const unsigned b = __ballot_sync(0xffffffffu, bits != 0);
      if (bits) dst[cnt + __popc(b & ((1u << lane) - 1u))] = static_cast<int32_t>(static_cast<uint32_t>(i) | (bits << 24));
      cnt += __popc(b);
    }
    if (lane == 0) q_count[c] = cnt;
  }
}

cudaError_t launch_sparse64_plan(const uint8_t *mask, int BH, int nq64, int nk64, int nq, int nk, int32_t *kv_list,
                                 int32_t *kv_count, int32_t *q_list, int32_t *q_count, cudaStream_t stream) {
  const int64_t warps = static_cast<int64_t>(BH) * (nq + nk);
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  sparse64_plan_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(mask, BH, nq64, nk64, nq, nk, kv_list,
                                                                          kv_count, q_list, q_count);
  return cudaGetLastError();
}

// Causal masking walks the lower triangle of tiles: key tiles 0..I for query
// tile I (the diagonal last), query tiles J..nt-1 for key tile J (the
// diagonal first).  One warp writes one list.
__global__ void __launch_bounds__(256) causal_plan_kernel(int BH, int nt, int32_t *__restrict__ kv_list,
                                                          int32_t *__restrict__ kv_count,
                                                          int32_t *__restrict__ q_list,
                                                          int32_t *__restrict__ q_count) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(BH) * nt;
  if (w < rows) {
    const int I = static_cast<int>(w % nt);
    for (int j = lane; j <= I; j += 32) kv_list[w * nt + j] = j;
    if (lane == 0) kv_count[w] = I + 1;
  } else if (w < 2 * rows) {
    const int64_t c = w - rows;
    const int J = static_cast<int>(c % nt);
    for (int i = J + lane; i < nt; i += 32) q_list[c * nt + (i - J)] = i;
    if (lane == 0) q_count[c] = nt - J;
  }
}

cudaError_t launch_causal_plan(int BH, int nt, int32_t *kv_list, int32_t *kv_count, int32_t *q_list,
                               int32_t *q_count, cudaStream_t stream) {
  const int64_t blocks = (static_cast<int64_t>(BH) * 2 * nt * 32 + 255) / 256;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  causal_plan_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(BH, nt, kv_list, kv_count, q_list, q_count);
  return cudaGetLastError();
}

// ------------------------------------------------------ key-tile selection --
//
// VSA selection (vsqa-test-1.3b metadata.json, "attention.selection": top-k
// key cubes per query cube; "precision.coarse": BF16, unquantized).  Each
// T-token tile (T = 128, or 64 for the tile-64 profile) is summarised by the
// mean of its valid rows, the coarse
// score of (query tile I, key tile J) is the dot product of the two means,
// and query tile I keeps the topk key tiles of highest score, ties to the
// lower J.  The ranking decides integers, so every step has a fixed float32
// order: rows summed in token order, one correctly rounded division by the
// row count, channels accumulated in order with one fused multiply-add each.

// One CTA per (tile, head), one thread per pair of channels (D/2 threads):
// means[bh][t][d], tiles t < nq of q, then nk tiles of k.  Each thread loads
// 32 rows of its two channels before adding any (2*D-byte rows, coalesced
// across the CTA), then adds them in token order.
__global__ void __launch_bounds__(64) tile_mean_kernel(const __nv_bfloat16 *__restrict__ q,
                                                       const __nv_bfloat16 *__restrict__ k, int Lq, int Lk,
                                                       int D, int T, int nq, int nk, float *__restrict__ means) {
  const int t = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int d = 2 * threadIdx.x;
  const bool isq = t < nq;
  const int L = isq ? Lq : Lk;
  const int r0 = (isq ? t : t - nq) * T;
  const int r1 = r0 + T < L ? r0 + T : L;
  const uint32_t *x =
      reinterpret_cast<const uint32_t *>((isq ? q : k) + static_cast<size_t>(bh) * L * D + d);
  float s0 = 0.0f, s1 = 0.0f;
  for (int r = r0; r < r1; r += 32) {
    uint32_t w[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) w[u] = r + u < r1 ? __ldg(x + static_cast<size_t>(r + u) * (D / 2)) : 0u;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      if (r + u < r1) {
        s0 = __fadd_rn(s0, __uint_as_float(w[u] << 16));
        s1 = __fadd_rn(s1, __uint_as_float(w[u] & 0xFFFF0000u));
      }
    }
  }
  const float cnt = static_cast<float>(r1 - r0);
  float2 *dst = reinterpret_cast<float2 *>(means + (static_cast<size_t>(bh) * (nq + nk) + t) * D + d);
  *dst = make_float2(__fdiv_rn(s0, cnt), __fdiv_rn(s1, cnt));
}

// Coarse scores: one CTA per (32 key tiles, 8 query tiles, head), a warp per
// query tile and a lane per key tile.  The CTA stages its means in shared
// memory (key rows padded to D + 1 floats, so that lane j reads its own
// bank); each score is the in-order chain of D fused multiply-adds.
constexpr int kScoreQ = 8;
__global__ void __launch_bounds__(32 * kScoreQ) tile_score_kernel(const float *__restrict__ means, int nq, int nk,
                                                                   int D, float *__restrict__ scores) {
  __shared__ float qs[kScoreQ][128];
  __shared__ float ks[32][129];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bh = blockIdx.z;
  const int I0 = blockIdx.y * kScoreQ, j0 = blockIdx.x * 32;
  const int nqr = nq - I0 < kScoreQ ? nq - I0 : kScoreQ, nkr = nk - j0 < 32 ? nk - j0 : 32;
  const float *qm = means + (bh * (nq + nk) + I0) * D;
  const float *km = means + (bh * (nq + nk) + nq + j0) * D;
  // every load in flight before any store: 32 key rows and 8 query rows of
  // at most 128 channels (16 and 4 per thread)
  float kv[16], qv[4];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int x = threadIdx.x + u * 32 * kScoreQ;
    kv[u] = x < nkr * D ? __ldg(km + x) : 0.0f;
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int x = threadIdx.x + u * 32 * kScoreQ;
    qv[u] = x < nqr * D ? __ldg(qm + x) : 0.0f;
  }
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int x = threadIdx.x + u * 32 * kScoreQ;
    if (x < nkr * D) ks[x / D][x % D] = kv[u];
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int x = threadIdx.x + u * 32 * kScoreQ;
    if (x < nqr * D) qs[x / D][x % D] = qv[u];
  }
  __syncthreads();
  if (warp < nqr && lane < nkr) {
    const float *qr = qs[warp], *kr = ks[lane];
    float acc = 0.0f;
#pragma unroll 16
    for (int d = 0; d < D; ++d) acc = __fmaf_rn(qr[d], kr[d], acc);
    scores[(bh * nq + I0 + warp) * nk + j0 + lane] = acc;
  }
}

// Top-k: one warp per (head, query tile), topk rounds of a warp-wide argmax
// (score descending, tile ascending) over the tiles not yet kept, with the
// taken tiles marked -inf in the score row (scores are finite for finite
// inputs).  SM: the warp copies its score row into shared memory first
// (nk <= kSelectSmemTiles); else it works on the row in global memory.  The
// mask row is written at the end (0 or 1 per tile).
constexpr int kSelectSmemTiles = 2048;
constexpr int kTopkWarps = 4;

template <bool SM>
__global__ void __launch_bounds__(32 * kTopkWarps) tile_topk_kernel(float *__restrict__ scores, int rows, int nk,
                                                                     int topk, uint8_t *__restrict__ mask) {
  extern __shared__ float sel_smem[];
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kTopkWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;  // warp-uniform; no CTA barrier follows
  float *g = scores + row * nk;
  float *sc = SM ? sel_smem + (threadIdx.x >> 5) * nk : g;
  if (SM) {
    for (int j = lane; j < nk; j += 32) sc[j] = g[j];
    __syncwarp();
  }
  const int kk = topk < nk ? topk : nk;
  for (int r = 0; r < kk; ++r) {
    float best = -INFINITY;
    int bj = -1;  // -1: no candidate
    for (int j = lane; j < nk; j += 32) {
      const float v = sc[j];
      if (v != -INFINITY && (bj < 0 || v > best)) {  // ascending j: equal scores keep the lower tile
        best = v;
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (oj >= 0 && (bj < 0 || ov > best || (ov == best && oj < bj))) {
        best = ov;
        bj = oj;
      }
    }
    if (lane == 0 && bj >= 0 && bj < nk) sc[bj] = -INFINITY;
    __syncwarp();
  }
  // kept tiles are the ones marked -inf
  uint8_t *mk = mask + row * nk;
  for (int j = lane; j < nk; j += 32) mk[j] = sc[j] == -INFINITY ? 1 : 0;
}

cudaError_t launch_vsa_select(const __nv_bfloat16 *q, const __nv_bfloat16 *k, int BH, int Lq, int Lk, int D, int T,
                              int topk, float *means, float *scores, uint8_t *mask, cudaStream_t stream) {
  const int nq = (Lq + T - 1) / T, nk = (Lk + T - 1) / T;
  if (BH > 65535 || D > 128 || (nq + kScoreQ - 1) / kScoreQ > 65535) return cudaErrorInvalidValue;
  tile_mean_kernel<<<dim3(nq + nk, BH), D / 2, 0, stream>>>(q, k, Lq, Lk, D, T, nq, nk, means);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  tile_score_kernel<<<dim3((nk + 31) / 32, (nq + kScoreQ - 1) / kScoreQ, BH), 32 * kScoreQ, 0, stream>>>(
      means, nq, nk, D, scores);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(BH) * nq;
  const int64_t blocks = (rows + kTopkWarps - 1) / kTopkWarps;
  if (blocks > 0x7fffffff || rows > 0x7fffffff) return cudaErrorInvalidValue;
  if (nk <= kSelectSmemTiles) {
    // the limit is raised once, to the most any call of this branch needs
    const int bytes = kTopkWarps * nk * static_cast<int>(sizeof(float));
    e = ensure_smem_attr(reinterpret_cast<const void *>(tile_topk_kernel<true>),
                         kTopkWarps * kSelectSmemTiles * static_cast<int>(sizeof(float)));
    if (e != cudaSuccess) return e;
    tile_topk_kernel<true><<<static_cast<unsigned>(blocks), 32 * kTopkWarps, bytes, stream>>>(
        scores, static_cast<int>(rows), nk, topk, mask);
  } else {
    tile_topk_kernel<false><<<static_cast<unsigned>(blocks), 32 * kTopkWarps, 0, stream>>>(
        scores, static_cast<int>(rows), nk, topk, mask);
  }
  return cudaGetLastError();
}

}  // namespace attnqat
