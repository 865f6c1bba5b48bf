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

}  // namespace attnqat
