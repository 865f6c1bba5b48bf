// selftest.cu -- attnqat_selftest_wait_timeout: runs the failure path of the
// library's bounded device waits on purpose, without a fault.
//
// Every wait of the attention kernels is an mbarrier wait bounded by
// %globaltimer: a wait that gives up sets the CTA's abort flag (so the other
// roles leave their loops), raises the device status word that
// attnqat_device_status() reports as ATTNQAT_ETIMEOUT, lets the copies
// already in flight land, and frees the CTA's TMEM before it exits.  The
// kernel here takes the same steps with the same helpers on a barrier that
// nothing ever arrives at, with a caller-chosen limit:
//   warp 1 allocates TMEM, as the attention kernels' TMEM owner does;
//   warp 0 starts a bulk copy into shared memory (completing on `full`),
//     then waits on `never` until the limit passes, sets the abort flag,
//     and drains the copy;
//   warp 2 waits on `never` as well and leaves when it sees the abort flag;
//   after a CTA barrier warp 1 frees the TMEM.
#include "common.cuh"
#include "internal.h"

namespace attnqat {

// Source of the self-test's bulk copy (16-byte aligned, 1 KB).
static __device__ __align__(16) unsigned char g_selftest_src[1024];

struct SelftestSmem {
  uint64_t full, never;
  uint32_t tmem_slot;
  int abort;
  alignas(16) unsigned char buf[1024];
};

__global__ void __launch_bounds__(96, 1) selftest_wait_kernel(unsigned long long limit_ns, int *waits_ended) {
  __shared__ SelftestSmem sm;
  volatile int *abort = &sm.abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sm.full, 1);
    mbar_init(&sm.never, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_slot, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0 && lane == 0) {
    mbar_arrive_expect_tx(&sm.full, sizeof sm.buf);
    bulk_load(sm.buf, g_selftest_src, sizeof sm.buf, &sm.full);
    // nothing arrives at `never`: the wait gives up after limit_ns
    if (!mbar_wait_for(&sm.never, 0, abort, limit_ns)) atomicAdd(waits_ended, 1);
    mbar_wait_drain(&sm.full, 0);  // the copy in flight lands before the CTA exits
  } else if (warp == 2 && lane == 0) {
    // a second role: it leaves its wait when the first sets the abort flag
    // (or after its own limit, ten times longer)
    if (!mbar_wait_for(&sm.never, 0, abort, 10 * limit_ns)) atomicAdd(waits_ended, 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(sm.tmem_slot, 32);
  }
}

}  // namespace attnqat

extern "C" int attnqat_selftest_wait_timeout(unsigned long long limit_ns, int *waits_ended, void *stream) {
  if (!waits_ended || (reinterpret_cast<uintptr_t>(waits_ended) & 3u)) return ATTNQAT_EINVAL;
  if (limit_ns < 1000 || limit_ns > attnqat::kWaitLimitNs) return ATTNQAT_EINVAL;
  const int st = attnqat::check_device();
  if (st != ATTNQAT_OK) return st;
  attnqat::selftest_wait_kernel<<<1, 96, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, waits_ended);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ATTNQAT_OK : attnqat::cuda_fail(e);
}
