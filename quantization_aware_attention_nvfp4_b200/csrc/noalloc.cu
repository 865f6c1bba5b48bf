// noalloc.cu -- attnqat_fwd_noalloc: the forward pass for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: a framework whose
// caching allocator has already reserved nearly all of the GPU's memory (a
// fresh cudaMalloc would fail or fragment its pool), code that runs inside an
// allocator or memory-pressure callback (allocating there would recurse or
// deadlock), and plain C hosts with no device allocator of their own.  This
// entry point needs nothing from them but the inputs and outputs: its
// workspace is a fixed block of device memory that the library itself
// carries as a file-scope __device__ array.
//
// Costs and limits:
//  - every GPU that loads this library holds the block (kNoAllocBytes) until
//    the process exits, whether or not this entry point is ever called;
//  - shapes whose workspace would exceed the block are rejected;
//  - all calls share the one block, so calls whose GPU work overlaps (two
//    streams, or two host threads on one device) race and corrupt each
//    other's results; serialise them on one stream;
//  - the block keeps whatever the previous call left; the parts that must
//    start at zero are cleared by the forward itself on the caller's stream.
#include "attnqat.h"
#include "internal.h"

#include <mutex>

namespace attnqat {

constexpr size_t kNoAllocBytes = ATTNQAT_NOALLOC_WS_MAX;

// The workspace block.  In host code this name only stands for the symbol:
// its device address comes from cudaGetSymbolAddress, per device.
static __device__ __align__(256) unsigned char g_noalloc_ws[kNoAllocBytes];

// Device address of g_noalloc_ws on the current device.  It is looked up
// (cudaGetSymbolAddress, with that device current) once per device and
// context: the cache is keyed by the driver's context ID, which is never
// reused within a process, so after a cudaDeviceReset the module is loaded
// again at a new address and the next call looks that address up afresh.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// ID of the current context, or 0 when there is none yet (or the driver
// entry points are unavailable, in which case every call looks up again).
static unsigned long long current_ctx_id() {
  static std::once_flag once;
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

static int noalloc_ws_address(void **out) {
  static std::mutex mu;
  static void *addr[64] = {};
  static unsigned long long ctx_of[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return ATTNQAT_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long id = current_ctx_id();
  if (!addr[dev] || id == 0 || id != ctx_of[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_ws);
    if (e != cudaSuccess) return cuda_fail(e);
    addr[dev] = p;
    ctx_of[dev] = current_ctx_id();  // the lookup has made the primary context current
  }
  *out = addr[dev];
  return ATTNQAT_OK;
}

}  // namespace attnqat

extern "C" int attnqat_fwd_noalloc(const void *q, const void *k, const void *v, int B, int H, int Lq, int Lk,
                                   int D, float sm_scale, uint32_t flags, void *o, float *lse, float *m,
                                   void *stream) {
  const size_t need = attnqat_workspace_size(B, H, Lq, Lk, D, flags);
  // an invalid shape: attnqat_fwd reports it with the code it gives any caller
  if (need == 0) return attnqat_fwd(q, k, v, B, H, Lq, Lk, D, sm_scale, flags, o, lse, m, nullptr, 0, stream);
  if (need > attnqat::kNoAllocBytes) return ATTNQAT_ENOSPC;
  int st = attnqat::check_device();
  if (st != ATTNQAT_OK) return st;
  void *ws = nullptr;
  st = attnqat::noalloc_ws_address(&ws);
  if (st != ATTNQAT_OK) return st;
  return attnqat_fwd(q, k, v, B, H, Lq, Lk, D, sm_scale, flags, o, lse, m, ws, attnqat::kNoAllocBytes, stream);
}
