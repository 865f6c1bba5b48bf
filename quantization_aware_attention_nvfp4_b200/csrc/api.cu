// api.cu -- the extern "C" boundary of libattnqat (declared in attnqat.h):
// host-side validation, workspace layout, TMA descriptor encoding and kernel
// launches.  Every step of the computation runs in the kernels of this
// library; there is no host or library fallback.
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>
#include <utility>

#include "attnqat.h"
#include "common.cuh"
#include "internal.h"

namespace attnqat {

static thread_local int g_last_cuda_error = 0;

static int cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return ATTNQAT_ECUDA;
}

// Raises a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device.  The largest limit set so far is remembered per (device,
// kernel): a later call asking for more sets it again.
cudaError_t ensure_smem_attr(const void *kernel, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void *>, int> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev, kernel);
  const auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

// ------------------------------------------------------- kernel timing --

// Optional instrumentation: while enabled, every kernel launch of
// attnqat_fwd / attnqat_bwd is bracketed by two CUDA events recorded on the
// caller's stream; attnqat_profile_read() returns the durations.
struct Profiler {
  std::mutex mu;
  bool on = false;
  struct Rec {
    const char *name;
    cudaEvent_t a, b;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  cudaEvent_t take() {
    if (used == pool.size()) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
      pool.push_back(e);
    }
    return pool[used++];
  }
};
static Profiler g_prof;

struct ProfScope {
  cudaStream_t s;
  bool on;
  cudaEvent_t b = nullptr;
  ProfScope(const char *name, cudaStream_t stream) : s(stream), on(false) {
    std::lock_guard<std::mutex> lock(g_prof.mu);
    if (!g_prof.on) return;
    cudaEvent_t a = g_prof.take();
    b = g_prof.take();
    if (!a || !b) return;
    cudaEventRecord(a, s);
    g_prof.recs.push_back({name, a, b});
    on = true;
  }
  ~ProfScope() {
    if (on) cudaEventRecord(b, s);
  }
};

// ----------------------------------------------------------- device check --

static int check_device() {
  static std::mutex mu;
  static int verdict[64];  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return ATTNQAT_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (verdict[dev] == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    verdict[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return verdict[dev] == 1 ? ATTNQAT_OK : ATTNQAT_EUNSUPPORTED;
}

// ------------------------------------------------------------ TMA encode --

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encoder() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D map over a [BH][L][D] tensor of 16-bit elements, 64 x 128 boxes
// (128 bytes x 128 rows), 128-byte swizzle; rows past L read as zeros.
static bool encode_bhld(CUtensorMap *map, const void *base, int BH, int L, int D, bool f16) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L) * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D map over packed NVFP4 codes [BH][L][D/2 bytes]: whole rows of D/2 bytes
// x 128 rows per box, swizzled by the row width (64 B for D = 128, 32 B for
// D = 64) as the block-scaled MMA's K-major descriptors expect; rows past L
// read as zeros.
static bool encode_codes(CUtensorMap *map, const void *base, int BH, int L, int D) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(D) / 2;
  cuuint64_t dims[3] = {row, static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {row, static_cast<cuuint64_t>(L) * row};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(row), 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D map over fq(V)'s packed codes [BH][D][Lk/2 bytes] (blocks of 16 tokens
// per channel): 128 tokens (64 bytes) x D channels per box, 64-byte swizzle,
// the K-major B operand of the NVFP4 P V product; tokens past Lk read as zeros.
static bool encode_vcodes(CUtensorMap *map, const void *base, int BH, int Lk, int D) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(Lk) / 2;
  cuuint64_t dims[3] = {row, static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {row, row * static_cast<cuuint64_t>(D)};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(D), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------- workspace --

struct Workspace {
  size_t qh, kh, vh16, o32, delta, stats, do16, qc, qsf, kc, ksf, vc, vsf, total;
  size_t qsf_bytes, ksf_bytes, vsf_bytes;
  size_t kv_list, kv_count, q_list, q_count;  // block-sparse tile lists
};

// With Q and K both quantized, S = fq(Q) fq(K)^T runs as a block-scaled NVFP4
// MMA on their packed codes (every product of two E2M1 codes and two E4M3
// scales is exact in float32).
static bool fp4s(uint32_t flags) { return (flags & ATTNQAT_QUANT_Q) && (flags & ATTNQAT_QUANT_K); }

// With every quantizer on, fq(P~) fq(V) is also a product of NVFP4 blocks
// along its K axis (keys for P~, tokens for V), so the forward's P V runs as
// a block-scaled NVFP4 MMA (M = 128 queries, N = D) on fq(V)'s packed codes
// [B*H][D][Lk/2] -- whose rows the TMA reads need 16-byte aligned:
// Lk % 32 == 0.
static bool pv_fp4(uint32_t flags, int Lk, int D) {
  (void)D;  // both head dimensions (N = 64 or 128)
  return (flags & ATTNQAT_QUANT_ALL) == ATTNQAT_QUANT_ALL && (Lk % 32) == 0;
}

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Statistics block (float32): [0] max_i |dO_i|_1, [1] max_i |Delta_i|,
// [2] max |fq(V)| (or max |V|), [3] max |dO|, [4] max |Q| and [5] max |K|
// (only when that operand is not quantized: the scales of their fp16 copies).
constexpr size_t kStatsBytes = 32;

// Every 16-bit operand of the attention MMAs is fp16: fq(Q), fq(K), fq(V)
// are exact in fp16 (values sign * E2M1 * E4M3 lie in [2^-10, 2688] with at
// most 7 significant bits), and an operand whose quantizer is off is copied as
// X * 2^e, a power of two that maps its max magnitude into [2^13, 2^14) (bf16
// has 8 significant bits, so the copy is exact for every element within 2^27
// of the largest).  dO gets the same copy.  So the backward feeds dS and the
// dV operand P/l as fp16 (11 significant bits) whatever the flags.
static Workspace layout(int B, int H, int Lq, int Lk, int D, uint32_t flags, bool sparse = false) {
  Workspace w{};
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t qbytes = BH * Lq * D * 2, kbytes = BH * Lk * D * 2;
  size_t off = 0;
  w.qh = off;
  off = align256(off + qbytes);
  w.kh = off;
  off = align256(off + kbytes);
  w.vh16 = off;
  off = align256(off + kbytes);
  w.o32 = off;
  off = align256(off + BH * Lq * D * 4);
  w.delta = off;
  off = align256(off + BH * Lq * 4);
  w.stats = off;
  off = align256(off + kStatsBytes);
  w.do16 = off;   // fp16 copy dO * 2^e
  off = align256(off + qbytes);
  // packed NVFP4 codes of fq(Q), fq(K) and their scales in 128-row tiles
  // (512 bytes per 128 rows x 64 columns), read by the S MMAs
  const size_t ntq = (static_cast<size_t>(Lq) + 127) / 128, ntk = (static_cast<size_t>(Lk) + 127) / 128;
  w.qsf_bytes = BH * ntq * (D / 64) * 512;
  w.ksf_bytes = BH * ntk * (D / 64) * 512;
  const bool fp4 = fp4s(flags);
  w.qc = off;
  if (fp4) off = align256(off + BH * Lq * D / 2);
  w.qsf = off;
  if (fp4) off = align256(off + w.qsf_bytes);
  w.kc = off;
  if (fp4) off = align256(off + BH * Lk * D / 2);
  w.ksf = off;
  if (fp4) off = align256(off + w.ksf_bytes);
  // fq(V)'s packed codes and its scales in 128-token tiles (1 KB per tile)
  const bool pv4 = pv_fp4(flags, Lk, D);
  w.vsf_bytes = BH * ntk * 1024;
  w.vc = off;
  if (pv4) off = align256(off + BH * Lk * D / 2);
  w.vsf = off;
  if (pv4) off = align256(off + w.vsf_bytes);
  // block-sparse: the tile lists the attention kernels walk (int32), built
  // from the caller's tile mask by every sparse call
  w.kv_list = off;
  if (sparse) off = align256(off + BH * ntq * ntk * 4);
  w.kv_count = off;
  if (sparse) off = align256(off + BH * ntq * 4);
  w.q_list = off;
  if (sparse) off = align256(off + BH * ntk * ntq * 4);
  w.q_count = off;
  if (sparse) off = align256(off + BH * ntk * 4);
  w.total = off;
  return w;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_shape(int B, int H, int Lq, int Lk, int D, float sm_scale, uint32_t flags) {
  if (B < 1 || H < 1 || Lq < 1 || Lk < 1) return ATTNQAT_EINVAL;
  if ((flags & ATTNQAT_CAUSAL) && Lq != Lk) return ATTNQAT_EINVAL;  // query i and key i are one token
  if (static_cast<int64_t>(B) * H > 65535) return ATTNQAT_EINVAL;  // grid.y
  const int64_t Lmax = Lq > Lk ? Lq : Lk;
  if (static_cast<int64_t>(B) * H * Lmax * 128 >= (int64_t(1) << 40)) return ATTNQAT_EINVAL;
  if (!(std::isfinite(sm_scale) && sm_scale > 0.0f)) return ATTNQAT_EINVAL;
  if (flags & ~(ATTNQAT_QUANT_ALL | ATTNQAT_CAUSAL | ATTNQAT_TILE64)) return ATTNQAT_EINVAL;
  if ((flags & ATTNQAT_TILE64) && (flags & ATTNQAT_CAUSAL)) return ATTNQAT_EINVAL;  // a mask, or causal
  if (D != 64 && D != 128) return ATTNQAT_EUNSUPPORTED;
  return ATTNQAT_OK;
}

// Writes the fp16 operands -- fq(Q), fq(K), fq(V), or the scaled copies of
// the operands whose quantizer is off -- and the packed NVFP4 codes into the
// workspace, and the max magnitudes that scale the copies into its
// statistics block.
static int prepare_operands(const void *q, const void *k, const void *v, int B, int H, int Lq, int Lk,
                            int D, uint32_t flags, uint8_t *ws, const Workspace &w,
                            cudaStream_t stream) {
  const int64_t BH = static_cast<int64_t>(B) * H;
  const bool fp4 = fp4s(flags);
  float *stats = reinterpret_cast<float *>(ws + w.stats);
  cudaError_t e = cudaMemsetAsync(stats, 0, kStatsBytes, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  // A quantized operand: one pass writes the exact fp16 fq and, with Q and K
  // both quantized, the packed codes with tiled scales (for the S MMAs);
  // scale tiles are cleared first when the last 128-row tile is partial, so
  // its padding rows carry zero scales.  An unquantized one: its max
  // magnitude, then the scaled fp16 copy.
  auto prep_qk = [&](const void *x, bool quantized, int L, size_t deq_off, size_t c_off, size_t sf_off,
                     size_t sf_bytes, float *amax, const char *qname, const char *aname,
                     const char *cname) -> int {
    uint16_t *dst = reinterpret_cast<uint16_t *>(ws + deq_off);
    if (quantized) {
      if (fp4 && (L % 128) != 0) {
        cudaError_t em = cudaMemsetAsync(ws + sf_off, 0, sf_bytes, stream);
        if (em != cudaSuccess) return cuda_fail(em);
      }
      ProfScope ps(qname, stream);
      cudaError_t eq = launch_quantize(static_cast<const uint16_t *>(x), 1, BH * L, D, 0, D, 1,
                                       fp4 ? ws + c_off : nullptr, fp4 ? ws + sf_off : nullptr, nullptr, dst,
                                       nullptr, stream, fp4 ? L : 0);
      return eq == cudaSuccess ? ATTNQAT_OK : cuda_fail(eq);
    }
    cudaError_t ea;
    {
      ProfScope ps(aname, stream);
      ea = launch_absmax(static_cast<const __nv_bfloat16 *>(x), BH * L * D, amax, stream);
    }
    if (ea != cudaSuccess) return cuda_fail(ea);
    ProfScope ps(cname, stream);
    ea = launch_scale_f16(static_cast<const __nv_bfloat16 *>(x), dst, BH * L * D, amax, stream);
    return ea == cudaSuccess ? ATTNQAT_OK : cuda_fail(ea);
  };
  int st = prep_qk(q, (flags & ATTNQAT_QUANT_Q) != 0, Lq, w.qh, w.qc, w.qsf, w.qsf_bytes, stats + 4, "quantize_q",
                   "absmax_q", "scale_q");
  if (st != ATTNQAT_OK) return st;
  st = prep_qk(k, (flags & ATTNQAT_QUANT_K) != 0, Lk, w.kh, w.kc, w.ksf, w.ksf_bytes, stats + 5, "quantize_k",
               "absmax_k", "scale_k");
  if (st != ATTNQAT_OK) return st;
  uint16_t *vdst = reinterpret_cast<uint16_t *>(ws + w.vh16);
  if (flags & ATTNQAT_QUANT_V) {
    // blocks of 16 consecutive tokens per channel: the transposed view
    const bool pv4 = pv_fp4(flags, Lk, D);
    if (pv4 && (Lk % 128) != 0) {
      e = cudaMemsetAsync(ws + w.vsf, 0, w.vsf_bytes, stream);
      if (e != cudaSuccess) return cuda_fail(e);
    }
    ProfScope ps("quantize_v", stream);
    e = launch_quantize(static_cast<const uint16_t *>(v), BH, D, Lk, static_cast<int64_t>(Lk) * D, 1, D,
                        pv4 ? ws + w.vc : nullptr, pv4 ? ws + w.vsf : nullptr, nullptr, vdst, stats + 2, stream, 0,
                        pv4);
    if (e != cudaSuccess) return cuda_fail(e);
  } else {
    {
      ProfScope ps("absmax_v", stream);
      e = launch_absmax(static_cast<const __nv_bfloat16 *>(v), BH * Lk * D, stats + 2, stream);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    ProfScope ps("scale_v", stream);
    e = launch_scale_f16(static_cast<const __nv_bfloat16 *>(v), vdst, BH * Lk * D, stats + 2, stream);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return ATTNQAT_OK;
}

// The max magnitudes that scale the fp16 copies of unquantized operands
// (null for a quantized operand: its fq copy is unscaled).
static void operand_amax(uint32_t flags, uint8_t *wsb, const Workspace &w, const float **aq, const float **ak,
                         const float **av) {
  const float *stats = reinterpret_cast<const float *>(wsb + w.stats);
  *aq = (flags & ATTNQAT_QUANT_Q) ? nullptr : stats + 4;
  *ak = (flags & ATTNQAT_QUANT_K) ? nullptr : stats + 5;
  *av = (flags & ATTNQAT_QUANT_V) ? nullptr : stats + 2;
}

}  // namespace attnqat

using namespace attnqat;

extern "C" {

const char *attnqat_strerror(int status) {
  switch (status) {
    case ATTNQAT_OK: return "success";
    case ATTNQAT_EINVAL: return "invalid argument (null or misaligned pointer, bad shape or scale)";
    case ATTNQAT_EUNSUPPORTED: return "unsupported (device is not sm_100 or head dimension not 64/128)";
    case ATTNQAT_ENOSPC: return "workspace too small";
    case ATTNQAT_ECUDA: return "CUDA error (see attnqat_last_cuda_error)";
    case ATTNQAT_ETIMEOUT: return "a device-side wait timed out";
    default: return "unknown status";
  }
}

int attnqat_last_cuda_error(void) { return g_last_cuda_error; }

int attnqat_profile_enable(int on) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  g_prof.on = on != 0;
  g_prof.recs.clear();
  g_prof.used = 0;
  return ATTNQAT_OK;
}

int attnqat_profile_read(const char **names, float *ms, int max_records) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  const int n = static_cast<int>(g_prof.recs.size());
  for (int i = 0; i < n && i < max_records; ++i) {
    const Profiler::Rec &r = g_prof.recs[i];
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e);
    float t = 0.0f;
    e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e);
    if (names) names[i] = r.name;
    if (ms) ms[i] = t;
  }
  g_prof.recs.clear();
  g_prof.used = 0;
  return n;
}

int attnqat_device_status(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof v);
  if (e != cudaSuccess) return cuda_fail(e);
  if (v == 0) return ATTNQAT_OK;
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero);
  if (e != cudaSuccess) return cuda_fail(e);
  return ATTNQAT_ETIMEOUT;
}

int attnqat_quantize(const void *x, int64_t batch, int64_t rows, int64_t cols, int64_t stride_batch,
                     int64_t stride_row, int64_t stride_col, uint8_t *codes, uint8_t *scales, void *deq,
                     void *stream) {
  if (!x || !codes || !scales) return ATTNQAT_EINVAL;
  if (batch < 1 || rows < 1 || cols < 16 || (cols % 16) != 0) return ATTNQAT_EINVAL;
  if (stride_batch < 0 || stride_row < 0 || stride_col < 0) return ATTNQAT_EINVAL;
  const int64_t lim = int64_t(1) << 40;
  if (batch > lim || rows > lim || cols > lim || batch * rows > lim / cols) return ATTNQAT_EINVAL;
  // codes are written as 8-byte groups (one 16-element block each)
  if ((reinterpret_cast<uintptr_t>(x) & 1u) || (deq && (reinterpret_cast<uintptr_t>(deq) & 1u)) ||
      (reinterpret_cast<uintptr_t>(codes) & 7u))
    return ATTNQAT_EINVAL;
  const int st = check_device();
  if (st != ATTNQAT_OK) return st;
  cudaError_t e = launch_quantize(static_cast<const uint16_t *>(x), batch, rows, cols, stride_batch,
                                  stride_row, stride_col, codes, scales, static_cast<uint16_t *>(deq),
                                  nullptr, nullptr, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTNQAT_OK : cuda_fail(e);
}

int attnqat_quantize_gs(const void *x, int64_t batch, int64_t rows, int64_t cols, int64_t stride_batch,
                        int64_t stride_row, int64_t stride_col, uint8_t *codes, uint8_t *scales, void *deq,
                        float *gscale, void *stream) {
  if (!x || !codes || !scales || !gscale) return ATTNQAT_EINVAL;
  if (batch < 1 || rows < 1 || cols < 16 || (cols % 16) != 0) return ATTNQAT_EINVAL;
  if (stride_batch < 0 || stride_row < 0 || stride_col < 0) return ATTNQAT_EINVAL;
  const int64_t lim = int64_t(1) << 40;
  if (batch > lim || rows > lim || cols > lim || batch * rows > lim / cols) return ATTNQAT_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x) & 1u) || (deq && (reinterpret_cast<uintptr_t>(deq) & 1u)) ||
      (reinterpret_cast<uintptr_t>(gscale) & 3u) || (reinterpret_cast<uintptr_t>(codes) & 7u))
    return ATTNQAT_EINVAL;
  const int st = check_device();
  if (st != ATTNQAT_OK) return st;
  cudaError_t e = launch_quantize_gs(static_cast<const uint16_t *>(x), batch, rows, cols, stride_batch, stride_row,
                                     stride_col, codes, scales, static_cast<uint16_t *>(deq), gscale,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTNQAT_OK : cuda_fail(e);
}

size_t attnqat_workspace_size(int B, int H, int Lq, int Lk, int D, uint32_t flags) {
  if ((flags & ATTNQAT_TILE64) || check_shape(B, H, Lq, Lk, D, 1.0f, flags) != ATTNQAT_OK) return 0;
  return layout(B, H, Lq, Lk, D, flags, (flags & ATTNQAT_CAUSAL) != 0).total;
}

}  // extern "C"

namespace attnqat {

// Builds the tile lists into the workspace: from the caller's mask
// (block-sparse; with tile64 a 64-token mask whose quadrants ride in the list
// entries), the lower triangle (causal), or nothing (dense).
static int plan_sparse(const uint8_t *mask, bool causal, bool tile64, int BH, int Lq, int Lk, uint8_t *wsb,
                       const Workspace &w, cudaStream_t s) {
  if (!mask && !causal) return ATTNQAT_OK;
  int32_t *kvl = reinterpret_cast<int32_t *>(wsb + w.kv_list), *kvc = reinterpret_cast<int32_t *>(wsb + w.kv_count);
  int32_t *ql = reinterpret_cast<int32_t *>(wsb + w.q_list), *qc = reinterpret_cast<int32_t *>(wsb + w.q_count);
  const int nq = (Lq + kBM - 1) / kBM, nk = (Lk + kBN - 1) / kBN;
  ProfScope ps(causal ? "causal_plan" : "sparse_plan", s);
  cudaError_t e;
  if (causal)
    e = launch_causal_plan(BH, nq, kvl, kvc, ql, qc, s);
  else if (tile64)
    e = launch_sparse64_plan(mask, BH, (Lq + 63) / 64, (Lk + 63) / 64, nq, nk, kvl, kvc, ql, qc, s);
  else
    e = launch_sparse_plan(mask, BH, nq, nk, kvl, kvc, ql, qc, s);
  return e == cudaSuccess ? ATTNQAT_OK : cuda_fail(e);
}

// attnqat_fwd (mask == nullptr) and attnqat_sparse_fwd.
static int run_fwd(const void *q, const void *k, const void *v, int B, int H, int Lq, int Lk, int D,
                   float sm_scale, uint32_t flags, const uint8_t *mask, void *o, float *lse, float *m, void *ws,
                   size_t ws_bytes, void *stream) {
  int st = check_shape(B, H, Lq, Lk, D, sm_scale, flags);
  if (st != ATTNQAT_OK) return st;
  const bool causal = (flags & ATTNQAT_CAUSAL) != 0;
  const bool tile64 = (flags & ATTNQAT_TILE64) != 0;
  if (causal && mask) return ATTNQAT_EINVAL;  // a tile selection and causal masking do not combine
  if (tile64 && !mask) return ATTNQAT_EINVAL;  // 64-token tiles describe a mask
  if (!q || !k || !v || !o || !lse || !m || !ws) return ATTNQAT_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(m) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return ATTNQAT_EINVAL;
  const Workspace w = layout(B, H, Lq, Lk, D, flags, mask != nullptr || causal);
  if (ws_bytes < w.total) return ATTNQAT_ENOSPC;
  st = check_device();
  if (st != ATTNQAT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  st = prepare_operands(q, k, v, B, H, Lq, Lk, D, flags, wsb, w, s);
  if (st != ATTNQAT_OK) return st;
  const int BH = B * H;
  st = plan_sparse(mask, causal, tile64, BH, Lq, Lk, wsb, w, s);
  if (st != ATTNQAT_OK) return st;
  const bool fp4 = fp4s(flags);
  const bool pv4 = pv_fp4(flags, Lk, D);
  CUtensorMap tq, tk, tv;
  const bool maps_ok = fp4 ? encode_codes(&tq, wsb + w.qc, BH, Lq, D) && encode_codes(&tk, wsb + w.kc, BH, Lk, D)
                           : encode_bhld(&tq, wsb + w.qh, BH, Lq, D, true) && encode_bhld(&tk, wsb + w.kh, BH, Lk, D, true);
  const bool vmap_ok = pv4 ? encode_vcodes(&tv, wsb + w.vc, BH, Lk, D) : encode_bhld(&tv, wsb + w.vh16, BH, Lk, D, true);
  if (!maps_ok || !vmap_ok) return cuda_fail(cudaErrorInvalidValue);
  FwdArgs a;
  a.Lq = Lq;
  a.Lk = Lk;
  a.nq_tiles = (Lq + kBM - 1) / kBM;
  a.nk_tiles = (Lk + kBN - 1) / kBN;
  a.sm_scale = sm_scale;
  a.scale_log2 = sm_scale * kLog2e;
  a.qsf = wsb + w.qsf;
  a.ksf = wsb + w.ksf;
  a.vsf = wsb + w.vsf;
  operand_amax(flags, wsb, w, &a.amax_q, &a.amax_k, &a.amax_v);
  a.o = static_cast<__nv_bfloat16 *>(o);
  a.o32 = reinterpret_cast<float *>(wsb + w.o32);
  a.lse = lse;
  a.m = m;
  const bool listed = mask != nullptr || causal;
  a.kv_list = listed ? reinterpret_cast<const int32_t *>(wsb + w.kv_list) : nullptr;
  a.kv_count = listed ? reinterpret_cast<const int32_t *>(wsb + w.kv_count) : nullptr;
  a.causal = causal ? 1 : 0;
  a.quad = tile64 ? 1 : 0;
  cudaError_t e;
  {
    ProfScope ps("attn_fwd", s);
    e = launch_fwd(D, fp4, pv4, (flags & ATTNQAT_QUANT_P) != 0, tq, tk, tv, a, BH, s);
  }
  return e == cudaSuccess ? ATTNQAT_OK : cuda_fail(e);
}

// attnqat_bwd (mask == nullptr) and attnqat_sparse_bwd.
static int run_bwd(const void *q, const void *k, const void *v, const float *lse, const float *m, const void *dO,
                   int B, int H, int Lq, int Lk, int D, float sm_scale, uint32_t flags, const uint8_t *mask,
                   void *dq, void *dk, void *dv, void *ws, size_t ws_bytes, void *stream) {
  int st = check_shape(B, H, Lq, Lk, D, sm_scale, flags);
  if (st != ATTNQAT_OK) return st;
  const bool causal = (flags & ATTNQAT_CAUSAL) != 0;
  const bool tile64 = (flags & ATTNQAT_TILE64) != 0;
  if (causal && mask) return ATTNQAT_EINVAL;
  if (tile64 && !mask) return ATTNQAT_EINVAL;
  if (!q || !k || !v || !lse || !m || !dO || !dq || !dk || !dv || !ws) return ATTNQAT_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(lse) || !aligned16(m) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return ATTNQAT_EINVAL;
  const Workspace w = layout(B, H, Lq, Lk, D, flags, mask != nullptr || causal);
  if (ws_bytes < w.total) return ATTNQAT_ENOSPC;
  st = check_device();
  if (st != ATTNQAT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  const int BH = B * H;
  st = plan_sparse(mask, causal, tile64, BH, Lq, Lk, wsb, w, s);
  if (st != ATTNQAT_OK) return st;
  float *delta = reinterpret_cast<float *>(wsb + w.delta);
  float *stats = reinterpret_cast<float *>(wsb + w.stats);
  // stats[2], [4], [5] come from the forward; [0], [1], [3] start at zero
  cudaError_t e = cudaMemsetAsync(stats, 0, 8, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(stats + 3, 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e);
  {
    ProfScope ps("delta", s);
    e = launch_delta(reinterpret_cast<const float *>(wsb + w.o32), static_cast<const __nv_bfloat16 *>(dO), delta,
                     static_cast<int64_t>(BH) * Lq, D, stats, s);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  {
    ProfScope ps("scale_do", s);
    e = launch_scale_f16(static_cast<const __nv_bfloat16 *>(dO), reinterpret_cast<uint16_t *>(wsb + w.do16),
                         static_cast<int64_t>(BH) * Lq * D, stats + 3, s);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  const bool fp4 = fp4s(flags);
  CUtensorMap tq, tk, tv, tdo;
  if (!encode_bhld(&tq, wsb + w.qh, BH, Lq, D, true) || !encode_bhld(&tk, wsb + w.kh, BH, Lk, D, true) ||
      !encode_bhld(&tv, wsb + w.vh16, BH, Lk, D, true) || !encode_bhld(&tdo, wsb + w.do16, BH, Lq, D, true))
    return cuda_fail(cudaErrorInvalidValue);
  BwdArgs a;
  a.Lq = Lq;
  a.Lk = Lk;
  a.nq_tiles = (Lq + kBM - 1) / kBM;
  a.nk_tiles = (Lk + kBN - 1) / kBN;
  a.sm_scale = sm_scale;
  a.scale_log2 = sm_scale * kLog2e;
  a.m = m;
  a.lse = lse;
  a.delta = delta;
  a.stats = stats;
  operand_amax(flags, wsb, w, &a.amax_q, &a.amax_k, &a.amax_v);
  a.qsf = wsb + w.qsf;
  a.ksf = wsb + w.ksf;
  a.dq = static_cast<__nv_bfloat16 *>(dq);
  a.dk = static_cast<__nv_bfloat16 *>(dk);
  a.dv = static_cast<__nv_bfloat16 *>(dv);
  const bool listed = mask != nullptr || causal;
  a.kv_list = listed ? reinterpret_cast<const int32_t *>(wsb + w.kv_list) : nullptr;
  a.kv_count = listed ? reinterpret_cast<const int32_t *>(wsb + w.kv_count) : nullptr;
  a.q_list = listed ? reinterpret_cast<const int32_t *>(wsb + w.q_list) : nullptr;
  a.q_count = listed ? reinterpret_cast<const int32_t *>(wsb + w.q_count) : nullptr;
  a.causal = causal ? 1 : 0;
  a.quad = tile64 ? 1 : 0;
  // with Q and K quantized, S runs on the packed NVFP4 codes
  CUtensorMap tq4, tk4;
  if (fp4 && !(encode_codes(&tq4, wsb + w.qc, BH, Lq, D) && encode_codes(&tk4, wsb + w.kc, BH, Lk, D)))
    return cuda_fail(cudaErrorInvalidValue);
  {
    ProfScope ps("attn_bwd_dkdv", s);
    e = launch_bwd_dkdv(D, fp4, (flags & ATTNQAT_QUANT_P) != 0, tq, fp4 ? tk4 : tk, tv, tdo, fp4 ? tq4 : tq, a, BH,
                        s);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  {
    ProfScope ps("attn_bwd_dq", s);
    // dS as an fp16 hi + lo pair unless every quantizer is on (measured: a
    // single fp16 dS keeps the all-quantized dQ within the bar with margin,
    // and the hot path keeps its one dQ product)
    const bool dsplit = (flags & ATTNQAT_QUANT_ALL) != ATTNQAT_QUANT_ALL;
    e = launch_bwd_dq(D, fp4, dsplit, fp4 ? tq4 : tq, tk, tv, tdo, fp4 ? tk4 : tk, a, BH, s);
  }
  return e == cudaSuccess ? ATTNQAT_OK : cuda_fail(e);
}

}  // namespace attnqat

extern "C" {

int attnqat_fwd(const void *q, const void *k, const void *v, int B, int H, int Lq, int Lk, int D,
                float sm_scale, uint32_t flags, void *o, float *lse, float *m, void *ws, size_t ws_bytes,
                void *stream) {
  return run_fwd(q, k, v, B, H, Lq, Lk, D, sm_scale, flags, nullptr, o, lse, m, ws, ws_bytes, stream);
}

int attnqat_bwd(const void *q, const void *k, const void *v, const float *lse, const float *m, const void *dO,
                int B, int H, int Lq, int Lk, int D, float sm_scale, uint32_t flags, void *dq, void *dk, void *dv,
                void *ws, size_t ws_bytes, void *stream) {
  return run_bwd(q, k, v, lse, m, dO, B, H, Lq, Lk, D, sm_scale, flags, nullptr, dq, dk, dv, ws, ws_bytes,
                 stream);
}

size_t attnqat_sparse_workspace_size(int B, int H, int Lq, int Lk, int D, uint32_t flags) {
  if ((flags & ATTNQAT_CAUSAL) || check_shape(B, H, Lq, Lk, D, 1.0f, flags) != ATTNQAT_OK) return 0;
  return layout(B, H, Lq, Lk, D, flags & ~ATTNQAT_TILE64, true).total;
}

int attnqat_sparse_fwd(const void *q, const void *k, const void *v, int B, int H, int Lq, int Lk, int D,
                       float sm_scale, uint32_t flags, const uint8_t *tile_mask, void *o, float *lse, float *m,
                       void *ws, size_t ws_bytes, void *stream) {
  if (!tile_mask) return ATTNQAT_EINVAL;
  return run_fwd(q, k, v, B, H, Lq, Lk, D, sm_scale, flags, tile_mask, o, lse, m, ws, ws_bytes, stream);
}

size_t attnqat_vsa_select_tiles_workspace_size(int B, int H, int Lq, int Lk, int D, int tile) {
  if ((tile != 64 && tile != 128) || check_shape(B, H, Lq, Lk, D, 1.0f, 0) != ATTNQAT_OK) return 0;
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t nq = (static_cast<size_t>(Lq) + tile - 1) / tile, nk = (static_cast<size_t>(Lk) + tile - 1) / tile;
  return align256(BH * (nq + nk) * D * 4) + align256(BH * nq * nk * 4);
}

size_t attnqat_vsa_select_workspace_size(int B, int H, int Lq, int Lk, int D) {
  return attnqat_vsa_select_tiles_workspace_size(B, H, Lq, Lk, D, ATTNQAT_SPARSE_TILE);
}

int attnqat_vsa_select_tiles(const void *q, const void *k, int B, int H, int Lq, int Lk, int D, int tile, int topk,
                             uint8_t *tile_mask, void *ws, size_t ws_bytes, void *stream) {
  int st = check_shape(B, H, Lq, Lk, D, 1.0f, 0);
  if (st != ATTNQAT_OK) return st;
  if (!q || !k || !tile_mask || !ws || topk < 1 || (tile != 64 && tile != 128)) return ATTNQAT_EINVAL;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return ATTNQAT_EINVAL;
  const size_t need = attnqat_vsa_select_tiles_workspace_size(B, H, Lq, Lk, D, tile);
  if (ws_bytes < need) return ATTNQAT_ENOSPC;
  st = check_device();
  if (st != ATTNQAT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t nq = (static_cast<size_t>(Lq) + tile - 1) / tile, nk = (static_cast<size_t>(Lk) + tile - 1) / tile;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  float *means = reinterpret_cast<float *>(wsb);
  float *scores = reinterpret_cast<float *>(wsb + align256(BH * (nq + nk) * D * 4));
  ProfScope ps("vsa_select", s);
  const cudaError_t e = launch_vsa_select(static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
                                          B * H, Lq, Lk, D, tile, topk, means, scores, tile_mask, s);
  return e == cudaSuccess ? ATTNQAT_OK : cuda_fail(e);
}

int attnqat_vsa_select(const void *q, const void *k, int B, int H, int Lq, int Lk, int D, int topk,
                       uint8_t *tile_mask, void *ws, size_t ws_bytes, void *stream) {
  return attnqat_vsa_select_tiles(q, k, B, H, Lq, Lk, D, ATTNQAT_SPARSE_TILE, topk, tile_mask, ws, ws_bytes, stream);
}

int attnqat_sparse_bwd(const void *q, const void *k, const void *v, const float *lse, const float *m,
                       const void *dO, int B, int H, int Lq, int Lk, int D, float sm_scale, uint32_t flags,
                       const uint8_t *tile_mask, void *dq, void *dk, void *dv, void *ws, size_t ws_bytes,
                       void *stream) {
  if (!tile_mask) return ATTNQAT_EINVAL;
  return run_bwd(q, k, v, lse, m, dO, B, H, Lq, Lk, D, sm_scale, flags, tile_mask, dq, dk, dv, ws, ws_bytes,
                 stream);
}

}  // extern "C"
