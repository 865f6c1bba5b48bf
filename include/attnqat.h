/*
 * attnqat.h -- C ABI of the B200 (sm_100a) Attn-QAT attention library.
 *
 * Attn-QAT training attention: multi-head attention whose operands are NVFP4
 * fake-quantized (fq) inside the op, with a straight-through backward --
 * non-causal as the pages' route (attnqat_fwd / attnqat_bwd), plus the VSA
 * block-sparse fine attention with its key-tile selection and causal masking
 * (declared further down).  The method and its format come from these pages:
 *  - FastVideo "Attn-QAT Training" guide, section "Architecture-specific
 *    Triton routing": non-causal BF16 attention, head dimension 128, query
 *    and key/value lengths may differ (K and V share one), the optimized
 *    backward needs a 16-aligned KV length, the backend fails loudly instead
 *    of falling back to dense attention ("Prerequisites").
 *  - vsqa-test-1.3b checkpoint metadata.json, "attention.precision": "NVFP4
 *    fake-quant with BF16 matmul", quant_p and quant_v on, no global scale
 *    (use_global_sf_p / use_global_sf_qkv false); "linear_quantization.format":
 *    E2M1 values, 16-element blocks, E4M3 block scales.
 *  - fastvideo-kernel triton_kernels commit (SM100 Attn-QAT route): full KV
 *    tiles without bounds masks plus a separate masked tail tile.
 *  - FastVideo PR #1457 review, finding F1: the softmax scale must be plumbed
 *    end to end, never replaced by a hidden 1/sqrt(D).
 *
 * fq(x) on a block of 16 elements along the contraction axis of the matmul
 * the operand feeds: s = E4M3(amax/6) (round to nearest even, saturating at
 * 448, subnormals kept, s = 0 zeroes the block), each element becomes
 * sign(x) * E2M1(|x|/s) * s (round to nearest even on {0,.5,1,1.5,2,3,4,6}).
 *
 * Forward:  S = fq(Q) fq(K)^T * sm_scale, m = exact row max of S,
 *           P~ = exp(S - m), l = sum_j P~ (unquantized),
 *           O = fq(P~) fq(V) / l with fq(P~) blocked along keys from key 0,
 *           LSE = m + ln l.
 * Backward: dV = (fq(P~)/l)^T dO, dP = dO fq(V)^T, Delta = rowsum(dO o O),
 *           dS = P o (dP - Delta) with P = P~/l, dQ = dS fq(K) sm_scale,
 *           dK = dS^T fq(Q) sm_scale.
 *
 * Conventions shared by every entry point:
 *  - Tensors are dense, contiguous, row-major bf16 in BHSD order:
 *    q, o, dO, dq: [B][H][Lq][D]; k, v, dk, dv: [B][H][Lk][D].  m, lse:
 *    float32 [B][H][Lq].  All pointers are device pointers unless stated.
 *  - The caller owns every buffer; no call allocates device memory.  The
 *    library's state: the driver entry points it looks up once per process
 *    (to encode TMA descriptors, to identify a context), the largest dynamic
 *    shared-memory size set so far per kernel and device, a per-device
 *    record of the device check, the device status word below, and one
 *    static block of ATTNQAT_NOALLOC_WS_MAX bytes per device that only
 *    attnqat_fwd_noalloc uses (held by every GPU that loads the library),
 *    with its device address kept per device and context.  Inputs are never
 *    written.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Work is enqueued asynchronously; all argument checks run on the
 *    host before any launch.  There is no CPU fallback.
 *  - Return value: 0 on success, else a negative ATTNQAT_E* code;
 *    attnqat_strerror() describes it.  On ATTNQAT_ECUDA the CUDA error is
 *    kept and returned by attnqat_last_cuda_error().
 *  - Device-side waits are bounded.  A wait that gives up sets a device flag,
 *    read (with a device synchronize) by attnqat_device_status().
 */
#ifndef ATTNQAT_H
#define ATTNQAT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define ATTNQAT_OK 0
#define ATTNQAT_EINVAL (-1)       /* null or misaligned pointer, bad shape, bad scale */
#define ATTNQAT_EUNSUPPORTED (-2) /* device is not sm_100 (B200) or D not in {64,128} */
#define ATTNQAT_ENOSPC (-3)       /* workspace smaller than attnqat_workspace_size() */
#define ATTNQAT_ECUDA (-4)        /* a CUDA call or launch failed */
#define ATTNQAT_ETIMEOUT (-5)     /* a device-side wait gave up (attnqat_device_status) */

/* ---- flags: which operands are fake-quantized (vsqa-test-1.3b
 * metadata.json, attention.precision: quant_p, quant_v; the fine attention
 * quantizes q/k as well).  A cleared bit makes that fq the identity. ---- */
#define ATTNQAT_QUANT_Q 1u
#define ATTNQAT_QUANT_K 2u
#define ATTNQAT_QUANT_V 4u
#define ATTNQAT_QUANT_P 8u
#define ATTNQAT_QUANT_ALL 15u
/* Causal masking (attnqat_fwd / attnqat_bwd / attnqat_workspace_size only;
 * needs Lq == Lk; any quantizer flags): query i attends to keys j <= i.  The
 * first keys' gradients gather every later row's contribution, which the
 * backward's fp16 dS and dV operands (11 significant bits) carry accurately.
 * The pages' training route is non-causal (FastVideo "Attn-QAT Training"
 * guide, "Architecture-specific Triton routing"); the mask is applied like a
 * tile selection: masked keys have P~ = 0 inside their fq(P~) blocks, m and l
 * run over the unmasked keys, and only the lower triangle of 128 x 128 tiles
 * is computed. */
#define ATTNQAT_CAUSAL 32u

/* Text for a status code (static storage). */
const char *attnqat_strerror(int status);

/* Last CUDA runtime error recorded by a failed call (cudaError_t as int). */
int attnqat_last_cuda_error(void);

/* Kernel timing (instrumentation).  attnqat_profile_enable(1) makes every
 * later attnqat_fwd / attnqat_bwd call record a CUDA event on its stream
 * before and after each kernel it launches (0 turns this off; both calls
 * discard what was recorded).  attnqat_profile_read() waits for the recorded
 * events, writes up to max_records kernel names (static strings) and
 * durations in milliseconds, clears the record and returns how many kernels
 * were recorded (or a negative status).  Not thread-safe across streams of
 * different devices; meant for benchmarks. */
int attnqat_profile_enable(int on);
int attnqat_profile_read(const char **names, float *ms, int max_records);

/* Synchronizes the current device, then returns ATTNQAT_OK if no device-side
 * wait of this library has timed out since the last call, else
 * ATTNQAT_ETIMEOUT (and clears the flag). */
int attnqat_device_status(void);

/* Self-test of that failure path (no counterpart on the pages: it checks the
 * library's own fail-loudly machinery).  Launches one small kernel on
 * `stream` that takes the steps an attention kernel takes when a wait gives
 * up, on an mbarrier nothing ever arrives at: it allocates TMEM, starts a
 * bulk copy into shared memory, waits limit_ns nanoseconds (1000 <= limit_ns
 * <= 2e9), sets its abort flag -- a second waiting role sees it and leaves --
 * lets the copy land, and frees the TMEM.  Each of the two waits that ends
 * without its barrier adds 1 to *waits_ended (a device int, 4-byte aligned),
 * and the device status word is raised, so the next attnqat_device_status()
 * returns ATTNQAT_ETIMEOUT.  No fault is raised and the context stays usable.
 * Errors: EINVAL (null or misaligned waits_ended, limit out of range),
 * EUNSUPPORTED, ECUDA. */
int attnqat_selftest_wait_timeout(unsigned long long limit_ns, int *waits_ended, void *stream);

/*
 * attnqat_quantize -- standalone NVFP4 quantizer (fq of a strided bf16 view).
 *
 * Defined by: vsqa-test-1.3b metadata.json, "linear_quantization.format"
 * (E2M1 values, 16-element blocks, E4M3 block scale) with the attention's
 * "no global scale" setting (attention.precision.use_global_sf_qkv = false).
 *
 * View: for batch index z in [0, batch), row r in [0, rows), column j in
 * [0, cols), the element is x[z*stride_batch + r*stride_row + j*stride_col]
 * (strides in elements, >= 0).  Each row is quantized in blocks of 16
 * consecutive columns; cols % 16 == 0 is required.
 *  - Q or K ([B,H,L,D] contiguous): batch = 1, rows = B*H*L, cols = D,
 *    strides (0, D, 1).
 *  - V blocked along tokens: batch = B*H, rows = D, cols = Lk,
 *    strides (Lk*D, 1, D)  (the transposed view of each head).
 * Outputs (device, dense, caller-owned):
 *  - codes  [batch][rows][cols/2] bytes, 8-byte aligned (each block's 16
 *    nibbles are written as one 8-byte group): element 2i in the low nibble and
 *    2i+1 in the high nibble; nibble = sign bit (bit 3, the input's sign,
 *    also for values that round to 0) | 3-bit E2M1 magnitude code.
 *  - scales [batch][rows][cols/16] bytes: E4M3 codes, sign bit 0.
 *  - deq    [batch][rows][cols] bf16 (may be NULL): the dequantized values
 *    sign * E2M1 * scale, which bf16 represents exactly.
 * Codes and scales are bit-exact round-to-nearest-even results of the exact
 * quotients amax/6 and |x|/s.  Inputs must be finite.
 * Errors: EINVAL for null x/codes/scales, codes not 8-byte aligned, cols % 16
 * != 0, non-positive rows/cols/batch, negative strides, or sizes above 2^40
 * elements.
 */
int attnqat_quantize(const void *x, int64_t batch, int64_t rows, int64_t cols,
                     int64_t stride_batch, int64_t stride_row,
                     int64_t stride_col, uint8_t *codes, uint8_t *scales,
                     void *deq, void *stream);

/*
 * attnqat_quantize_gs -- NVFP4 with an FP32 global scale (the format's
 * linear-layer variant).
 *
 * Defined by: vsqa-test-1.3b metadata.json, "linear_quantization": "NVFP4
 * W4A4: E2M1 values, 16-element blocks, FP8 E4M3 block scales, FP32 global
 * scale", the activation global scale "dynamic, 448*6/max|X| recomputed every
 * forward".  The steps the page leaves open are read as:
 *   G   = float32 2688 / max|x| over the whole view (1 if every element is
 *         zero; the largest finite float32 if the quotient overflows);
 *   k_b = E4M3 code nearest to a_b * G / 6 (a_b = the block's max |x|), ties
 *         to even, saturating at 448;  s_b = its value;
 *   c   = E2M1 code nearest to |x| * G / s_b, ties to even, saturating at 6;
 *   deq = sign * E2M1(c) * s_b / G, rounded to bf16 (nearest, ties to even).
 * Every rounding is exact (a_b G and |x| G are exact in float64).
 *
 * View, codes, scales and deq (bf16, may be NULL): as attnqat_quantize, with
 * scales holding the k_b.  gscale: one device float32, caller-owned, that
 * receives G; it also holds the max-magnitude reduction while the call runs,
 * so it must not alias another argument.  The work is three launches on
 * `stream` (reduce max|x|, quantize, finish G).
 * Errors: as attnqat_quantize, plus EINVAL for a null or misaligned gscale.
 */
int attnqat_quantize_gs(const void *x, int64_t batch, int64_t rows,
                        int64_t cols, int64_t stride_batch, int64_t stride_row,
                        int64_t stride_col, uint8_t *codes, uint8_t *scales,
                        void *deq, float *gscale, void *stream);

/*
 * attnqat_workspace_size -- bytes of device workspace attnqat_fwd and
 * attnqat_bwd need for this shape and flag set (0 for invalid shapes).  Every
 * 16-bit operand of the attention's matrix products is fp16, so the
 * workspace holds fp16 copies of Q, K, V and dO: fq(X) for a quantized
 * operand (exact: sign * E2M1 * E4M3 values lie in [2^-10, 2688] with at most
 * 7 significant bits), else X * 2^e with 2^e a power of two that maps max |X|
 * into [2^13, 2^14) (exact for every element within 2^27 of the largest).  It
 * also holds a float32 copy of O written by the forward, the backward's Delta,
 * 32 bytes of statistics (the max magnitudes behind those powers of two and
 * the bound on |dS|), and -- with Q and K quantized -- their packed NVFP4
 * codes (D/2 bytes per row) with scale tiles (512 bytes per 128 rows x 64
 * columns) for the block-scaled S = fq(Q) fq(K)^T; with all four quantizers
 * on and Lk % 32 == 0 also fq(V)'s packed codes ([B*H][D][Lk/2]
 * bytes, blocks along tokens) and scale tiles (1 KB per 128 tokens) for the
 * forward's block-scaled fq(P~) fq(V).  Every region is 256-byte aligned.
 */
size_t attnqat_workspace_size(int B, int H, int Lq, int Lk, int D,
                              uint32_t flags);

/*
 * attnqat_fwd -- Attn-QAT forward.
 *
 * Inputs q [B,H,Lq,D], k and v [B,H,Lk,D] (bf16, 16-byte aligned), softmax
 * scale sm_scale (finite, > 0; used exactly as given -- FastVideo PR #1457
 * review F1), flags (ATTNQAT_QUANT_*).  Outputs o [B,H,Lq,D] bf16,
 * lse [B,H,Lq] float32 (natural-log LSE of the scaled scores), m [B,H,Lq]
 * float32 (the exact row max of the scaled scores).  ws/ws_bytes: device
 * workspace of at least attnqat_workspace_size(B,H,Lq,Lk,D,flags) bytes,
 * 256-byte aligned; it must be passed unchanged to attnqat_bwd.
 * flags may add ATTNQAT_CAUSAL (then Lq == Lk is required).
 * Shapes: B, H >= 1; B*H <= 65535; Lq >= 1; Lk >= 1; D in {64, 128};
 * B*H*max(Lq,Lk)*128 below 2^40 (offsets are 64-bit).  Lq is arbitrary (the last query tile is masked); a partial
 * last KV tile runs the separate masked tail step.  Lk need not be 16-aligned
 * (the pages' SM100 backward requires it; here a ragged last block of 16 keys
 * or tokens is zero-padded: its missing keys get P~ = 0 and its missing V
 * tokens count as zeros in their fq(V) block).
 * Errors: EINVAL, EUNSUPPORTED (not sm_100, D unsupported), ENOSPC, ECUDA.
 */
int attnqat_fwd(const void *q, const void *k, const void *v, int B, int H,
                int Lq, int Lk, int D, float sm_scale, uint32_t flags, void *o,
                float *lse, float *m, void *ws, size_t ws_bytes, void *stream);

/*
 * attnqat_bwd -- Attn-QAT backward (straight-through estimator).
 *
 * Inputs: q, k, v as given to attnqat_fwd; lse, m as it returned them;
 * dO [B,H,Lq,D] bf16; the same shape, sm_scale and flags; ws as left by
 * attnqat_fwd (it holds fq(Q), fq(K), fq(V) and the float32 O).  Outputs
 * dq [B,H,Lq,D], dk and dv [B,H,Lk,D], bf16.  Delta = rowsum(dO o O) is
 * taken from the forward's float32 O, not from the bf16 o: where a softmax
 * row is peaked, dP - Delta cancels and would amplify the bf16 rounding of
 * O about thirtyfold.
 * Errors as attnqat_fwd.
 */
int attnqat_bwd(const void *q, const void *k, const void *v, const float *lse,
                const float *m, const void *dO, int B, int H, int Lq, int Lk,
                int D, float sm_scale, uint32_t flags, void *dq, void *dk,
                void *dv, void *ws, size_t ws_bytes, void *stream);

/*
 * Block-sparse fine attention (VSA).
 *
 * Defined by: vsqa-test-1.3b metadata.json, "attention": backend
 * VSA_QAT_TRAIN_C128, kind "vsa", cube_shape 4 x 4 x 8 (128-token cubes),
 * "fine": "NVFP4 fake-quant with BF16 matmul" (quantize_fine, quant_p,
 * quant_v), key blocks chosen per query block by a top-k "selection"
 * (effective_topk = max(1, min(ceil((1 - sparsity) * num_blocks),
 * num_blocks)), sparsity 0.9).  Each query tile of ATTNQAT_SPARSE_TILE tokens
 * attends only to the keys of its selected key tiles: the computation above
 * with the softmax (exact max m, sum l, fq(P~) blocks) over those keys alone;
 * fq(Q), fq(K), fq(V) do not depend on the selection.  A query tile with no
 * selected key tile gets O = 0 and m = LSE = -infinity, dQ = 0; a key tile no
 * query tile selects gets dK = dV = 0.  Choosing the tiles (the coarse
 * branch), its gates and the token-to-cube layout belong to the caller:
 * tokens are taken in cube order.
 *
 * tile_mask: device bytes [B][H][ceil(Lq/128)][ceil(Lk/128)], caller-owned,
 * nonzero = the query tile attends the key tile; read, never written.  The
 * backward must receive the mask the forward used.  Other arguments and
 * errors are those of attnqat_fwd / attnqat_bwd (plus EINVAL for a null
 * tile_mask); the workspace is attnqat_sparse_workspace_size() bytes (the
 * dense workspace plus int32 tile lists, 8 * B*H*nq*nk + 4 * B*H*(nq + nk)
 * bytes, rebuilt from the mask by every call), passed unchanged from
 * attnqat_sparse_fwd to attnqat_sparse_bwd.  ATTNQAT_CAUSAL is not accepted
 * here (EINVAL; the workspace size is 0).
 */
#define ATTNQAT_SPARSE_TILE 128
/* The tile-64 profile (fastvideo-kernel triton_kernels commit: the FP4
 * sparse-attention emulator's tile-64 and tile-128 profiles; vsqa-test-1.3b
 * metadata.json, attention.physical_block_tokens = 64): with this flag on the
 * sparse calls, tile_mask has 64-token granularity,
 * [B][H][ceil(Lq/64)][ceil(Lk/64)], and query block I attends exactly the
 * keys of its selected 64-token key blocks; everything else is as for
 * 128-token tiles (the workspace size is the same).  Not accepted by the
 * dense calls or with ATTNQAT_CAUSAL (EINVAL). */
#define ATTNQAT_TILE64 64u
size_t attnqat_sparse_workspace_size(int B, int H, int Lq, int Lk, int D,
                                     uint32_t flags);
int attnqat_sparse_fwd(const void *q, const void *k, const void *v, int B,
                       int H, int Lq, int Lk, int D, float sm_scale,
                       uint32_t flags, const uint8_t *tile_mask, void *o,
                       float *lse, float *m, void *ws, size_t ws_bytes,
                       void *stream);
int attnqat_sparse_bwd(const void *q, const void *k, const void *v,
                       const float *lse, const float *m, const void *dO, int B,
                       int H, int Lq, int Lk, int D, float sm_scale,
                       uint32_t flags, const uint8_t *tile_mask, void *dq,
                       void *dk, void *dv, void *ws, size_t ws_bytes,
                       void *stream);

/*
 * attnqat_vsa_select -- the key tiles each query tile of the block-sparse
 * attention attends to (the tile mask attnqat_sparse_fwd takes).
 *
 * Defined by: vsqa-test-1.3b metadata.json, "attention.selection": top-k key
 * cubes per query cube, effective_topk = max(1, min(ceil((1 - sparsity) *
 * num_blocks), num_blocks)) at sparsity 0.9 (the "top-p" mode field stands
 * beside that count); "attention.precision.coarse": BF16, not quantized.
 * The page names the fields, not the arithmetic; read as: each 128-token tile
 * is summarised by the mean of its valid rows; the coarse score of (query tile
 * I, key tile J) is the dot product of the two means (a softmax and its scale
 * keep the order); query tile I keeps the `topk` key tiles of highest score,
 * ties to the lower J (topk above the tile count keeps every tile).  The
 * ranking is computed in float32 with every step ordered -- rows summed in
 * token order, one correctly rounded division by the row count, channels
 * accumulated in order with one fused multiply-add each -- so it is
 * reproducible bit for bit.
 *
 * q [B,H,Lq,D], k [B,H,Lk,D] bf16 (16-byte aligned); topk >= 1 (the caller
 * evaluates the page's effective_topk); tile_mask: device bytes
 * [B][H][ceil(Lq/128)][ceil(Lk/128)], written with 0 or 1.  ws: device
 * workspace of attnqat_vsa_select_workspace_size() bytes, 256-byte aligned
 * (tile means and scores).  Two launches on `stream`.  Inputs must be finite.
 * Errors: EINVAL (null or misaligned pointer, bad shape, topk < 1),
 * EUNSUPPORTED, ENOSPC, ECUDA.
 */
size_t attnqat_vsa_select_workspace_size(int B, int H, int Lq, int Lk, int D);
int attnqat_vsa_select(const void *q, const void *k, int B, int H, int Lq,
                       int Lk, int D, int topk, uint8_t *tile_mask, void *ws,
                       size_t ws_bytes, void *stream);

/* The same selection over `tile`-token tiles, tile = 128 (as above) or 64
 * (the tile-64 profile, whose mask feeds the sparse calls with
 * ATTNQAT_TILE64): tile_mask is [B][H][ceil(Lq/tile)][ceil(Lk/tile)] and topk
 * counts tile-token key tiles.  The workspace (tile means and scores) is
 * attnqat_vsa_select_tiles_workspace_size() bytes (0 for a tile other than
 * 64 or 128).  Errors as attnqat_vsa_select, plus EINVAL for another tile. */
size_t attnqat_vsa_select_tiles_workspace_size(int B, int H, int Lq, int Lk,
                                               int D, int tile);
int attnqat_vsa_select_tiles(const void *q, const void *k, int B, int H,
                             int Lq, int Lk, int D, int tile, int topk,
                             uint8_t *tile_mask, void *ws, size_t ws_bytes,
                             void *stream);

/*
 * attnqat_fwd_noalloc -- attnqat_fwd for callers that cannot allocate.
 *
 * The pages have no counterpart of this entry point; it exists for callers
 * that cannot hand the library a device workspace -- e.g. a framework whose
 * caching allocator already holds nearly all device memory, code running
 * inside an allocator or memory-pressure callback, or a plain C host without
 * a device allocator.  It computes exactly what attnqat_fwd computes, with the
 * same arguments minus ws/ws_bytes: the workspace is a fixed block of
 * ATTNQAT_NOALLOC_WS_MAX bytes of device memory that the library carries as a
 * static __device__ array (held on every GPU that loads the library, until
 * the process exits).  It calls no cudaMalloc, cudaFree or other allocating
 * routine.
 *  - Shapes with attnqat_workspace_size(...) > ATTNQAT_NOALLOC_WS_MAX return
 *    ATTNQAT_ENOSPC; invalid arguments return the code attnqat_fwd returns
 *    for them (EINVAL, or EUNSUPPORTED for a head dimension it lacks or a
 *    device that is not sm_100).
 *  - The first call on each device looks up the block's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before capturing the stream into a CUDA graph.  The address is kept per
 *    device and CUDA context: after a cudaDeviceReset the next call looks it
 *    up again (so, again, before any capture).
 *  - All calls share the block and it keeps the last call's contents (the
 *    parts that must start at zero are cleared on the caller's stream).
 *    Calls whose GPU work overlaps -- two streams, or several host threads on
 *    one device -- race on it: serialise them.
 *  - The workspace is internal, so the result cannot be passed to
 *    attnqat_bwd; use attnqat_fwd for training.
 */
#define ATTNQAT_NOALLOC_WS_MAX ((size_t)32 << 20)
int attnqat_fwd_noalloc(const void *q, const void *k, const void *v, int B,
                        int H, int Lq, int Lk, int D, float sm_scale,
                        uint32_t flags, void *o, float *lse, float *m,
                        void *stream);

#ifdef __cplusplus
}
#endif
#endif /* ATTNQAT_H */
