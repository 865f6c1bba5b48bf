// fwd.cu -- Attn-QAT forward kernel for sm_100a.
//
// One CTA per (128-query tile, batch*head).  384 threads in four roles:
//   warp 0      TMA producer: the Q tile once, then K tiles for the row-max
//               sweep and K, fq(V) tiles for the output sweep.  With Q and K
//               quantized these are the packed NVFP4 codes plus their scale
//               tiles (8-stage K ring) and S is a block-scaled NVFP4 MMA;
//               otherwise fp16 tiles.  fq(V): with every quantizer on (Lk %
//               32 == 0) its packed codes and scale tiles (4-stage ring) for
//               a block-scaled NVFP4 P V (N = D), else fp16 tiles (2-stage
//               ring, 128-byte swizzle);
//   warps 1, 10 tcgen05.mma issuers (one thread each; warp 1 owns TMEM): A
//               issues even row-max tiles and the output sweep's S, B the odd
//               row-max tiles and P V (one thread alone cannot issue fast
//               enough to keep the tensor pipe busy);
//   warps 2..9  row warps, two per TMEM lane quarter: each query row (TMEM
//               lane) has two threads owning 64 columns each -- row max, exp,
//               row sum, in-register NVFP4 fq of P~ in 16-key blocks, the P
//               tile (packed codes and scale bytes, or fp16 values) to
//               shared memory, and the O epilogue; the pair merges its
//               partial max and sum through shared memory.
// Every 16-bit MMA operand is fp16: fq(Q), fq(K), fq(V) and fq(P~) are exact
// in fp16 as they are; an operand whose quantizer is off is copied as
// X * 2^e (a power of two that maps its max magnitude into [2^13, 2^14),
// exact for every element within 2^27 of the largest), and the powers of two
// are divided out of S and O.
//   warp 11     idle (pads the CTA to whole groups of four warps).
// TMEM columns: S buffers [0,256) (plus [256,384) during the row-max sweep,
// before O exists), O accumulator [256, 256+D), scale factors from 384.
//
// The row max is exact over all keys, taken in a first sweep of S = Q K^T,
// so fq(P~) sees the reference-order statistics and O needs no rescaling
// (FastVideo "Attn-QAT Training" guide, "Architecture-specific Triton
// routing": FWD_EXACT_M recomputes reference-order softmax statistics).  Full
// KV tiles run without bounds masks; the partial last KV tile runs a
// separate masked step (fastvideo-kernel triton_kernels commit, SM100
// Attn-QAT route).
//
// Block-sparse (VSA fine attention): with a.kv_list set, the CTA walks only
// the key tiles listed for its query tile, in both sweeps, so m is the exact
// max over the selected keys; a query tile with no key tile writes O = 0 and
// m = LSE = -inf.  Causal masking walks the lower triangle the same way and
// masks its last tile, the diagonal, to keys <= the query row.
#include "common.cuh"
#include "internal.h"

namespace attnqat {

// Shared-memory and TMEM layout of the forward.  With FP4S the Q and K tiles
// are packed NVFP4 codes (D/2 bytes per row, TMA swizzle of D/2 bytes) and
// their 16-element scales (512-byte scale-factor blocks per 64 columns); S is
// then a block-scaled kind::mxf4nvf4 MMA.  Otherwise Q and K are fp16 tiles.
// With PV4 the P V product is block-scaled NVFP4 too: fq(P~) blocks run along
// keys and fq(V) blocks along tokens, both the K axis of P V, so the P tile
// holds packed codes (64 bytes per query row, 64-byte swizzle) plus scale
// blocks, and the V stages hold fq(V)'s codes ([D][128 keys / 2]) and scales.
template <int D, int FP4S, int PV4>
struct FwdLayout {
  // K ring stages: the row-max sweep consumes a K tile every few hundred ns,
  // so the 9 KB NVFP4 stages are kept deep enough to cover the TMA latency
  static constexpr int kNSK = FP4S ? 8 : 2;
  static constexpr int kNSV = PV4 ? 4 : 2;              // V ring stages
  static constexpr int kQKRow = FP4S ? D / 2 : 2 * D;   // bytes per Q/K row
  static constexpr int kQK = 128 * kQKRow;              // bytes per Q/K tile
  static constexpr int kSF = FP4S ? (D / 64) * 512 : 0;  // scale-factor bytes per tile
  static constexpr int kVT = PV4 ? D * 64 : Tile<D>::kBytes;
  static constexpr int kVSF = PV4 ? 1024 : 0;           // 128 keys = two 64-key scale blocks
  static constexpr int kPBytes = PV4 ? kBM * 64 : kBM * kBN * 2;
  static constexpr int kPSF = PV4 ? 1024 : 0;
  // P slots: three for the 8 KB NVFP4 P tiles (the rows then never wait for
  // the P V two tiles back), two for fp16 P (or one P split into hi and lo)
  static constexpr int kNPB = PV4 ? 3 : 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQK;
  static constexpr int kV = (kK + kNSK * kQK + 1023) / 1024 * 1024;
  static constexpr int kP = kV + kNSV * kVT;
  static constexpr int kQSF = kP + kNPB * kPBytes;
  static constexpr int kKSF = kQSF + kSF;
  static constexpr int kVSFo = kKSF + kNSK * kSF;
  static constexpr int kPSFo = kVSFo + kNSV * kVSF;
  static constexpr int kBar = kPSFo + kNPB * kPSF;
  static constexpr int kBarBytes = 2048;  // FwdBars (checked at the launch)
  static constexpr int kBytes = kBar + kBarBytes;
  static constexpr int kDynSmem = kBytes + 1024;        // slack for 1024-byte alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 256;
  static constexpr uint32_t kSFCols = (D / 64) * 4;     // TMEM columns of one tile's scales
  // sweep 1 (row max) rotates S through three buffers: columns 0, 128 and
  // 256 (the O accumulator's columns, unused until sweep 2's first P V);
  // sweep 2 uses the first two.  Scale factors sit above all of them.
  static constexpr int kNS1 = 3;
  static constexpr uint32_t kTmemSFA = 384;
  static constexpr uint32_t kTmemSFB = kTmemSFA + kSFCols;            // kNSK stages
  static constexpr uint32_t kTmemSFP = kTmemSFB + kNSK * kSFCols;     // PV4: kNPB P slots x 8
  static constexpr uint32_t kTmemSFV = kTmemSFP + (PV4 ? 8 * kNPB : 0);  // PV4: kNSV stages x 8
  static constexpr uint32_t kTmemEnd = kTmemSFV + (PV4 ? 8 * kNSV : 0);
  // UMMA layout of the packed tiles: 64-byte rows swizzle 64B, 32-byte rows 32B
  static constexpr uint32_t kCodeLayout = (D / 2 == 64) ? 4u : 6u;
  static constexpr uint32_t kCodeSBO = 8 * (D / 2);
};

// Row warps per TMEM lane quarter in the forward: 2, each owning 64 of the
// 128 columns.  (4 per quarter, 32 columns each, measured no faster: the
// forward is not limited by how many row warps hide latency.)
constexpr int kFwdG = 2;

struct FwdBars {
  uint64_t qfull;
  uint64_t kfull[8], kempty[8], vfull[4], vempty[4];   // sized for the deepest rings
  uint64_t sfull1[3], sempty1[3];   // sweep-1 S buffers
  uint64_t sfull[2], sempty[2], pfull[3], pempty[3];
  uint64_t ofull;
  uint64_t sfa_ready;   // issuer A's copy of the Q scales into TMEM has landed
  uint64_t adone;       // issuer A's MMAs have completed (drained before TMEM is freed)
  uint32_t tmem_slot;
  int abort;
  float part[kFwdG][kBM];   // per-row partial max / sum of the column groups
};

// Row max over this thread's NC columns (col0..col0+NC-1) of one S tile.
template <bool MASKED, int NC>
__device__ __forceinline__ float row_max_cols(uint32_t taddr, int col0, int valid) {
  float mx = -INFINITY;
  uint32_t r[NC / 32][32];
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) tmem_ld32(taddr + col0 + 32 * c, r[c]);
  tmem_ld_wait();
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float a = (!MASKED || col0 + 32 * c + i < valid) ? __uint_as_float(r[c][i]) : -INFINITY;
      const float b = (!MASKED || col0 + 32 * c + i + 1 < valid) ? __uint_as_float(r[c][i + 1]) : -INFINITY;
      mx = fmax3(mx, a, b);
    }
  }
  return mx;
}

// Sweep-2 work for this thread's NC columns of one S tile: P~ = exp2(S*cl +
// nml), partial row sum, and fq(P~) (or P~ itself) written as columns
// col0..col0+NC-1 of row `row` of the P tile at `pbase`.
// PV4 selects the P tile's form: packed NVFP4 codes (64-byte rows, 64-byte
// swizzle) with the E4M3 scale bytes at `psf` in the layout tcgen05.cp moves
// into TMEM; otherwise fp16 values in 128-byte swizzled chunks of 64 columns.
// With P unquantized (QP = 0) P~ itself is the operand and fp16 would round
// it to 11 bits; the product is then taken as hi V + lo V with hi = fp16(P~)
// and lo = fp16(P~ - hi), stored as two tiles (`lo_off` bytes apart), which
// carries P~ to about 22 bits.  (Where dP - Delta cancels, Delta = dO . O
// would otherwise inherit the fp16 rounding of P~ about thirtyfold.)
// ZERO: every column of the thread is masked (an unselected 64 x 64
// quadrant; warp-uniform): no TMEM load, zeros stored, l += 0.
template <int PV4, int QP, bool MASKED, int NC, bool ZERO = false>
__device__ __forceinline__ float prob_cols(uint32_t taddr, int col0, int valid, float cl, float nml,
                                           uint32_t pbase, uint32_t psf, uint32_t row, uint32_t lo_off) {
  static_assert(!PV4 || (QP && NC == 64), "NVFP4 P V needs quantized P and 64 columns per thread");
  uint32_t sfw = 0;  // PV4: this thread's four scale bytes
  float2 lsum = make_float2(0.0f, 0.0f);
  const float2 cl2 = make_float2(cl, cl), nml2 = make_float2(nml, nml);
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) {
    uint32_t r[32];
    if (!ZERO) {
      tmem_ld32(taddr + col0 + c * 32, r);
      tmem_ld_wait();
    }
    float p[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (ZERO) {
        p[2 * i] = p[2 * i + 1] = 0.0f;
        continue;
      }
      const float2 x = fma2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), cl2, nml2);
      const float e0 = ex2_approx(x.x), e1 = ex2_approx(x.y);
      p[2 * i] = (!MASKED || col0 + c * 32 + 2 * i < valid) ? e0 : 0.0f;
      p[2 * i + 1] = (!MASKED || col0 + c * 32 + 2 * i + 1 < valid) ? e1 : 0.0f;
      lsum = add2(lsum, make_float2(p[2 * i], p[2 * i + 1]));
    }
    if (PV4) {
      // two 16-key blocks -> 16 bytes of codes (the 16-byte unit cc/32 of the
      // row's 64 bytes, swizzled as TMA's 64-byte mode) and two scale bytes
      uint32_t cw[4] = {0u, 0u, 0u, 0u};
      uint32_t s0 = 0u, s1 = 0u;
      if (!ZERO) {
        s0 = fq4_probs(p, *reinterpret_cast<uint32_t(*)[2]>(cw));
        s1 = fq4_probs(p + 16, *reinterpret_cast<uint32_t(*)[2]>(cw + 2));
      }
      sfw |= (s0 | (s1 << 8)) << (16 * c);
      const int unit = (col0 + 32 * c) >> 5;
      st_shared_v4(pbase + (row >> 3) * 512 + (row & 7) * 64 + ((unit ^ ((row >> 1) & 3)) << 4), cw[0], cw[1],
                   cw[2], cw[3]);
    } else {
      uint32_t w[16], wl[16];
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        if (ZERO) {
#pragma unroll
          for (int i = 0; i < 8; ++i) w[8 * b + i] = wl[8 * b + i] = 0u;
        } else if (QP) {
          uint32_t rr[8];
          const uint32_t s2 = f16x2_broadcast(fq16_probs(p + 16 * b, rr));
#pragma unroll
          for (int i = 0; i < 8; ++i) w[8 * b + i] = hmul2_u32(rr[i], s2);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 x = make_float2(p[16 * b + 2 * i], p[16 * b + 2 * i + 1]);
            w[8 * b + i] = pack_f16x2(x.x, x.y);
            const float2 h = unpack_f16x2(w[8 * b + i]);
            wl[8 * b + i] = pack_f16x2(x.x - h.x, x.y - h.y);  // x - h is exact in float
          }
        }
      }
      // 32 keys = four 16-byte units of the 64-key swizzled chunk holding them
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int cc = col0 + 32 * c;
        const uint32_t addr = pbase + static_cast<uint32_t>(cc >> 6) * kChunkBytes +
                              sw128_offset(row, ((cc & 63) >> 3) + u);
        st_shared_v4(addr, w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        if (!QP) st_shared_v4(addr + lo_off, wl[4 * u], wl[4 * u + 1], wl[4 * u + 2], wl[4 * u + 3]);
      }
    }
  }
  if (PV4) {
    // this thread's 64 keys are one 64-key scale block (k-chunk col0 / 64):
    // row r's four bytes at (r % 32) * 16 + (r / 32) * 4
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(psf + static_cast<uint32_t>(col0 >> 6) * 512 + (row & 31) * 16 +
                                                   (row >> 5) * 4),
                 "r"(sfw)
                 : "memory");
  }
  return lsum.x + lsum.y;
}

// Synchronises the G row warps of one TMEM lane quarter (named barrier
// 1 + lane quarter), around the shared-memory merge of per-row partials.
template <int G>
__device__ __forceinline__ void group_sync(int wq) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + wq), "n"(32 * G) : "memory");
}

// Threads of a forward CTA with G row warps per TMEM lane quarter: producer,
// MMA issuer A, 4G row warps, MMA issuer B (warp 2 + 4G), padded to whole
// groups of four warps.
template <int G>
constexpr int fwd_threads() { return (2 + 4 * G + 1 + 3) / 4 * 128; }

// SP: 0 dense; 1 block-sparse (walks a.kv_list); 2 causal (walks the
// lower-triangle lists and masks the diagonal); 3 block-sparse with 64-token
// masks (list entries carry quadrant bits).  Separate instantiations, so the
// dense kernel carries none of the list handling.
template <int D, int FP4S, int PV4, int QP, int G, int SP>
__global__ void __launch_bounds__(fwd_threads<G>(), 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using L = FwdLayout<D, FP4S, PV4>;
  // unquantized P: one P slot holding the hi and lo tiles (the two P buffers'
  // space), handed over once per key tile
  constexpr bool PSPLIT = !QP;
  // P slots in use: one (hi at the slot, lo at the next), else the layout's
  constexpr int kNP = PSPLIT ? 1 : L::kNPB;
  static_assert(!(PSPLIT && PV4), "the NVFP4 P V takes quantized P");
  static_assert(G <= kFwdG, "column groups beyond the partial-sum block");
  static_assert(L::kNSK <= 8 && L::kNSV <= 4, "ring deeper than its barrier arrays");
  constexpr int kNSK = L::kNSK, kNSV = L::kNSV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  FwdBars *bars = reinterpret_cast<FwdBars *>(smem + L::kBar);
  volatile int *abort = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x;
  const int bh = blockIdx.y;
  const int nk = a.nk_tiles;
  // the key tiles this query tile visits: all nk, or its block-sparse list
  const size_t qrow = static_cast<size_t>(bh) * a.nq_tiles + qt;
  const int32_t *kvl = SP ? a.kv_list + qrow * nk : nullptr;
  const int n = SP ? a.kv_count[qrow] : nk;
  // SP 3 (64-token masks): list entries carry quadrant bits in the top byte
  auto ktile = [&](int j) -> int { return SP == 3 ? (__ldg(kvl + j) & 0xFFFFFF) : (SP ? __ldg(kvl + j) : j); };

  if (threadIdx.x == 0) {
    mbar_init(&bars->qfull, 1);
    for (int s = 0; s < kNSK; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
    }
    for (int s = 0; s < kNSV; ++s) {
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&bars->sfull1[b], 1);
      mbar_init(&bars->sempty1[b], 4 * G);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->sfull[b], 1);
      mbar_init(&bars->sempty[b], 4 * G);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&bars->pfull[b], 4 * G);
      mbar_init(&bars->pempty[b], 1);
    }
    mbar_init(&bars->ofull, 1);
    mbar_init(&bars->sfa_ready, 1);
    mbar_init(&bars->adone, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      // Q (or its packed codes and scales) once
      auto load_qk = [&](uint8_t *dst, const CUtensorMap *map, uint64_t *bar, int row0) {
        if (FP4S) {
          tma_load_3d(dst, map, bar, 0, row0, bh);
        } else {
          for (int c = 0; c < Tile<D>::kChunks; ++c) tma_load_3d(dst + c * kChunkBytes, map, bar, c * 64, row0, bh);
        }
      };
      mbar_arrive_expect_tx(&bars->qfull, L::kQK + L::kSF);
      load_qk(smem + L::kQ, &tmQ, &bars->qfull, qt * kBM);
      if (FP4S)
        bulk_load(smem + L::kQSF, a.qsf + (static_cast<size_t>(bh) * a.nq_tiles + qt) * L::kSF, L::kSF,
                  &bars->qfull);
      int kissued = 0, vissued = 0;
      for (int t = 0; t < 2 * n; ++t) {
        const int j = ktile(t < n ? t : t - n);
        const int st = t % kNSK;
        if (t >= kNSK && !mbar_wait(&bars->kempty[st], ((t / kNSK) - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars->kfull[st], L::kQK + L::kSF);
        load_qk(smem + L::kK + st * L::kQK, &tmK, &bars->kfull[st], j * kBN);
        if (FP4S)
          bulk_load(smem + L::kKSF + st * L::kSF, a.ksf + (static_cast<size_t>(bh) * nk + j) * L::kSF, L::kSF,
                    &bars->kfull[st]);
        kissued = t + 1;
        if (t >= n) {
          const int u = t - n;
          const int vs = u % kNSV;
          if (u >= kNSV && !mbar_wait(&bars->vempty[vs], ((u / kNSV) - 1) & 1, abort)) break;
          mbar_arrive_expect_tx(&bars->vfull[vs], L::kVT + L::kVSF);
          if (PV4) {
            // fq(V) codes [D][128 keys / 2] and the tile's two scale blocks
            tma_load_3d(smem + L::kV + vs * L::kVT, &tmV, &bars->vfull[vs], j * (kBN / 2), 0, bh);
            bulk_load(smem + L::kVSFo + vs * L::kVSF, a.vsf + (static_cast<size_t>(bh) * nk + j) * L::kVSF, L::kVSF,
                      &bars->vfull[vs]);
          } else {
            for (int c = 0; c < Tile<D>::kChunks; ++c)
              tma_load_3d(smem + L::kV + vs * L::kVT + c * kChunkBytes, &tmV, &bars->vfull[vs],
                          c * 64, j * kBN, bh);
          }
          vissued = u + 1;
        }
      }
      if (*abort) {
        // let the copies already issued land before the CTA exits
        for (int t = (kissued > kNSK ? kissued - kNSK : 0); t < kissued; ++t)
          mbar_wait_drain(&bars->kfull[t % kNSK], (t / kNSK) & 1);
        for (int u = (vissued > kNSV ? vissued - kNSV : 0); u < vissued; ++u)
          mbar_wait_drain(&bars->vfull[u % kNSV], (u / kNSV) & 1);
      }
    }
  } else if (warp == 1 || warp == 2 + 4 * G) {
    // ---------------------------------------------------------------- MMA --
    // Two issuing threads (one thread issues a tcgen05 instruction only every
    // ~50-60 cycles): A issues the even tiles of the row-max sweep and every
    // S of the output sweep, B the odd row-max tiles and every P V.
    if (lane == 0) {
      const bool issuer_a = warp == 1;
      constexpr uint32_t idS = FP4S ? idesc_mxf4(kBM, kBN) : idesc_f16(kBM, kBN, false, false, false);
      constexpr uint32_t idPV = idesc_f16(kBM, D, false, false, true);
      const uint32_t qaddr = sbase + L::kQ;
      bool ok = mbar_wait(&bars->qfull, 0, abort);
      if (FP4S) {
        if (issuer_a) {
          // scales of the Q tile into TMEM once; B waits for them to land
          if (ok) {
            tc_fence_after();
            for (int kc = 0; kc < D / 64; ++kc)
              tmem_cp_32x128b_x4(tmem + L::kTmemSFA + kc * 4, sdesc_make(sbase + L::kQSF + kc * 512, 16, 128, 0));
          }
          umma_commit(&bars->sfa_ready);
        } else {
          ok = ok && mbar_wait(&bars->sfa_ready, 0, abort);
        }
      }
      // operand descriptors of the tiles' base addresses
      const uint64_t dQ = FP4S ? sdesc_make(qaddr, 16, L::kCodeSBO, L::kCodeLayout) : desc_k(qaddr);
      const uint64_t dK = FP4S ? sdesc_make(sbase + L::kK, 16, L::kCodeSBO, L::kCodeLayout) : desc_k(sbase + L::kK);
      const uint64_t dKSF = sdesc_make(sbase + L::kKSF, 16, 128, 0);
      const uint64_t dP = desc_k(sbase + L::kP), dV = desc_mn(sbase + L::kV);
      const uint64_t dP4 = sdesc_make(sbase + L::kP, 16, 512, 4), dV4 = sdesc_make(sbase + L::kV, 16, 512, 4);
      const uint64_t dPSF = sdesc_make(sbase + L::kPSFo, 16, 128, 0), dVSF = sdesc_make(sbase + L::kVSFo, 16, 128, 0);
      constexpr uint32_t idPV4 = idesc_mxf4(kBM, D);
      // S tile t (the t-th K tile loaded) into TMEM column dcol, signalling `full`
      auto issue_s = [&](int t, uint32_t dcol, uint64_t *full) -> bool {
        const int st = t % kNSK;
        if (!mbar_wait(&bars->kfull[st], (t / kNSK) & 1, abort)) return false;
        tc_fence_after();
        const uint64_t dKs = sdesc_add(dK, st * L::kQK);
        if (FP4S) {
          const uint32_t sfb = tmem + L::kTmemSFB + st * L::kSFCols;
#pragma unroll
          for (int kc = 0; kc < D / 64; ++kc) tmem_cp_32x128b_x4(sfb + kc * 4, sdesc_add(dKSF, st * L::kSF + kc * 512));
#pragma unroll
          for (int kk = 0; kk < D / 64; ++kk)
            umma_fp4(tmem + dcol, sdesc_add(dQ, kk * 32), sdesc_add(dKs, kk * 32), idS, tmem + L::kTmemSFA + kk * 4,
                     sfb + kk * 4, kk > 0 ? 1u : 0u);
        } else {
          mma_kmajor<D / 16>(tmem + dcol, dQ, dKs, idS, false);
        }
        umma_commit(&bars->kempty[st]);
        umma_commit(full);
        return true;
      };
      // row-max sweep: three S buffers, tiles alternating between A and B
      for (int t = issuer_a ? 0 : 1; ok && t < n; t += 2) {
        const int b = t % L::kNS1;
        if (t >= L::kNS1 && !mbar_wait(&bars->sempty1[b], ((t / L::kNS1) - 1) & 1, abort)) { ok = false; break; }
        ok = issue_s(t, b * kBN, &bars->sfull1[b]);
      }
      if (issuer_a) {
        // every row-max buffer read before the output sweep reuses columns 0..255
        for (int t = (n > L::kNS1 ? n - L::kNS1 : 0); ok && t < n; ++t)
          ok = mbar_wait(&bars->sempty1[t % L::kNS1], (t / L::kNS1) & 1, abort);
        // output sweep: S into two buffers
        for (int j = 0; ok && j < n; ++j) {
          const int sb = j & 1;
          if (j >= 2 && !mbar_wait(&bars->sempty[sb], ((j >> 1) - 1) & 1, abort)) { ok = false; break; }
          ok = issue_s(n + j, sb * kBN, &bars->sfull[sb]);
        }
        // TMEM is freed by this warp: let its own MMAs finish first
        umma_commit(&bars->adone);
        mbar_wait_drain(&bars->adone, 0);
      } else {
        // output sweep: O += fq(P~)_j fq(V)_j as the rows hand over each P tile
        // (the first P V runs after every row-max tile was read, so it may
        // overwrite the third S buffer's columns)
        for (int j = 0; ok && j < n; ++j) {
          const int pb = j % kNP;
          const int vs = j % kNSV;
          const uint32_t pph = (j / kNP) & 1;
          if (!mbar_wait(&bars->pfull[pb], pph, abort) || !mbar_wait(&bars->vfull[vs], (j / kNSV) & 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (PV4) {
            // scales of this P tile and V stage into TMEM (their previous
            // users, P V two and kNSV tiles back, have completed: the rows
            // and the producer waited for them before refilling)
            const uint32_t sfp = tmem + L::kTmemSFP + pb * 8, sfv = tmem + L::kTmemSFV + vs * 8;
#pragma unroll
            for (int kc = 0; kc < 2; ++kc) {
              tmem_cp_32x128b_x4(sfp + kc * 4, sdesc_add(dPSF, pb * L::kPSF + kc * 512));
              tmem_cp_32x128b_x4(sfv + kc * 4, sdesc_add(dVSF, vs * L::kVSF + kc * 512));
            }
            const uint64_t dPs = sdesc_add(dP4, pb * L::kPBytes), dVs = sdesc_add(dV4, vs * L::kVT);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              umma_fp4(tmem + L::kTmemO, sdesc_add(dPs, kk * 32), sdesc_add(dVs, kk * 32), idPV4, sfp + kk * 4,
                       sfv + kk * 4, (j > 0 || kk > 0) ? 1u : 0u);
          } else {
            mma_a_k_b_mn<kBN / 16>(tmem + L::kTmemO, sdesc_add(dP, pb * L::kPBytes), sdesc_add(dV, vs * L::kVT),
                                   idPV, j > 0);
            // the lo tile (second P buffer): O += lo V
            if (PSPLIT)
              mma_a_k_b_mn<kBN / 16>(tmem + L::kTmemO, sdesc_add(dP, L::kPBytes), sdesc_add(dV, vs * L::kVT), idPV,
                                     true);
          }
          umma_commit(&bars->vempty[vs]);
          umma_commit(&bars->pempty[pb]);
        }
        // ofull tracks completion of every P V, so the epilogue and the TMEM
        // release never race one in flight (the rows have read every S)
        umma_commit(&bars->ofull);
      }
    }
  } else if (warp >= 2 && warp < 2 + 4 * G) {
    // ---------------------------------------------------------- row warps --
    constexpr int NC = kBN / G;  // columns per thread
    const RowRole rr(warp, lane);
    const int col0 = rr.half * NC;
    const int last_valid = a.Lk - (nk - 1) * kBN;  // keys in the last KV tile
    // the lists ascend, so only the last tile visited can be the partial one;
    // with causal masking the last tile is the diagonal, where row r keeps
    // keys 0..r (which also covers a partial diagonal tile: Lq == Lk)
    const bool tail_last = SP == 2 ? true : (n > 0 && ktile(n - 1) == nk - 1 && last_valid < kBN);
    const int last_cols = SP == 2 ? static_cast<int>(rr.row) + 1 : last_valid;
    // SP 3: this thread's quadrant bit (its query half, its 64-key half); a
    // clear bit masks every column it owns (valid bound = col0).  The bit is
    // the same for the 32 rows and the column group of one warp, and so is
    // "last tile": the branch between the masked and the plain column loops
    // is taken on those two alone, never on the per-row bound, because both
    // loops hold warp-collective TMEM loads (a causal diagonal row 127 has
    // bound kBN but must stay on its warp's masked path).
    static_assert(SP != 3 || NC == 64, "quadrant masks need 64 columns per thread");
    const int qbit = (static_cast<int>(rr.row) >> 6) * 2 + (col0 >> 6);
    auto quad_clear = [&](int j) -> bool { return SP == 3 && !((__ldg(kvl + j) >> (24 + qbit)) & 1); };
    float mrow = -INFINITY;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int b = j % L::kNS1;
      const bool clear = quad_clear(j);
      const bool masked = clear || (tail_last && j == n - 1);  // warp-uniform
      const int vb = clear ? col0 : last_cols;
      if (!mbar_wait(&bars->sfull1[b], (j / L::kNS1) & 1, abort)) { ok = false; break; }
      tc_fence_after();
      const uint32_t taddr = tmem + rr.lane_addr + b * kBN;
      // an unselected quadrant adds -inf without reading S
      const float mx = clear ? -INFINITY
                             : (masked ? row_max_cols<true, NC>(taddr, col0, vb) : row_max_cols<false, NC>(taddr, col0, kBN));
      mrow = fmaxf(mrow, mx);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->sempty1[b]);
    }
    // every column group of a row sees every tile, so all reach this merge
    bars->part[rr.half][rr.row] = mrow;
    group_sync<G>(rr.wq);
#pragma unroll
    for (int g = 0; g < G; ++g) mrow = fmaxf(mrow, bars->part[g][rr.row]);
    group_sync<G>(rr.wq);
    // S arrives as S * 2^(eq + ek) when Q or K is a scaled fp16 copy (both
    // factors are 1 for quantized operands): dividing the powers of two out
    // of c is exact, so m and P~ are the same bits either way
    const float sqk = FP4S ? 1.0f : operand_scale(a.amax_q) * operand_scale(a.amax_k);
    const float m_scaled = mrow * (a.sm_scale / sqk);
    const float nml = -(m_scaled * kLog2e);
    const float cl = a.scale_log2 / sqk;
    float lsum = 0.0f;
    for (int j = 0; ok && j < n; ++j) {
      const int sb = j & 1;
      const int pb = j % kNP;
      const bool clear = quad_clear(j);
      const bool masked = clear || (tail_last && j == n - 1);  // warp-uniform
      const int vb = clear ? col0 : last_cols;
      if (!mbar_wait(&bars->sfull[sb], (j >> 1) & 1, abort)) { ok = false; break; }
      if (j >= kNP && !mbar_wait(&bars->pempty[pb], ((j / kNP) - 1) & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + rr.lane_addr + sb * kBN;
      const uint32_t pbase = sbase + L::kP + pb * L::kPBytes;
      const uint32_t psf = sbase + L::kPSFo + pb * L::kPSF;
      if (SP == 3 && clear)  // an unselected quadrant: zeros, without reading S
        lsum += prob_cols<PV4, QP, true, NC, true>(taddr, col0, vb, cl, nml, pbase, psf, rr.row, L::kPBytes);
      else if (masked)
        lsum += prob_cols<PV4, QP, true, NC>(taddr, col0, vb, cl, nml, pbase, psf, rr.row, L::kPBytes);
      else
        lsum += prob_cols<PV4, QP, false, NC>(taddr, col0, kBN, cl, nml, pbase, psf, rr.row, L::kPBytes);
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->sempty[sb]);
        mbar_arrive(&bars->pfull[pb]);
      }
    }
    // ------------------------------------------------------------ epilogue --
    if (ok && mbar_wait(&bars->ofull, 0, abort)) {
      bars->part[rr.half][rr.row] = lsum;
      group_sync<G>(rr.wq);
      lsum = 0.0f;
#pragma unroll
      for (int g = 0; g < G; ++g) lsum += bars->part[g][rr.row];
      tc_fence_after();
      const int q = qt * kBM + static_cast<int>(rr.row);
      // no key tile selected: O = 0 (the accumulator was never written),
      // m = LSE = -inf.  A scaled fp16 copy of V leaves O * 2^ev in TMEM.
      // With quadrant masks a row may select no key inside its listed tiles:
      // l = 0 there, and it is treated the same way.
      const float inv_l = (1.0f / lsum) / (PV4 ? 1.0f : operand_scale(a.amax_v));
      const bool has_keys = SP == 3 ? (n > 0 && lsum > 0.0f) : n > 0;
      const size_t rowoff = (static_cast<size_t>(bh) * a.Lq + q) * D;
      constexpr int DC = D / G;            // output columns per thread
      constexpr int W = DC < 32 ? DC : 32;  // columns per TMEM load
#pragma unroll
      for (int c = 0; c < DC / W; ++c) {
        const int col = rr.half * DC + c * W;
        uint32_t r[32];
        if (W == 32) {
          tmem_ld32(tmem + rr.lane_addr + L::kTmemO + col, r);
        } else {
          tmem_ld16(tmem + rr.lane_addr + L::kTmemO + col, *reinterpret_cast<uint32_t(*)[16]>(r));
        }
        tmem_ld_wait();
        if (q < a.Lq) {
          float f[W];
#pragma unroll
          for (int i = 0; i < W; ++i) f[i] = has_keys ? __uint_as_float(r[i]) * inv_l : 0.0f;
          uint32_t w[W / 2];
#pragma unroll
          for (int i = 0; i < W / 2; ++i) w[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
          uint4 *dst = reinterpret_cast<uint4 *>(a.o + rowoff + col);
#pragma unroll
          for (int i = 0; i < W / 8; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          float4 *d32 = reinterpret_cast<float4 *>(a.o32 + rowoff + col);
#pragma unroll
          for (int i = 0; i < W / 4; ++i) d32[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
        }
      }
      if (q < a.Lq && rr.half == 0) {
        a.m[static_cast<size_t>(bh) * a.Lq + q] = has_keys ? m_scaled : -INFINITY;
        a.lse[static_cast<size_t>(bh) * a.Lq + q] = has_keys ? m_scaled + logf(lsum) : -INFINITY;
      }
    } else {
      // keep the MMA issuer's final commit from outliving the CTA
      mbar_wait_drain(&bars->ofull, 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int D, int FP4S, int PV4, int QP, int SP>
static cudaError_t launch_fwd_sp(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                 const FwdArgs &a, int BH, cudaStream_t stream) {
  using L = FwdLayout<D, FP4S, PV4>;
  static_assert(L::kDynSmem <= 232448, "forward shared memory over the 227 KB limit");
  static_assert(sizeof(FwdBars) <= L::kBarBytes, "forward barrier block larger than its reservation");
  static_assert(!FP4S || L::kTmemEnd <= L::kTmemCols, "forward TMEM over 512 columns");
  auto kern = attn_fwd_kernel<D, FP4S, PV4, QP, kFwdG, SP>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kern), L::kDynSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nq_tiles, BH);
  kern<<<grid, fwd_threads<kFwdG>(), L::kDynSmem, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

template <int D, int FP4S, int PV4, int QP>
static cudaError_t launch_fwd_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                const FwdArgs &a, int BH, cudaStream_t stream) {
  if (!a.kv_list) return launch_fwd_sp<D, FP4S, PV4, QP, 0>(tq, tk, tv, a, BH, stream);
  if (a.quad) return launch_fwd_sp<D, FP4S, PV4, QP, 3>(tq, tk, tv, a, BH, stream);
  return a.causal ? launch_fwd_sp<D, FP4S, PV4, QP, 2>(tq, tk, tv, a, BH, stream)
                  : launch_fwd_sp<D, FP4S, PV4, QP, 1>(tq, tk, tv, a, BH, stream);
}

template <int D, int FP4S>
static cudaError_t fwd_dispatch(bool pv4, bool quant_p, const CUtensorMap &tq, const CUtensorMap &tk,
                                const CUtensorMap &tv, const FwdArgs &a, int BH, cudaStream_t stream) {
  // the NVFP4 P V needs every quantizer (FP4S included)
  if (FP4S && pv4) return launch_fwd_t<D, FP4S, 1, 1>(tq, tk, tv, a, BH, stream);
  return quant_p ? launch_fwd_t<D, FP4S, 0, 1>(tq, tk, tv, a, BH, stream)
                 : launch_fwd_t<D, FP4S, 0, 0>(tq, tk, tv, a, BH, stream);
}

cudaError_t launch_fwd(int D, bool fp4s, bool pv4, bool quant_p, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const FwdArgs &a, int BH, cudaStream_t stream) {
  // quantized Q and K: S runs on the NVFP4 tensor-core path
  if (D == 128)
    return fp4s ? fwd_dispatch<128, 1>(pv4, quant_p, tq, tk, tv, a, BH, stream)
                : fwd_dispatch<128, 0>(pv4, quant_p, tq, tk, tv, a, BH, stream);
  return fp4s ? fwd_dispatch<64, 1>(pv4, quant_p, tq, tk, tv, a, BH, stream)
              : fwd_dispatch<64, 0>(pv4, quant_p, tq, tk, tv, a, BH, stream);
}

}  // namespace attnqat
