// bwd.cu -- Attn-QAT backward kernels for sm_100a (straight-through
// estimator: every fq is the identity for the gradient).
//
//   dK/dV kernel: one CTA per (128-key tile, batch*head), looping over query
//     tiles.  Per query tile: S = fq(Q) fq(K)^T, then dP = dO fq(V)^T, into
//     one TMEM buffer; the row warps (a query row per TMEM lane) rebuild
//     P~ = exp(S - m) and fq(P~) exactly as the forward does (same blocks of
//     16 keys), form (fq(P~)/l)^T and dS^T = (P o (dP - Delta))^T in shared
//     memory (two buffers where they fit), and the tensor cores accumulate
//     dV += (fq(P~)/l)^T dO and dK += dS^T fq(Q) in TMEM.
//   dQ kernel: one CTA per (128-query tile, batch*head), looping over key
//     tiles: S, dP as above, dS = P o (dP - Delta) with P = exp(S - LSE),
//     dQ += dS fq(K).
//
// The split into a dK/dV and a dQ kernel follows the fastvideo-kernel
// triton_kernels commit (SM100 Attn-QAT route: separate dQ and dK/dV tiles);
// the tiles here are 128 x 128 tcgen05 tiles with TMEM accumulators.
// Roles (384 threads): warp 0 TMA producer; warp 1 TMEM owner and MMA issuer
// (one thread); in the dQ kernel warp 10 is a second MMA-issuing thread, A
// issuing S and dP and B the dQ products (one thread alone issues a
// tcgen05.mma only every ~58 cycles, too slowly to keep the tensor pipe busy
// there), and in the dK/dV kernel warp 10 loads the 16-bit Q tiles; warps
// 2..9 row warps: two per TMEM lane quarter, so every query row (TMEM lane)
// has two threads, each owning 64 of the tile's 128 columns; the remaining
// warp idles.
//
// Block-sparse (VSA fine attention): with a.q_list / a.kv_list set, the dK/dV
// kernel walks only the query tiles that selected its key tile and the dQ
// kernel only the key tiles its query tile selected; a CTA with an empty list
// writes zero gradients.  Causal masking walks the lower triangle of tiles and
// masks the diagonal tile (the dK/dV kernel's first, the dQ kernel's last) to
// keys <= the query row.
#include "common.cuh"
#include "internal.h"

namespace attnqat {

// dK/dV kernel layout.  One TMEM buffer holds S_i, then dP_i, then S_{i+1}
// (each released as soon as the row warps have read it into registers), so
// the TMEM left over holds the scale factors of the NVFP4 S = fq(Q) fq(K)^T
// (FP4S: Q and K quantized).  With FP4S the K codes stay resident and Q codes
// stream through their own ring, so S never waits on the 16-bit Q tile,
// which only dK = dS^T fq(Q) reads, late in the tile.
template <int D, int FP4S>
struct DkdvLayout {
  static constexpr int kTile = Tile<D>::kBytes;
  static constexpr int kXBytes = kBM * kBN * 2;
  static constexpr int kCode = 128 * (D / 2);  // one packed NVFP4 tile
  static constexpr int kSF = (D / 64) * 512;   // its scale-factor blocks
  static constexpr int kK = 0;                 // 16-bit K, or K codes + scales (FP4S)
  static constexpr int kKSF = kK + kCode;      // FP4S
  static constexpr int kV = FP4S ? (kKSF + kSF + 1023) / 1024 * 1024 : kK + kTile;
  static constexpr int kQ4 = kV + kTile;       // FP4S: 2 stages of Q codes
  static constexpr int kQSF = kQ4 + (FP4S ? 2 * kCode : 0);
  static constexpr int kQ = (kQSF + (FP4S ? 2 * kSF : 0) + 1023) / 1024 * 1024;  // kNQ stages
  static constexpr int kBarBytes = 256;  // BwdBars (checked at the launch)
  // Two X buffers (P^T in one, dS^T in the other) let the rows store both
  // operands of a query tile without waiting for dV to finish reading P^T.
  // Where two of them and two 16-bit Q stages do not fit (D = 128), the
  // NVFP4-S build keeps one Q stage (its Q tile feeds dK alone, the last MMA
  // of a query tile, so one stage has a whole tile's row work to refill);
  // the 16-bit-S build, whose S also reads that tile, keeps one X buffer.
  static constexpr bool kFitBoth = kQ + 4 * kTile + 2 * kXBytes + kBarBytes + 1024 <= 232448;
  static constexpr int kNQ = (kFitBoth || !FP4S) ? 2 : 1;  // 16-bit Q stages
  static constexpr int kXB = (kFitBoth || FP4S) ? 2 : 1;   // X buffers
  static constexpr int kDO = kQ + kNQ * kTile;  // 2 stages
  static constexpr int kX = kDO + 2 * kTile;    // kXB buffers: P^T (and dS^T in the last)
  static constexpr int kBar = kX + kXB * kXBytes;
  static constexpr int kBytes = kBar + kBarBytes;
  static constexpr int kDynSmem = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemBuf = 0, kTmemDV = 128, kTmemDK = 128 + D;
  static constexpr uint32_t kSFCols = (D / 64) * 4;
  static constexpr uint32_t kTmemSFA = 128 + 2 * D;         // 2 stages (Q codes)
  static constexpr uint32_t kTmemSFB = kTmemSFA + 2 * kSFCols;  // K codes
  static constexpr uint32_t kCodeLayout = (D / 2 == 64) ? 4u : 6u;  // SW64 / SW32
  static constexpr uint32_t kCodeSBO = 8 * (D / 2);
};

struct BwdBars {
  uint64_t kvfull;
  uint64_t afull[2], aempty[2];   // Q tiles (dK/dV kernel) or K tiles (dQ kernel)
  uint64_t bfull[2], bempty[2];   // dO tiles (dK/dV kernel) or V tiles (dQ kernel)
  uint64_t cfull[2], cempty[2];   // packed NVFP4 Q (dK/dV kernel) or K (dQ kernel) codes + scales
  // dK/dV kernel: the TMEM buffer's fills S_0, dP_0, S_1, ... one phase each;
  // dQ kernel: S and dP filled together, released together
  uint64_t sfull, sempty;
  uint64_t xfull[2], xempty[2];   // X buffers (the dQ kernel uses the first)
  uint64_t done;
  uint64_t adone;   // issuer A's MMAs have completed (drained before TMEM is freed)
  uint32_t tmem_slot;
  int abort;
};

// a_users / b_users: MMA-issuing threads that commit to aempty / bempty (a
// ring slot is free once every MMA reading it has completed).
__device__ __forceinline__ void init_bwd_bars(BwdBars *b, int a_users, int b_users, int row_warps = kSoftWarps) {
  mbar_init(&b->kvfull, 1);
  for (int s = 0; s < 2; ++s) {
    mbar_init(&b->afull[s], 1);
    mbar_init(&b->aempty[s], a_users);
    mbar_init(&b->bfull[s], 1);
    mbar_init(&b->bempty[s], b_users);
    mbar_init(&b->cfull[s], 1);
    mbar_init(&b->cempty[s], 1);
  }
  mbar_init(&b->sfull, 1);
  mbar_init(&b->sempty, row_warps);
  for (int s = 0; s < 2; ++s) {
    mbar_init(&b->xfull[s], row_warps);
    mbar_init(&b->xempty[s], 1);
  }
  mbar_init(&b->done, 1);
  mbar_init(&b->adone, 1);
  b->abort = 0;
  fence_mbar_init();
}

// Loads one 128-row x D tile (D/64 swizzled chunks) with TMA.
template <int D>
__device__ __forceinline__ void load_tile(uint8_t *dst, const CUtensorMap *map, uint64_t *bar, int row0,
                                          int bh) {
  for (int c = 0; c < Tile<D>::kChunks; ++c) tma_load_3d(dst + c * kChunkBytes, map, bar, c * 64, row0, bh);
}

// ----------------------------------------------------------- dK / dV ------

// Power-of-two scale for the fp16 dS operand: 2^e with e chosen so that the
// bound |dS| <= max_i|dO_i|_1 * max|fq(V)| + max_i|Delta_i| maps to at most
// 2^14 (fp16 max is 65504); the float range of dS below that keeps full fp16
// precision over 29 binades.  Returns 1 for a zero bound.
__device__ __forceinline__ float ds_scale(const float *stats) {
  const float bound = fmaf(stats[0], stats[2], stats[1]);
  if (!(bound > 0.0f)) return 1.0f;
  int e = 14 - (static_cast<int>((__float_as_uint(bound) >> 23) & 0xFF) - 127) - 1;
  e = e < -120 ? -120 : (e > 120 ? 120 : e);
  return __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}

// S and dP of one thread's 64 columns (starting at col0) from TMEM into
// registers.  The caller releases the TMEM tiles right after, so the next
// tile's S and dP MMAs run while this tile's row math proceeds.
__device__ __forceinline__ void load_sdp(uint32_t tS, uint32_t tDP, int col0, uint32_t (&sv)[64],
                                         uint32_t (&dv)[64]) {
  tmem_ld32(tS + col0, *reinterpret_cast<uint32_t(*)[32]>(sv));
  tmem_ld32(tS + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
  tmem_ld32(tDP + col0, *reinterpret_cast<uint32_t(*)[32]>(dv));
  tmem_ld32(tDP + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(dv + 32));
  tmem_ld_wait();
}

// 64 columns (one thread's half row) of one 32-bit TMEM tile into registers.
__device__ __forceinline__ void load_cols64(uint32_t taddr, uint32_t (&v)[64]) {
  tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(v));
  tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
  tmem_ld_wait();
}

// NC (32 or 64) columns of one 32-bit TMEM tile into registers.
template <int NC>
__device__ __forceinline__ void load_cols(uint32_t taddr, uint32_t (&v)[NC]) {
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) tmem_ld32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
  tmem_ld_wait();
}

// dK/dV kernel, first half of a query tile for one thread (one query row, NC
// key columns from col0): P~ = exp2(S cl + nml) -- rebuilt exactly as the
// forward builds it (same bits, same blocks of 16 keys) -- and the dV
// operand row in fp16: fq(P~)/l * 2^14 (r times the per-block factor
// s/l * 2^14), or P~/l * 2^14 when P is not quantized, with 11 significant
// bits and in fp16's normal range for every value above 2^-28 (all nonzero
// fq(P~)/l while Lk <= 2^17).  P~ stays in float32 for dS.  Rows past Lq come
// in with nml = -inf, so their P~ is 0 without a per-element test.
template <int QP, bool MASKED, int NC>
__device__ __forceinline__ void dkdv_probs(const uint32_t (&sv)[NC], int col0, int valid_k, float cl, float nml,
                                           float vf, float (&p)[NC], uint32_t (&pw)[NC / 2]) {
  const float2 cl2 = make_float2(cl, cl), nml2 = make_float2(nml, nml);
#pragma unroll
  for (int i = 0; i < NC / 2; ++i) {
    const float2 x = fma2(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), cl2, nml2);
    const float e0 = ex2_approx(x.x), e1 = ex2_approx(x.y);
    p[2 * i] = (!MASKED || col0 + 2 * i < valid_k) ? e0 : 0.0f;
    p[2 * i + 1] = (!MASKED || col0 + 2 * i + 1 < valid_k) ? e1 : 0.0f;
  }
  if (QP) {
#pragma unroll
    for (int b = 0; b < NC / 16; ++b) {
      uint32_t rr[8];
      const uint32_t s2 = f16x2_broadcast(fq16_probs(p + 16 * b, rr) * vf);
#pragma unroll
      for (int i = 0; i < 8; ++i) pw[8 * b + i] = hmul2_u32(rr[i], s2);
    }
  } else {
    const float2 vf2 = make_float2(vf, vf);
#pragma unroll
    for (int i = 0; i < NC / 2; ++i) {
      const float2 x = mul2(make_float2(p[2 * i], p[2 * i + 1]), vf2);
      pw[i] = pack_f16x2(x.x, x.y);
    }
  }
}

// Second half: dS = (P~/l)(dP - Delta) in float32, scaled by the fp16
// operand's power of two dsc and packed for the dK operand.  dP arrives as
// dP' = dP 2^e (the fp16 copies of dO and V carry powers of two), so
// dS * dsc = P~/l * (dP' 2^-e - Delta) * dsc = P~ * fma(dP', a1, b1) with
// a1 = 2^-e dsc / l, b1 = -Delta dsc / l.
template <int NC>
__device__ __forceinline__ void dkdv_ds(const float (&p)[NC], const uint32_t (&dv)[NC], float a1, float b1,
                                        uint32_t (&dsw)[NC / 2]) {
  const float2 a12 = make_float2(a1, a1), b12 = make_float2(b1, b1);
#pragma unroll
  for (int i = 0; i < NC / 2; ++i) {
    const float2 g = fma2(make_float2(__uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1])), a12, b12);
    const float2 d = mul2(make_float2(p[2 * i], p[2 * i + 1]), g);
    dsw[i] = pack_f16x2(d.x, d.y);
  }
}

// Row warps per TMEM lane quarter of the dK/dV kernel, and its CTA size
// (producer, MMA issuer, 4 * RG row warps, the 16-bit Q producer; 12 warps
// for RG = 2, one of them idle).  RG = 4 (32 columns per thread) measured
// slower at the H6 L31200 shape, 5.23 against 5.08 ms: with 18 warps one
// scheduler holds five of them, which caps registers at 96 per thread.
constexpr int kDkdvRG = 2;
template <int RG>
constexpr int dkdv_threads() { return RG == 2 ? kThreads : 32 * (3 + 4 * RG); }

// SP: 0 dense; 1 block-sparse (walks a.q_list); 2 causal (lower-triangle
// lists, diagonal masked).  Separate instantiations, so the dense kernel
// carries none of the list handling.
template <int D, int QP, int FP4S, int SP, int RG>
__global__ void __launch_bounds__(dkdv_threads<RG>(), 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const __grid_constant__ CUtensorMap tmQ4, const BwdArgs a) {
  using L = DkdvLayout<D, FP4S>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  BwdBars *bars = reinterpret_cast<BwdBars *>(smem + L::kBar);
  volatile int *abort = &bars->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kt = blockIdx.x;
  const int bh = blockIdx.y;
  const int nq = a.nq_tiles;
  // the query tiles this key tile meets: all nq, or those that selected it
  const size_t krow = static_cast<size_t>(bh) * a.nk_tiles + kt;
  const int32_t *ql = SP ? a.q_list + krow * nq : nullptr;
  const int n = SP ? a.q_count[krow] : nq;
  // SP 3 (64-token masks): list entries carry quadrant bits in the top byte
  auto qtile = [&](int i) -> int { return SP == 3 ? (__ldg(ql + i) & 0xFFFFFF) : (SP ? __ldg(ql + i) : i); };

  constexpr int NC = kBN / RG;  // key columns per row-warp thread
  if (threadIdx.x == 0) init_bwd_bars(bars, 1, 1, 4 * RG);
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDO);
      if (FP4S) prefetch_tmap(&tmQ4);
      mbar_arrive_expect_tx(&bars->kvfull, (FP4S ? L::kCode + L::kSF : L::kTile) + L::kTile);
      if (FP4S) {
        tma_load_3d(smem + L::kK, &tmK, &bars->kvfull, 0, kt * kBN, bh);
        bulk_load(smem + L::kKSF, a.ksf + (static_cast<size_t>(bh) * a.nk_tiles + kt) * L::kSF, L::kSF,
                  &bars->kvfull);
      } else {
        load_tile<D>(smem + L::kK, &tmK, &bars->kvfull, kt * kBN, bh);
      }
      load_tile<D>(smem + L::kV, &tmV, &bars->kvfull, kt * kBN, bh);
      // per query tile, in the order the MMAs need them: Q codes (S), dO (dP,
      // then dV); the 16-bit Q ring (dK; with !FP4S also S) has its own
      // producer warp, so a wait for its slot never holds these back
      int nc = 0, nd = 0;  // tiles issued per ring
      for (int i = 0; i < n; ++i) {
        const int st = i & 1;
        const int ph = ((i >> 1) - 1) & 1;
        const int qi = qtile(i);
        if (FP4S) {
          if (i >= 2 && !mbar_wait(&bars->cempty[st], ph, abort)) break;
          mbar_arrive_expect_tx(&bars->cfull[st], L::kCode + L::kSF);
          tma_load_3d(smem + L::kQ4 + st * L::kCode, &tmQ4, &bars->cfull[st], 0, qi * kBM, bh);
          bulk_load(smem + L::kQSF + st * L::kSF, a.qsf + (static_cast<size_t>(bh) * nq + qi) * L::kSF, L::kSF,
                    &bars->cfull[st]);
          nc = i + 1;
        }
        if (i >= 2 && !mbar_wait(&bars->bempty[st], ph, abort)) break;
        mbar_arrive_expect_tx(&bars->bfull[st], L::kTile);
        load_tile<D>(smem + L::kDO + st * L::kTile, &tmDO, &bars->bfull[st], qi * kBM, bh);
        nd = i + 1;
      }
      if (*abort) {
        mbar_wait_drain(&bars->kvfull, 0);
        for (int i = (nc > 2 ? nc - 2 : 0); i < nc; ++i) mbar_wait_drain(&bars->cfull[i & 1], (i >> 1) & 1);
        for (int i = (nd > 2 ? nd - 2 : 0); i < nd; ++i) mbar_wait_drain(&bars->bfull[i & 1], (i >> 1) & 1);
      }
    }
  } else if (warp == 2 + 4 * RG) {
    // ------------------------------------------------ 16-bit Q producer --
    if (lane == 0) {
      constexpr int NQ = L::kNQ;
      prefetch_tmap(&tmQ);
      int nqh = 0;
      for (int i = 0; i < n; ++i) {
        const int sq = i % NQ;
        if (i >= NQ && !mbar_wait(&bars->aempty[sq], ((i / NQ) - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars->afull[sq], L::kTile);
        load_tile<D>(smem + L::kQ + sq * L::kTile, &tmQ, &bars->afull[sq], qtile(i) * kBM, bh);
        nqh = i + 1;
      }
      if (*abort)
        for (int i = (nqh > NQ ? nqh - NQ : 0); i < nqh; ++i) mbar_wait_drain(&bars->afull[i % NQ], (i / NQ) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = FP4S ? idesc_mxf4(kBM, kBN) : idesc_f16(kBM, kBN, false, false, false);  // Q K^T
      constexpr uint32_t idDP = idesc_f16(kBM, kBN, false, false, false);  // dO V^T
      constexpr uint32_t idV = idesc_f16(kBN, D, false, true, true);       // P^T dO
      constexpr uint32_t idK = idesc_f16(kBN, D, false, true, true);       // dS^T Q
      const uint32_t kaddr = sbase + L::kK;
      const uint32_t tbuf = tmem + L::kTmemBuf;
      // operand descriptors of the tiles' base addresses
      const uint64_t dK = FP4S ? sdesc_make(kaddr, 16, L::kCodeSBO, L::kCodeLayout) : desc_k(kaddr);
      const uint64_t dQ4 = sdesc_make(sbase + L::kQ4, 16, L::kCodeSBO, L::kCodeLayout);
      const uint64_t dQSF = sdesc_make(sbase + L::kQSF, 16, 128, 0);
      const uint64_t dQk = desc_k(sbase + L::kQ), dQmn = desc_mn(sbase + L::kQ);
      const uint64_t dDOk = desc_k(sbase + L::kDO), dDOmn = desc_mn(sbase + L::kDO);
      const uint64_t dVk = desc_k(sbase + L::kV);
      // X buffers: P^T in the first, dS^T in the last (the same one when
      // there is one, used twice per query tile)
      constexpr int XB = L::kXB;
      const uint64_t dXP = desc_mn(sbase + L::kX), dXS = desc_mn(sbase + L::kX + (XB - 1) * L::kXBytes);
      // One issuing thread here (a second one measured slower: this kernel is
      // bound by its row warps, whose scheduler the second poller shares).
      // Order per query tile: dP_i (once the rows have read S_i), S_{i+1}
      // (once the rows have read dP_i, ahead of the two accumulations so that
      // the rows find it ready when they finish tile i), dV_i, dK_i.
      bool ok = mbar_wait(&bars->kvfull, 0, abort);
      if (ok && FP4S) {
        tc_fence_after();
        for (int kc = 0; kc < D / 64; ++kc)
          tmem_cp_32x128b_x4(tmem + L::kTmemSFB + kc * 4, sdesc_make(sbase + L::kKSF + kc * 512, 16, 128, 0));
      }
      // S_i into the TMEM buffer (fill 2i); the buffer's previous fill
      // (dP_{i-1}) has been released by the caller's wait
      auto issue_s = [&](int i) -> bool {
        const int st = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        static_assert(FP4S || L::kNQ == 2, "16-bit S reads the 16-bit Q ring");
        if (FP4S) {
          if (!mbar_wait(&bars->cfull[st], ph, abort)) return false;
          tc_fence_after();
          const uint32_t sfa = tmem + L::kTmemSFA + st * L::kSFCols;
          const uint64_t dQs = sdesc_add(dQ4, st * L::kCode);
#pragma unroll
          for (int kc = 0; kc < D / 64; ++kc)
            tmem_cp_32x128b_x4(sfa + kc * 4, sdesc_add(dQSF, st * L::kSF + kc * 512));
#pragma unroll
          for (int kk = 0; kk < D / 64; ++kk)
            umma_fp4(tbuf, sdesc_add(dQs, kk * 32), sdesc_add(dK, kk * 32), idS, sfa + kk * 4,
                     tmem + L::kTmemSFB + kk * 4, kk > 0 ? 1u : 0u);
          umma_commit(&bars->cempty[st]);
        } else {
          if (!mbar_wait(&bars->afull[st], ph, abort)) return false;
          tc_fence_after();
          mma_kmajor<D / 16>(tbuf, sdesc_add(dQk, st * L::kTile), dK, idS, false);
        }
        umma_commit(&bars->sfull);
        return true;
      };
      if (ok && n > 0) ok = issue_s(0);
      for (int i = 0; ok && i < n; ++i) {
        const int st = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        const int sq = i % L::kNQ;  // 16-bit Q stage
        const uint32_t phq = (i / L::kNQ) & 1;
        // uses of the X buffers so far: P^T_i is use up of the first, dS^T_i
        // use us of the last
        const int up = XB == 2 ? i : 2 * i, us = XB == 2 ? i : 2 * i + 1;
        // dP_i once the rows have read S_i (fill 2i)
        if (!mbar_wait(&bars->sempty, (2 * i) & 1, abort) || !mbar_wait(&bars->bfull[st], ph, abort)) break;
        tc_fence_after();
        mma_kmajor<D / 16>(tbuf, sdesc_add(dDOk, st * L::kTile), dVk, idDP, false);
        umma_commit(&bars->sfull);
        // S_{i+1} once the rows have read dP_i (fill 2i+1)
        if (i + 1 < n && !(mbar_wait(&bars->sempty, (2 * i + 1) & 1, abort) && issue_s(i + 1))) break;
        // dV += (fq(P~)/l)^T dO_i : A = X (M = keys, MN-major), B = dO (N = D, MN-major)
        if (!mbar_wait(&bars->xfull[0], up & 1, abort)) break;
        tc_fence_after();
        mma_mn_mn<kBM / 16>(tmem + L::kTmemDV, dXP, sdesc_add(dDOmn, st * L::kTile), idV, i > 0);
        umma_commit(&bars->xempty[0]);
        umma_commit(&bars->bempty[st]);
        // dK += dS^T Q_i
        if (!mbar_wait(&bars->xfull[XB - 1], us & 1, abort)) break;
        if (FP4S && !mbar_wait(&bars->afull[sq], phq, abort)) break;
        tc_fence_after();
        mma_mn_mn<kBM / 16>(tmem + L::kTmemDK, dXS, sdesc_add(dQmn, sq * L::kTile), idK, i > 0);
        umma_commit(&bars->xempty[XB - 1]);
        umma_commit(&bars->aempty[sq]);
      }
      umma_commit(&bars->done);
    }
  } else if (warp >= 2 && warp < 2 + 4 * RG) {
    const RowRole rr(warp, lane);
    const int col0 = rr.half * NC;
    const int valid_k = a.Lk - kt * kBN;  // >= 128 for full key tiles
    // causal: the first query tile visited is the diagonal, where query row r
    // keeps keys 0..r (a partial key tile only ever meets its diagonal)
    const int diag_k = static_cast<int>(rr.row) + 1;
    // the fp16 copies of unquantized operands carry powers of two: S arrives
    // as S 2^(eq+ek), dP as dP 2^(edo+ev) (all exact to divide out)
    const float sq = operand_scale(a.amax_q), sk = operand_scale(a.amax_k);
    const float cl = FP4S ? a.scale_log2 : a.scale_log2 / (sq * sk);
    const float dsc = ds_scale(a.stats);
    const float dos = do_scale(a.stats) * operand_scale(a.amax_v);
    constexpr int XB = L::kXB;
    const uint32_t xaddr_p = sbase + L::kX, xaddr_s = sbase + L::kX + (XB - 1) * L::kXBytes;
    const uint32_t tbuf = tmem + rr.lane_addr + L::kTmemBuf + col0;
    bool ok = true;
    // row statistics of the current query tile, prefetched one tile ahead
    auto load_stats = [&](int i, float &m, float &lse, float &delta) {
      const int qg = (i < n ? qtile(i) : 0) * kBM + static_cast<int>(rr.row);
      const bool vq = i < n && qg < a.Lq;
      const size_t si = static_cast<size_t>(bh) * a.Lq + (vq ? qg : 0);
      m = vq ? a.m[si] : 0.0f;
      lse = vq ? a.lse[si] : 0.0f;
      delta = vq ? a.delta[si] : 0.0f;
    };
    // SP 3: this thread's quadrant bit (its query half, its 64-key half)
    const int qbit = (static_cast<int>(rr.row) >> 6) * 2 + (col0 >> 6);
    float m_n, lse_n, delta_n;
    load_stats(0, m_n, lse_n, delta_n);
    for (int i = 0; i < n; ++i) {
      const int up = XB == 2 ? i : 2 * i, us = XB == 2 ? i : 2 * i + 1;  // X buffer uses, as the issuer counts them
      // with quadrant masks a row may have selected no key at all (m = -inf):
      // it contributes nothing, like a row past Lq
      const bool vq = qtile(i) * kBM + static_cast<int>(rr.row) < a.Lq && (SP != 3 || m_n > -INFINITY);
      const float m = m_n, lse = lse_n, delta = delta_n;
      load_stats(i + 1, m_n, lse_n, delta_n);
      const float inv_l = vq ? ex2_approx((m - lse) * kLog2e) : 0.0f;
      float p[NC];
      uint32_t pw[NC / 2], dsw[NC / 2];
      // SP 3: an unselected quadrant (warp-uniform) reads neither S nor dP
      // and stores zero operands
      const bool clear = SP == 3 && !((__ldg(ql + i) >> (24 + qbit)) & 1);
      {
        // S_i: read, release the buffer for dP_i, build P~ and the dV operand
        if (!mbar_wait(&bars->sfull, (2 * i) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        if (clear) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->sempty);
#pragma unroll
          for (int k = 0; k < NC / 2; ++k) pw[k] = 0u;
        } else {
          uint32_t sv[NC];
          load_cols<NC>(tbuf, sv);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->sempty);
          const bool masked = SP == 2 ? i == 0 : valid_k < kBN;
          const int vk = SP == 2 ? diag_k : valid_k;
          const float nml = vq ? -(m * kLog2e) : -INFINITY;
          const float vf = inv_l * 16384.0f;  // fq(P~)/l scaled by 2^14 for the fp16 dV operand
          if (masked)
            dkdv_probs<QP, true, NC>(sv, col0, vk, cl, nml, vf, p, pw);
          else
            dkdv_probs<QP, false, NC>(sv, col0, vk, cl, nml, vf, p, pw);
        }
      }
      // X_P = (fq(P~)/l)^T once the buffer's previous use has been read
      // (dV_{i-1}; with one buffer, dK_{i-1} reading dS^T_{i-1})
      if (up >= 1 && !mbar_wait(&bars->xempty[0], (up - 1) & 1, abort)) { ok = false; break; }
      store_row_cols<NC>(xaddr_p, rr.row, col0, pw);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->xfull[0]);
      {
        // dP_i: read, release the buffer for S_{i+1}, build dS
        if (!mbar_wait(&bars->sfull, (2 * i + 1) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        if (clear) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->sempty);
#pragma unroll
          for (int k = 0; k < NC / 2; ++k) dsw[k] = 0u;
        } else {
          uint32_t dv[NC];
          load_cols<NC>(tbuf, dv);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->sempty);
          dkdv_ds<NC>(p, dv, inv_l * dsc / dos, -delta * inv_l * dsc, dsw);
        }
      }
      // X_S = dS^T once the buffer's previous use has been read (dK_{i-1};
      // with one buffer, dV_i reading P^T_i)
      if (us >= 1 && !mbar_wait(&bars->xempty[XB - 1], (us - 1) & 1, abort)) { ok = false; break; }
      store_row_cols<NC>(xaddr_s, rr.row, col0, dsw);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->xfull[XB - 1]);
    }
    if (ok && mbar_wait(&bars->done, 0, abort)) {
      tc_fence_after();
      // TMEM lanes of dV/dK are keys; each thread stores D/RG columns of its key row
      const int kg = kt * kBN + static_cast<int>(rr.row);
      const size_t rowoff = (static_cast<size_t>(bh) * a.Lk + kg) * D;
      const float kscale = a.sm_scale / (dsc * sq);  // exact: power-of-two divisors
      const float vscale = (1.0f / 16384.0f) / do_scale(a.stats);  // exact: powers of two
      constexpr int DC = D / RG;            // output columns per thread
      constexpr int W = DC < 32 ? DC : 32;  // columns per TMEM load
#pragma unroll
      for (int c = 0; c < DC / W; ++c) {
        const int col = rr.half * DC + c * W;
        uint32_t r[32], s[32];
        if (W == 32) {
          tmem_ld32(tmem + rr.lane_addr + L::kTmemDV + col, r);
          tmem_ld32(tmem + rr.lane_addr + L::kTmemDK + col, s);
        } else {
          tmem_ld16(tmem + rr.lane_addr + L::kTmemDV + col, *reinterpret_cast<uint32_t(*)[16]>(r));
          tmem_ld16(tmem + rr.lane_addr + L::kTmemDK + col, *reinterpret_cast<uint32_t(*)[16]>(s));
        }
        tmem_ld_wait();
        if (kg < a.Lk) {
          uint4 *dv = reinterpret_cast<uint4 *>(a.dv + rowoff + col);
          uint4 *dk = reinterpret_cast<uint4 *>(a.dk + rowoff + col);
#pragma unroll
          for (int i = 0; i < W / 8; ++i) {
            uint32_t w[4], x[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              w[k] = pack_bf16x2(__uint_as_float(r[8 * i + 2 * k]) * vscale,
                                 __uint_as_float(r[8 * i + 2 * k + 1]) * vscale);
              x[k] = pack_bf16x2(__uint_as_float(s[8 * i + 2 * k]) * kscale,
                                 __uint_as_float(s[8 * i + 2 * k + 1]) * kscale);
            }
            // a key tile no query tile selected: the accumulators were never written
            dv[i] = n > 0 ? make_uint4(w[0], w[1], w[2], w[3]) : make_uint4(0, 0, 0, 0);
            dk[i] = n > 0 ? make_uint4(x[0], x[1], x[2], x[3]) : make_uint4(0, 0, 0, 0);
          }
        }
      }
    } else {
      mbar_wait_drain(&bars->done, 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ----------------------------------------------------------------- dQ -----

// dQ kernel layout.  With FP4S (Q and K quantized) S = fq(Q) fq(K)^T is a
// block-scaled NVFP4 MMA: the Q codes and scales stay resident and K codes
// stream through their own small 2-stage ring, so S never waits on the
// 16-bit K slot that the dQ MMA holds; the 16-bit Q tile is then not needed.
// With DSPLIT, dS is fed as two fp16 tiles, hi = fp16(dS) and lo =
// fp16(dS - hi) (about 22 significant bits: dQ = sum_j dS_ij K_j cancels,
// since sum_j dS_ij is 0 up to the quantization of P, and amplifies the
// rounding of an 11-bit dS); the second tile's 32 KB come from running the V
// ring, which only dP reads, with one stage.
template <int D, int FP4S, int DSPLIT>
struct DqLayout {
  static constexpr int kTile = Tile<D>::kBytes;
  static constexpr int kXBytes = kBM * kBN * 2;
  static constexpr int kCode = 128 * (D / 2);   // one packed NVFP4 tile
  static constexpr int kSF = (D / 64) * 512;    // its scale-factor blocks
  static constexpr int kNV = DSPLIT ? 1 : 2;    // V ring stages
  static constexpr int kQ = 0;                  // 16-bit Q tile, or Q codes (FP4S)
  static constexpr int kQSF = kQ + (FP4S ? kCode : kTile);
  static constexpr int kDO = (kQSF + (FP4S ? kSF : 0) + 1023) / 1024 * 1024;
  static constexpr int kK = kDO + kTile;        // 2 stages of 16-bit K
  static constexpr int kV = kK + 2 * kTile;     // kNV stages
  static constexpr int kX = kV + kNV * kTile;   // dS (DSPLIT: its hi part, the lo part follows)
  static constexpr int kK4 = kX + (DSPLIT ? 2 : 1) * kXBytes;  // FP4S: 2 stages of K codes
  static constexpr int kKSF = kK4 + (FP4S ? 2 * kCode : 0);
  static constexpr int kBar = kKSF + (FP4S ? 2 * kSF : 0);
  static constexpr int kBarBytes = 256;  // BwdBars (checked at the launch)
  static constexpr int kBytes = kBar + kBarBytes;
  static constexpr int kDynSmem = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemS = 0, kTmemDP = 128, kTmemDQ = 256;
  static constexpr uint32_t kSFCols = (D / 64) * 4;
  static constexpr uint32_t kTmemSFA = 256 + D, kTmemSFB = kTmemSFA + kSFCols;  // 2 stages
  static constexpr uint32_t kCodeLayout = (D / 2 == 64) ? 4u : 6u;  // SW64 / SW32
  static constexpr uint32_t kCodeSBO = 8 * (D / 2);
};

// One key tile for one thread of the dQ kernel (one query row, 64 key
// columns starting at col0), from S and dP in registers: P = exp2(S cl +
// nlse) in float32 and dS = P (dP - Delta), scaled by the fp16 operand's
// power of two dsc and packed as fp16 for dQ = dS fq(K).  dP arrives as
// dP' = dP 2^e (the fp16 copies of dO and V carry powers of two), so
// dS * dsc = P (dP' 2^-e - Delta) dsc = P * fma(dP', a1, b1) with
// a1 = 2^-e dsc, b1 = -Delta dsc.  Rows past Lq come in with nlse = -inf.
template <bool MASKED, int DSPLIT>
__device__ __forceinline__ void dq_tile(const uint32_t (&sv)[64], const uint32_t (&dv)[64], int col0, int valid_k,
                                        float cl, float nlse, float a1, float b1, uint32_t (&dsw)[32],
                                        uint32_t (&dsl)[32]) {
  const float2 cl2 = make_float2(cl, cl), nl2 = make_float2(nlse, nlse);
  const float2 a12 = make_float2(a1, a1), b12 = make_float2(b1, b1);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float2 x = fma2(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), cl2, nl2);
    float p0 = ex2_approx(x.x);
    float p1 = ex2_approx(x.y);
    if (MASKED && col0 + 2 * i >= valid_k) p0 = 0.0f;
    if (MASKED && col0 + 2 * i + 1 >= valid_k) p1 = 0.0f;
    const float2 g = fma2(make_float2(__uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1])), a12, b12);
    const float2 d = mul2(make_float2(p0, p1), g);
    dsw[i] = pack_f16x2(d.x, d.y);
    if (DSPLIT) {
      const float2 h = unpack_f16x2(dsw[i]);
      dsl[i] = pack_f16x2(d.x - h.x, d.y - h.y);  // d - h is exact in float
    }
  }
}

// SP: 0 dense, 1 block-sparse (walks a.kv_list), 2 causal, as for the dK/dV
// kernel.
template <int D, int FP4S, int DSPLIT, int SP>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmK4, const BwdArgs a) {
  using L = DqLayout<D, FP4S, DSPLIT>;
  constexpr int kNV = L::kNV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  BwdBars *bars = reinterpret_cast<BwdBars *>(smem + L::kBar);
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

  if (threadIdx.x == 0) init_bwd_bars(bars, 1, 1);
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDO);
      if (FP4S) prefetch_tmap(&tmK4);
      mbar_arrive_expect_tx(&bars->kvfull, (FP4S ? L::kCode + L::kSF : L::kTile) + L::kTile);
      if (FP4S) {
        tma_load_3d(smem + L::kQ, &tmQ, &bars->kvfull, 0, qt * kBM, bh);
        bulk_load(smem + L::kQSF, a.qsf + (static_cast<size_t>(bh) * a.nq_tiles + qt) * L::kSF, L::kSF,
                  &bars->kvfull);
      } else {
        load_tile<D>(smem + L::kQ, &tmQ, &bars->kvfull, qt * kBM, bh);
      }
      load_tile<D>(smem + L::kDO, &tmDO, &bars->kvfull, qt * kBM, bh);
      int n4 = 0, nv = 0, nkh = 0;  // tiles issued per ring
      for (int j = 0; j < n; ++j) {
        const int st = j & 1;
        const int ph = ((j >> 1) - 1) & 1;
        const int kj = ktile(j);
        if (FP4S) {
          if (j >= 2 && !mbar_wait(&bars->cempty[st], ph, abort)) break;
          mbar_arrive_expect_tx(&bars->cfull[st], L::kCode + L::kSF);
          tma_load_3d(smem + L::kK4 + st * L::kCode, &tmK4, &bars->cfull[st], 0, kj * kBN, bh);
          bulk_load(smem + L::kKSF + st * L::kSF, a.ksf + (static_cast<size_t>(bh) * nk + kj) * L::kSF, L::kSF,
                    &bars->cfull[st]);
          n4 = j + 1;
        }
        const int vs = j % kNV;
        if (j >= kNV && !mbar_wait(&bars->bempty[vs], ((j / kNV) - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars->bfull[vs], L::kTile);
        load_tile<D>(smem + L::kV + vs * L::kTile, &tmV, &bars->bfull[vs], kj * kBN, bh);
        nv = j + 1;
        if (j >= 2 && !mbar_wait(&bars->aempty[st], ph, abort)) break;
        mbar_arrive_expect_tx(&bars->afull[st], L::kTile);
        load_tile<D>(smem + L::kK + st * L::kTile, &tmK, &bars->afull[st], kj * kBN, bh);
        nkh = j + 1;
      }
      if (*abort) {
        mbar_wait_drain(&bars->kvfull, 0);
        for (int j = (n4 > 2 ? n4 - 2 : 0); j < n4; ++j) mbar_wait_drain(&bars->cfull[j & 1], (j >> 1) & 1);
        for (int j = (nv > kNV ? nv - kNV : 0); j < nv; ++j) mbar_wait_drain(&bars->bfull[j % kNV], (j / kNV) & 1);
        for (int j = (nkh > 2 ? nkh - 2 : 0); j < nkh; ++j) mbar_wait_drain(&bars->afull[j & 1], (j >> 1) & 1);
      }
    }
  } else if (warp == 1 || warp == kMmaB2) {
    if (lane == 0) {
      constexpr uint32_t idS = FP4S ? idesc_mxf4(kBM, kBN) : idesc_f16(kBM, kBN, false, false, false);  // Q K^T
      constexpr uint32_t idDP = idesc_f16(kBM, kBN, false, false, false);  // dO V^T
      constexpr uint32_t idQ = idesc_f16(kBM, D, false, false, true);     // dS (K-major) * K (MN-major)
      const uint32_t qaddr = sbase + L::kQ;
      // operand descriptors of the tiles' base addresses
      const uint64_t dQ = FP4S ? sdesc_make(qaddr, 16, L::kCodeSBO, L::kCodeLayout) : desc_k(qaddr);
      const uint64_t dDO = desc_k(sbase + L::kDO), dVk = desc_k(sbase + L::kV);
      const uint64_t dK4 = sdesc_make(sbase + L::kK4, 16, L::kCodeSBO, L::kCodeLayout);
      const uint64_t dKSF = sdesc_make(sbase + L::kKSF, 16, 128, 0);
      const uint64_t dKk = desc_k(sbase + L::kK), dKmn = desc_mn(sbase + L::kK), dX = desc_k(sbase + L::kX);
      if (warp == 1) {
        // issuer A: dP_j, then S_j; one commit signals both
        bool ok = mbar_wait(&bars->kvfull, 0, abort);
        if (ok && FP4S) {
          tc_fence_after();
          for (int kc = 0; kc < D / 64; ++kc)
            tmem_cp_32x128b_x4(tmem + L::kTmemSFA + kc * 4, sdesc_make(sbase + L::kQSF + kc * 512, 16, 128, 0));
        }
        auto issue_sdp = [&](int j) -> bool {
          const int st = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          const int vs = j % kNV;
          if (!mbar_wait(&bars->bfull[vs], (j / kNV) & 1, abort)) return false;
          tc_fence_after();
          mma_kmajor<D / 16>(tmem + L::kTmemDP, dDO, sdesc_add(dVk, vs * L::kTile), idDP, false);
          umma_commit(&bars->bempty[vs]);
          if (FP4S) {
            if (!mbar_wait(&bars->cfull[st], ph, abort)) return false;
            tc_fence_after();
            const uint32_t sfb = tmem + L::kTmemSFB + st * L::kSFCols;
            const uint64_t dKs = sdesc_add(dK4, st * L::kCode);
#pragma unroll
            for (int kc = 0; kc < D / 64; ++kc)
              tmem_cp_32x128b_x4(sfb + kc * 4, sdesc_add(dKSF, st * L::kSF + kc * 512));
#pragma unroll
            for (int kk = 0; kk < D / 64; ++kk)
              umma_fp4(tmem + L::kTmemS, sdesc_add(dQ, kk * 32), sdesc_add(dKs, kk * 32), idS,
                       tmem + L::kTmemSFA + kk * 4, sfb + kk * 4, kk > 0 ? 1u : 0u);
            umma_commit(&bars->cempty[st]);
          } else {
            if (!mbar_wait(&bars->afull[st], ph, abort)) return false;
            tc_fence_after();
            mma_kmajor<D / 16>(tmem + L::kTmemS, dQ, sdesc_add(dKk, st * L::kTile), idS, false);
          }
          umma_commit(&bars->sfull);
          return true;
        };
        if (ok && n > 0) ok = issue_sdp(0);
        for (int j = 1; ok && j < n; ++j) ok = mbar_wait(&bars->sempty, (j - 1) & 1, abort) && issue_sdp(j);
        // TMEM is freed by this warp: let its own MMAs finish first
        umma_commit(&bars->adone);
        mbar_wait_drain(&bars->adone, 0);
      } else {
        // issuer B: dQ += dS_j K_j.  K_j goes back to the producer after dQ_j
        // (without FP4S, S_j read it too; the rows have read S_j by then).
        for (int j = 0; j < n; ++j) {
          const int st = j & 1;
          if (!mbar_wait(&bars->xfull[0], j & 1, abort) || !mbar_wait(&bars->afull[st], (j >> 1) & 1, abort)) break;
          tc_fence_after();
          mma_a_k_b_mn<kBN / 16>(tmem + L::kTmemDQ, dX, sdesc_add(dKmn, st * L::kTile), idQ, j > 0);
          if (DSPLIT)  // the lo tile of dS
            mma_a_k_b_mn<kBN / 16>(tmem + L::kTmemDQ, sdesc_add(dX, L::kXBytes), sdesc_add(dKmn, st * L::kTile), idQ,
                                   true);
          umma_commit(&bars->xempty[0]);
          umma_commit(&bars->aempty[st]);
        }
        umma_commit(&bars->done);
      }
    }
  } else if (warp >= 2 && warp < 2 + kSoftWarps) {
    const RowRole rr(warp, lane);
    const int col0 = rr.half * 64;
    const int q = qt * kBM + static_cast<int>(rr.row);
    const size_t si = static_cast<size_t>(bh) * a.Lq + (q < a.Lq ? q : 0);
    // with quadrant masks a row may have selected no key at all (LSE = -inf):
    // its dQ is 0, like a row past Lq
    const bool vq = q < a.Lq && (SP != 3 || a.lse[si] > -INFINITY);
    const float lse = vq ? a.lse[si] : 0.0f;
    const float delta = vq ? a.delta[si] : 0.0f;
    const float nlse = vq ? -(lse * kLog2e) : -INFINITY;
    // the fp16 copies of unquantized operands carry powers of two: S arrives
    // as S 2^(eq+ek), dP as dP 2^(edo+ev) (all exact to divide out)
    const float sk = operand_scale(a.amax_k);
    const float cl = FP4S ? a.scale_log2 : a.scale_log2 / (operand_scale(a.amax_q) * sk);
    const float dsc = ds_scale(a.stats);
    const float a1 = dsc / (do_scale(a.stats) * operand_scale(a.amax_v));
    const float b1 = -delta * dsc;
    const int last_valid = a.Lk - (nk - 1) * kBN;
    // the lists ascend, so only the last tile visited can be the partial one;
    // with causal masking the last tile is the diagonal, where row r keeps
    // keys 0..r
    const bool tail_last = SP == 2 ? true : (n > 0 && ktile(n - 1) == nk - 1 && last_valid < kBN);
    const int last_cols = SP == 2 ? static_cast<int>(rr.row) + 1 : last_valid;
    const int qbit = (static_cast<int>(rr.row) >> 6) * 2 + (col0 >> 6);  // SP 3: this thread's quadrant
    const uint32_t xaddr = sbase + L::kX;
    const uint32_t tS = tmem + rr.lane_addr + L::kTmemS, tDP = tmem + rr.lane_addr + L::kTmemDP;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      uint32_t dsw[32], dsl[32];
      uint32_t sv[64], dv[64];
      const bool tail = tail_last && j == n - 1;
      const int vk = last_cols;
      // SP 3: an unselected quadrant (warp-uniform) reads neither S nor dP
      // and stores zero dS
      const bool clear = SP == 3 && !((__ldg(kvl + j) >> (24 + qbit)) & 1);
      if (!mbar_wait(&bars->sfull, j & 1, abort)) { ok = false; break; }
      tc_fence_after();
      if (clear) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->sempty);
#pragma unroll
        for (int k = 0; k < 32; ++k) dsw[k] = dsl[k] = 0u;
      } else {
        load_sdp(tS, tDP, col0, sv, dv);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->sempty);
        if (tail)
          dq_tile<true, DSPLIT>(sv, dv, col0, vk, cl, nlse, a1, b1, dsw, dsl);
        else
          dq_tile<false, DSPLIT>(sv, dv, col0, kBN, cl, nlse, a1, b1, dsw, dsl);
      }
      if (j >= 1 && !mbar_wait(&bars->xempty[0], (j - 1) & 1, abort)) { ok = false; break; }
      store_row_half(xaddr, rr.row, rr.half, dsw);
      if (DSPLIT) store_row_half(xaddr + L::kXBytes, rr.row, rr.half, dsl);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->xfull[0]);
    }
    if (ok && mbar_wait(&bars->done, 0, abort)) {
      tc_fence_after();
      const size_t rowoff = (static_cast<size_t>(bh) * a.Lq + q) * D;
      const float qscale = a.sm_scale / (dsc * sk);  // exact: power-of-two divisors
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const int col = rr.half * (D / 2) + c * 32;
        uint32_t r[32];
        tmem_ld32(tmem + rr.lane_addr + L::kTmemDQ + col, r);
        tmem_ld_wait();
        // every row in range is written; a row with no selected key (SP 3)
        // accumulated only zeros
        if (q < a.Lq) {
          uint4 *dst = reinterpret_cast<uint4 *>(a.dq + rowoff + col);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              w[k] = pack_bf16x2(__uint_as_float(r[8 * i + 2 * k]) * qscale,
                                 __uint_as_float(r[8 * i + 2 * k + 1]) * qscale);
            // no key tile selected: the accumulator was never written
            dst[i] = n > 0 ? make_uint4(w[0], w[1], w[2], w[3]) : make_uint4(0, 0, 0, 0);
          }
        }
      }
    } else {
      mbar_wait_drain(&bars->done, 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ------------------------------------------------------------- launchers --

template <int D, int QP, int FP4S, int SP>
static cudaError_t launch_dkdv_sp(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const CUtensorMap &tdo, const CUtensorMap &tq4, const BwdArgs &a, int BH,
                                  cudaStream_t stream) {
  using L = DkdvLayout<D, FP4S>;
  static_assert(L::kDynSmem <= 232448, "dK/dV shared memory over the 227 KB limit");
  static_assert(sizeof(BwdBars) <= L::kBarBytes, "dK/dV barrier block larger than its reservation");
  static_assert(L::kTmemSFB + L::kSFCols <= L::kTmemCols, "dK/dV TMEM over 512 columns");
  auto kern = attn_bwd_dkdv_kernel<D, QP, FP4S, SP, kDkdvRG>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kern), L::kDynSmem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.nk_tiles, BH), dkdv_threads<kDkdvRG>(), L::kDynSmem, stream>>>(tq, tk, tv, tdo, tq4, a);
  return cudaGetLastError();
}

template <int D, int QP, int FP4S>
static cudaError_t launch_dkdv_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                 const CUtensorMap &tdo, const CUtensorMap &tq4, const BwdArgs &a, int BH,
                                 cudaStream_t stream) {
  if (!a.q_list) return launch_dkdv_sp<D, QP, FP4S, 0>(tq, tk, tv, tdo, tq4, a, BH, stream);
  if (a.quad) return launch_dkdv_sp<D, QP, FP4S, 3>(tq, tk, tv, tdo, tq4, a, BH, stream);
  return a.causal ? launch_dkdv_sp<D, QP, FP4S, 2>(tq, tk, tv, tdo, tq4, a, BH, stream)
                  : launch_dkdv_sp<D, QP, FP4S, 1>(tq, tk, tv, tdo, tq4, a, BH, stream);
}

template <int D>
static cudaError_t dkdv_dispatch(bool fp4s, bool quant_p, const CUtensorMap &tq, const CUtensorMap &tk,
                                 const CUtensorMap &tv, const CUtensorMap &tdo, const CUtensorMap &tq4,
                                 const BwdArgs &a, int BH, cudaStream_t stream) {
  if (fp4s)
    return quant_p ? launch_dkdv_t<D, 1, 1>(tq, tk, tv, tdo, tq4, a, BH, stream)
                   : launch_dkdv_t<D, 0, 1>(tq, tk, tv, tdo, tq4, a, BH, stream);
  return quant_p ? launch_dkdv_t<D, 1, 0>(tq, tk, tv, tdo, tq4, a, BH, stream)
                 : launch_dkdv_t<D, 0, 0>(tq, tk, tv, tdo, tq4, a, BH, stream);
}

cudaError_t launch_bwd_dkdv(int D, bool fp4s, bool quant_p, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, const CUtensorMap &tdo, const CUtensorMap &tq4,
                            const BwdArgs &a, int BH, cudaStream_t stream) {
  return D == 128 ? dkdv_dispatch<128>(fp4s, quant_p, tq, tk, tv, tdo, tq4, a, BH, stream)
                  : dkdv_dispatch<64>(fp4s, quant_p, tq, tk, tv, tdo, tq4, a, BH, stream);
}

template <int D, int FP4S, int DSPLIT, int SP>
static cudaError_t launch_dq_sp(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                const CUtensorMap &tdo, const CUtensorMap &tk4, const BwdArgs &a, int BH,
                                cudaStream_t stream) {
  using L = DqLayout<D, FP4S, DSPLIT>;
  static_assert(L::kDynSmem <= 232448, "dQ shared memory over the 227 KB limit");
  static_assert(sizeof(BwdBars) <= L::kBarBytes, "dQ barrier block larger than its reservation");
  static_assert(L::kTmemSFB + 2 * L::kSFCols <= L::kTmemCols, "dQ TMEM over 512 columns");
  auto kern = attn_bwd_dq_kernel<D, FP4S, DSPLIT, SP>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kern), L::kDynSmem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.nq_tiles, BH), kThreads, L::kDynSmem, stream>>>(tq, tk, tv, tdo, tk4, a);
  return cudaGetLastError();
}

template <int D, int FP4S, int DSPLIT>
static cudaError_t launch_dq_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                               const CUtensorMap &tdo, const CUtensorMap &tk4, const BwdArgs &a, int BH,
                               cudaStream_t stream) {
  if (!a.kv_list) return launch_dq_sp<D, FP4S, DSPLIT, 0>(tq, tk, tv, tdo, tk4, a, BH, stream);
  if (a.quad) return launch_dq_sp<D, FP4S, DSPLIT, 3>(tq, tk, tv, tdo, tk4, a, BH, stream);
  return a.causal ? launch_dq_sp<D, FP4S, DSPLIT, 2>(tq, tk, tv, tdo, tk4, a, BH, stream)
                  : launch_dq_sp<D, FP4S, DSPLIT, 1>(tq, tk, tv, tdo, tk4, a, BH, stream);
}

template <int D>
static cudaError_t dq_dispatch(bool fp4s, bool dsplit, const CUtensorMap &tq, const CUtensorMap &tk,
                               const CUtensorMap &tv, const CUtensorMap &tdo, const CUtensorMap &tk4,
                               const BwdArgs &a, int BH, cudaStream_t stream) {
  if (!fp4s) return launch_dq_t<D, 0, 1>(tq, tk, tv, tdo, tk4, a, BH, stream);
  return dsplit ? launch_dq_t<D, 1, 1>(tq, tk, tv, tdo, tk4, a, BH, stream)
                : launch_dq_t<D, 1, 0>(tq, tk, tv, tdo, tk4, a, BH, stream);
}

cudaError_t launch_bwd_dq(int D, bool fp4s, bool dsplit, const CUtensorMap &tq, const CUtensorMap &tk,
                          const CUtensorMap &tv, const CUtensorMap &tdo, const CUtensorMap &tk4, const BwdArgs &a,
                          int BH, cudaStream_t stream) {
  return D == 128 ? dq_dispatch<128>(fp4s, dsplit, tq, tk, tv, tdo, tk4, a, BH, stream)
                  : dq_dispatch<64>(fp4s, dsplit, tq, tk, tv, tdo, tk4, a, BH, stream);
}

}  // namespace attnqat
