// Forward pass of exact attention on sm_100a: O = softmax(scale Q K^T [causal]) V
// and the row log-sum-exp, tile by tile, with no N x N matrix in HBM.
//
// Sources (page title, section):
//   "Flash Attention spiegata: una guida completa" (datacamp), "Tiling": Q, K
//   and V are split into tiles that sit in fast on-chip memory and each tile is
//   processed end to end with the softmax applied incrementally.
//   "FlashAttention-2" (systems-analysis.info wiki), "Техническая архитектура и
//   принципы работы": (1) fewer non-matmul operations -- here the running
//   maximum is only applied to the output when it grows by more than 2^8, and
//   the 1/l normalisation happens once at the end; (2) parallelism over the
//   sequence -- every CTA owns up to 256 query rows of one (batch, head); (3)
//   work split across warps so that softmax statistics never go through shared
//   memory -- here one thread owns one query row, read straight from TMEM.
//   "Flash Attention spiegata", "Specializzazione dei warp" and "TMA":
//   producer and consumer warps and asynchronous tile copies (Hopper-era prior
//   art, restated for tcgen05).
//
// CTA layout (384 threads, three warpgroups):
//   warps 0-3  softmax warpgroup for query tile 0 (rows r0 .. r0+127)
//   warps 4-7  softmax warpgroup for query tile 1 (rows r0+128 .. r0+255)
//   warp  8    TMA producer (Q once, then a ring of K and V tiles)
//   warp  9    MMA issuer (tcgen05, one thread)
//   warps 10-11 idle (they complete the third warpgroup)
// The kernel is compiled for 168 registers per thread (384 x 168 = 64512); the
// third warpgroup gives registers back (down to 72) and the two softmax
// warpgroups take them (up to 216): 2 x 128 x 216 + 128 x 72 = 64512, so the
// re-split never asks for more than the launch holds.  (232 / 40 and 224 / 56
// made the MMA issuer spill.)  The host refuses to launch a build whose register
// count is not 168.
//
// TMEM (512 columns x 128 lanes, fp32): S_t at column 128 t, O_t at 256 + D t.
// P_t (16-bit) overwrites the first 64 columns of S_t and feeds the P V MMA
// straight from TMEM.  The MMA warp alternates between the two query tiles so
// that one warpgroup's softmax overlaps the other tile's matrix products.  At
// D = 64 the two P have columns of their own (384 and 448), so S of step j + 1
// is computed as soon as the softmax has read S of step j.
//
// A CTA with one query tile -- short or decode-like queries, and every CTA at
// tile widths D = 192 / 256, where two D-column accumulators would not fit TMEM
// -- instead uses both S column blocks as a double buffer (S of step j + 1 is
// computed while the softmax of step j runs) and its idle second Q slot, if
// any, as one more V stage.  Decode-like calls may also cut the keys into
// stretches (one per blockIdx.y) and replicate up to 64 queries down the tile
// so every softmax warp has rows to work on; both write partial results that
// fa2_decode.cuh merges.  With 8-bit inputs (F8) the tiles are 128 bytes wide,
// the products are kind::f8f6f4 MMAs and P is rounded to E4M3, four per TMEM
// column.
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace fa2 {

struct FwdParams {
  void* O;                     // [BH][Nq][d] 16-bit (unused when the keys are split)
  float* LSE;                  // [BH][Nq]            (unused when the keys are split)
  int d;                       // head dim: 16-bit inputs D - 64 < d <= D, a multiple of 8;
                               // 8-bit inputs a multiple of 16 up to 128 (columns past d
                               // of the tiles are TMA zero fill and are never stored)
  int Nq;                      // query rows per (batch, head)
  int Nk;                      // key / value rows per (batch, head)
  int off;                     // causal only: query row i sees keys <= i + off (Nk - Nq)
  int BH;                      // batch * heads
  int n_qblk;                  // ceil(Nq / (128 QT)): query blocks per (batch, head)
  int head_group;              // heads per group of the block order (1 .. BH)
  float scale_log2;            // scale * log2(e)
  unsigned int* status;        // device status word
  unsigned long long wait_ns;  // budget of one bounded wait
  int fault;                   // test hook: 1 = skip the first K load
  int window;                  // causal only: row i sees keys i+off-window+1..i+off (0 = none)
  float o_scale;               // 8-bit inputs: the scale of V, applied with 1/l
  // Split keys (blockIdx.y = split): CTA y covers key tiles [y kv_per_split,
  // (y + 1) kv_per_split) and writes its rows' partial results, normalised by
  // its own row sums, to O_part [split][BH][Nq][D] (D columns, the padding
  // included) and LSE_part [split][BH][Nq]
  // (float, -inf for a row that sees no key of the split).  kv_per_split = 0:
  // all key tiles.  O_part = nullptr: O and LSE are written directly.
  int kv_per_split;
  float* O_part;
  float* LSE_part;
};

template <int D, bool F8 = false, bool ONE = false>
struct FwdCfg {
  static_assert(D == 64 || D == 128 || D == 192 || D == 256, "tile head dims");
  static_assert(!F8 || D == 128, "8-bit inputs use 128-byte tiles");
  static constexpr int ESZ = F8 ? 1 : 2;          // bytes per Q/K/V element
  static constexpr int KE = 32 / ESZ;             // K elements per MMA instruction (32 bytes)
  static constexpr int CHUNK_COLS = 128 / ESZ;    // elements per 128-byte swizzle row
  static constexpr int BM = 128;                  // query rows per tile
  static constexpr int BN = 128;                  // keys per tile
  // Query tiles per CTA: two (ping-pong) up to D = 128; one above, where two
  // D-column output accumulators and two S blocks would exceed TMEM's 512
  // columns (S double buffer 256 + O D <= 512 still fits).  ONE asks for one
  // query tile at D <= 128 too: twice the CTAs, for grids that would otherwise
  // leave SMs idle.
  static constexpr int QT = (D <= 128 && !ONE) ? 2 : 1;
  static constexpr int KCH = D * ESZ / 128;       // 128-byte swizzle chunks along d
  static constexpr int CHUNK = 128 * 128;         // bytes of one 128-row x 128-byte chunk
  static constexpr int TILE = 128 * D * ESZ;      // bytes of one 128-row tile
  // K and V ring stages within 227 KB of shared memory (by tile size: 16, 32,
  // 48 or 64 KB).
  static constexpr int KS = (TILE == 16384) ? 4 : (TILE == 65536 ? 1 : 2);
  static constexpr int VS = (TILE == 16384) ? 4 : (TILE == 32768 ? 2 : 1);
  // With one query tile in the CTA, the second Q slot (if any) is one more V stage.
  static constexpr int VX = (QT == 2) ? 1 : 0;
  static constexpr int SMEM = (QT + KS + VS) * TILE + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static constexpr int THREADS = 384;
  static constexpr int LAUNCH_REGS = 168;  // per thread, as compiled (checked on the host)
#ifndef FA2_FWD_SOFT_REGS
#define FA2_FWD_SOFT_REGS 216
#endif
  static constexpr int SOFT_REGS = FA2_FWD_SOFT_REGS;
  static constexpr int OTHER_REGS = (THREADS * LAUNCH_REGS - 2 * 128 * SOFT_REGS) / 128 / 8 * 8;
  static_assert(2 * 128 * SOFT_REGS + 128 * OTHER_REGS <= THREADS * LAUNCH_REGS,
                "register re-split exceeds the launch allocation");
  static constexpr uint32_t S_COL0 = 0, S_COL1 = 128;
  static constexpr uint32_t O_COL0 = 256, O_COL1 = 256 + D;
  // D = 64 with two query tiles: each tile's P has its own 64 columns after the
  // two O blocks, so the S block is free as soon as the softmax has read it.
  static constexpr bool SEP_P = (D == 64);
  static constexpr uint32_t P_COL0 = 384, P_COL1 = 448;
};

// Pairs i of a score row with (i & 3) >= kPolyFrom take the polynomial exp2
// (4: none, 3: one pair in four, 2: half).  Measured on B200 (d = 128): the FMA
// and ALU pipes, not the MUFU unit, bound the softmax, and moving exponentials
// onto them slows the kernel (one in four: -13 %, half: -20 %), so none do.
#ifndef FA2_POLY_FROM
#define FA2_POLY_FROM 4
#endif
constexpr int kPolyFrom = FA2_POLY_FROM;
// The same split for 8-bit inputs, whose matrix products take half the tensor
// time, leaving the exponential unit the busiest pipe.
#ifndef FA2_POLY_FROM_F8
#define FA2_POLY_FROM_F8 4
#endif
constexpr int kPolyFromF8 = FA2_POLY_FROM_F8;

// Wait-site ids reported through the status word.
enum FwdSite : uint32_t {
  kSiteProdKEmpty = 1, kSiteProdVEmpty, kSiteMmaQ, kSiteMmaK, kSiteMmaV, kSiteMmaP,
  kSiteMmaDrain, kSiteSoftS, kSiteSoftO, kSiteSoftOEnd, kSiteProdDrain
};

// F8: Q, K, V are E4M3 bytes (D = 128-byte tiles, REP = 1), the products are
// kind::f8f6f4 MMAs, P is rounded to E4M3 for P V, and O is bf16 (BF16 = true);
// the per-tensor scales of Q and K are folded into scale_log2 and that of V into
// o_scale.
// REP: query copies (1, 2 or 4; > 1 only with Nq <= 128 / REP and partial
// results).  The 128-row Q tile then holds REP copies of the Nq queries, loaded
// through tmQr (boxes of 128 / REP rows), and copy c scores only key columns
// [c 128 / REP, (c + 1) 128 / REP) of every key tile, as partial result
// blockIdx.y * REP + c: a lone query keeps four softmax warps busy, not one.
template <int D, bool BF16, bool CAUSAL, int REP, bool F8 = false, bool ONE = false>
__global__ void __launch_bounds__(384, 1)
fa2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQr,
               const FwdParams p) {
  static_assert(!F8 || (BF16 && REP == 1), "8-bit inputs: bf16 output, no query copies");
  using C = FwdCfg<D, F8, ONE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::QT * C::TILE;
  uint8_t* sV = sK + C::KS * C::TILE;

  __shared__ uint64_t bar_q, k_full[C::KS], k_empty[C::KS], v_full[C::VS + C::VX],
      v_empty[C::VS + C::VX];
  __shared__ uint64_t s_full[2], s_free[2], p_ready[2], o_done[2], drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  // A merge kernel queued behind this grid (decode-like calls) may launch now:
  // it waits for this grid's completion before reading anything.
  griddep_launch_dependents();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int Nq = p.Nq, Nk = p.Nk;
  const int off = CAUSAL ? p.off : 0;
  const bool split = p.kv_per_split > 0;    // keys cut into stretches (blockIdx.y)
  const bool partial = p.O_part != nullptr;  // partial results, merged by a second kernel

  // Block order: head group by head group (head_group heads each, the last group
  // possibly smaller), and within a group the heaviest query blocks first (they
  // see the most keys when causal).  A group spans about two waves of CTAs, so the
  // CTAs running at any one time share a few heads and their K and V tiles come
  // from L2 (head_group = BH orders every head's blocks together).
  const int qb_bh_x = static_cast<int>(blockIdx.x);
  const int grp_blocks = p.head_group * p.n_qblk;
  const int hgrp = qb_bh_x / grp_blocks;
  const int hpos = qb_bh_x - hgrp * grp_blocks;
  const int hcnt = min(p.head_group, p.BH - hgrp * p.head_group);
  const int qb = p.n_qblk - 1 - hpos / hcnt;
  const int bh = hgrp * p.head_group + hpos % hcnt;
  const int n_kv_all = (Nk + C::BN - 1) / C::BN;
  // Key tiles of this CTA's split (all of them when the keys are not split).
  const int s_lo = split ? static_cast<int>(blockIdx.y) * p.kv_per_split : 0;
  const int s_hi = split ? min(n_kv_all, s_lo + p.kv_per_split) : n_kv_all;
  // Key tiles [j_lo[t], j_hi[t]) are the ones query tile t needs: all of them,
  // or (causal) up to the one holding the last key its last row sees, and
  // (sliding window) from the tile that holds the first key its first row still
  // sees; then cut to the split.  Tiles past Nq have an empty range.
  int row0[2], j_lo[2], j_hi[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    row0[t] = qb * (C::QT * C::BM) + t * C::BM;
    j_lo[t] = 0;
    if (row0[t] >= Nq || t >= C::QT) {
      j_hi[t] = 0;
    } else if (CAUSAL) {
      j_hi[t] = min(n_kv_all, (min(row0[t] + C::BM - 1, Nq - 1) + off) / C::BN + 1);
      if (p.window > 0) j_lo[t] = max(0, row0[t] + off - p.window + 1) / C::BN;
    } else {
      j_hi[t] = n_kv_all;
    }
    j_lo[t] = max(j_lo[t], s_lo);
    j_hi[t] = min(j_hi[t], s_hi);
    if (j_hi[t] <= j_lo[t]) j_lo[t] = j_hi[t] = 0;  // nothing to do for this tile
  }
  const bool has0 = j_hi[0] > 0, has1 = j_hi[1] > 0;
  // The CTA walks key tiles j0 .. j1-1; the K/V ring is indexed from j0.
  const int j0 = has0 ? (has1 ? min(j_lo[0], j_lo[1]) : j_lo[0]) : j_lo[1];
  const int j1 = max(j_hi[0], j_hi[1]);
  const int n_steps = j1 - j0;
  // A CTA with one query tile runs it double-buffered (see the MMA issuer).
  const bool single = C::QT == 1 || !has1;
  // Two query tiles at D = 64: P in its own columns, S(j + 1) issued once S(j) is read.
  const bool sep = C::SEP_P && !single;

  WaitCtl wc{p.status, &abort_flag, p.wait_ns};

  // The producer thread sets up the barriers and sends Q and the first K tile out
  // at once, so that their latency overlaps the TMEM allocation and the block-wide
  // barrier (a CTA's set-up up to its first scores took 2.8 us on the training
  // shape, 0.9 us of it before the first load).
  const bool prod0 = warp == 8 && lane == 0;
  bool k0_early = false;  // K tile 0 issued in the set-up
  if (prod0) {
    abort_flag = 0;
    mbar_init(&bar_q, 1);
    for (int s = 0; s < C::KS; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < C::VS + C::VX; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_free[t], 4);
      mbar_init(&p_ready[t], 4);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(&drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    uint32_t q_bytes = 0;
    for (int t = 0; t < 2; ++t) q_bytes += (j_hi[t] > 0) ? C::TILE : 0;
    // (A CTA whose split holds no key any of its rows sees loads nothing.)
    mbar_arrive_expect_tx(&bar_q, q_bytes);
    if constexpr (REP > 1) {
      // REP copies of rows 0 .. 128/REP - 1 (tile 0 only), one box each.
      if (j_hi[0] > 0) {
        tma_prefetch_desc(&tmQr);
        constexpr int qr = C::BM / REP;
        for (int r = 0; r < REP; ++r)
          for (int c = 0; c < C::KCH; ++c)
            tma_load_3d(sQ + c * C::CHUNK + r * qr * 128, &tmQr, &bar_q, c * C::CHUNK_COLS, 0, bh);
      }
    } else {
      for (int t = 0; t < 2; ++t) {
        if (j_hi[t] == 0) continue;
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sQ + t * C::TILE + c * C::CHUNK, &tmQ, &bar_q, c * C::CHUNK_COLS, row0[t], bh);
      }
    }
    if (n_steps > 0 && p.fault != 1) {  // the test hook skips K tile 0 (see load_k)
      const uint64_t keep = policy_evict_last();
      mbar_arrive_expect_tx(&k_full[0], C::TILE);
      for (int c = 0; c < C::KCH; ++c)
        tma_load_3d_hint(sK + c * C::CHUNK, &tmK, &k_full[0], c * 64, j0 * C::BN, bh, keep);
      k0_early = true;
    }
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;

  if (warp >= 8) {
  // Third warpgroup: every warp executes the same register release first.
  regs_dec<C::OTHER_REGS>();
  if (warp >= 10) {
    // idle warps of the third warpgroup
  } else if (warp == 8) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      // Q and K tile 0 went out in the set-up.
      const uint64_t keep = policy_evict_last();
      // With one query tile the second Q slot (if any) is one more V stage.
      const int vring = single ? C::VS + C::VX : C::VS;
      int k_issued = 0, v_issued = 0;  // loads issued so far
      auto load_k = [&](int jj) -> bool {
        if (jj == 0 && k0_early) {
          k_issued = 1;
          return true;
        }
        const int ks = jj % C::KS;
        if (jj >= C::KS && !mbar_wait(&k_empty[ks], ((jj / C::KS) - 1) & 1, wc, kSiteProdKEmpty))
          return false;
        if (!(p.fault == 1 && jj == 0)) {
          mbar_arrive_expect_tx(&k_full[ks], C::TILE);
          for (int c = 0; c < C::KCH; ++c)
            tma_load_3d_hint(sK + ks * C::TILE + c * C::CHUNK, &tmK, &k_full[ks], c * 64,
                             (j0 + jj) * C::BN, bh, keep);
          k_issued = jj + 1;
        }
        return true;
      };
      auto load_v = [&](int jj) -> bool {
        const int vs = jj % vring;
        if (jj >= vring && !mbar_wait(&v_empty[vs], ((jj / vring) - 1) & 1, wc, kSiteProdVEmpty))
          return false;
        uint8_t* dst = vs < C::VS ? sV + vs * C::TILE : sQ + C::TILE;
        mbar_arrive_expect_tx(&v_full[vs], C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d_hint(dst + c * C::CHUNK, &tmV, &v_full[vs], c * C::CHUNK_COLS, (j0 + jj) * C::BN, bh,
                           keep);
        v_issued = jj + 1;
        return true;
      };
      // Loads go out in the order the MMA warp consumes them: with one query
      // tile, K of step jj + 1 (for S) is needed before V of step jj, and a V
      // slot waiting for its P V product must not hold back the next K.
      bool ok = true;
      if (single) {
        ok = n_steps == 0 || load_k(0);
        for (int jj = 0; jj < n_steps && ok; ++jj)
          ok = (jj + 1 >= n_steps || load_k(jj + 1)) && load_v(jj);
      } else {
        for (int jj = 0; jj < n_steps && ok; ++jj) ok = load_k(jj) && load_v(jj);
      }
      if (!ok) {
        // Let every copy already issued land before the CTA exits.
        volatile int no_abort = 0;
        WaitCtl dw{p.status, &no_abort, 100000000ull};
        // The last load put into each ring slot is load jj; its phase is jj / stages.
        for (int jj = max(0, k_issued - C::KS); jj < k_issued; ++jj)
          if (!(p.fault == 1 && jj == 0))
            mbar_wait(&k_full[jj % C::KS], (jj / C::KS) & 1, dw, kSiteProdDrain);
        for (int jj = max(0, v_issued - vring); jj < v_issued; ++jj)
          mbar_wait(&v_full[jj % vring], (jj / vring) & 1, dw, kSiteProdDrain);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_qk =
          F8 ? idesc_e4m3(128, 128, false, false) : idesc_f16(128, 128, BF16, false, false);
      constexpr uint32_t id_pv =
          F8 ? idesc_e4m3(128, D, false, true) : idesc_f16(128, D, BF16, false, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);

      // S = Q_t K^T into S buffer b; O_t += P_b V.
      // K steps of 32 bytes: 4 per 128-byte swizzle row, then the next chunk.
      auto issue_qk = [&](int t, int b, int ks) {
#pragma unroll
        for (int kk = 0; kk < D / C::KE; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          const uint32_t dt = tbase + (b ? C::S_COL1 : C::S_COL0);
          const uint64_t da = sdesc_sw128(sQa + t * C::TILE + off, 16, 1024);
          const uint64_t db = sdesc_sw128(sKa + ks * C::TILE + off, 16, 1024);
          if constexpr (F8) umma_ss_f8(dt, da, db, id_qk, kk > 0);
          else umma_ss(dt, da, db, id_qk, kk > 0);
        }
      };
      // V ring slot vs: the V stages, then (one query tile) the second Q slot.
      auto v_addr = [&](int vs) -> uint32_t {
        return vs < C::VS ? sVa + vs * C::TILE : sQa + C::TILE;
      };
      // P from TMEM (8 columns = 32 bytes of keys per step), V MN-major: a step
      // of KE keys advances KE rows of 128 bytes.
      auto issue_pv = [&](int t, uint32_t a_col, int vs, bool acc) {
        const uint32_t va = v_addr(vs);
#pragma unroll
        for (int kk = 0; kk < C::BN / C::KE; ++kk) {
          const uint32_t dt = tbase + (t ? C::O_COL1 : C::O_COL0);
          const uint32_t at = tbase + a_col + kk * 8;
          const uint64_t db = sdesc_sw128(va + kk * C::KE * 128, C::CHUNK, 1024);
          if constexpr (F8) umma_ts_f8(dt, at, db, id_pv, (acc || kk > 0) ? 1u : 0u);
          else umma_ts(dt, at, db, id_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      const int lo0 = j_lo[0], hi0 = j_hi[0], lo1 = j_lo[1], hi1 = j_hi[1];

      bool ok = n_steps > 0 && mbar_wait(&bar_q, 0, wc, kSiteMmaQ) &&
                mbar_wait(&k_full[0], 0, wc, kSiteMmaK);
      if (single) {
        // One query tile: S is double-buffered in the two S column blocks, and
        // S of step jj + 1 is issued before P of step jj is awaited, so the
        // softmax of one step overlaps the P V product of the one before.
        if (ok) {
          tc_fence_after();
          issue_qk(0, 0, 0);
          umma_commit(&s_full[0]);
          umma_commit(&k_empty[0]);
        }
        for (int jj = 0; jj < n_steps && ok; ++jj) {
          const int b = jj & 1;
          if (jj + 1 < n_steps) {
            // Buffer b^1 held P of step jj - 1, consumed by the P V product
            // issued (in order, before this) in the previous iteration.
            const int ks1 = (jj + 1) % C::KS;
            if (!mbar_wait(&k_full[ks1], ((jj + 1) / C::KS) & 1, wc, kSiteMmaK)) { ok = false; break; }
            tc_fence_after();
            issue_qk(0, b ^ 1, ks1);
            umma_commit(&s_full[b ^ 1]);
            umma_commit(&k_empty[ks1]);
          }
          constexpr int VR = C::VS + C::VX;  // V ring with the second Q slot
          const int vs = jj % VR;
          if (!mbar_wait(&v_full[vs], (jj / VR) & 1, wc, kSiteMmaV) ||
              !mbar_wait(&p_ready[b], (jj >> 1) & 1, wc, kSiteMmaP)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(0, b ? C::S_COL1 : C::S_COL0, vs, jj > 0);
          umma_commit(&o_done[0]);
          umma_commit(&v_empty[vs]);
        }
        ok = false;  // the two-tile loop below is skipped
      }
      if (ok) {
        tc_fence_after();
        // Tiles whose key range starts at j0 get their first S now.
        if (hi0 > lo0 && lo0 == j0) {
          issue_qk(0, 0, 0);
          umma_commit(&s_full[0]);
        }
        if (hi1 > lo1 && lo1 == j0) {
          issue_qk(1, 1, 0);
          umma_commit(&s_full[1]);
        }
        umma_commit(&k_empty[0]);
      }
      for (int jj = 0; jj < n_steps && ok; ++jj) {
        const int j = j0 + jj;
        const int vs = jj % C::VS;
        const int ks1 = (jj + 1) % C::KS;
        const bool has_next = jj + 1 < n_steps;
        bool k_next_ready = false;
        if (!mbar_wait(&v_full[vs], (jj / C::VS) & 1, wc, kSiteMmaV)) { ok = false; break; }
        auto next_s = [&](int t, int lo, int hi) -> bool {
          // S for step j + 1 (this tile's next step, or its first when its range
          // starts there).
          if (j + 1 >= lo && j + 1 < hi) {
            if (sep && j >= lo) {
              // The S block still holds S of step j until the softmax has read it.
              if (!mbar_wait(&s_free[t], (j - lo) & 1, wc, kSiteMmaP)) return false;
              tc_fence_after();
            }
            if (!k_next_ready) {
              if (!mbar_wait(&k_full[ks1], ((jj + 1) / C::KS) & 1, wc, kSiteMmaK)) return false;
              tc_fence_after();
              k_next_ready = true;
            }
            issue_qk(t, t, ks1);
            umma_commit(&s_full[t]);
          }
          return true;
        };
        auto pv = [&](int t, int lo, int hi) -> bool {
          if (j >= lo && j < hi) {
            const int step = j - lo;  // this tile's own step count
            if (!mbar_wait(&p_ready[t], step & 1, wc, kSiteMmaP)) return false;
            tc_fence_after();
            const uint32_t a_col = sep ? (t ? C::P_COL1 : C::P_COL0) : (t ? C::S_COL1 : C::S_COL0);
            issue_pv(t, a_col, vs, step > 0);
            umma_commit(&o_done[t]);
          }
          return true;
        };
        if (sep) {
          // Both tiles' next S as soon as their scores are read, then the P V products.
          ok = next_s(0, lo0, hi0) && next_s(1, lo1, hi1) && pv(0, lo0, hi0) && pv(1, lo1, hi1);
        } else {
          // P of step j sits in the S block: P V first, then the next S over it.
          ok = pv(0, lo0, hi0) && next_s(0, lo0, hi0) && pv(1, lo1, hi1) && next_s(1, lo1, hi1);
        }
        if (ok && has_next && !k_next_ready)  // a slot is only released once its load landed
          ok = mbar_wait(&k_full[ks1], ((jj + 1) / C::KS) & 1, wc, kSiteMmaK);
        if (!ok) break;
        umma_commit(&v_empty[vs]);
        if (has_next) umma_commit(&k_empty[ks1]);
      }
      // Every MMA issued above completes before TMEM is released.
      umma_commit(&drain);
      volatile int no_abort = 0;
      WaitCtl dw{p.status, &no_abort, p.wait_ns};
      mbar_wait(&drain, 0, dw, kSiteMmaDrain);
    }
    __syncwarp();
  }
  } else {
    // ------------------------------------------------------------------ softmax
    regs_inc<C::SOFT_REGS>();
    const int t = warp >> 2;      // query tile of this warpgroup
    const int wq = warp & 3;      // TMEM lane quadrant
    const int r_loc = wq * 32 + lane;
    const int my_row0 = t ? row0[1] : row0[0];
    const int my_lo = t ? j_lo[1] : j_lo[0];
    const int my_nkv = (t ? j_hi[1] : j_hi[0]) - my_lo;  // steps of this tile
    // With REP > 1 the tile holds REP copies of its QR = 128 / REP query rows;
    // copy qcopy (warp-uniform) owns key columns qcopy * 128 / REP onwards.
    constexpr int QR = C::BM / REP;
    const int qcopy = r_loc / QR;
    const int row = my_row0 + r_loc % QR;
    const uint32_t o_col = t ? C::O_COL1 : C::O_COL0;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32);
    const float sl2 = p.scale_log2;  // > 0 (checked on the host)
    float m = -INFINITY;  // running max, log2 units of scaled scores
    float l = 0.f;        // running sum of exp2(s * sl2 - m): the log-sum-exp
    // Running sum of the same values as rounded to 16 bits, the weights the P V
    // product actually applies: O is divided by this one, so that it is an exact
    // weighted average of V rows.  (Dividing by the unrounded sum adds the rounding
    // error of P to O: up to 2^-9 |v| on a row dominated by one key, which the
    // long-context workload with its x8 key outliers shows.)  8-bit inputs keep the
    // unrounded sum.
    float lr = 0.f;
    bool ok = my_nkv > 0;
    const int win = p.window;
    // A warp whose 32 rows are all past Nq only keeps the barrier count: its P
    // rows feed output rows that are never stored.
    const bool live = my_row0 + (wq * 32) % QR < Nq;

    // One step of the online softmax over the NC key columns this warp owns:
    // S from TMEM, masks, running max (with the lazy output rescale), P back to
    // TMEM in 16-bit over the first 64 columns of the S buffer -- zeros in the
    // columns of the other copies -- and the running sum.  False if a wait ran out.
    auto soft_step = [&](auto nc_tag, int step, uint32_t s_col) -> bool {
      constexpr int NC = decltype(nc_tag)::value;
      constexpr int EPC = 4 / C::ESZ;             // P values per 32-bit TMEM column
      constexpr int NP = NC / EPC;                // packed columns of P
      constexpr int G = NP < 32 ? NP : 32;        // columns per TMEM store
      const int col0 = qcopy * NC;
      uint32_t sr[NC];
#pragma unroll
      for (int c = 0; c < NC / 32; ++c)
        tmem_ld32(tmem_addr(tbase, lane_base, s_col + col0 + 32 * c),
                  *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
      tmem_wait_ld();
      reg_fence(sr);
      if (sep) {  // the S block may now take the next scores
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[t]);
      }
      const int kc0 = (my_lo + step) * C::BN + col0;  // key of column 0 of sr
      // Keys after the row's last one (causal), past Nk, or before the row's
      // window start.
      const bool need_mask = (CAUSAL && kc0 + NC - 1 > my_row0 + off) || (kc0 + NC > Nk) ||
                             (CAUSAL && win > 0 && kc0 < my_row0 + off + 127 - win + 1);
      if (need_mask) {
        const int hi_lim = CAUSAL ? min(row + off - kc0 + 1, Nk - kc0) : (Nk - kc0);
        const int lo_lim = (CAUSAL && win > 0) ? row + off - win + 1 - kc0 : 0;
#pragma unroll
        for (int i = 0; i < NC; ++i)
          if (i >= hi_lim || i < lo_lim) sr[i] = __float_as_uint(-INFINITY);
      }
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mx[k] = fmax3(__uint_as_float(sr[k]), __uint_as_float(sr[k + 8]), __uint_as_float(sr[k + 16]));
#pragma unroll
      for (int i = 24; i + 24 <= NC; i += 16)  // elements 24 .. NC - 9
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mx[k] = fmax3(mx[k], __uint_as_float(sr[i + k]), __uint_as_float(sr[i + k + 8]));
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmaxf(mx[k], __uint_as_float(sr[NC - 8 + k]));
      mx[0] = fmax3(mx[0], mx[1], mx[2]);
      mx[3] = fmax3(mx[3], mx[4], mx[5]);
      mx[6] = fmaxf(mx[6], mx[7]);
      mx[0] = fmax3(mx[0], mx[3], mx[6]);
      const float m_new = fmaxf(m, mx[0] * sl2);
      if (step == 0) {
        m = m_new;  // -inf when the window hides this whole tile from the row
      } else {
        // Lazy rescale: the stale maximum is kept unless it fell behind by more
        // than 8 (a factor 256 in the exponentials); the output accumulator is
        // only touched in that case, after the previous P V product landed.
        // (The product before that one finished before this step's S, which
        // this warp has seen, so the barrier is at most one phase behind.)
        const bool need = m_new - m > 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? ex2_approx(m - m_new) : 1.0f;
          if (need) m = m_new;
          l *= f;
          lr *= f;
          if (!__all_sync(0xffffffffu, mbar_wait(&o_done[t], (step - 1) & 1, wc, kSiteSoftO)))
            return false;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tbase, lane_base, o_col + 32 * c), r);
            tmem_wait_ld();
            reg_fence(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
            tmem_st32(tmem_addr(tbase, lane_base, o_col + 32 * c), r);
          }
        }
      }
      // P = 2^(s * scale * log2 e - m): arguments two at a time (f32x2),
      // exponentials on the MUFU unit (or the polynomial, see kPolyFrom).
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      // A row that has seen no key yet (m = -inf) gets exp2(-inf) = 0 everywhere.
      const float neg_m = (m == -INFINITY) ? 0.f : -m;
      const uint64_t negm2 = f2_pack(neg_m, neg_m);
      uint64_t sum2[4] = {0, 0, 0, 0};
      [[maybe_unused]] uint64_t sumr2[4] = {0, 0, 0, 0};  // of the 16-bit P values
      // With its own P columns the previous P V product may still be reading them.
      if (sep && step > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(&o_done[t], (step - 1) & 1, wc, kSiteSoftO)))
          return false;
        tc_fence_after();
      }
      const uint32_t p_col = sep ? (t ? C::P_COL1 : C::P_COL0) : s_col;
#pragma unroll
      for (int h = 0; h < NP / G; ++h) {
        uint32_t pk[G];
#pragma unroll
        for (int i = 0; i < G; ++i) {
          float e[EPC];
#pragma unroll
          for (int q = 0; q < EPC / 2; ++q) {
            const int k = EPC * (G * h + i) + 2 * q;  // first of the pair in sr
            const int pi = (EPC / 2) * i + q;         // pair count within the store
            const uint64_t arg = f2_fma(
                f2_pack(__uint_as_float(sr[k]), __uint_as_float(sr[k + 1])), sl2x2, negm2);
            float a, b;
            f2_unpack(arg, a, b);
            if ((pi & 3) >= (F8 ? kPolyFromF8 : kPolyFrom)) {
              a = exp2_poly3(a);
              b = exp2_poly3(b);
            } else {
              a = ex2_approx(a);
              b = ex2_approx(b);
            }
            sum2[pi & 3] = f2_add(sum2[pi & 3], f2_pack(a, b));
            e[2 * q] = a;
            e[2 * q + 1] = b;
          }
          if constexpr (F8) {
            pk[i] = pack4_e4m3(e[0], e[1], e[2], e[3]);
          } else {
            pk[i] = pack2<BF16>(e[0], e[1]);
            float r0, r1;
            unpack2<BF16>(pk[i], r0, r1);
            sumr2[i & 3] = f2_add(sumr2[i & 3], f2_pack(r0, r1));
          }
        }
        const uint32_t dst = tmem_addr(tbase, lane_base, p_col + col0 / EPC + G * h);
        if constexpr (G == 32) tmem_st32(dst, pk); else tmem_st16(dst, pk);
      }
      if constexpr (NC < 128) {
        // The other copies' key columns contribute nothing to this copy's rows.
        uint32_t zero[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) zero[i] = 0u;
#pragma unroll
        for (int b = 0; b < 128 / NC; ++b) {
          if (b == qcopy) continue;
          const uint32_t dst = tmem_addr(tbase, lane_base, s_col + b * NP);
          if constexpr (NP == 32) tmem_st32(dst, zero); else tmem_st16(dst, zero);
        }
      }
      {
        const uint64_t s01 = f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3]));
        float lo, hi;
        f2_unpack(s01, lo, hi);
        l += lo + hi;
        if constexpr (F8) {
          lr = l;
        } else {
          const uint64_t r01 = f2_add(f2_add(sumr2[0], sumr2[1]), f2_add(sumr2[2], sumr2[3]));
          f2_unpack(r01, lo, hi);
          lr += lo + hi;
        }
      }
      return true;
    };

    for (int step = 0; step < my_nkv && ok; ++step) {
      // S buffer of this step and the phase of its barriers: one buffer per
      // tile, or (one tile in the CTA) the two buffers in turn.
      const int buf = single ? (step & 1) : t;
      const uint32_t par = single ? ((step >> 1) & 1) : (step & 1);
      const uint32_t s_col = buf ? C::S_COL1 : C::S_COL0;
      // Warp-uniform wait: the TMEM loads and stores below are warp-collective.
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[buf], par, wc, kSiteSoftS));
      if (!ok) break;
      if (live) {
        tc_fence_after();
        ok = soft_step(std::integral_constant<int, C::BN / REP>{}, step, s_col);
        if (!ok) break;
        tmem_wait_st();
        tc_fence_before();
        // One tile per CTA: S of the last step was issued before the P V product
        // of the step before it (phase my_nkv - 2), which may still be pending.
        // Wait for it here, before this warp hands over the last P: no later
        // product can complete until then, so the barrier is at most one phase
        // behind now and at the final wait below.  (Waiting after the hand-over
        // could find both products complete, two phases on, where a parity wait
        // no longer tells them apart.)
        if (single && step == my_nkv - 1 && step >= 1) {
          ok = __all_sync(0xffffffffu, mbar_wait(&o_done[t], (step - 1) & 1, wc, kSiteSoftOEnd));
          if (!ok) break;
        }
      } else if (sep) {
        // Keep the barrier counts: S read; and, like the live warps (which wait
        // for the previous P V product before writing P), arrive for this step's
        // P only once the previous step's P was complete and consumed.
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[t]);
        if (step > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(&o_done[t], (step - 1) & 1, wc, kSiteSoftO));
          if (!ok) break;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[buf]);
    }
    // Wait for the last P V product.  A phase-parity wait is only sound while the
    // barrier is at most one phase behind: every earlier product has been seen
    // complete (with one tile per CTA, the one before it inside the last step).
    if (ok && live)
      ok = __all_sync(0xffffffffu, mbar_wait(&o_done[t], (my_nkv - 1) & 1, wc, kSiteSoftOEnd));
    if (ok && live) {
      tc_fence_after();
      // A row can see no key of a split (l = 0): it contributes nothing.
      // (8-bit inputs: the scale of V is applied here, once per output element.)
      const float inv_l = (l > 0.f && lr > 0.f) ? (F8 ? p.o_scale : 1.0f) / lr : 0.f;
      const float lse = (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const size_t orow_idx = static_cast<size_t>(bh) * Nq + row;
      if (!partial) {
        const int d = p.d;
        uint8_t* orow = reinterpret_cast<uint8_t*>(p.O) + orow_idx * (d * 2);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem_addr(tbase, lane_base, o_col + 32 * c), r);
          tmem_wait_ld();
          reg_fence(r);
          uint4 v[4];
          uint32_t* pv = reinterpret_cast<uint32_t*>(v);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pv[i] = pack2<BF16>(__uint_as_float(r[2 * i]) * inv_l,
                                __uint_as_float(r[2 * i + 1]) * inv_l);
          if (row < Nq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (c * 32 + 8 * i < d) dst[i] = v[i];  // 8 columns per store; d % 8 == 0
          }
        }
        if (row < Nq) p.LSE[orow_idx] = lse;
      } else {
        const size_t part = static_cast<size_t>(blockIdx.y * REP + qcopy) * p.BH * Nq + orow_idx;
        float* orow = p.O_part + part * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem_addr(tbase, lane_base, o_col + 32 * c), r);
          tmem_wait_ld();
          reg_fence(r);
          if (row < Nq && l > 0.f) {
            float4* dst = reinterpret_cast<float4*>(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv_l, __uint_as_float(r[4 * i + 1]) * inv_l,
                                   __uint_as_float(r[4 * i + 2]) * inv_l,
                                   __uint_as_float(r[4 * i + 3]) * inv_l);
          }
        }
        if (row < Nq) p.LSE_part[part] = lse;
      }
    } else if (partial && my_nkv == 0 && row < Nq && t < C::QT) {
      // The split holds no key this tile's rows see.  (With one query tile per
      // CTA, the second warpgroup's rows belong to the next CTA: it writes nothing.)
      p.LSE_part[static_cast<size_t>(blockIdx.y * REP + qcopy) * p.BH * Nq +
                 static_cast<size_t>(bh) * Nq + row] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace fa2
