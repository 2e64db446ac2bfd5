// dQ of the backward pass on sm_100a, query-stationary, for 128-wide tiles.
//
// Source: "Flash Attention spiegata: una guida completa" (datacamp), section
// "Ricomputazione": the backward pass rebuilds the probabilities from Q, K and the
// saved log-sum-exp instead of storing them.  For one 128-row query tile Q_i:
//   for each key tile j it sees:  S = Q_i K_j^T,  P = exp(scale S - LSE_i),
//                                 dP = dO_i V_j^T,  dS = P * (dP - D_i),
//                                 dQ_i += dS K_j,
//   dQ_i = scale dQ_i,  with D_i = rowsum(dO_i * O_i).
//
// At head dims above 64 the dK/dV products and a per-step dQ product do not fit
// tensor memory together (S^T, dP^T, dV and dK take all 512 columns), so the
// backward runs as two kernels: this one computes dQ (plus the per-row D and
// LSE * log2 e that the other needs), and fa2_bwd_kernel computes dK and dV.  The
// scores and dP are computed twice (seven products per tile pair instead of
// five), in exchange for no float atomics, no accumulator in global memory and
// a software pipeline in both kernels; dQ is summed in TMEM in a fixed order, so
// it is bitwise repeatable.
//
// CTA layout (320 threads), one CTA per (query tile, batch*head), heaviest causal
// tiles first:
//   warps 0-7 two compute warpgroups g = 0, 1.  Thread r of warpgroup g owns query
//             row r of the tile and key columns 64 g .. 64 g + 63 of S, P, dP, dS;
//             D_r and LSE_r sit in its registers.  At the start the same threads
//             copy the Q tile (their row, head columns 64 g ..) into TMEM;
//   warp  8   TMA producer: dO_i once, then a 4-stage K ring and a 2-stage V ring
//             in the order the MMA warp consumes them;
//   warp  9   tcgen05 MMA issuer (one thread).
// TMEM (fp32 columns): S [0,128); Q packed 16-bit [128,192) (A operand of S, so
// that shared memory holds one more K stage); dS packed 16-bit [192,256), warpgroup
// g in [192 + 32 g, + 32); dP [256,384); dQ [384,512).
// Products per key tile (M = 128 query rows, K = 16 per instruction):
//   S  = Q  K_j^T   (A = Q TMEM, B = K smem K-major)
//   dP = dO V_j^T   (A = dO smem K-major, B = V smem K-major)
//   dQ += dS K_j    (A = dS TMEM, B = K smem MN-major)
// Issue order per step j: S(j + 1) as soon as the P stage has read S(j) (s_free),
// dP(j + 1) as soon as the dS stage has read dP(j) (dp_free), dQ(j) once dS(j) is
// packed (ds_ready).  The products of step j + 1 thus run during the exponentials
// and the dS of step j, and the compute warps only wait for the tensor core when
// it is the slower side.  dS(j + 1) is written once dQ(j) has read dS(j) (dq_step).
#pragma once

#include "ptx.cuh"

namespace fa2 {

struct BwdDqParams {
  void* dQ;              // [BH][N][d] 16-bit (out)
  const uint16_t* Q;     // [BH][N][d] 16-bit
  const uint16_t* O;     // [BH][N][d] 16-bit
  const uint16_t* dO;    // [BH][N][d] 16-bit
  const float* LSE;      // [BH][N]
  float* Dg;             // [BH][Npad] out: D_i (0 on rows past N)
  float* Lg;             // [BH][Npad] out: LSE_i * log2 e (+inf on rows past N)
  int d;                 // head dim, 64 < d <= 128, a multiple of 8
  int N, Npad, BH, n_q;  // n_q = Npad / 128 query (and key) tiles per head
  int window;            // causal only: query i sees keys i - window + 1 .. i (0 = none)
  float scale, scale_log2;
  unsigned int* status;
  unsigned long long wait_ns;
  int fault;             // test hook: 1 = skip the first K load (a wait runs out)
  unsigned int* tile_ctr;  // the dK/dV kernel's tile counter, zeroed here (it runs next)
};

struct BwdDqCfg {
  static constexpr int D = 128;
  static constexpr int KCH = D / 64;           // 128-byte swizzle chunks along d
  static constexpr int CHUNK = 128 * 128;      // bytes of a 128-row x 64-column chunk
  static constexpr int TILE = 128 * D * 2;     // bytes of a 128-row tile
  static constexpr int KS = 4, VS = 2;         // K and V ring stages
  static constexpr int CTRL_BYTES = 1280;      // barriers, TMEM address, D exchange
  static constexpr int SMEM = (1 + KS + VS) * TILE + CTRL_BYTES;  // dO, K ring, V ring
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static constexpr int THREADS = 320;
  static constexpr uint32_t C_S = 0, C_Q = 128, C_DS = 192, C_DP = 256, C_DQ = 384;
};

struct BwdDqCtrl {
  uint64_t bar_qdo, k_full[BwdDqCfg::KS], k_empty[BwdDqCfg::KS], v_full[BwdDqCfg::VS],
      v_empty[BwdDqCfg::VS];
  uint64_t q_ready, s_full, s_free, dp_full, dp_free, ds_ready, dq_step, dq_full, drain;
  uint32_t tmem_slot;
  int abort_flag;
  float dpart[2][128];  // each warpgroup's half of rowsum(dO * O)
};

enum BwdDqSite : uint32_t {
  kQSiteAlign = 63, kQSiteProdK = 64, kQSiteProdV, kQSiteMmaQ, kQSiteMmaK, kQSiteMmaV,
  kQSiteMmaDS, kQSiteMmaDPFree, kQSiteCmpS, kQSiteCmpDP, kQSiteCmpDQ, kQSiteMmaDrain, kQSiteProdDrain,
  kQSiteMmaSFree, kQSiteCmpDQStep
};

template <bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(320, 1)
fa2_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdDqParams p) {
  using C = BwdDqCfg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    // The swizzled tiles need a 1024-byte aligned base; report and do nothing.
    if (threadIdx.x == 0) atomicCAS(p.status, 0u, 4u | (kQSiteAlign << 8));
    return;
  }
  // The dK/dV kernel queued behind this grid may launch once every CTA of this one
  // has started; it waits for this grid to complete before it reads D and L.
  griddep_launch_dependents();
  uint8_t* sdO = smem_raw;
  uint8_t* sK = sdO + C::TILE;               // KS stages
  uint8_t* sV = sK + C::KS * C::TILE;        // VS stages
  BwdDqCtrl& ctl = *reinterpret_cast<BwdDqCtrl*>(sV + C::VS * C::TILE);
  static_assert(sizeof(BwdDqCtrl) <= C::CTRL_BYTES, "control block too large");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = p.N, BH = p.BH;
  // Heaviest query tiles first (a causal tile i sees key tiles 0 .. i).
  const int qt = p.n_q - 1 - static_cast<int>(blockIdx.x) / BH;
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int row0 = qt * 128;
  const int win = p.window;
  // Key tiles [j_lo, j_lo + n) the tile's rows see: all, or (causal) up to the
  // diagonal tile, and (sliding window) from the tile holding the first key its
  // first row still sees.  n >= 1 always (a row sees at least its own key).
  int j_lo = 0, j_hi = p.n_q;
  if (CAUSAL) {
    j_hi = qt + 1;
    if (win > 0) j_lo = max(0, row0 - win + 1) / 128;
  }
  const int n = j_hi - j_lo;

  WaitCtl wc{p.status, &ctl.abort_flag, p.wait_ns};

  if (threadIdx.x == 0) {
    ctl.abort_flag = 0;
    mbar_init(&ctl.bar_qdo, 1);
    mbar_init(&ctl.q_ready, 8);
    for (int s = 0; s < C::KS; ++s) { mbar_init(&ctl.k_full[s], 1); mbar_init(&ctl.k_empty[s], 1); }
    for (int s = 0; s < C::VS; ++s) { mbar_init(&ctl.v_full[s], 1); mbar_init(&ctl.v_empty[s], 1); }
    mbar_init(&ctl.s_full, 1);
    mbar_init(&ctl.s_free, 8);
    mbar_init(&ctl.dp_full, 1);
    mbar_init(&ctl.dp_free, 8);
    mbar_init(&ctl.ds_ready, 8);
    mbar_init(&ctl.dq_step, 1);
    mbar_init(&ctl.dq_full, 1);
    mbar_init(&ctl.drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ctl.tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl.tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      // Nothing is read before the previous grid on the stream (the forward that
      // wrote O and LSE, typically) has completed; the counter is zeroed after it
      // too (that grid may be the previous call's dK/dV kernel, still using it).
      griddep_wait();
      if (blockIdx.x == 0) *p.tile_ctr = 0u;
      mbar_arrive_expect_tx(&ctl.bar_qdo, C::TILE);
      for (int c = 0; c < C::KCH; ++c)
        tma_load_3d(sdO + c * C::CHUNK, &tmdO, &ctl.bar_qdo, c * 64, row0, bh);
      const uint64_t keep = policy_evict_last();
      int k_issued = 0, v_issued = 0;
      auto load_k = [&](int jj) -> bool {
        const int s = jj % C::KS;
        if (jj >= C::KS && !mbar_wait(&ctl.k_empty[s], ((jj / C::KS) - 1) & 1, wc, kQSiteProdK))
          return false;
        if (!(p.fault == 1 && jj == 0)) {
          mbar_arrive_expect_tx(&ctl.k_full[s], C::TILE);
          for (int c = 0; c < C::KCH; ++c)
            tma_load_3d_hint(sK + s * C::TILE + c * C::CHUNK, &tmK, &ctl.k_full[s], c * 64,
                             (j_lo + jj) * 128, bh, keep);
          k_issued = jj + 1;
        }
        return true;
      };
      auto load_v = [&](int jj) -> bool {
        const int s = jj % C::VS;
        if (jj >= C::VS && !mbar_wait(&ctl.v_empty[s], ((jj / C::VS) - 1) & 1, wc, kQSiteProdV))
          return false;
        mbar_arrive_expect_tx(&ctl.v_full[s], C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d_hint(sV + s * C::TILE + c * C::CHUNK, &tmV, &ctl.v_full[s], c * 64,
                           (j_lo + jj) * 128, bh, keep);
        v_issued = jj + 1;
        return true;
      };
      // Consumption order: S(0) K0, dP(0) V0, then per step j: S(j + 1) K(j + 1),
      // dP(j + 1) V(j + 1), dQ(j) K(j).
      bool ok = load_k(0) && load_v(0);
      for (int jj = 0; jj + 1 < n && ok; ++jj) ok = load_k(jj + 1) && load_v(jj + 1);
      if (!ok) {
        // Every copy already issued lands before the CTA exits.
        volatile int no_abort = 0;
        WaitCtl dw{p.status, &no_abort, 100000000ull};
        for (int jj = max(0, k_issued - C::KS); jj < k_issued; ++jj)
          if (!(p.fault == 1 && jj == 0))
            mbar_wait(&ctl.k_full[jj % C::KS], (jj / C::KS) & 1, dw, kQSiteProdDrain);
        for (int jj = max(0, v_issued - C::VS); jj < v_issued; ++jj)
          mbar_wait(&ctl.v_full[jj % C::VS], (jj / C::VS) & 1, dw, kQSiteProdDrain);
      }
      // dO lands before exit too (issued unconditionally above).
      volatile int no_abort = 0;
      WaitCtl dw{p.status, &no_abort, 100000000ull};
      mbar_wait(&ctl.bar_qdo, 0, dw, kQSiteProdDrain);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16(128, 128, BF16, false, false);     // S, dP
      constexpr uint32_t id_dq = idesc_f16(128, C::D, BF16, false, true);    // dQ (B MN-major)
      const uint32_t adO = smem_u32(sdO), aK = smem_u32(sK), aV = smem_u32(sV);
      const uint64_t kdO = sdesc_sw128(adO, 16, 1024);
      const uint64_t kK = sdesc_sw128(aK, 16, 1024), kV = sdesc_sw128(aV, 16, 1024);
      const uint64_t mK = sdesc_sw128(aK, C::CHUNK, 1024);
      auto mma_s = [&](int jj) {  // S(jj) = Q K(jj)^T (Q from TMEM: 8 columns per K step)
        const uint32_t ko = static_cast<uint32_t>((jj % C::KS) * C::TILE);
#pragma unroll
        for (int kk = 0; kk < C::D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          umma_ts(tbase + C::C_S, tbase + C::C_Q + 8u * kk, sdesc_add(kK, ko + off), id_s, kk > 0);
        }
        umma_commit(&ctl.s_full);
      };
      auto mma_dp = [&](int jj) {  // dP(jj) = dO V(jj)^T
        const uint32_t vo = static_cast<uint32_t>((jj % C::VS) * C::TILE);
#pragma unroll
        for (int kk = 0; kk < C::D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          umma_ss(tbase + C::C_DP, sdesc_add(kdO, off), sdesc_add(kV, vo + off), id_s, kk > 0);
        }
        umma_commit(&ctl.dp_full);
        umma_commit(&ctl.v_empty[jj % C::VS]);  // V(jj) is read by dP(jj) only
      };
      auto mma_dq = [&](int jj) {  // dQ += dS(jj) K(jj); keys 16 kk ..: warpgroup kk / 4
        const uint32_t ko = static_cast<uint32_t>((jj % C::KS) * C::TILE);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tbase + C::C_DQ, tbase + C::C_DS + 32u * (kk >> 2) + (kk & 3) * 8,
                  sdesc_add(mK, ko + kk * 2048), id_dq, (jj > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&ctl.k_empty[jj % C::KS]);  // K(jj): last read by dQ(jj)
        umma_commit(&ctl.dq_step);              // the dS columns may take dS(jj + 1)
      };
      bool ok = mbar_wait(&ctl.q_ready, 0, wc, kQSiteMmaQ) &&
                mbar_wait(&ctl.bar_qdo, 0, wc, kQSiteMmaQ) &&
                mbar_wait(&ctl.k_full[0], 0, wc, kQSiteMmaK);
      if (ok) {
        tc_fence_after();
        mma_s(0);
        ok = mbar_wait(&ctl.v_full[0], 0, wc, kQSiteMmaV);
      }
      if (ok) {
        tc_fence_after();
        mma_dp(0);
      }
      for (int jj = 0; jj < n && ok; ++jj) {
        if (jj + 1 < n) {  // S(jj + 1) once the P stage has read S(jj)
          const int s = (jj + 1) % C::KS;
          if (!mbar_wait(&ctl.s_free, jj & 1, wc, kQSiteMmaSFree) ||
              !mbar_wait(&ctl.k_full[s], ((jj + 1) / C::KS) & 1, wc, kQSiteMmaK)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_s(jj + 1);
          // dP(jj + 1) once the dS stage has read dP(jj)
          const int v = (jj + 1) % C::VS;
          if (!mbar_wait(&ctl.dp_free, jj & 1, wc, kQSiteMmaDPFree) ||
              !mbar_wait(&ctl.v_full[v], ((jj + 1) / C::VS) & 1, wc, kQSiteMmaV)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_dp(jj + 1);
        }
        if (!mbar_wait(&ctl.ds_ready, jj & 1, wc, kQSiteMmaDS)) { ok = false; break; }
        tc_fence_after();
        mma_dq(jj);
      }
      if (ok) umma_commit(&ctl.dq_full);
      // Every product issued above completes before TMEM is released.
      umma_commit(&ctl.drain);
      volatile int no_abort = 0;
      WaitCtl dw{p.status, &no_abort, p.wait_ns};
      mbar_wait(&ctl.drain, 0, dw, kQSiteMmaDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ compute
    const int g = warp >> 2;                   // key columns 64 g .. 64 g + 63
    const int wq = warp & 3;                   // TMEM lane quadrant
    const int r = wq * 32 + lane;              // query row within the tile
    const int q = row0 + r;                    // query row within the head
    const uint32_t lb = static_cast<uint32_t>(wq * 32);
    const uint32_t wg_bar = 1 + g;             // named barrier of this warpgroup
    const int d = p.d;
    griddep_wait();  // O, dO and LSE come from the kernels before this one
    // Q row q, head columns 64 g .. 64 g + 63, into TMEM as 32 packed columns (the A
    // operand of S); D_r = sum_c dO_rc O_rc, warpgroup g summing the same columns.
    // Rows past N and columns past d are zero.
    float D_r, L_r;
    {
      float acc = 0.f;
      uint32_t qw[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) qw[i] = 0u;
      if (q < N) {
        const size_t base = (static_cast<size_t>(bh) * N + q) * d;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = 64 * g + 8 * u;
          if (c < d) {
            const uint4 qv = *reinterpret_cast<const uint4*>(p.Q + base + c);
            qw[4 * u] = qv.x;
            qw[4 * u + 1] = qv.y;
            qw[4 * u + 2] = qv.z;
            qw[4 * u + 3] = qv.w;
            const uint4 a = *reinterpret_cast<const uint4*>(p.O + base + c);
            const uint4 b = *reinterpret_cast<const uint4*>(p.dO + base + c);
            const uint32_t* pa = reinterpret_cast<const uint32_t*>(&a);
            const uint32_t* pb = reinterpret_cast<const uint32_t*>(&b);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float a0, a1, b0, b1;
              unpack2<BF16>(pa[i], a0, a1);
              unpack2<BF16>(pb[i], b0, b1);
              acc = fmaf(a0, b0, acc);
              acc = fmaf(a1, b1, acc);
            }
          }
        }
      }
      tmem_st32(tmem_addr(tbase, lb, C::C_Q + 32u * g), qw);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.q_ready);
      ctl.dpart[g][r] = acc;
      named_bar_sync(3, 256);
      D_r = q < N ? ctl.dpart[0][r] + ctl.dpart[1][r] : 0.f;
      L_r = q < N ? p.LSE[static_cast<size_t>(bh) * N + q] * 1.4426950408889634f : INFINITY;
      if (g == 0) {  // the rows the dK/dV kernel reads (it waits for this grid)
        p.Dg[static_cast<size_t>(bh) * p.Npad + q] = D_r;
        p.Lg[static_cast<size_t>(bh) * p.Npad + q] = L_r;
      }
    }
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint64_t negl2 = f2_pack(-L_r, -L_r);  // -inf past N: P = 0 there
    bool ok = true;
    for (int jj = 0; jj < n && ok; ++jj) {
      const int j = j_lo + jj;
      // ---- P = exp2(S * scale * log2 e - LSE * log2 e), this warpgroup's 64 keys
      ok = named_bar_and(wg_bar, 128, mbar_wait(&ctl.s_full, jj & 1, wc, kQSiteCmpS));
      if (!ok) break;
      tc_fence_after();
      float pr[64];
      {
        uint32_t srr[2][32];
        tmem_ld32(tmem_addr(tbase, lb, C::C_S + 64u * g), srr[0]);
        tmem_ld32(tmem_addr(tbase, lb, C::C_S + 64u * g + 32u), srr[1]);
        tmem_wait_ld();
        reg_fence(srr[0]);
        reg_fence(srr[1]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.s_free);  // the S columns may take S(jj + 1)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(srr[c][2 * e]), __uint_as_float(srr[c][2 * e + 1])),
                             sl2x2, negl2),
                      x0, x1);
            if ((e & 3) >= kBwdPolyFrom) {  // FMA-pipe exp2 for this pair (see kBwdPolyFrom)
              pr[32 * c + 2 * e] = exp2_poly3(x0);
              pr[32 * c + 2 * e + 1] = exp2_poly3(x1);
            } else {
              pr[32 * c + 2 * e] = ex2_approx(x0);
              pr[32 * c + 2 * e + 1] = ex2_approx(x1);
            }
          }
        }
      }
      // Keys after the query (causal, the diagonal tile), past N, or before the
      // window: one branch per tile, not a compare per element.
      const int key0 = j * 128 + 64 * g;
      const bool masked = (CAUSAL && j == qt) || key0 + 63 >= N ||
                          (CAUSAL && win > 0 && row0 + 127 - j * 128 >= win);
      if (masked) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int key = key0 + c;
          if ((CAUSAL && key > q) || key >= N || (CAUSAL && win > 0 && q - key >= win)) pr[c] = 0.f;
        }
      }
      // ---- dS = P * (dP - D), packed to 16 bits into this warpgroup's dS columns
      ok = named_bar_and(wg_bar, 128, mbar_wait(&ctl.dp_full, jj & 1, wc, kQSiteCmpDP));
      if (!ok) break;
      tc_fence_after();
      {
        const uint64_t negd2 = f2_pack(-D_r, -D_r);
        uint32_t dr[2][32];
        tmem_ld32(tmem_addr(tbase, lb, C::C_DP + 64u * g), dr[0]);
        tmem_ld32(tmem_addr(tbase, lb, C::C_DP + 64u * g + 32u), dr[1]);
        tmem_wait_ld();
        reg_fence(dr[0]);
        reg_fence(dr[1]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.dp_free);  // the dP columns may take dP(jj + 1)
        uint32_t dsk[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t t = f2_add(f2_pack(__uint_as_float(dr[c][2 * e]), __uint_as_float(dr[c][2 * e + 1])),
                                      negd2);
            float a0, a1;
            f2_unpack(f2_mul(f2_pack(pr[32 * c + 2 * e], pr[32 * c + 2 * e + 1]), t), a0, a1);
            dsk[16 * c + e] = pack2<BF16>(a0, a1);
          }
        }
        // dS(jj - 1) in these columns must have been read by dQ(jj - 1)
        if (jj > 0) {
          ok = named_bar_and(wg_bar, 128, mbar_wait(&ctl.dq_step, (jj - 1) & 1, wc, kQSiteCmpDQStep));
          if (!ok) break;
          tc_fence_after();
        }
        tmem_st32(tmem_addr(tbase, lb, C::C_DS + 32u * g), dsk);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.ds_ready);
    }
    // ---- epilogue: dQ_i = scale * accumulator, 16-bit, head columns 64 g ..
    if (ok) ok = named_bar_and(wg_bar, 128, mbar_wait(&ctl.dq_full, 0, wc, kQSiteCmpDQ));
    if (ok) {
      tc_fence_after();
      uint8_t* row = reinterpret_cast<uint8_t*>(p.dQ) + (static_cast<size_t>(bh) * N + q) * (d * 2);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t rr[32];
        tmem_ld32(tmem_addr(tbase, lb, C::C_DQ + 64u * g + 32u * c), rr);
        tmem_wait_ld();
        reg_fence(rr);
        uint4 v[4];
        uint32_t* pv = reinterpret_cast<uint32_t*>(v);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pv[e] = pack2<BF16>(__uint_as_float(rr[2 * e]) * p.scale,
                              __uint_as_float(rr[2 * e + 1]) * p.scale);
        if (q < N) {
          const int col = 64 * g + 32 * c;
          uint4* dst = reinterpret_cast<uint4*>(row + col * 2);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (col + 8 * e < d) dst[e] = v[e];  // 8 columns per store; d % 8 == 0
        }
      }
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
