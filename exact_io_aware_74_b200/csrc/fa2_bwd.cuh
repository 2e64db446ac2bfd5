// Backward pass of exact attention on sm_100a.
//
// Source: "Flash Attention spiegata: una guida completa" (datacamp), section
// "Ricomputazione": instead of keeping the probabilities for the backward pass,
// the scores are recomputed from Q and K (cheap next to the memory traffic they
// would cost).  Here P is rebuilt from the saved log-sum-exp, so no N x N matrix
// is ever stored.  With dO = dL/dO:
//   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,
//   dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Kernels per call, all on the caller's stream, chained by programmatic dependent
// launch (each reads nothing before its griddepcontrol.wait).  Tile width 64 for
// d <= 64, 128 for 64 < d <= 128.
//   default mode:
//   1. fa2_bwd_pre_kernel  : D and LSE * log2(e) per query row (padded to a
//                            multiple of 128 rows), a zeroed fp32 dQ accumulator
//                            and a zeroed tile counter;
//   2. fa2_bwd_kernel      : persistent, at most one CTA per SM, over the list of
//                            key tiles (128 keys, batch*head; see the tile
//                            scheduler); each tile loops over the query tiles that
//                            see its keys, accumulates dV and dK in TMEM and adds
//                            its dQ partials into the accumulator (TMA reduce-add);
//   3. fa2_bwd_dq_finalise_kernel : dQ = scale * accumulator, rounded to 16 bits.
//   deterministic mode (tile width 128 at every d):
//   1. fa2_bwd_dq_kernel (fa2_bwd_dq.cuh): dQ, query-stationary, summed in TMEM in a
//                            fixed order; it also writes the D and LSE * log2(e)
//                            rows and zeroes the tile counter;
//   2. fa2_bwd_kernel      : as above, dK and dV only.
//
// Main kernel, CTA layout (320 threads):
//   warps 0-7 two compute warpgroups g = 0, 1.  Thread r of warpgroup g owns key
//             row r of the tile for the query columns 64 g .. 64 g + 63 of P^T
//             and dS^T, and query row r of the current query tile for the head
//             columns g D/2 .. (g+1) D/2 - 1 when it moves the dQ partial from TMEM
//             through shared memory into the fp32 accumulator (one TMA reduce-add
//             per 128 x 32 tile).  Splitting every row between the two warpgroups
//             halves the per-step chain P^T -> dS^T -> dQ drain that the products
//             wait on;
//   warp  8   TMA producer: K_j and V_j per tile (two buffers at D = 64, the next
//             tile's loaded during the current one), the (Q_i, dO_i) tiles and LSE /
//             D rows of each step in 2-stage rings, across the CTA's tiles;
//   warp  9   tcgen05 MMA issuer (one thread).
// TMEM (fp32 columns): S^T [0,128); dP^T [128,256); dV [256, 256 + D); dK
// [256 + D, 256 + 2 D).
//   D = 64: dQ [384,448); packed P^T of warpgroup g at [448 + 32 g, + 32), its dS^T
//     over its own dP^T columns [128 + 64 g, + 32).  The steps are software-
//     pipelined: the scores of step i + 1 go out right after step i's dV product and
//     its dP^T right after step i's dK product, so that the next step's products
//     overlap this step's dS.
//   D = 128 with dQ: no free columns; packed P^T and dS^T of warpgroup g over its
//     own score columns [64 g, + 32), [64 g + 32, + 32); the dQ partial over dP^T.
//     Each step runs its products in order (S^T, dP^T, dV, dQ, dK).
//   D = 128, dK/dV only: packed dS^T and P^T over warpgroup g's dP^T columns, so
//     that step i + 1's scores run during step i's exponentials.
// Products (M = 128 rows of the first operand, K = 16 per instruction):
//   S^T  = K_j  Q_i^T   (A = K smem K-major, B = Q smem K-major)
//   dP^T = V_j  dO_i^T  (A = V smem K-major, B = dO smem K-major)
//   dV  += P^T  dO_i    (A = P^T TMEM, B = dO smem MN-major)
//   dK  += dS^T Q_i     (A = dS^T TMEM, B = Q smem MN-major)
//   dQ_i = dS   K_j     (A = dS^T smem MN-major, B = K smem MN-major)
#pragma once

#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>

#include "fa2_bwd_dq.cuh"
#include "ptx.cuh"

namespace fa2 {

// Workspace: D [BH][Npad] f32 | L2 = LSE*log2(e) [BH][Npad] f32 | dQacc [BH][N][Dt] f32
// | tile counter (256 bytes), Dt the kernel's tile head dim (64 or 128).  The
// deterministic mode sums dQ in TMEM (fa2_bwd_dq_kernel) and uses the row statistics
// and the counter alone.  The counter hands out the key tiles of the persistent grid
// (see the tile scheduler); the first kernel of a call zeroes it.
inline size_t bwd_npad(int N) { return (static_cast<size_t>(N) + 127) / 128 * 128; }
inline size_t bwd_rowstat_bytes(size_t BH, int N) {
  return (2 * BH * bwd_npad(N) * 4 + 255) / 256 * 256;
}
// Kernel head dim for a head dim d <= 128: the tiles are 64 or 128 columns wide.
inline int bwd_tile_dim(int d) { return d <= 64 ? 64 : 128; }
inline size_t bwd_workspace_bytes(size_t BH, int N, int d, bool deterministic = false) {
  const size_t acc =
      deterministic ? 0 : (BH * static_cast<size_t>(N) * bwd_tile_dim(d) * 4 + 255) / 256 * 256;
  return bwd_rowstat_bytes(BH, N) + acc + 256;
}
// Kernels one backward call launches: preprocess, main and dQ finalisation; in the
// deterministic mode the dQ kernel and the dK/dV kernel.
inline int bwd_kernels_per_call(bool deterministic) { return deterministic ? 2 : 3; }

// ------------------------------------------------------------------------------------
// 1. preprocess
// ------------------------------------------------------------------------------------

template <int D, bool BF16>
__global__ void __launch_bounds__(256)
fa2_bwd_pre_kernel(const uint16_t* __restrict__ O, const uint16_t* __restrict__ dO,
                   const float* __restrict__ LSE, float* __restrict__ Dg,
                   float* __restrict__ Lg, float* __restrict__ dQacc, unsigned int* __restrict__ tile_ctr,
                   int N, int Npad, long long total_rows, int d) {
  constexpr int TPR = D / 8;  // threads per row, 8 elements (16 bytes) each
  constexpr int RPB = 256 / TPR;
  // Launched behind the caller's previous kernel (the forward, typically) with
  // programmatic serialisation: let the main kernel start its set-up, then wait
  // for O and LSE.
  griddep_launch_dependents();
  griddep_wait();
  if (blockIdx.x == 0 && threadIdx.x == 0) *tile_ctr = 0u;
  const int sub = threadIdx.x % TPR;
  const long long r = static_cast<long long>(blockIdx.x) * RPB + threadIdx.x / TPR;
  const bool in_range = r < total_rows;  // no early exit: the shuffle below is warp-wide
  const long long bh = in_range ? r / Npad : 0;
  const int q = in_range ? static_cast<int>(r % Npad) : N;
  float acc = 0.f;
  if (q < N && sub * 8 < d) {  // O, dO rows have d (a multiple of 8) columns
    const size_t off = (static_cast<size_t>(bh) * N + q) * d + sub * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(O + off);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + off);
    const uint32_t* pa = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* pb = reinterpret_cast<const uint32_t*>(&b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a0, a1, b0, b1;
      if constexpr (BF16) {
        a0 = __uint_as_float(pa[i] << 16); a1 = __uint_as_float(pa[i] & 0xFFFF0000u);
        b0 = __uint_as_float(pb[i] << 16); b1 = __uint_as_float(pb[i] & 0xFFFF0000u);
      } else {
        const __half2 ha = *reinterpret_cast<const __half2*>(&pa[i]);
        const __half2 hb = *reinterpret_cast<const __half2*>(&pb[i]);
        a0 = __low2float(ha); a1 = __high2float(ha);
        b0 = __low2float(hb); b1 = __high2float(hb);
      }
      acc = fmaf(a0, b0, acc);
      acc = fmaf(a1, b1, acc);
    }
  }
  if (q < N) {  // the accumulator has D columns, the padding included
    float4* z = reinterpret_cast<float4*>(dQacc + (static_cast<size_t>(bh) * N + q) * D + sub * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int o = TPR / 2; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, TPR);
  if (in_range && sub == 0) {
    Dg[r] = q < N ? acc : 0.f;
    Lg[r] = q < N ? LSE[static_cast<size_t>(bh) * N + q] * 1.4426950408889634f : INFINITY;
  }
}

// ------------------------------------------------------------------------------------
// 3. dQ finalise
// ------------------------------------------------------------------------------------

template <bool BF16>
__global__ void __launch_bounds__(256)
fa2_bwd_dq_finalise_kernel(const float* __restrict__ dQacc, uint16_t* __restrict__ dQ, float scale,
                  long long n8, int D, int d) {
  // Thread i converts 8 accumulator columns (group i % (D/8) of row i / (D/8));
  // groups past the head dim d are padding and are dropped.
  griddep_wait();  // the main kernel's reductions are complete and visible
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const long long row = i / (D / 8);
  const int g = static_cast<int>(i % (D / 8));
  if (g * 8 >= d) return;
  const float4 a = reinterpret_cast<const float4*>(dQacc)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(dQacc)[2 * i + 1];
  uint4 out;
  out.x = pack2<BF16>(a.x * scale, a.y * scale);
  out.y = pack2<BF16>(a.z * scale, a.w * scale);
  out.z = pack2<BF16>(b.x * scale, b.y * scale);
  out.w = pack2<BF16>(b.z * scale, b.w * scale);
  *reinterpret_cast<uint4*>(dQ + row * d + g * 8) = out;
}

// ------------------------------------------------------------------------------------
// 2. main kernel
// ------------------------------------------------------------------------------------

struct BwdParams {
  const float* Dg;    // [BH][Npad]
  const float* Lg;    // [BH][Npad]
  float* dQacc;       // [BH][N][D] (D columns, the padding included)
  void* dK;           // [BH][N][d] 16-bit
  void* dV;           // [BH][N][d] 16-bit
  int d;              // head dim (multiple of 8, <= D); tile columns past d are zero fill
  int N, Npad, BH, n_kv;
  int head_group;     // heads per group of the tile list (see the tile scheduler)
  int window;         // causal only: query i sees keys i-window+1..i (0 = no window)
  float scale, scale_log2;
  unsigned int* status;
  unsigned long long wait_ns;
  int fault;          // test hook: 1 = skip the K, V load (a consumer's wait runs out)
  unsigned int* tile_ctr;  // tiles handed out past the first two rounds (zeroed by the first kernel)
  int dynamic;        // 1: tiles past the first two rounds from tile_ctr; 0: snake order
};

template <int D, bool DQ_>
struct BwdCfg {
  static constexpr int KCH = D / 64;
  static constexpr int CHUNK = 128 * 128;
  static constexpr int TILE = 128 * D * 2;
  static constexpr int ST = 2;                 // (Q, dO) ring stages; dO ring at tile width 128
  // K/V buffers: a CTA runs several key tiles in turn.  At D = 64 the next tile's
  // K and V load into a buffer of their own while the current tile runs; at
  // D = 128 there is room for one, reloaded once the tile's last product has read it.
  static constexpr int KVB = (D == 64) ? 2 : 1;
  // DQ: dQ partials from this kernel, added into a float accumulator (the default
  // mode); otherwise (the deterministic mode, D = 128) fa2_bwd_dq_kernel computes
  // dQ and this kernel computes dK and dV only.
  static constexpr bool DQ = DQ_;
  static_assert(DQ || D == 128, "the dK/dV-only kernel uses 128-wide tiles");
  // Software-pipelined steps with the dQ product: at D = 64, where TMEM has room.
  static constexpr bool PIPE = DQ && D == 64;
  static constexpr int DS_BYTES = DQ ? 128 * 128 * 2 : 0;  // dS^T in shared memory, for dQ
  // Q tiles: in the (Q, dO) ring at tile width 64; a ring of their own at 128,
  // released by dK (their last reader).  Without dQ that ring is one stage deeper
  // than dO's: the next step's scores are issued as soon as this step's have been
  // read, so the next Q must already be resident then, while dO is first needed
  // later, by dP^T.  With dQ (D = 128) the dO tile of a step is released later than
  // its Q: it doubles as a staging tile of the step's dQ reduce (see the drain).
  static constexpr int QS = DQ ? ST : 3;
  // LSE*log2e and D rows of each stage: loaded with Q in the fused D = 128 kernel,
  // with dO otherwise.
  static constexpr int LD_BYTES = ST * 2 * 128 * 4;
  static constexpr int CTRL_BYTES = 512;  // barriers, tile ring, TMEM address, abort flag
  // No alignment slack: the dynamic region must start 1024-byte aligned (checked).
  static constexpr int SMEM = (2 * KVB + QS + ST) * TILE + DS_BYTES + LD_BYTES + CTRL_BYTES;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static constexpr int THREADS = 320;
  static constexpr uint32_t C_S = 0, C_DP = 128;
  // Packed P^T and dS^T of warpgroup g:
  //   D = 64 (pipelined): P^T in columns 448 + 32 g .. + 31 (free at D = 64), dS^T
  //     over its own dP^T columns 128 + 64 g .. + 31, so the score columns are free
  //     as soon as the scores have been read and the next step's scores are
  //     computed during this step's dS;
  //   D = 128 with dQ: both inside its own score columns, 64 g + (0 | 32) .. + 31
  //     (no free columns: dP^T also holds the dQ partial);
  //   D = 128, dK/dV only: both over its own dP^T columns, dS^T at 128 + 64 g, P^T
  //     at 128 + 64 g + 32 (P stays in registers until then), so the next step's
  //     scores are computed during this step's exponentials.
  __host__ __device__ static constexpr uint32_t C_P(int g) {
    return D == 64 ? 448u + 32u * g : (DQ ? 64u * g : C_DP + 64u * g + 32u);
  }
  __host__ __device__ static constexpr uint32_t C_DS(int g) {
    return (D == 128 && DQ) ? 64u * g + 32u : C_DP + 64u * g;
  }
  static constexpr uint32_t C_DV = 256, C_DK = 256 + D;
  static constexpr uint32_t C_DQ = (D == 128) ? 128 : 384;  // D = 128: shares dP^T's columns
};

// Control block at the end of the dynamic shared memory (no static shared memory,
// so that the 1024-byte aligned tiles start at the base of the window).
// Depth of the ring through which the producer hands the CTA's tile sequence to the
// MMA and compute roles.
constexpr int kTileRing = 4;

template <int ST>
struct BwdCtrl {
  uint64_t bar_kv[2], kv_empty[2], acc_free, qdo_full[ST], qdo_empty[ST], q_full[3], q_empty[3];
  uint64_t s_full, s_read, dp_full, p_ready, ds_ready, dq_full, dq_drained, drain, fin;
  uint64_t tile_full[kTileRing], tile_empty[kTileRing];
  int tile_ring[kTileRing];
  uint32_t tmem_slot;
  int abort_flag;
};

__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gmem_src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

enum BwdSite : uint32_t {
  kBSiteAlign = 31, kBSiteProdEmpty = 32, kBSiteMmaKV, kBSiteMmaQ, kBSiteMmaDrained, kBSiteMmaP, kBSiteMmaDS,
  kBSiteMmaDrain, kBSiteCmpQ, kBSiteCmpS, kBSiteCmpDP, kBSiteCmpDQ, kBSiteProdDrain, kBSiteMmaAcc,
  kBSiteProdKV, kBSiteProdTile, kBSiteMmaTile, kBSiteCmpTile
};

template <int D, bool BF16, bool CAUSAL, bool DQ>
__global__ void __launch_bounds__(320, 1)
fa2_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
               const __grid_constant__ CUtensorMap tmdQ, const BwdParams p) {
  using C = BwdCfg<D, DQ>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    // The swizzled tiles need a 1024-byte aligned base; report and do nothing.
    if (threadIdx.x == 0) atomicCAS(p.status, 0u, 4u | (kBSiteAlign << 8));
    return;
  }
  // The dQ finalisation queued behind this grid may launch now; it waits for
  // this grid to complete before reading the accumulator.
  griddep_launch_dependents();
  uint8_t* smem = smem_raw;
  uint8_t* sK = smem;                        // KVB tiles
  uint8_t* sV = sK + C::KVB * C::TILE;       // KVB tiles
  uint8_t* sQ = sV + C::KVB * C::TILE;       // QS tiles
  uint8_t* sdO = sQ + C::QS * C::TILE;       // ST tiles
  uint8_t* sDS = sdO + C::ST * C::TILE;      // dS^T, MN-major for the dQ product
  float* sLD = reinterpret_cast<float*>(sDS + C::DS_BYTES);  // [ST][2][128]: L, D
  BwdCtrl<C::ST>& ctl = *reinterpret_cast<BwdCtrl<C::ST>*>(sDS + C::DS_BYTES + C::LD_BYTES);
  static_assert(sizeof(BwdCtrl<C::ST>) <= C::CTRL_BYTES, "control block too large");
  uint64_t* bar_kv = ctl.bar_kv;
  uint64_t* kv_empty = ctl.kv_empty;
  uint64_t& acc_free = ctl.acc_free;
  uint64_t* qdo_full = ctl.qdo_full;
  uint64_t* qdo_empty = ctl.qdo_empty;
  uint64_t* q_full = ctl.q_full;    // tile width 128: the Q ring
  uint64_t* q_empty = ctl.q_empty;
  uint64_t& s_full = ctl.s_full;
  uint64_t& dp_full = ctl.dp_full;
  uint64_t& p_ready = ctl.p_ready;
  uint64_t& s_read = ctl.s_read;
  uint64_t& ds_ready = ctl.ds_ready;
  uint64_t& dq_full = ctl.dq_full;
  uint64_t& dq_drained = ctl.dq_drained;
  uint64_t& drain = ctl.drain;
  uint64_t& fin = ctl.fin;
  uint32_t& tmem_slot = ctl.tmem_slot;
  int& abort_flag = ctl.abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = p.N;
  const int n_q = p.n_kv;
  // Tile scheduler.  The key tiles (j, bh) are listed head group by head group (HG
  // heads each, the last group possibly smaller), and within a group heaviest first
  // (causal: key tile j is seen by query tiles j .. n - 1, so the work falls with
  // j): list position t of group g0 = t / (HG n) is tile j = p / hg of head
  // g0 HG + p % hg, p = t mod HG n, hg the group's head count.  The grid has at most
  // one CTA per SM; CTA c starts with positions c and 2G - 1 - c (G CTAs: a heavy
  // and a light tile of the first two rounds).  Its later tiles (p.dynamic) are the
  // next free positions of the list, taken from a counter in global memory by the
  // producer as the CTA starts the tile two before (the atomic's latency stays off
  // the critical path, and the next tile's K and V can be loaded ahead): the CTAs
  // work down the list together, each taking new work as it finishes, so that they
  // end within about a tile of each other whatever the mix of tile sizes.  Otherwise
  // they continue the snake, 2G + c, 4G - 1 - c, ..., which balances lists of equal
  // tiles and short lists.  The CTAs running at any one time share a few heads,
  // whose K, V, Q, dO and dQ accumulator rows then stay in L2 (HG = BH lists every
  // head at once).  With the counter, the producer passes tiles 2, 3, ... to the
  // other roles through a ring in shared memory (-1 ends the sequence); snake
  // positions every role computes itself.
  // (The helpers below copy what they need from p: capturing the kernel parameter
  // itself would take its address and copy it to local memory.)
  const int G = static_cast<int>(gridDim.x);
  const int cta = static_cast<int>(blockIdx.x);
  const int BH = p.BH;
  const int win = p.window;
  const int T = n_q * BH;
  const bool dyn = p.dynamic != 0;
  auto snake_tile = [=](int k) {  // the CTA's tile k in snake order (-1: none)
    const long long t = static_cast<long long>(k) * G + ((k & 1) ? G - 1 - cta : cta);
    return t < T ? static_cast<int>(t) : -1;
  };
  const int HG = p.head_group;
  auto tile_j = [=](int t) {  // key tile of list position t
    const int g0 = t / (HG * n_q), pp = t - g0 * (HG * n_q);
    return pp / min(HG, BH - g0 * HG);
  };
  auto tile_bh = [=](int t) {  // batch * head of list position t
    const int g0 = t / (HG * n_q), pp = t - g0 * (HG * n_q);
    return g0 * HG + pp % min(HG, BH - g0 * HG);
  };
  // Query tiles that see key tile j: from j on when causal, and with a sliding
  // window up to the last query that sees its last key, j*128 + 127 + window - 1.
  auto q_begin = [](int j) { return CAUSAL ? j : 0; };
  auto q_end = [=](int j) {
    return (CAUSAL && win > 0) ? min(n_q, (j * 128 + 127 + win - 1) / 128 + 1) : n_q;
  };
  // bar_kv[b] and kv_empty[b] complete once per tile that uses buffer b: the
  // phase parity of tile k's turn on its buffer.
  auto kv_par = [](int k) { return static_cast<uint32_t>((C::KVB == 2 ? (k >> 1) : k) & 1); };

  WaitCtl wc{p.status, &abort_flag, p.wait_ns};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar_kv[b], 1);
      mbar_init(&kv_empty[b], 1);
    }
    mbar_init(&acc_free, 8);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(&qdo_full[s], 1);
      mbar_init(&qdo_empty[s], (C::DQ && !C::PIPE) ? 2 : 1);
    }
    for (int s = 0; s < 3; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1); }
    // a tile id is read by the MMA thread and by the 8 compute warps
    for (int s = 0; s < kTileRing; ++s) { mbar_init(&ctl.tile_full[s], 1); mbar_init(&ctl.tile_empty[s], 9); }
    mbar_init(&s_full, 1);
    mbar_init(&dp_full, 1);
    mbar_init(&p_ready, 8);
    mbar_init(&s_read, 8);
    mbar_init(&ds_ready, 8);
    mbar_init(&dq_full, 1);
    mbar_init(&dq_drained, 8);
    mbar_init(&drain, 1);
    mbar_init(&fin, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      int last_kv0 = -1, last_kv1 = -1;  // the last of the CTA's tiles whose K, V went to buffer 0, 1
      // K and V of the CTA's tile k into its buffer (the test hook skips them: a
      // consumer's wait then runs out).
      const bool skip_kv = p.fault == 1;
      auto load_kv = [&](int k, int t) {
        if (skip_kv) return;
        const int b = k % C::KVB;
        const int row = tile_j(t) * 128, bh = tile_bh(t);
        mbar_arrive_expect_tx(&bar_kv[b], 2 * C::TILE);
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_3d(sK + b * C::TILE + c * C::CHUNK, &tmK, &bar_kv[b], c * 64, row, bh);
          tma_load_3d(sV + b * C::TILE + c * C::CHUNK, &tmV, &bar_kv[b], c * 64, row, bh);
        }
        if (b == 0) last_kv0 = k; else last_kv1 = k;
      };
      // Nothing is read before the wait for the preprocess grid: its completion
      // also covers the kernels before it, one of which (the caller's, launched
      // with an early trigger) may still be writing K or V.  The L, D rows and the
      // zeroed dQ accumulator come from the preprocess itself.
      const uint64_t keep = policy_evict_last();
      // The CTA's tile kk >= 2 (-1 past the end of the list): the next free list
      // position past the first two rounds, or the snake's; and tile k's id into the
      // ring.
      auto grab = [&](int kk) -> int {
        if (!dyn) return snake_tile(kk);
        const long long t = 2LL * G + atomicAdd(p.tile_ctr, 1u);
        return t < T ? static_cast<int>(t) : -1;
      };
      // Tiles 0 and 1 are the snake's in both modes: the ring carries tiles 2, 3, ...
      auto publish = [&](int k, int t) -> bool {
        if (!dyn) return true;  // the other roles follow the snake themselves
        const int q = k - 2, s = q % kTileRing;
        if (q >= kTileRing &&
            !mbar_wait(&ctl.tile_empty[s], ((q / kTileRing) - 1) & 1, wc, kBSiteProdTile))
          return false;
        ctl.tile_ring[s] = t;
        mbar_arrive(&ctl.tile_full[s]);
        return true;
      };
      griddep_wait();  // also orders the counter's zeroing before the first grab
      // Tiles k, k + 1 and k + 2 of the CTA (-1: none).
      int t_cur = snake_tile(0);
      int t_nx = t_cur >= 0 ? snake_tile(1) : -1;
      int t_nx2 = -1;
      bool ok = true;
      if (t_cur >= 0) load_kv(0, t_cur);
      if (C::KVB == 2 && t_nx >= 0) load_kv(1, t_nx);
      int gs = 0;  // query steps issued so far (ring slot and phase)
      int gq = 0;  // tile width 128: Q loads issued (may run one ahead of gs on an abort)
      for (int k = 0; ok && t_cur >= 0; ++k) {
        const int t = t_cur;
        const int bh = tile_bh(t);
        const int i0 = q_begin(tile_j(t)), n_it = q_end(tile_j(t)) - i0;
        for (int it = 0; it < n_it; ++it) {
          const int st = gs % C::ST;
          const int row = (i0 + it) * 128;
          if constexpr (!C::PIPE) {
            // Q in a ring of its own (released by dK), loaded before this step's dO.
            const int qs = gs % C::QS;
            if (gs >= C::QS &&
                !mbar_wait(&q_empty[qs], ((gs / C::QS) - 1) & 1, wc, kBSiteProdEmpty)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&q_full[qs], C::TILE + (C::DQ ? 2 * 512 : 0));
            if constexpr (C::DQ) {
              const size_t stq = static_cast<size_t>(bh) * p.Npad + row;
              bulk_load_1d(sLD + qs * 256, p.Lg + stq, 512, &q_full[qs]);
              bulk_load_1d(sLD + qs * 256 + 128, p.Dg + stq, 512, &q_full[qs]);
            }
            for (int c = 0; c < C::KCH; ++c)
              tma_load_3d_hint(sQ + qs * C::TILE + c * C::CHUNK, &tmQ, &q_full[qs], c * 64, row, bh,
                               keep);
            ++gq;
          }
          if (gs >= C::ST &&
              !mbar_wait(&qdo_empty[st], ((gs / C::ST) - 1) & 1, wc, kBSiteProdEmpty)) {
            ok = false;
            break;
          }
          constexpr bool LD_WITH_Q = C::DQ && !C::PIPE;
          mbar_arrive_expect_tx(&qdo_full[st], (C::PIPE ? 2 : 1) * C::TILE + (LD_WITH_Q ? 0 : 2 * 512));
          if constexpr (!LD_WITH_Q) {
            const size_t stat = static_cast<size_t>(bh) * p.Npad + row;
            bulk_load_1d(sLD + st * 256, p.Lg + stat, 512, &qdo_full[st]);
            bulk_load_1d(sLD + st * 256 + 128, p.Dg + stat, 512, &qdo_full[st]);
          }
          for (int c = 0; c < C::KCH; ++c) {
            if constexpr (C::PIPE)
              tma_load_3d_hint(sQ + st * C::TILE + c * C::CHUNK, &tmQ, &qdo_full[st], c * 64, row,
                               bh, keep);
            tma_load_3d_hint(sdO + st * C::TILE + c * C::CHUNK, &tmdO, &qdo_full[st], c * 64,
                             row, bh, keep);
          }
          ++gs;
          // Tile k + 2 is taken once tile k's first loads are out, and handed on at
          // the end of tile k (the atomic's result is not waited for before then).
          if (it == 0 && t_nx >= 0) t_nx2 = grab(k + 2);
          // The next K, V load.  Two buffers: tile k + 1's, a step or two into tile
          // k, once tile k - 1 has released the buffer.  One buffer: tile k's own,
          // right after its first (Q, dO) load, once tile k - 1's last product has
          // read the buffer.
          int nk = -1, nt = -1;
          if (C::KVB == 2) {
            if (k >= 1 && it == min(C::ST, n_it - 1) && t_nx >= 0) nk = k + 1, nt = t_nx;
          } else if (k >= 1 && it == 0) {
            nk = k, nt = t;
          }
          if (nk >= 0) {
            if (!mbar_wait(&kv_empty[nk % C::KVB], kv_par(nk - C::KVB), wc, kBSiteProdKV)) {
              ok = false;
              break;
            }
            load_kv(nk, nt);
          }
        }
        if (!ok) break;
        if (t_nx >= 0 && !publish(k + 2, t_nx2)) {
          ok = false;
          break;
        }
        t_cur = t_nx;
        t_nx = t_nx2;
        t_nx2 = -1;
      }
      volatile int no_abort = 0;
      WaitCtl dw{p.status, &no_abort, 100000000ull};
      if (!ok) {
        for (int q = max(0, gs - C::ST); q < gs; ++q)
          mbar_wait(&qdo_full[q % C::ST], (q / C::ST) & 1, dw, kBSiteProdDrain);
        if constexpr (!C::PIPE) {
          for (int q = max(0, gq - C::QS); q < gq; ++q)
            mbar_wait(&q_full[q % C::QS], (q / C::QS) & 1, dw, kBSiteProdDrain);
        }
      }
      // Every K, V load lands before exit, even on an aborted run (one at most is
      // in flight per buffer: a reload waits for the previous one to be consumed).
      if (last_kv0 >= 0) mbar_wait(&bar_kv[0], kv_par(last_kv0), dw, kBSiteProdDrain);
      if (last_kv1 >= 0) mbar_wait(&bar_kv[1], kv_par(last_kv1), dw, kBSiteProdDrain);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_f16(128, 128, BF16, false, false);  // S^T, dP^T
      constexpr uint32_t id_tb = idesc_f16(128, D, BF16, false, true);     // dV, dK (B MN-major)
      constexpr uint32_t id_dq = idesc_f16(128, D, BF16, true, true);      // dQ (A, B MN-major)
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ),
                     adO = smem_u32(sdO), aDS = smem_u32(sDS);
      // Base descriptors; a K step, a ring stage or a K/V buffer only moves the
      // start address.
      const uint64_t kK = sdesc_sw128(aK, 16, 1024), kV = sdesc_sw128(aV, 16, 1024);
      const uint64_t kQ = sdesc_sw128(aQ, 16, 1024), kdO = sdesc_sw128(adO, 16, 1024);
      const uint64_t mQ = sdesc_sw128(aQ, C::CHUNK, 1024), mdO = sdesc_sw128(adO, C::CHUNK, 1024);
      const uint64_t mK = sdesc_sw128(aK, C::CHUNK, 1024), mDS = sdesc_sw128(aDS, C::CHUNK, 1024);
      // The products of a step; `st` is its ring slot, `kvo` the tile's K/V buffer.
      auto mma_s = [&](int st, uint32_t kvo) {  // S^T = K Q^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          umma_ss(tbase + C::C_S, sdesc_add(kK, kvo + off), sdesc_add(kQ, st * C::TILE + off),
                  id_kk, kk > 0);
        }
        umma_commit(&s_full);
      };
      auto mma_dp = [&](int st, uint32_t kvo) {  // dP^T = V dO^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          umma_ss(tbase + C::C_DP, sdesc_add(kV, kvo + off), sdesc_add(kdO, st * C::TILE + off),
                  id_kk, kk > 0);
        }
        umma_commit(&dp_full);
      };
      auto mma_dv = [&](int st, bool first) {  // dV += P^T dO (queries 16 kk ..: warpgroup kk / 4)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tbase + C::C_DV, tbase + C::C_P(kk >> 2) + (kk & 3) * 8,
                  sdesc_add(mdO, st * C::TILE + kk * 2048), id_tb, (!first || kk > 0) ? 1u : 0u);
        // Without dQ, dV is dO's last reader (its L, D rows were read before
        // ds_ready).  With dQ at D = 128 the compute warpgroups release dO instead,
        // once the dQ reduce staged in its tile has been read.
        if constexpr (!C::DQ) umma_commit(&qdo_empty[st]);
      };
      auto mma_dq = [&](uint32_t kvo) {  // dQ_i = dS K
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tbase + C::C_DQ, sdesc_add(mDS, kk * 2048), sdesc_add(mK, kvo + kk * 2048),
                  id_dq, kk > 0);
        umma_commit(&dq_full);
      };
      // dK += dS^T Q; the step's last read of Q (and, at tile width 64, of its dO).
      // qs: the Q slot -- the (Q, dO) ring's at tile width 64, the Q ring's at 128.
      auto mma_dk = [&](int qs, bool first) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tbase + C::C_DK, tbase + C::C_DS(kk >> 2) + (kk & 3) * 8,
                  sdesc_add(mQ, qs * C::TILE + kk * 2048), id_tb, (!first || kk > 0) ? 1u : 0u);
        umma_commit(C::PIPE ? &qdo_empty[qs] : &q_empty[qs]);
      };
      bool ok = true;
      int gs = 0;  // query steps so far
      for (int k = 0; ok; ++k) {
        int t = snake_tile(k);
        if (dyn && k >= 2) {
          const int ts = (k - 2) % kTileRing;
          if (!mbar_wait(&ctl.tile_full[ts], ((k - 2) / kTileRing) & 1, wc, kBSiteMmaTile)) { ok = false; break; }
          t = ctl.tile_ring[ts];
          mbar_arrive(&ctl.tile_empty[ts]);
        }
        if (t < 0) break;
        const int n_it = q_end(tile_j(t)) - q_begin(tile_j(t));
        const int b = k % C::KVB;
        const uint32_t kvo = static_cast<uint32_t>(b * C::TILE);  // this tile's K, V buffer
        if (!mbar_wait(&bar_kv[b], kv_par(k), wc, kBSiteMmaKV)) { ok = false; break; }
        if constexpr (C::DQ && !C::PIPE) {
          // Tile width 128 with dQ: TMEM has no free columns, so each step runs in
          // order -- S^T, dP^T (once the previous dQ partial, in the same columns,
          // is drained), dV (P^T ready), dQ and dK (dS^T ready).
          for (int it = 0; it < n_it; ++it, ++gs) {
            const int st = gs % C::ST;
            if (!mbar_wait(&q_full[st], (gs / C::QS) & 1, wc, kBSiteMmaQ)) { ok = false; break; }
            tc_fence_after();
            mma_s(st, kvo);
            if (gs > 0) {
              if (!mbar_wait(&dq_drained, (gs - 1) & 1, wc, kBSiteMmaDrained)) { ok = false; break; }
              tc_fence_after();
            }
            if (!mbar_wait(&qdo_full[st], (gs / C::ST) & 1, wc, kBSiteMmaQ)) { ok = false; break; }
            tc_fence_after();
            mma_dp(st, kvo);
            if (!mbar_wait(&p_ready, gs & 1, wc, kBSiteMmaP)) { ok = false; break; }
            tc_fence_after();
            if (k > 0 && it == 0) {
              if (!mbar_wait(&acc_free, (k - 1) & 1, wc, kBSiteMmaAcc)) { ok = false; break; }
              tc_fence_after();
            }
            mma_dv(st, it == 0);
            // dQ_i = dS K first (the drain needs only this one), then dK += dS^T Q (A
            // from TMEM, so the dQ staging that reuses the dS^T tile of shared memory
            // cannot race it).
            if (!mbar_wait(&ds_ready, gs & 1, wc, kBSiteMmaDS)) { ok = false; break; }
            tc_fence_after();
            mma_dq(kvo);
            if (it == n_it - 1) umma_commit(&kv_empty[b]);
            mma_dk(st, it == 0);
          }
        } else if constexpr (C::DQ) {
          // Tile width 64: step g + 1's scores go out once the compute warps have
          // read step g's and written P^T (p_ready), right after step g's dV product,
          // so that they overlap step g's dS; step g + 1's dP^T follows step g's dK,
          // whose dS^T operand sits in the dP^T columns.
          if (!mbar_wait(&qdo_full[gs % C::ST], (gs / C::ST) & 1, wc, kBSiteMmaQ)) { ok = false; break; }
          tc_fence_after();
          mma_s(gs % C::ST, kvo);
          mma_dp(gs % C::ST, kvo);
          for (int it = 0; it < n_it; ++it, ++gs) {
            const int st = gs % C::ST;
            if (!mbar_wait(&p_ready, gs & 1, wc, kBSiteMmaP)) { ok = false; break; }
            tc_fence_after();
            if (k > 0 && it == 0) {
              // A tile's first dV and dK products overwrite the accumulators: the
              // previous tile's epilogue must have read them out.
              if (!mbar_wait(&acc_free, (k - 1) & 1, wc, kBSiteMmaAcc)) { ok = false; break; }
              tc_fence_after();
            }
            mma_dv(st, it == 0);
            if (it + 1 < n_it) {
              const int st1 = (gs + 1) % C::ST;
              if (!mbar_wait(&qdo_full[st1], ((gs + 1) / C::ST) & 1, wc, kBSiteMmaQ)) { ok = false; break; }
              tc_fence_after();
              mma_s(st1, kvo);
            }
            if (!mbar_wait(&ds_ready, gs & 1, wc, kBSiteMmaDS)) { ok = false; break; }
            tc_fence_after();
            if (gs > 0) {  // the dQ columns hold the previous partial until drained
              if (!mbar_wait(&dq_drained, (gs - 1) & 1, wc, kBSiteMmaDrained)) { ok = false; break; }
              tc_fence_after();
            }
            mma_dq(kvo);
            // The tile's K, V have been read for the last time: release the buffer.
            if (it == n_it - 1) umma_commit(&kv_empty[b]);
            mma_dk(st, it == 0);
            if (it + 1 < n_it) mma_dp((gs + 1) % C::ST, kvo);
          }
        } else {
          // Tile width 128: S^T(g + 1) as soon as the compute warps have read S^T(g)
          // (s_read), so that it runs during their exponentials; dV(g) and dK(g) once
          // P^T and dS^T are packed over the dP^T columns (ds_ready); dP^T(g + 1)
          // after them, in issue order, since it overwrites those columns.
          if (!mbar_wait(&q_full[gs % C::QS], (gs / C::QS) & 1, wc, kBSiteMmaQ)) { ok = false; break; }
          tc_fence_after();
          mma_s(gs % C::QS, kvo);
          if (!mbar_wait(&qdo_full[gs % C::ST], (gs / C::ST) & 1, wc, kBSiteMmaQ)) { ok = false; break; }
          tc_fence_after();
          mma_dp(gs % C::ST, kvo);
          // The tile's last reads of K and V are its last S^T and dP^T: the buffer can
          // take the next tile's K, V during the last dV, dK.
          if (n_it == 1) umma_commit(&kv_empty[b]);
          for (int it = 0; it < n_it; ++it, ++gs) {
            const int st = gs % C::ST;
            if (it + 1 < n_it) {
              const int qs1 = (gs + 1) % C::QS;
              if (!mbar_wait(&s_read, gs & 1, wc, kBSiteMmaP) ||
                  !mbar_wait(&q_full[qs1], ((gs + 1) / C::QS) & 1, wc, kBSiteMmaQ)) {
                ok = false;
                break;
              }
              tc_fence_after();
              mma_s(qs1, kvo);
            }
            if (!mbar_wait(&ds_ready, gs & 1, wc, kBSiteMmaDS)) { ok = false; break; }
            tc_fence_after();
            if (k > 0 && it == 0) {
              // A tile's first dV and dK products overwrite the accumulators: the
              // previous tile's epilogue must have read them out.
              if (!mbar_wait(&acc_free, (k - 1) & 1, wc, kBSiteMmaAcc)) { ok = false; break; }
              tc_fence_after();
            }
            mma_dv(st, it == 0);
            mma_dk(gs % C::QS, it == 0);
            if (it + 1 < n_it) {
              const int st1 = (gs + 1) % C::ST;
              if (!mbar_wait(&qdo_full[st1], ((gs + 1) / C::ST) & 1, wc, kBSiteMmaQ)) { ok = false; break; }
              tc_fence_after();
              mma_dp(st1, kvo);
              if (it + 1 == n_it - 1) umma_commit(&kv_empty[b]);
            }
          }
        }
        if (!ok) break;
        umma_commit(&drain);  // the tile's dK and dV are final once this lands
      }
      umma_commit(&fin);  // every product issued has landed once this does
      volatile int no_abort = 0;
      WaitCtl dw{p.status, &no_abort, p.wait_ns};
      mbar_wait(&fin, 0, dw, kBSiteMmaDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ compute
    griddep_wait();  // the accumulator this role adds into was zeroed by the preprocess
    const int g = warp >> 2;                   // warpgroup: query columns 64 g .. 64 g + 63
    const int wq = warp & 3;                   // TMEM lane quadrant
    const int r = wq * 32 + lane;              // key row (P^T, dS^T) / query row (dQ)
    const uint32_t lb = static_cast<uint32_t>(wq * 32);
    const float sl2 = p.scale_log2;
    const int qoff = 64 * g;
    const uint32_t wg_bar = 1 + g;             // named barrier of this warpgroup
    bool ok = true;
    int gs = 0;  // query steps so far
    float pr[64];  // this warpgroup's P^T of a step, from its P stage to its dS stage
    // The three stages of query step gp (query tile ip of key tile j).  Every wait
    // of a compute warpgroup ends in a warpgroup-wide vote, so that all of its 128
    // threads leave together on a timeout (the named barriers have no time limit and
    // must never be left waiting).
    auto stage_p = [&](int gp, int ip, int j, int key) -> bool {
      const int stp = gp % C::ST;
      // The step's LSE*log2e and D rows arrive in shared memory with Q_i (fused
      // D = 128 kernel) or with dO_i.
      const float4* L4 = reinterpret_cast<const float4*>(sLD + stp * 256 + qoff);
      constexpr bool LD_WITH_Q = C::DQ && !C::PIPE;
      uint64_t* ld_full = LD_WITH_Q ? &q_full[gp % C::QS] : &qdo_full[stp];
      const uint32_t ld_par = static_cast<uint32_t>((gp / (LD_WITH_Q ? C::QS : C::ST)) & 1);
      if (!named_bar_and(wg_bar, 128, mbar_wait(ld_full, ld_par, wc, kBSiteCmpQ))) return false;
      if (!named_bar_and(wg_bar, 128, mbar_wait(&s_full, gp & 1, wc, kBSiteCmpS))) return false;
      tc_fence_after();
      // P^T (this warpgroup's 64 query columns): exp2(S^T * scale * log2e - LSE * log2e),
      // zero where the key comes after the query or lies past N.
      // Masking (key after query on the diagonal tile, or key past N) is rare: one
      // branch per tile, not a compare per element.
      const bool masked = (CAUSAL && ip == j) || key >= N ||
                          (CAUSAL && win > 0 && ip * 128 + 127 - j * 128 >= win);
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      uint32_t srr[2][32];
      tmem_ld32(tmem_addr(tbase, lb, C::C_S + qoff), srr[0]);
      tmem_ld32(tmem_addr(tbase, lb, C::C_S + qoff + 32), srr[1]);
      tmem_wait_ld();
      reg_fence(srr[0]);
      reg_fence(srr[1]);
      if constexpr (!C::DQ) {
        // Tile width 128: the score columns may take the next step's scores now.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_read);
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint32_t (&sr)[32] = srr[c];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 l4 = L4[c * 8 + v];
          const uint64_t a01 = f2_fma(f2_pack(__uint_as_float(sr[v * 4]), __uint_as_float(sr[v * 4 + 1])),
                                      sl2x2, f2_pack(-l4.x, -l4.y));
          const uint64_t a23 = f2_fma(f2_pack(__uint_as_float(sr[v * 4 + 2]), __uint_as_float(sr[v * 4 + 3])),
                                      sl2x2, f2_pack(-l4.z, -l4.w));
          float x0, x1, x2, x3;
          f2_unpack(a01, x0, x1);
          f2_unpack(a23, x2, x3);
          const int q0 = c * 32 + v * 4;
          if ((v & 3) >= kBwdPolyFrom) {  // FMA-pipe exp2 for this group of four
            pr[q0 + 0] = exp2_poly3(x0);
            pr[q0 + 1] = exp2_poly3(x1);
            pr[q0 + 2] = exp2_poly3(x2);
            pr[q0 + 3] = exp2_poly3(x3);
          } else {
            pr[q0 + 0] = ex2_approx(x0);
            pr[q0 + 1] = ex2_approx(x1);
            pr[q0 + 2] = ex2_approx(x2);
            pr[q0 + 3] = ex2_approx(x3);
          }
        }
      }
      if (masked) {
#pragma unroll
        for (int qc = 0; qc < 64; ++qc)
          if ((CAUSAL && ip == j && qoff + qc < r) || key >= N ||
              (CAUSAL && win > 0 && ip * 128 + qoff + qc - key >= win))
            pr[qc] = 0.f;
      }
      if constexpr (C::DQ) {
        // Tile width 64: P^T goes to its own columns now (dV can start).  At 128 it
        // stays in registers and is written with dS^T.
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack2<BF16>(pr[2 * e], pr[2 * e + 1]);
        tmem_st32(tmem_addr(tbase, lb, C::C_P(g)), pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_ready);
      }
      return true;
    };
    // dS^T = P^T * (dP^T - D), 32 queries at a time, written to TMEM (A operand
    // of dK) and to shared memory (A operand of dQ).  The shared copy is
    // MN-major with 128-byte swizzle: chunk g holds queries 64 g .. 64 g + 63 of
    // every key row; 16-byte unit u of row r sits at unit u ^ (r % 8).
    auto stage_ds = [&](int gd) -> bool {
      const float4* D4 = reinterpret_cast<const float4*>(sLD + (gd % C::ST) * 256 + 128 + qoff);
      if (!named_bar_and(wg_bar, 128, mbar_wait(&dp_full, gd & 1, wc, kBSiteCmpDP))) return false;
      tc_fence_after();
      if constexpr (!C::DQ) {
        // Tile width 128: all 64 dP^T columns of this warpgroup into registers, then
        // packed dS^T and P^T over them (the A operands of dK and dV).
        uint32_t dr[2][32];
        tmem_ld32(tmem_addr(tbase, lb, C::C_DP + qoff), dr[0]);
        tmem_ld32(tmem_addr(tbase, lb, C::C_DP + qoff + 32), dr[1]);
        tmem_wait_ld();
        reg_fence(dr[0]);
        reg_fence(dr[1]);
        uint32_t dsk[32], pk[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float4 d4 = D4[c * 8 + v];
            const int q0 = c * 32 + v * 4;
            const uint64_t t01 = f2_sub(f2_pack(__uint_as_float(dr[c][v * 4]), __uint_as_float(dr[c][v * 4 + 1])),
                                        f2_pack(d4.x, d4.y));
            const uint64_t t23 = f2_sub(f2_pack(__uint_as_float(dr[c][v * 4 + 2]), __uint_as_float(dr[c][v * 4 + 3])),
                                        f2_pack(d4.z, d4.w));
            float a0, a1, a2, a3;
            f2_unpack(f2_mul(f2_pack(pr[q0], pr[q0 + 1]), t01), a0, a1);
            f2_unpack(f2_mul(f2_pack(pr[q0 + 2], pr[q0 + 3]), t23), a2, a3);
            dsk[q0 / 2] = pack2<BF16>(a0, a1);
            dsk[q0 / 2 + 1] = pack2<BF16>(a2, a3);
            pk[q0 / 2] = pack2<BF16>(pr[q0], pr[q0 + 1]);
            pk[q0 / 2 + 1] = pack2<BF16>(pr[q0 + 2], pr[q0 + 3]);
          }
        }
        tmem_st32(tmem_addr(tbase, lb, C::C_DS(g)), dsk);
        tmem_st32(tmem_addr(tbase, lb, C::C_P(g)), pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_ready);
        return true;
      }
      if (C::DQ && gd > 0) {
        // This warpgroup's dS^T chunk (and, at D = 128, its half of the previous
        // step's dO tile) held the previous step's dQ reduce: the bulk copies must
        // have finished reading it.  At D = 128 the dO tile then goes back to the
        // producer.
        if (r == 0) {
          tma_store_wait_read();
          if constexpr (!C::PIPE) mbar_arrive(&qdo_empty[(gd - 1) % C::ST]);
        }
        named_bar_sync(wg_bar, 128);
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dr[32];
        tmem_ld32(tmem_addr(tbase, lb, C::C_DP + qoff + 32 * c), dr);
        tmem_wait_ld();
        reg_fence(dr);
        uint32_t dsk[16];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 d4 = D4[c * 8 + v];
          const int q0 = c * 32 + v * 4;
          const uint64_t t01 = f2_sub(f2_pack(__uint_as_float(dr[v * 4]), __uint_as_float(dr[v * 4 + 1])),
                                      f2_pack(d4.x, d4.y));
          const uint64_t t23 = f2_sub(f2_pack(__uint_as_float(dr[v * 4 + 2]), __uint_as_float(dr[v * 4 + 3])),
                                      f2_pack(d4.z, d4.w));
          float a0, a1, a2, a3;
          f2_unpack(f2_mul(f2_pack(pr[q0], pr[q0 + 1]), t01), a0, a1);
          f2_unpack(f2_mul(f2_pack(pr[q0 + 2], pr[q0 + 3]), t23), a2, a3);
          dsk[2 * v] = pack2<BF16>(a0, a1);
          dsk[2 * v + 1] = pack2<BF16>(a2, a3);
        }
        tmem_st16(tmem_addr(tbase, lb, C::C_DS(g) + 16 * c), dsk);
        if constexpr (C::DQ) {
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) {
            const int u = c * 4 + uu;
            const uint4 val = make_uint4(dsk[4 * uu], dsk[4 * uu + 1], dsk[4 * uu + 2], dsk[4 * uu + 3]);
            *reinterpret_cast<uint4*>(sDS + g * C::CHUNK + r * 128 + ((u ^ (r & 7)) << 4)) = val;
          }
        }
      }
      if constexpr (C::DQ) fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_ready);
      return true;
    };
    auto stage_dq = [&](int gq, int iq, int bh) -> bool {
      if (!named_bar_and(wg_bar, 128, mbar_wait(&dq_full, gq & 1, wc, kBSiteCmpDQ))) return false;
      tc_fence_after();
      // dQ partial, head columns g D/2 .. (g+1) D/2 - 1, in 32-column tiles: TMEM ->
      // shared memory, laid out as a 128-row x 32-float tile with 128-byte swizzle
      // -> one TMA reduce-add per tile into the fp32 accumulator (rows past N are
      // clipped by the tensor map).  The first tile goes to this warpgroup's dS^T
      // chunk (free: the dQ product that read it has completed).
      constexpr int HALF = D / 2;
      constexpr int NCH = HALF / 32;
      uint8_t* stage = sDS + g * C::CHUNK;
      if constexpr (C::PIPE) {
        // One 32-column tile, 16 columns at a time: the next step's P^T is live
        // beside it.  The columns are released once both halves are read.
        static_assert(NCH == 1, "pipelined steps assume D = 64");
  #pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t q16[16];
          tmem_ld16(tmem_addr(tbase, lb, C::C_DQ + g * HALF + 16 * h), q16);
          tmem_wait_ld();
          reg_fence(q16);
          if (h == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dq_drained);
          }
  #pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(stage + r * 128 + (((4 * h + u) ^ (r & 7)) << 4)) =
                make_uint4(q16[4 * u], q16[4 * u + 1], q16[4 * u + 2], q16[4 * u + 3]);
        }
        fence_proxy_async_smem();
        named_bar_sync(wg_bar, 128);
        if (r == 0) {
          tma_reduce_add_3d(&tmdQ, stage, g * HALF, iq * 128, bh);
          tma_store_commit();
        }
        __syncwarp();
      } else {
        // All of this warpgroup's TMEM columns first, so that the region is released
        // (dq_drained) before any staging starts.  The second tile goes to this
        // warpgroup's half of the step's dO tile (dP^T and dV, its readers, have
        // completed before dQ; the producer reloads it only after the next step's
        // release), so that both reduces leave together: with a single staging tile
        // the second would wait for the first to be read (~1.4k cycles when every SM
        // is adding into L2).
        uint32_t qr[NCH][32];
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          tmem_ld32(tmem_addr(tbase, lb, C::C_DQ + g * HALF + 32 * c), qr[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < NCH; ++c) reg_fence(qr[c]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dq_drained);
        static_assert(NCH == 2, "two staging tiles");
        uint8_t* stg[2] = {stage, sdO + (gq % C::ST) * C::TILE + g * C::CHUNK};
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(stg[c] + r * 128 + ((u ^ (r & 7)) << 4)) =
                make_uint4(qr[c][4 * u], qr[c][4 * u + 1], qr[c][4 * u + 2], qr[c][4 * u + 3]);
        }
        fence_proxy_async_smem();
        named_bar_sync(wg_bar, 128);
        if (r == 0) {
          tma_reduce_add_3d(&tmdQ, stg[0], g * HALF, iq * 128, bh);
          tma_reduce_add_3d(&tmdQ, stg[1], g * HALF + 32, iq * 128, bh);
          tma_store_commit();
        }
        __syncwarp();
      }
      return true;
    };
    // dV (warpgroup 0) and dK (warpgroup 1) of the tile are final once its
    // products have landed: read them out of TMEM, hand the columns to the next
    // tile's products, then store them.
    auto epilogue = [&](int k, int key, int bh) -> bool {
      if (!named_bar_and(wg_bar, 128, mbar_wait(&drain, k & 1, wc, kBSiteCmpDQ))) return false;
      tc_fence_after();
      const uint32_t col = g ? C::C_DK : C::C_DV;
      const float mul = g ? p.scale : 1.0f;
      const int d = p.d;
      uint8_t* row = reinterpret_cast<uint8_t*>(g ? p.dK : p.dV) +
                     (static_cast<size_t>(bh) * N + key) * (d * 2);
      // 32 columns at a time: TMEM -> 16-bit -> global (stores do not wait), the
      // columns handed back once the last chunk is in registers.
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(tmem_addr(tbase, lb, col + 32 * c), rr);
        tmem_wait_ld();
        reg_fence(rr);
        if (c == D / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_free);
        }
        uint4 v[4];
        uint32_t* pv = reinterpret_cast<uint32_t*>(v);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pv[e] = pack2<BF16>(__uint_as_float(rr[2 * e]) * mul, __uint_as_float(rr[2 * e + 1]) * mul);
        if (key < N) {
          uint4* dst4 = reinterpret_cast<uint4*>(row + c * 64);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (c * 32 + 8 * e < d) dst4[e] = v[e];  // 8 columns per store; d % 8 == 0
        }
      }
      return true;
    };
    for (int k = 0; ok; ++k) {
      int t = snake_tile(k);
      if (dyn && k >= 2) {
        const int ts = (k - 2) % kTileRing;
        if (!named_bar_and(wg_bar, 128,
                           mbar_wait(&ctl.tile_full[ts], ((k - 2) / kTileRing) & 1, wc, kBSiteCmpTile))) {
          ok = false;
          break;
        }
        t = ctl.tile_ring[ts];
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.tile_empty[ts]);
      }
      if (t < 0) break;
      const int j = tile_j(t), bh = tile_bh(t);
      const int key = j * 128 + r;
      const int i_begin = q_begin(j);
      const int n_it = q_end(j) - i_begin;
      // Pipelined order: P of step 0, then per step i: dS(i), P(i + 1), dQ drain(i)
      // (tile width 64; without dQ no drain), so that step i's dQ product and step
      // i + 1's dP product run while the softmax works.
      const int g0 = gs;
      if constexpr (C::DQ && !C::PIPE) {
        // Tile width 128 with dQ: P, dS, dQ drain of each step in turn.
        for (int it = 0; it < n_it && ok; ++it) {
          ok = stage_p(g0 + it, i_begin + it, j, key);
          if (!ok) break;
          ok = stage_ds(g0 + it);
          if (!ok) break;
          ok = stage_dq(g0 + it, i_begin + it, bh);
        }
      } else {
        ok = stage_p(g0, i_begin, j, key);
        for (int it = 0; it < n_it && ok; ++it) {
          ok = stage_ds(g0 + it);
          if (!ok) break;
          if (it + 1 < n_it) {
            ok = stage_p(g0 + it + 1, i_begin + it + 1, j, key);
            if (!ok) break;
          }
          if constexpr (C::DQ) ok = stage_dq(g0 + it, i_begin + it, bh);
        }
      }
      gs = g0 + n_it;
      if (!ok) break;
      ok = epilogue(k, key, bh);
    }
    // All reductions complete before the CTA (and its shared memory) goes away.
    if (r == 0) tma_store_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------------------------------
// host launcher
// ------------------------------------------------------------------------------------

// [BH][N][d] 16-bit tensor as a 3-D TMA map, box_rows x 64-column boxes, 128-byte
// swizzle; fp32 accumulator map with 128 x 32 boxes (both defined with the host API).
bool make_tile_map(CUtensorMap* map, const void* base, int BH, int N, int d, bool bf16,
                   int box_rows = 128);
bool make_acc_map(CUtensorMap* map, float* base, int BH, int N, int d);

// Raises a kernel's dynamic shared memory limit once per device (the attribute is
// host state, set before the first launch on each device, not per call).  Every
// kernel instantiation passes flags of its own (a static array in its launcher).
constexpr int kSmemFlagDevices = 64;
template <typename Kern>
bool set_smem_once(Kern kern, int smem, std::atomic<bool> (&done)[kSmemFlagDevices]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSmemFlagDevices) {
    cudaGetLastError();
    return false;
  }
  if (done[dev].load(std::memory_order_acquire)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  done[dev].store(true, std::memory_order_release);
  return true;
}

// Launch with programmatic stream serialisation: the kernel may start while the
// previous kernel on the stream finishes; it waits (griddepcontrol.wait) before
// touching that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, int smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) cudaGetLastError();
  return e;
}

template <int D, bool BF16, bool CAUSAL, bool DQ>
int launch_bwd_t(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, void* dQ, void* dK, void* dV, void* workspace, int BH, int N,
                 int d, float scale, int window, unsigned int* status, unsigned long long wait_ns,
                 int fault, int max_ctas, cudaStream_t stream) {
  using Cfg = BwdCfg<D, DQ>;
  const int Npad = static_cast<int>(bwd_npad(N));
  // The tile list (key tiles x heads) is indexed with 32-bit ints in the kernel.
  if (static_cast<long long>(Npad / 128) * BH > (1ll << 30)) return 1;  // FA2_ERR_INVALID_ARG
  float* Dg = static_cast<float*>(workspace);
  float* Lg = Dg + static_cast<size_t>(BH) * Npad;
  unsigned int* tile_ctr = reinterpret_cast<unsigned int*>(
      static_cast<uint8_t*>(workspace) +
      bwd_workspace_bytes(static_cast<size_t>(BH), N, d, !Cfg::DQ) - 256);
  // The fp32 dQ accumulator (tile width 64 only) follows the row statistics.
  float* dQacc = Cfg::DQ ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                    bwd_rowstat_bytes(static_cast<size_t>(BH), N))
                         : nullptr;
  CUtensorMap mq, mk, mv, mdo, mdq;
  if (!make_tile_map(&mq, Q, BH, N, d, BF16) || !make_tile_map(&mk, K, BH, N, d, BF16) ||
      !make_tile_map(&mv, V, BH, N, d, BF16) || !make_tile_map(&mdo, dO, BH, N, d, BF16))
    return 4;  // FA2_ERR_CUDA
  if constexpr (Cfg::DQ) {
    if (!make_acc_map(&mdq, dQacc, BH, N, D)) return 4;
  } else {
    mdq = mq;  // not read
  }
  if constexpr (!Cfg::DQ) {
    // 1. dQ (and the D, LSE * log2 e rows), one CTA per (query tile, batch*head)
    const long long grid = static_cast<long long>(Npad / 128) * BH;
    if (grid > 0x7fffffffll) return 1;  // FA2_ERR_INVALID_ARG
    auto kq = fa2_bwd_dq_kernel<BF16, CAUSAL>;
    static std::atomic<bool> smem_q[kSmemFlagDevices];
    if (!set_smem_once(kq, BwdDqCfg::SMEM, smem_q)) return 4;
    BwdDqParams qp{};
    qp.dQ = dQ;
    qp.Q = static_cast<const uint16_t*>(Q);
    qp.O = static_cast<const uint16_t*>(O);
    qp.dO = static_cast<const uint16_t*>(dO);
    qp.LSE = LSE;
    qp.Dg = Dg;
    qp.Lg = Lg;
    qp.d = d;
    qp.N = N;
    qp.Npad = Npad;
    qp.BH = BH;
    qp.n_q = Npad / 128;
    qp.window = window;
    qp.scale = scale;
    qp.scale_log2 = scale * 1.4426950408889634f;
    qp.status = status;
    qp.wait_ns = wait_ns;
    qp.fault = fault;
    qp.tile_ctr = tile_ctr;
    if (launch_pdl(kq, dim3(static_cast<unsigned int>(grid)), dim3(BwdDqCfg::THREADS),
                   BwdDqCfg::SMEM, stream, mq, mk, mv, mdo, qp) != cudaSuccess)
      return 4;
  } else {
    // 1. preprocess
    const long long rows = static_cast<long long>(BH) * Npad;
    constexpr int RPB = 256 / (D / 8);
    const unsigned int grid = static_cast<unsigned int>((rows + RPB - 1) / RPB);
    if (launch_pdl(fa2_bwd_pre_kernel<D, BF16>, dim3(grid), dim3(256), 0, stream,
                   static_cast<const uint16_t*>(O), static_cast<const uint16_t*>(dO), LSE, Dg, Lg,
                   dQacc, tile_ctr, N, Npad, rows, d) != cudaSuccess)
      return 4;
  }
  // 2. main (dK, dV; and, by default, the dQ partials)
  {
    auto kern = fa2_bwd_kernel<D, BF16, CAUSAL, DQ>;
    static std::atomic<bool> smem_set[kSmemFlagDevices];  // this instantiation's flags
    if (!set_smem_once(kern, Cfg::SMEM, smem_set)) return 4;
    BwdParams bp{};
    bp.Dg = Dg;
    bp.Lg = Lg;
    bp.dQacc = dQacc;
    bp.dK = dK;
    bp.dV = dV;
    bp.d = d;
    bp.N = N;
    bp.Npad = Npad;
    bp.BH = BH;
    bp.n_kv = Npad / 128;
    bp.scale = scale;
    bp.scale_log2 = scale * 1.4426950408889634f;
    bp.window = window;
    bp.status = status;
    bp.wait_ns = wait_ns;
    bp.fault = fault;
    bp.tile_ctr = tile_ctr;
    // Persistent grid: one CTA per SM at most (the kernel's shared memory and TMEM
    // admit one per SM), each running its share of the tile list.
    int dev = 0, n_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n_sm <= 0) {
      cudaGetLastError();
      return 4;
    }
    long long ctas = std::min(static_cast<long long>(bp.n_kv) * BH, static_cast<long long>(n_sm));
    if (max_ctas > 0) ctas = std::min(ctas, static_cast<long long>(max_ctas));
    // Tiles past the first two rounds from the counter (dynamic) on causal lists of
    // at least 8 tiles per CTA, whose tile sizes vary; the snake otherwise (equal
    // tiles, or too few for the counter to pay).  Heads per group: dynamic, about
    // 192 MB of K, V, Q, dO (16-bit) and fp32 dQ rows, and at least two rounds of
    // tiles; snake, about two rounds, capped at ~32 MB of rows.  Measured on B200
    // (backward, ms; snake with the capped groups -> dynamic): training shape B8 H16
    // N4096 d128 causal 1.772 (5 heads) -> 1.729 (32), its deterministic mode 2.236
    // -> 2.160 (32), B1 H16 N16384 causal 3.69 (1) -> 2.99 (8); dynamic with the
    // snake's groups was slower on the training shape (1.82) and the counter on the
    // d = 64 bench shape B4 H16 N1024 (512 tiles) 70.6 -> 80.9 us.  The snake's
    // groups: every head at once -> two rounds took the training shape from 2.08 to
    // 1.87 ms; one round gave 1.83 ms but slowed the d = 64 shape 72.7 -> 80.9 us,
    // hence the 32 MB cap (5 heads there, that shape's 37 untouched).
    {
      const long long T = static_cast<long long>(bp.n_kv) * BH;
      bp.dynamic = (CAUSAL && T >= 8 * ctas) ? 1 : 0;
      const long long per_head = 12LL * N * D;  // bytes of one head's rows (see above)
      const long long two_rounds = (2 * ctas + bp.n_kv - 1) / bp.n_kv;
      const long long hg = bp.dynamic ? std::max(two_rounds, (192LL << 20) / per_head)
                                      : std::min(two_rounds, (32LL << 20) / per_head);
      bp.head_group = static_cast<int>(std::min<long long>(BH, std::max<long long>(1, hg)));
    }
    const unsigned int grid = static_cast<unsigned int>(ctas);
    if (launch_pdl(kern, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM, stream, mq, mk, mv, mdo, mdq,
                   bp) != cudaSuccess)
      return 4;
  }
  // 3. dQ finalise
  if constexpr (Cfg::DQ) {
    const long long n8 = static_cast<long long>(BH) * N * D / 8;
    const unsigned int grid = static_cast<unsigned int>((n8 + 255) / 256);
    if (launch_pdl(fa2_bwd_dq_finalise_kernel<BF16>, dim3(grid), dim3(256), 0, stream, dQacc,
                   static_cast<uint16_t*>(dQ), scale, n8, D, d) != cudaSuccess)
      return 4;
  }
  return 0;
}

// deterministic: dQ by fa2_bwd_dq_kernel (summed in TMEM in a fixed order) and dK,
// dV by the dK/dV-only kernel, on 128-wide tiles at every head dim; otherwise the
// main kernel adds dQ partials into the workspace's accumulator.
inline int launch_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                      const float* LSE, void* dQ, void* dK, void* dV, void* workspace, int BH,
                      int N, int d, float scale, bool causal, bool bf16, unsigned int* status,
                      unsigned long long wait_ns, cudaStream_t s, int window = 0,
                      int fault = 0, int max_ctas = 0, bool deterministic = false) {
#define FA2_BWD_CALL(D_, BF_, CA_, DQ_)                                                         \
  return launch_bwd_t<D_, BF_, CA_, DQ_>(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, BH, N, d,   \
                                         scale, window, status, wait_ns, fault, max_ctas, s)
  if (deterministic) {
    if (bf16) { if (causal) FA2_BWD_CALL(128, true, true, false); FA2_BWD_CALL(128, true, false, false); }
    if (causal) FA2_BWD_CALL(128, false, true, false);
    FA2_BWD_CALL(128, false, false, false);
  }
  if (d <= 64) {
    if (bf16) { if (causal) FA2_BWD_CALL(64, true, true, true); FA2_BWD_CALL(64, true, false, true); }
    if (causal) FA2_BWD_CALL(64, false, true, true);
    FA2_BWD_CALL(64, false, false, true);
  }
  if (bf16) { if (causal) FA2_BWD_CALL(128, true, true, true); FA2_BWD_CALL(128, true, false, true); }
  if (causal) FA2_BWD_CALL(128, false, true, true);
  FA2_BWD_CALL(128, false, false, true);
#undef FA2_BWD_CALL
}

}  // namespace fa2
