// Host side of libfa2.so: argument validation, TMA descriptor encoding, kernel
// launch and the device status word.  Declarations and the contract of every
// entry point are in include/fa2.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "../../include/fa2.h"
#include "fa2_bwd.cuh"
#include "fa2_decode.cuh"
#include "fa2_fwd.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned int kDefaultWaitMs = 2000;

std::mutex g_mu;
unsigned int* g_status[kMaxDevices] = {};  // one device word per device, lazily allocated
std::atomic<int> g_fault{0};
std::atomic<unsigned int> g_wait_ms{kDefaultWaitMs};
std::atomic<int> g_bwd_ctas{0};  // test hook: cap on the backward grid (0 = one CTA per SM)
std::atomic<int> g_fwd_tiles{0};  // test hook: forward query tiles per CTA (0 = chosen, 1, 2)
std::atomic<unsigned long long> g_launches{0};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

}  // namespace

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// True when [a, a + a_bytes) and [b, b + b_bytes) share a byte.
bool overlaps(const void* a, size_t a_bytes, const void* b, size_t b_bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + b_bytes && y < x + a_bytes;
}

// Head dims: multiples of 8 (16-byte rows for TMA) up to 256 in the forward and
// 128 in the backward.
constexpr int kMaxFwdHeadDim = 256;
constexpr int kMaxBwdHeadDim = 128;

// Common checks of fa2_fwd / fa2_bwd that need no CUDA call.
int check_sizes(int B, int H, int N, int d, float scale, int causal, int dtype,
                int max_d = kMaxFwdHeadDim) {
  if (B < 1 || H < 1 || N < 1) return FA2_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA2_ERR_INVALID_ARG;
  if (dtype != FA2_FP16 && dtype != FA2_BF16) return FA2_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA2_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > (1ll << 30) || N > (1 << 30)) return FA2_ERR_INVALID_ARG;
  if (d < 8 || d > max_d || d % 8 != 0) return FA2_ERR_UNSUPPORTED;
  return FA2_OK;
}

// Forward kernel head dim (tile width) for head dim d: the next of 64, 128, 192, 256.
int fwd_tile_dim(int d) { return d <= 64 ? 64 : (d <= 128 ? 128 : (d <= 192 ? 192 : 256)); }
// Query rows per forward CTA: two 128-row tiles up to a tile width of 128, one above.
int fwd_rows_per_cta(int d) { return fwd_tile_dim(d) <= 128 ? 256 : 128; }

// Query tiles per CTA of a plain (or sliding-window) forward on sm_count SMs:
// two 128-row tiles (ping-pong), or one (twice the CTAs) when that fills the SMs
// better.  Causal items shrink with their position, so one-tile items pack well
// once the two-tile grid is under one wave; equal items (not causal, or a sliding
// window) only gain while the one-tile grid itself fits in one wave.  Measured on
// B200 (two -> one tile): causal 1 x 16 x 2048, d = 64: 37.4 -> 29.1 us, d = 128:
// 43.2 -> 31.2 us; not causal 1 x 32 x 1024, d = 64: 23.0 -> 29.1 us (kept at two).
int fwd_tiles_per_cta(long long BH, int N, int d, bool causal, int window, int sm_count) {
  if (fwd_tile_dim(d) > 128) return 1;
  const int mode = g_fwd_tiles.load();
  if (mode != 0) return mode;
  const long long two = static_cast<long long>((N + 255) / 256) * BH;
  const bool one = (causal && window == 0) ? two < sm_count : 2 * two <= sm_count;
  return one ? 1 : 2;
}

// Current device must be compute capability 10.0; returns its ordinal in *dev.
int check_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  if (major != 10 || minor != 0) return FA2_ERR_ARCH;
  if (*dev < 0 || *dev >= kMaxDevices) return FA2_ERR_CUDA;
  return FA2_OK;
}

unsigned int* status_word(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status[dev]) {
    void* p = nullptr;
    if (cudaMalloc(&p, 256) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, 256) != cudaSuccess) return nullptr;
    g_status[dev] = static_cast<unsigned int*>(p);
  }
  return g_status[dev];
}

}  // namespace

namespace fa2 {

// [BH][N][d] 16-bit tensor viewed as a 3-D TMA map with box_rows x 64-column
// boxes and 128-byte swizzle; rows past N read as zeros.
bool make_tile_map(CUtensorMap* map, const void* base, int BH, int N, int d, bool bf16,
                   int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType ty =
      bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return enc(map, ty, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [BH][N][d] 8-bit tensor as a 3-D TMA map with 128-row x 128-column boxes and
// 128-byte swizzle; columns past d and rows past N read as zeros.
bool make_u8_map(CUtensorMap* map, const void* base, int BH, int N, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d),
                                 static_cast<cuuint64_t>(N) * d};
  const cuuint32_t box[3] = {128, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [BH][N][d] accumulator as a 3-D TMA map with 128-row x 32-column boxes
// and 128-byte swizzle, for tiled reduce-adds; rows past N are clipped.
bool make_acc_map(CUtensorMap* map, float* base, int BH, int N, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(N) * d * 4};
  const cuuint32_t box[3] = {32, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace fa2

namespace {

bool make_map(CUtensorMap* map, const void* base, int BH, int N, int d, int dtype,
              int box_rows = 128) {
  return fa2::make_tile_map(map, base, BH, N, d, dtype == FA2_BF16, box_rows);
}

unsigned long long wait_ns() { return static_cast<unsigned long long>(g_wait_ms.load()) * 1000000ull; }

template <int D, bool BF16, bool CAUSAL, int REP, bool F8 = false, bool ONE = false>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const CUtensorMap& mqr, const fa2::FwdParams& p, int n_split,
               cudaStream_t stream) {
  using Cfg = fa2::FwdCfg<D, F8, ONE>;
  auto kern = fa2::fa2_fwd_kernel<D, BF16, CAUSAL, REP, F8, ONE>;
  // The kernel re-splits its registers between warpgroups; that is only sound
  // when every thread was launched with exactly Cfg::LAUNCH_REGS registers.
  static const bool regs_ok = [&] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, kern) == cudaSuccess && fa.numRegs == Cfg::LAUNCH_REGS;
  }();
  if (!regs_ok) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  static std::atomic<bool> smem_set[fa2::kSmemFlagDevices];  // this instantiation's flags
  if (!fa2::set_smem_once(kern, Cfg::SMEM, smem_set)) return FA2_ERR_CUDA;
  const dim3 grid(static_cast<unsigned int>(p.n_qblk) * static_cast<unsigned int>(p.BH),
                  static_cast<unsigned int>(n_split));
  kern<<<grid, Cfg::THREADS, Cfg::SMEM, stream>>>(mq, mk, mv, mqr, p);
  if (cudaGetLastError() != cudaSuccess) return FA2_ERR_CUDA;
  g_launches.fetch_add(1);
  return FA2_OK;
}

// Instantiation of the forward for the runtime flags (one: one query tile per
// CTA at D <= 128, plain calls only).
template <int D>
int launch_fwd_any(bool bf, bool causal, int rep, bool one, const CUtensorMap& mq,
                   const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mqr,
                   const fa2::FwdParams& p, int n_split, cudaStream_t s) {
  if constexpr (D <= 128) {
    if (one) {
      if (rep != 1 || n_split != 1) return FA2_ERR_INVALID_ARG;
      if (bf) {
        return causal ? launch_fwd<D, true, true, 1, false, true>(mq, mk, mv, mqr, p, 1, s)
                      : launch_fwd<D, true, false, 1, false, true>(mq, mk, mv, mqr, p, 1, s);
      }
      return causal ? launch_fwd<D, false, true, 1, false, true>(mq, mk, mv, mqr, p, 1, s)
                    : launch_fwd<D, false, false, 1, false, true>(mq, mk, mv, mqr, p, 1, s);
    }
  }
#define FA2_FWD_REP(BF, CA)                                                        \
  switch (rep) {                                                                   \
    case 4: return launch_fwd<D, BF, CA, 4>(mq, mk, mv, mqr, p, n_split, s);       \
    case 2: return launch_fwd<D, BF, CA, 2>(mq, mk, mv, mqr, p, n_split, s);       \
    default: return launch_fwd<D, BF, CA, 1>(mq, mk, mv, mqr, p, n_split, s);      \
  }
  if (bf) {
    if (causal) { FA2_FWD_REP(true, true) }
    FA2_FWD_REP(true, false)
  }
  if (causal) { FA2_FWD_REP(false, true) }
  FA2_FWD_REP(false, false)
#undef FA2_FWD_REP
}

template <int D, bool BF16>
int launch_combine(const float* O_part, const float* LSE_part, void* O, float* LSE,
                   long long rows, int n_split, int d, cudaStream_t stream) {
  // Programmatic serialisation: the merge may launch while the forward runs and
  // waits on the device (griddepcontrol.wait) for it to finish.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned int>((rows + 7) / 8));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fa2::fa2_decode_combine_kernel<D, BF16>, O_part, LSE_part, O, LSE,
                         rows, n_split, d) != cudaSuccess) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  g_launches.fetch_add(1);
  return FA2_OK;
}

}  // namespace

namespace {

// Shared by every forward entry point.  Query rows [BH][Nq], key rows [BH][Nk];
// off = Nk - Nq aligns the causal mask to the bottom right; window = 0 means no
// sliding window.  The key tiles are cut into n_split stretches of kv_per_split
// and the queries replicated rep times (1, 2 or 4, rep > 1 only for
// Nq <= 128 / rep); with n_split x rep = 1 O and LSE are written directly,
// otherwise the n_split x rep partials go to O_part / LSE_part and a second
// kernel merges them into O and LSE.
int fwd_core(const void* Q, const void* K, const void* V, void* O, float* LSE, int BH, int Nq,
             int Nk, int d, float scale, int causal, int window, int dtype, int n_split,
             int kv_per_split, int rep, float* O_part, float* LSE_part, fa2_stream_t stream,
             bool one = false) {
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != FA2_OK) return rc;
  unsigned int* st = status_word(dev);
  if (!st) return FA2_ERR_CUDA;

  CUtensorMap mq, mk, mv, mqr;
  if (!make_map(&mq, Q, BH, Nq, d, dtype) || !make_map(&mk, K, BH, Nk, d, dtype) ||
      !make_map(&mv, V, BH, Nk, d, dtype))
    return FA2_ERR_CUDA;
  if (rep > 1) {
    if (!make_map(&mqr, Q, BH, Nq, d, dtype, 128 / rep)) return FA2_ERR_CUDA;
  } else {
    mqr = mq;  // not read
  }
  const int n_part = n_split * rep;
  // One CTA per (query block, batch*head) in x, one per key stretch in y.
  const int rows_per_cta = one ? 128 : fwd_rows_per_cta(d);
  const long long n_qblk = (Nq + rows_per_cta - 1) / rows_per_cta;
  if (n_qblk * BH > 0x7fffffffll || n_split > 65535) return FA2_ERR_INVALID_ARG;

  fa2::FwdParams p{};
  p.O = O;
  p.LSE = LSE;
  p.d = d;
  p.Nq = Nq;
  p.Nk = Nk;
  p.off = Nk - Nq;
  p.BH = BH;
  p.n_qblk = static_cast<int>(n_qblk);
  p.head_group = BH;
  if (n_split == 1 && window == 0) {
    // Heads per group of the block order: a group spans about two waves of CTAs
    // (one CTA per SM), so that the CTAs running together share a few heads.
    // Measured on B200: headline shape 2.135 -> 2.022 ms, long-context causal 9.15 ->
    // 8.77 ms, training shape 0.654 -> 0.648 ms; sliding windows (whose blocks read
    // only their window's keys) 0.397 -> 0.410 ms, so they keep the plain order.
    int dev_sm = 0;
    if (cudaDeviceGetAttribute(&dev_sm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        dev_sm > 0) {
      const long long hg = (2LL * dev_sm + n_qblk - 1) / n_qblk;
      p.head_group = static_cast<int>(std::min<long long>(BH, std::max<long long>(1, hg)));
    } else {
      cudaGetLastError();
    }
  }
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = st;
  p.wait_ns = wait_ns();
  p.fault = g_fault.load();
  p.window = window;
  p.kv_per_split = n_split > 1 ? kv_per_split : 0;
  p.O_part = n_part > 1 ? O_part : nullptr;
  p.LSE_part = n_part > 1 ? LSE_part : nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = dtype == FA2_BF16;
  const bool ca = causal != 0;
  switch (fwd_tile_dim(d)) {
    case 64: rc = launch_fwd_any<64>(bf, ca, rep, one, mq, mk, mv, mqr, p, n_split, s); break;
    case 128: rc = launch_fwd_any<128>(bf, ca, rep, one, mq, mk, mv, mqr, p, n_split, s); break;
    case 192: rc = launch_fwd_any<192>(bf, ca, rep, one, mq, mk, mv, mqr, p, n_split, s); break;
    default: rc = launch_fwd_any<256>(bf, ca, rep, one, mq, mk, mv, mqr, p, n_split, s); break;
  }
  if (rc != FA2_OK || n_part == 1) return rc;
  const long long rows = static_cast<long long>(BH) * Nq;
#define FA2_COMBINE(D_)                                                                   \
  return bf ? launch_combine<D_, true>(O_part, LSE_part, O, LSE, rows, n_part, d, s)      \
            : launch_combine<D_, false>(O_part, LSE_part, O, LSE, rows, n_part, d, s)
  switch (fwd_tile_dim(d)) {
    case 64: FA2_COMBINE(64);
    case 128: FA2_COMBINE(128);
    case 192: FA2_COMBINE(192);
    default: FA2_COMBINE(256);
  }
#undef FA2_COMBINE
}

// Shared by fa2_fwd and fa2_fwd_window; window = 0 means no sliding window.
int fwd_impl(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H,
             int N, int d, float scale, int causal, int window, int dtype, fa2_stream_t stream) {
  if (!Q || !K || !V || !O || !LSE) return FA2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
    return FA2_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, N, d, scale, causal, dtype);
  if (rc != FA2_OK) return rc;
  const int BH = B * H;
  const size_t bytes = static_cast<size_t>(BH) * N * d * 2;
  const size_t lse_bytes = static_cast<size_t>(BH) * N * sizeof(float);
  if (overlaps(O, bytes, Q, bytes) || overlaps(O, bytes, K, bytes) ||
      overlaps(O, bytes, V, bytes) || overlaps(LSE, lse_bytes, O, bytes) ||
      overlaps(LSE, lse_bytes, Q, bytes) || overlaps(LSE, lse_bytes, K, bytes) ||
      overlaps(LSE, lse_bytes, V, bytes))
    return FA2_ERR_INVALID_ARG;
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  const bool one = fwd_tile_dim(d) <= 128 && fwd_tiles_per_cta(BH, N, d, causal != 0, window, n_sm) == 1;
  return fwd_core(Q, K, V, O, LSE, BH, N, N, d, scale, causal, window, dtype, 1, 0, 1, nullptr,
                  nullptr, stream, one);
}

// Key tiles per split when the n_kv key tiles are cut into n_split stretches,
// and the number of non-empty stretches that gives.
int kv_tiles_per_split(int n_kv, int n_split) { return (n_kv + n_split - 1) / n_split; }
int effective_splits(int n_kv, int n_split) {
  const int per = kv_tiles_per_split(n_kv, n_split);
  return (n_kv + per - 1) / per;
}

constexpr int kMaxSplits = 1024;

// Query copies fa2_fwd_decode uses: 4 for up to 32 queries, 2 for up to 64.
int decode_rep(int Nq) { return Nq <= 32 ? 4 : (Nq <= 64 ? 2 : 1); }

// Checks of fa2_fwd_decode's sizes that need no CUDA call.
int check_decode_sizes(int B, int H, int Nq, int Nk, int d, float scale, int causal, int dtype) {
  if (Nq < 1 || Nk < Nq) return FA2_ERR_INVALID_ARG;
  return check_sizes(B, H, Nk, d, scale, causal, dtype);
}

}  // namespace

extern "C" {

int fa2_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H,
            int N, int d, float scale, int causal, int dtype, fa2_stream_t stream) {
  return fwd_impl(Q, K, V, O, LSE, B, H, N, d, scale, causal, 0, dtype, stream);
}

int fa2_fwd_window(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                   int H, int N, int d, float scale, int window, int dtype, fa2_stream_t stream) {
  if (window < 1) return FA2_ERR_INVALID_ARG;
  // A window as long as the sequence is plain causal attention.
  return fwd_impl(Q, K, V, O, LSE, B, H, N, d, scale, 1, window >= N ? 0 : window, dtype,
                  stream);
}

int fa2_fwd_tiles_per_cta(int B, int H, int N, int d, int causal, int window, int sm_count) {
  if (check_sizes(B, H, N, d, 1.0f, causal, FA2_BF16) != FA2_OK || window < 0) return 0;
  if (sm_count <= 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sm_count <= 0) {
      cudaGetLastError();
      return 0;
    }
  }
  // fa2_fwd_window treats a window as long as the sequence as plain causal.
  const int w = (causal && window > 0 && window < N) ? window : 0;
  return fwd_tiles_per_cta(static_cast<long long>(B) * H, N, d, causal != 0, w, sm_count);
}

int fa2_fwd_decode_splits(int B, int H, int Nq, int Nk, int d, int sm_count) {
  if (check_decode_sizes(B, H, Nq, Nk, d, 1.0f, 0, FA2_BF16) != FA2_OK) return 0;
  if (sm_count <= 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sm_count <= 0) {
      cudaGetLastError();
      return 0;
    }
  }
  // One forward CTA runs per SM (its TMEM allocation is the whole SM's).  As
  // many splits as still fit the CTAs in one wave, and at least 4 key tiles per
  // split: measured on B200, a second wave or shorter stretches cost more in
  // per-CTA set-up and the merge than they gain in parallelism.
  const long long ctas = static_cast<long long>((Nq + fwd_rows_per_cta(d) - 1) /
                                               fwd_rows_per_cta(d)) * B * H;
  const int n_kv = (Nq > 0) ? (Nk + 127) / 128 : 1;
  long long sp = sm_count / ctas;
  const long long cap = n_kv / 4;
  if (sp > cap) sp = cap;
  if (sp > kMaxSplits) sp = kMaxSplits;
  if (sp < 1) sp = 1;
  return static_cast<int>(sp);
}

size_t fa2_fwd_decode_workspace_size(int B, int H, int Nq, int Nk, int d, int n_splits) {
  if (check_decode_sizes(B, H, Nq, Nk, d, 1.0f, 0, FA2_BF16) != FA2_OK) return 0;
  if (n_splits < 1 || n_splits > kMaxSplits) return 0;
  const int parts = effective_splits((Nk + 127) / 128, n_splits) * decode_rep(Nq);
  if (parts == 1) return 0;
  return fa2::decode_workspace_bytes(static_cast<size_t>(parts), static_cast<size_t>(B) * H,
                                     static_cast<size_t>(Nq), fwd_tile_dim(d));
}

int fa2_fwd_decode(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                   int H, int Nq, int Nk, int d, float scale, int causal, int dtype, int n_splits,
                   void* workspace, size_t workspace_bytes, fa2_stream_t stream) {
  if (!Q || !K || !V || !O || !LSE) return FA2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
    return FA2_ERR_INVALID_ARG;
  int rc = check_decode_sizes(B, H, Nq, Nk, d, scale, causal, dtype);
  if (rc != FA2_OK) return rc;
  if (n_splits < 1 || n_splits > kMaxSplits) return FA2_ERR_INVALID_ARG;
  const int BH = B * H;
  const size_t q_bytes = static_cast<size_t>(BH) * Nq * d * 2;
  const size_t kv_bytes = static_cast<size_t>(BH) * Nk * d * 2;
  const size_t lse_bytes = static_cast<size_t>(BH) * Nq * sizeof(float);
  if (overlaps(O, q_bytes, Q, q_bytes) || overlaps(O, q_bytes, K, kv_bytes) ||
      overlaps(O, q_bytes, V, kv_bytes) || overlaps(LSE, lse_bytes, O, q_bytes) ||
      overlaps(LSE, lse_bytes, Q, q_bytes) || overlaps(LSE, lse_bytes, K, kv_bytes) ||
      overlaps(LSE, lse_bytes, V, kv_bytes))
    return FA2_ERR_INVALID_ARG;
  const int n_kv = (Nk + 127) / 128;
  const int eff = effective_splits(n_kv, n_splits);
  const int rep = decode_rep(Nq);
  const int parts = eff * rep;
  float* O_part = nullptr;
  float* LSE_part = nullptr;
  if (parts > 1) {
    const size_t need = fa2::decode_workspace_bytes(static_cast<size_t>(parts),
                                                    static_cast<size_t>(BH), Nq, fwd_tile_dim(d));
    if (!workspace || workspace_bytes < need ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return FA2_ERR_WORKSPACE;
    const void* bufs[5] = {Q, K, V, O, LSE};
    const size_t buf_bytes[5] = {q_bytes, kv_bytes, kv_bytes, q_bytes, lse_bytes};
    for (int i = 0; i < 5; ++i)
      if (overlaps(workspace, need, bufs[i], buf_bytes[i])) return FA2_ERR_WORKSPACE;
    O_part = static_cast<float*>(workspace);
    LSE_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                        fa2::decode_opart_bytes(static_cast<size_t>(parts),
                                                                static_cast<size_t>(BH), Nq,
                                                                fwd_tile_dim(d)));
  }
  return fwd_core(Q, K, V, O, LSE, BH, Nq, Nk, d, scale, causal, 0, dtype, eff,
                  kv_tiles_per_split(n_kv, n_splits), rep, O_part, LSE_part, stream);
}

int fa2_fwd_fp8(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H,
                int N, int d, float scale, int causal, float q_scale, float k_scale,
                float v_scale, fa2_stream_t stream) {
  if (!Q || !K || !V || !O || !LSE) return FA2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
    return FA2_ERR_INVALID_ARG;
  for (float f : {q_scale, k_scale, v_scale})
    if (!std::isfinite(f) || !(f > 0.f)) return FA2_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, N, 64, scale, causal, FA2_BF16);
  if (rc != FA2_OK) return rc;
  if (d < 16 || d > 128 || d % 16 != 0) return FA2_ERR_UNSUPPORTED;
  const float sl2 = scale * q_scale * k_scale * 1.4426950408889634f;
  if (!std::isfinite(sl2) || !(sl2 > 0.f)) return FA2_ERR_INVALID_ARG;
  const int BH = B * H;
  const size_t in_bytes = static_cast<size_t>(BH) * N * d;  // one byte per element
  const size_t o_bytes = in_bytes * 2;
  const size_t lse_bytes = static_cast<size_t>(BH) * N * sizeof(float);
  if (overlaps(O, o_bytes, Q, in_bytes) || overlaps(O, o_bytes, K, in_bytes) ||
      overlaps(O, o_bytes, V, in_bytes) || overlaps(LSE, lse_bytes, O, o_bytes) ||
      overlaps(LSE, lse_bytes, Q, in_bytes) || overlaps(LSE, lse_bytes, K, in_bytes) ||
      overlaps(LSE, lse_bytes, V, in_bytes))
    return FA2_ERR_INVALID_ARG;
  int dev = 0;
  rc = check_device(&dev);
  if (rc != FA2_OK) return rc;
  unsigned int* st = status_word(dev);
  if (!st) return FA2_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  if (!fa2::make_u8_map(&mq, Q, BH, N, d) || !fa2::make_u8_map(&mk, K, BH, N, d) ||
      !fa2::make_u8_map(&mv, V, BH, N, d))
    return FA2_ERR_CUDA;
  fa2::FwdParams p{};
  p.O = O;
  p.LSE = LSE;
  p.d = d;
  p.Nq = N;
  p.Nk = N;
  p.off = 0;
  p.BH = BH;
  if (static_cast<long long>((N + 255) / 256) * BH > 0x7fffffffll) return FA2_ERR_INVALID_ARG;
  p.n_qblk = (N + 255) / 256;
  p.head_group = BH;
  p.scale_log2 = sl2;
  p.status = st;
  p.wait_ns = wait_ns();
  p.fault = g_fault.load();
  p.window = 0;
  p.o_scale = v_scale;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return causal ? launch_fwd<128, true, true, 1, true>(mq, mk, mv, mq, p, 1, s)
                : launch_fwd<128, true, false, 1, true>(mq, mk, mv, mq, p, 1, s);
}

size_t fa2_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_sizes(B, H, N, d, 1.0f, 0, FA2_BF16, kMaxBwdHeadDim) != FA2_OK) return 0;
  return fa2::bwd_workspace_bytes(static_cast<size_t>(B) * H, N, d);
}

}  // extern "C"

namespace {

// Shared by fa2_bwd, fa2_bwd_window and fa2_bwd_ex; window = 0 means no sliding
// window.
int bwd_impl(const void* Q, const void* K, const void* V, const void* O, const void* dO,
             const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
             size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
             int window, int dtype, fa2_stream_t stream, bool deterministic = false) {
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return FA2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) ||
      !aligned16(LSE) || !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return FA2_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, N, d, scale, causal, dtype, kMaxBwdHeadDim);
  if (rc != FA2_OK) return rc;
  const int BH = B * H;
  const size_t bytes = static_cast<size_t>(BH) * N * d * 2;
  const size_t lse_bytes = static_cast<size_t>(BH) * N * sizeof(float);
  const void* ins[6] = {Q, K, V, O, dO, LSE};
  const size_t in_bytes[6] = {bytes, bytes, bytes, bytes, bytes, lse_bytes};
  void* outs[3] = {dQ, dK, dV};
  for (void* o : outs) {
    for (int i = 0; i < 6; ++i)
      if (overlaps(o, bytes, ins[i], in_bytes[i])) return FA2_ERR_INVALID_ARG;
  }
  if (overlaps(dQ, bytes, dK, bytes) || overlaps(dQ, bytes, dV, bytes) ||
      overlaps(dK, bytes, dV, bytes))
    return FA2_ERR_INVALID_ARG;
  const size_t need = fa2::bwd_workspace_bytes(static_cast<size_t>(BH), N, d, deterministic);
  if (!workspace || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FA2_ERR_WORKSPACE;
  int dev = 0;
  rc = check_device(&dev);
  if (rc != FA2_OK) return rc;
  unsigned int* st = status_word(dev);
  if (!st) return FA2_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  rc = fa2::launch_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, BH, N, d, scale, causal != 0,
                       dtype == FA2_BF16, st, wait_ns(), s, window, g_fault.load(),
                       g_bwd_ctas.load(), deterministic);
  if (rc == FA2_OK) g_launches.fetch_add(fa2::bwd_kernels_per_call(deterministic));
  return rc;
}

}  // namespace

extern "C" {

int fa2_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
            const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
            size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
            int dtype, fa2_stream_t stream) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes, B, H, N, d, scale,
                  causal, 0, dtype, stream);
}

int fa2_bwd_window(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                   const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
                   size_t workspace_bytes, int B, int H, int N, int d, float scale, int window,
                   int dtype, fa2_stream_t stream) {
  if (window < 1) return FA2_ERR_INVALID_ARG;
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes, B, H, N, d, scale,
                  1, window >= N ? 0 : window, dtype, stream);
}

size_t fa2_bwd_ex_workspace_size(int B, int H, int N, int d, int flags) {
  if ((flags & ~FA2_BWD_DETERMINISTIC) != 0) return 0;
  if (check_sizes(B, H, N, d, 1.0f, 0, FA2_BF16, kMaxBwdHeadDim) != FA2_OK) return 0;
  return fa2::bwd_workspace_bytes(static_cast<size_t>(B) * H, N, d,
                                  (flags & FA2_BWD_DETERMINISTIC) != 0);
}

int fa2_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* dO,
               const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
               size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
               int window, int flags, int dtype, fa2_stream_t stream) {
  if ((flags & ~FA2_BWD_DETERMINISTIC) != 0) return FA2_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && causal != 1)) return FA2_ERR_INVALID_ARG;
  // A window as long as the sequence is plain causal attention.
  const int w = (window > 0 && window < N) ? window : 0;
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes, B, H, N, d, scale,
                  causal, w, dtype, stream, (flags & FA2_BWD_DETERMINISTIC) != 0);
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// Allocation-free backward.
//
// Some callers cannot call cudaMalloc: runtimes that hand out device memory only
// from their own fixed pool, and latency-critical code that must not take the
// device-wide synchronisation an allocation can cause.  They cannot provide the
// workspace fa2_bwd asks for, so fa2_bwd_noalloc uses this file-scope buffer
// instead.  Every GPU that loads the library holds it until the process exits.
// ------------------------------------------------------------------------------------

namespace {

constexpr size_t kNoAllocBytes = static_cast<size_t>(32) << 20;  // 32 MiB
constexpr size_t kNoAllocStatusBytes = 256;  // the buffer's own status word, then the scratch

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch, per device.  In host code the symbol's
// name is only a host-side stand-in; the device address comes from
// cudaGetSymbolAddress, called with that device current.
void* g_noalloc_base[kMaxDevices] = {};

void* noalloc_base(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_noalloc_base[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_base[dev] = p;
  }
  return g_noalloc_base[dev];
}

// The status word in the buffer (its first 256 bytes), or null before the first
// fa2_bwd_noalloc call on the device.
unsigned int* noalloc_status_word(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  return static_cast<unsigned int*>(g_noalloc_base[dev]);
}

}  // namespace

extern "C" {

int fa2_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                    const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d,
                    float scale, int causal, int dtype, fa2_stream_t stream) {
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return FA2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) ||
      !aligned16(LSE) || !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return FA2_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, N, d, scale, causal, dtype, kMaxBwdHeadDim);
  if (rc != FA2_OK) return rc;
  const int BH = B * H;
  const size_t bytes = static_cast<size_t>(BH) * N * d * 2;
  const size_t lse_bytes = static_cast<size_t>(BH) * N * sizeof(float);
  const void* ins[6] = {Q, K, V, O, dO, LSE};
  const size_t in_bytes[6] = {bytes, bytes, bytes, bytes, bytes, lse_bytes};
  void* outs[3] = {dQ, dK, dV};
  for (void* o : outs) {
    for (int i = 0; i < 6; ++i)
      if (overlaps(o, bytes, ins[i], in_bytes[i])) return FA2_ERR_INVALID_ARG;
  }
  if (overlaps(dQ, bytes, dK, bytes) || overlaps(dQ, bytes, dV, bytes) ||
      overlaps(dK, bytes, dV, bytes))
    return FA2_ERR_INVALID_ARG;
  const size_t need = fa2::bwd_workspace_bytes(static_cast<size_t>(BH), N, d);
  if (need > kNoAllocBytes - kNoAllocStatusBytes) return FA2_ERR_WORKSPACE;
  int dev = 0;
  rc = check_device(&dev);
  if (rc != FA2_OK) return rc;
  uint8_t* base = static_cast<uint8_t*>(noalloc_base(dev));  // first call on a device: set-up
  if (!base) return FA2_ERR_CUDA;
  // Timeouts go to the word at the start of the buffer, which
  // fa2_get_device_status reads and clears along with the library's own word.
  unsigned int* st = reinterpret_cast<unsigned int*>(base);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  rc = fa2::launch_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, base + kNoAllocStatusBytes, BH, N, d,
                       scale, causal != 0, dtype == FA2_BF16, st, wait_ns(), s, 0, g_fault.load(),
                       g_bwd_ctas.load());
  if (rc == FA2_OK) g_launches.fetch_add(fa2::bwd_kernels_per_call(false));
  return rc;
}

int fa2_get_device_status(fa2_stream_t stream, int* site) {
  if (site) *site = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA2_ERR_CUDA;
  // Two words may exist: the one the calls with caller-provided memory write (created
  // by the first of them) and the one in fa2_bwd_noalloc's buffer.  Both are read and
  // cleared; nothing is allocated here, so a word that does not exist yet has had no
  // kernel to write it.  The first failure recorded (the library's word first) is
  // the one returned.
  unsigned int* words[2] = {nullptr, nullptr};
  {
    std::lock_guard<std::mutex> lock(g_mu);
    words[0] = g_status[dev];
  }
  words[1] = noalloc_status_word(dev);
  unsigned int first = 0;
  for (unsigned int* st : words) {
    if (!st) continue;
    unsigned int w = 0;
    if (cudaMemcpy(&w, st, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return FA2_ERR_CUDA;
    if (w != 0 && cudaMemset(st, 0, sizeof(w)) != cudaSuccess) return FA2_ERR_CUDA;
    if (first == 0) first = w;
  }
  if (site) *site = static_cast<int>((first >> 8) & 0xFFu);
  const unsigned int code = first & 0xFFu;
  return code == 0 ? FA2_OK : static_cast<int>(code);
}

const char* fa2_status_string(int status) {
  switch (status) {
    case FA2_OK: return "FA2_OK";
    case FA2_ERR_INVALID_ARG: return "FA2_ERR_INVALID_ARG";
    case FA2_ERR_UNSUPPORTED: return "FA2_ERR_UNSUPPORTED";
    case FA2_ERR_ARCH: return "FA2_ERR_ARCH";
    case FA2_ERR_CUDA: return "FA2_ERR_CUDA";
    case FA2_ERR_TIMEOUT: return "FA2_ERR_TIMEOUT";
    case FA2_ERR_WORKSPACE: return "FA2_ERR_WORKSPACE";
    default: return "FA2_ERR_UNKNOWN";
  }
}

void fa2_debug_set(int fault, unsigned int wait_limit_ms) {
  g_fault.store(fault == 1 ? 1 : 0);
  g_wait_ms.store(wait_limit_ms == 0 ? kDefaultWaitMs : wait_limit_ms);
}

void fa2_debug_set_bwd_grid(int max_ctas) { g_bwd_ctas.store(max_ctas > 0 ? max_ctas : 0); }

void fa2_debug_set_fwd_tiles(int tiles) { g_fwd_tiles.store(tiles == 1 || tiles == 2 ? tiles : 0); }

unsigned long long fa2_launch_count(void) { return g_launches.load(); }

}  // extern "C"
