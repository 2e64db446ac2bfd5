// Decode-like forward: a few query rows against a long key/value sequence.
//
// Source (page title, section): "Flash Attention spiegata: una guida completa"
// (datacamp), "Parallelismo lungo la lunghezza della sequenza": with small
// batches and long sequences the batch x heads grid alone leaves most of the GPU
// idle, so the work is also split along the sequence.  With few query rows the
// only long dimension left is the keys, so they are split: every CTA of the
// forward kernel takes one stretch of key tiles and writes its rows' partial
// results (output normalised by its own row sum, and its own log-sum-exp); this
// file merges them.  For one row with partials (O_s, L_s), s = 1..S:
//
//     M = max_s L_s,   w_s = exp(L_s - M),   O = sum_s w_s O_s / sum_s w_s,
//     LSE = M + ln sum_s w_s,
//
// which is the same rescaling the online softmax applies tile by tile, taken
// across splits instead of across tiles (each O_s already carries its 1/l_s and
// exp(L_s) = e^{m_s} l_s).  A split in which the row sees no key has L_s = -inf
// and drops out.
#pragma once

#include <cstddef>
#include <cstdint>

#include "ptx.cuh"

namespace fa2 {

// Bytes of the partial buffers for S splits: O_part float [S][BH][Nq][D], then
// LSE_part float [S][BH][Nq] at the next 256-byte boundary.
inline size_t decode_opart_bytes(size_t S, size_t BH, size_t Nq, int D) {
  return (S * BH * Nq * static_cast<size_t>(D) * 4 + 255) / 256 * 256;
}
inline size_t decode_workspace_bytes(size_t S, size_t BH, size_t Nq, int D) {
  return decode_opart_bytes(S, BH, Nq, D) + (S * BH * Nq * 4 + 255) / 256 * 256;
}

// One warp per output row (bh, i); lane c owns D/32 consecutive columns of the
// D-column partials and writes those below the head dim d (a multiple of 8).
// Launched behind the forward with programmatic serialisation: it may start
// while the forward still runs and waits for it before touching the partials.
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
fa2_decode_combine_kernel(const float* __restrict__ O_part, const float* __restrict__ LSE_part,
                          void* __restrict__ O, float* __restrict__ LSE, long long rows,
                          int n_split, int d) {
  constexpr int PER = D / 32;  // columns per lane: 2, 4, 6 or 8
  constexpr int U = 8;         // partial rows in flight per lane
  griddep_wait();
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;  // whole warp leaves together
  constexpr float kLog2e = 1.4426950408889634f;

  float M = -INFINITY;
  for (int s = lane; s < n_split; s += 32) M = fmaxf(M, LSE_part[s * rows + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));

  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (M != -INFINITY) {
    for (int s0 = 0; s0 < n_split; s0 += 32) {
      // Lane c weighs split s0 + c; the weights are then broadcast, and U
      // partial rows are loaded before any is used.  A split the row sees no
      // key of has weight 0 and its (unwritten) partial row is not read.
      const int s = s0 + lane;
      const float L = (s < n_split) ? LSE_part[s * rows + row] : -INFINITY;
      const float w = (L == -INFINITY) ? 0.f : exp2f((L - M) * kLog2e);
      wsum += w;
      const int cnt = min(32, n_split - s0);
      for (int c0 = 0; c0 < cnt; c0 += U) {
        float wc[U], v[U][PER];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = c0 + u;
          wc[u] = __shfl_sync(0xffffffffu, w, c & 31);
          if (c >= cnt) wc[u] = 0.f;
#pragma unroll
          for (int i = 0; i < PER; ++i) v[u][i] = 0.f;
          if (wc[u] != 0.f) {  // warp-uniform
            const float* src = O_part + ((s0 + c) * rows + row) * D + lane * PER;
#pragma unroll
            for (int i = 0; i < PER / 2; ++i) {  // 8-byte aligned pairs
              const float2 t = reinterpret_cast<const float2*>(src)[i];
              v[u][2 * i] = t.x;
              v[u][2 * i + 1] = t.y;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int i = 0; i < PER; ++i) acc[i] = fmaf(wc[u], v[u][i], acc[i]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  }
  const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
  uint32_t packed[PER / 2];
#pragma unroll
  for (int i = 0; i < PER / 2; ++i) packed[i] = pack2<BF16>(acc[2 * i] * inv, acc[2 * i + 1] * inv);
  uint32_t* dst = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(O) + (row * d + lane * PER) * 2);
#pragma unroll
  for (int i = 0; i < PER / 2; ++i)
    if (lane * PER + 2 * i < d) dst[i] = packed[i];  // d is even: whole pairs
  if (lane == 0) LSE[row] = (wsum > 0.f) ? M + logf(wsum) : -INFINITY;
}

}  // namespace fa2
