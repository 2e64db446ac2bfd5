// Backward pass (placeholder launcher while the kernels are written).
#pragma once
#include "ptx.cuh"
namespace fa2 {
constexpr int kBwdKernelsPerCall = 3;
inline size_t bwd_workspace_bytes(size_t BH, int N, int d) {
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  size_t b = 2 * BH * npad * 4;
  b = (b + 255) / 256 * 256;
  b += BH * static_cast<size_t>(N) * d * 4;
  return (b + 255) / 256 * 256;
}
inline int launch_bwd(const void*, const void*, const void*, const void*, const void*, const float*,
                      void*, void*, void*, void*, int, int, int, float, bool, bool, unsigned int*,
                      unsigned long long, cudaStream_t) {
  return 2;
}
}  // namespace fa2
