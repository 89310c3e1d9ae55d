// K0: parent indices -> stacked bit-planes (PagedWeight, "Composants Clés" 1: weights as
// superposed bit-planes).  Plane p holds bit (n-1-p) of every index; column 32w+j of a row is
// bit j of word w.  One warp builds the n words of a 32-column group with one ballot per plane.
#pragma once
#include "pw_common.cuh"

namespace pw {

__global__ void __launch_bounds__(256) pack_bitplanes_kernel(const uint8_t* __restrict__ idx,
                                                             int rows, int cols, int n,
                                                             uint32_t* __restrict__ planes) {
  const int lane = threadIdx.x & 31;
  const long long words_per_row = cols >> 5;
  const long long total_words = static_cast<long long>(rows) * words_per_row;
  const long long plane_stride = total_words;
  const long long warp0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long w = warp0; w < total_words; w += nwarps) {
    const long long r = w / words_per_row;
    const long long c = (w - r * words_per_row) * 32 + lane;
    const uint32_t v = idx[r * cols + c];
    for (int p = 0; p < n; ++p) {
      const uint32_t word = __ballot_sync(0xffffffffu, (v >> (n - 1 - p)) & 1u);
      if (lane == 0) planes[p * plane_stride + w] = word;
    }
  }
}

}  // namespace pw
