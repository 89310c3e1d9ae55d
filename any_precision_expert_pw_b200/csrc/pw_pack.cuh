// K0: parent indices -> stacked bit-planes (PagedWeight, "Composants Clés" 1: weights as
// superposed bit-planes).  Plane p holds bit (n-1-p) of every index; column 32w+j of a row is
// bit j of word w.  One warp builds the n words of a 32-column group with one ballot per plane
// and stores them in the requested layout (PW_LAYOUT_ROWS, or the FFN's tiled layouts, where
// the top planes of a 32-row tile and a 512-column stage are one contiguous run).
#pragma once
#include "pw_common.cuh"

namespace pw {

// uint32 index of word w of plane p, block row r, in a tiled layout (see pw_block in pw.h).
__host__ __device__ __forceinline__ long long tiled_index(int layout, int rows, int cols, int n,
                                                          int r, int w, int p) {
  int t, i;
  if (layout == PW_LAYOUT_TILED_GATE_UP) {
    const int half = rows >> 1;
    const bool up = r >= half;
    const int rr = up ? r - half : r;
    t = rr >> 4;
    i = (rr & 15) + (up ? 16 : 0);
  } else {
    t = r >> 5;
    i = r & 31;
  }
  return tiled_word(t, w / kTileStageWords, p, w % kTileStageWords, i, n, cols >> 5);
}

__global__ void __launch_bounds__(256) pack_bitplanes_kernel(const uint8_t* __restrict__ idx,
                                                             int rows, int cols, int n,
                                                             int layout,
                                                             uint32_t* __restrict__ planes) {
  const int lane = threadIdx.x & 31;
  const long long words_per_row = cols >> 5;
  const long long total_words = static_cast<long long>(rows) * words_per_row;
  const long long plane_stride = total_words;
  const long long warp0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long w = warp0; w < total_words; w += nwarps) {
    const long long r = w / words_per_row;
    const long long wc = w - r * words_per_row;
    const uint32_t v = idx[r * cols + wc * 32 + lane];
    for (int p = 0; p < n; ++p) {
      const uint32_t word = __ballot_sync(0xffffffffu, (v >> (n - 1 - p)) & 1u);
      if (lane == 0) {
        const long long o = layout == PW_LAYOUT_ROWS
                                ? p * plane_stride + w
                                : tiled_index(layout, rows, cols, n, static_cast<int>(r),
                                              static_cast<int>(wc), p);
        planes[o] = word;
      }
    }
  }
}

}  // namespace pw
