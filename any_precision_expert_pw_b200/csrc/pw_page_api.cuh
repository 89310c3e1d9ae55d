// Host side of page movement and bitwidth planning (pw_page_copy, pw_plan_bitwidths,
// pw_page_update; PagedWeight, "Composants Clés" 1 to 3).  Included once, by pw_lib.cu, after
// its launch helpers: the library is one translation unit so that every kernel shares one
// device status word.
#pragma once

extern "C" {

pw_status pw_page_copy(const uint32_t* src, int src_bits, uint32_t* dst, int dst_bits, int rows,
                       int cols, int q, pw_stream_t stream) {
  if (!src || !dst || rows <= 0 || cols <= 0 || rows % 32 || cols % 128) return PW_ERR_INVALID_ARG;
  if (src_bits < 1 || src_bits > PW_MAX_BITS || dst_bits < 1 || dst_bits > PW_MAX_BITS)
    return PW_ERR_INVALID_ARG;
  if (q < 1 || q > src_bits || q > dst_bits) return PW_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(src) % 16 || reinterpret_cast<uintptr_t>(dst) % 16)
    return PW_ERR_INVALID_ARG;
  // one pitched copy per stage index s: the runs (t, s) of every tile t are evenly spaced by
  // the tile stride in both buffers; each copies its first q planes
  const size_t W = static_cast<size_t>(cols) / 32, tiles = static_cast<size_t>(rows) / 32;
  const size_t src_tile = static_cast<size_t>(src_bits) * 32 * W * 4;
  const size_t dst_tile = static_cast<size_t>(dst_bits) * 32 * W * 4;
  const size_t SW = pw::kTileStageWords;
  const size_t nst = (W + SW - 1) / SW;
  for (size_t s = 0; s < nst; ++s) {
    const size_t ws = std::min<size_t>(SW, W - SW * s);
    const size_t width = static_cast<size_t>(q) * 32 * ws * 4;
    const uint8_t* sp = reinterpret_cast<const uint8_t*>(src) + s * src_bits * 32 * SW * 4;
    uint8_t* dp = reinterpret_cast<uint8_t*>(dst) + s * dst_bits * 32 * SW * 4;
    if (cudaMemcpy2DAsync(dp, dst_tile, sp, src_tile, width, tiles, cudaMemcpyDefault,
                          as_cuda(stream)) != cudaSuccess)
      return PW_ERR_CUDA;
  }
  return PW_OK;
}

pw_status pw_plan_bitwidths(int nblocks, const double* damage, const uint64_t* bytes,
                            const uint8_t* qmin, const uint8_t* qmax, uint64_t budget,
                            uint8_t* q_out) {
  if (nblocks < 1 || !damage || !bytes || !qmin || !qmax || !q_out) return PW_ERR_INVALID_ARG;
  constexpr int kQ = PW_MAX_BITS + 1;
  uint64_t total = 0;
  for (int i = 0; i < nblocks; ++i) {
    if (qmin[i] < 1 || qmax[i] > PW_MAX_BITS || qmin[i] > qmax[i]) return PW_ERR_INVALID_ARG;
    q_out[i] = qmax[i];
    total += bytes[static_cast<size_t>(i) * kQ + qmax[i]];
  }
  // marginal cost of lowering block i from q to q - 1: damage added per byte saved
  struct Step {
    double ratio;
    int block;
  };
  auto worse = [](const Step& a, const Step& b) {  // heap top = smallest ratio, lowest block
    return a.ratio > b.ratio || (a.ratio == b.ratio && a.block > b.block);
  };
  auto step_of = [&](int i) {
    const int q = q_out[i];
    const double dd = damage[static_cast<size_t>(i) * kQ + q - 1] -
                      damage[static_cast<size_t>(i) * kQ + q];
    const uint64_t hi = bytes[static_cast<size_t>(i) * kQ + q];
    const uint64_t lo = bytes[static_cast<size_t>(i) * kQ + q - 1];
    const double db = hi > lo ? static_cast<double>(hi - lo) : 0.0;
    return Step{db > 0.0 ? dd / db : INFINITY, i};
  };
  std::priority_queue<Step, std::vector<Step>, decltype(worse)> heap(worse);
  for (int i = 0; i < nblocks; ++i)
    if (q_out[i] > qmin[i]) heap.push(step_of(i));
  while (total > budget && !heap.empty()) {
    const Step st = heap.top();
    heap.pop();
    const int i = st.block, q = q_out[i];
    total -= bytes[static_cast<size_t>(i) * kQ + q] - bytes[static_cast<size_t>(i) * kQ + q - 1];
    q_out[i] = static_cast<uint8_t>(q - 1);
    if (q_out[i] > qmin[i]) heap.push(step_of(i));
  }
  return total <= budget ? PW_OK : PW_ERR_UNSUPPORTED;
}

pw_status pw_page_update(pw_page_table* pt_dev, int num_blocks, const pw_page_update_t* updates,
                         int count, pw_stream_t stream) {
  if (!pt_dev || !updates || count < 0 || num_blocks < 1) return PW_ERR_INVALID_ARG;
  if (count == 0) return PW_OK;
  pw::page_update_kernel<<<(count + 255) / 256, 256, 0, as_cuda(stream)>>>(pt_dev, num_blocks,
                                                                           updates, count);
  return launch_status();
}

pw_status pw_pack_bitplanes(const uint8_t* idx, int rows, int cols, int n, int layout,
                            uint32_t* planes, pw_stream_t stream) {
  if (!idx || !planes || rows <= 0 || cols <= 0 || cols % 32 || n < 1 || n > 8)
    return PW_ERR_INVALID_ARG;
  if (layout != PW_LAYOUT_ROWS && layout != PW_LAYOUT_TILED_GATE_UP &&
      layout != PW_LAYOUT_TILED_DOWN)
    return PW_ERR_INVALID_ARG;
  if (layout != PW_LAYOUT_ROWS && (rows % 32 || cols % 128)) return PW_ERR_INVALID_ARG;
  const long long words = static_cast<long long>(rows) * (cols / 32);
  const long long blocks = (words + 7) / 8;
  const int grid = static_cast<int>(blocks < 65535LL * 16 ? blocks : 65535LL * 16);
  pw::pack_bitplanes_kernel<<<grid, 256, 0, as_cuda(stream)>>>(idx, rows, cols, n, layout,
                                                                planes);
  return launch_status();
}

}  // extern "C"
