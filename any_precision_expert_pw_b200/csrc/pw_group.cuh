// K2: token -> expert grouping and activation staging for the grouped FFN.
// Assignment a = t*k + slot.  Within an expert the assignments are kept in ascending a (the
// set of experts to load grows with the batch -- LYNX, 1 "Énoncé du Problème").
#pragma once
#include "pw_common.cuh"
#include "pw_ffn.cuh"

namespace pw {

constexpr int kGroupThreads = 1024;
constexpr int kMaxAssign = 8192;  // T * k handled by the single-CTA grouping step

// counts[E], offsets[E+1], perm[T*k] (grouped position -> assignment), inv[T*k] (assignment ->
// grouped position, -1 for an invalid expert id), active[E] (experts with work, ascending),
// meta[0] = number of active experts, meta[1] = number of valid assignments.
__global__ void __launch_bounds__(kGroupThreads) group_kernel(const int32_t* __restrict__ idx,
                                                              int TK, int E,
                                                              int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ offsets,
                                                              int32_t* __restrict__ perm,
                                                              int32_t* __restrict__ inv,
                                                              int32_t* __restrict__ active,
                                                              int32_t* __restrict__ meta) {
  __shared__ int cnt[PW_MAX_EXPERTS];
  __shared__ int off[PW_MAX_EXPERTS + 1];
  __shared__ int act_pos[PW_MAX_EXPERTS + 1];
  __shared__ int16_t eid[kMaxAssign];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int a = tid; a < TK; a += blockDim.x) {
    int e = idx[a];
    if (e < 0 || e >= E) {
      set_status(PW_ERR_BAD_EXPERT);
      e = -1;
    } else {
      atomicAdd(&cnt[e], 1);
    }
    eid[a] = static_cast<int16_t>(e);
  }
  __syncthreads();
  if (tid == 0) {  // E <= 1024: a serial scan is a few hundred cycles
    int o = 0, na = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = o;
      act_pos[e] = na;
      o += cnt[e];
      na += (cnt[e] > 0);
    }
    off[E] = o;
    act_pos[E] = na;
    meta[0] = na;
    meta[1] = o;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    counts[e] = cnt[e];
    offsets[e] = off[e];
    if (cnt[e] > 0) active[act_pos[e]] = e;
  }
  if (tid == 0) offsets[E] = off[E];
  for (int a = tid; a < TK; a += blockDim.x) {
    const int e = eid[a];
    if (e < 0) {
      inv[a] = -1;
      continue;
    }
    int r = 0;
    for (int b = 0; b < a; ++b) r += (eid[b] == e);
    const int pos = off[e] + r;
    perm[pos] = a;
    inv[a] = pos;
  }
}

// X[pos][xslot(c)] = x[token(pos)][c] as fp32 for c < H and 0 for H <= c < ldx;
// Hbuf[pos][c] = 0 for I <= c < ldh.  The FFN streams whole 1024-column stages, so the padding
// must read as zero, and it reads activations in its decode order (xslot, a permutation inside
// each 32-column group that keeps padding groups whole).
__global__ void prep_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
                            const int32_t* __restrict__ meta, int k, int H, int ldx,
                            float* __restrict__ X, int I, int ldh, float* __restrict__ Hbuf) {
  const int n_valid = meta[1];
  const int pos = blockIdx.y;
  if (pos >= n_valid) return;
  const int t = perm[pos] / k;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < ldx; c += gridDim.x * blockDim.x) {
    X[static_cast<size_t>(pos) * ldx + k4::xslot(c)] =
        (c < H) ? bf16_to_f32(x[static_cast<size_t>(t) * H + c]) : 0.0f;
  }
  for (int c = I + blockIdx.x * blockDim.x + threadIdx.x; c < ldh; c += gridDim.x * blockDim.x)
    Hbuf[static_cast<size_t>(pos) * ldh + c] = 0.0f;
}

// y[t][r] = sum over slots (in slot order) of gate[t][s] * o[t, s][r], where o is the sum of
// the down projection's k-slice partials (in slice order).  fp32.
__global__ void combine_kernel(const float* __restrict__ O, const int32_t* __restrict__ inv,
                               const float* __restrict__ gate, const int32_t* __restrict__ meta,
                               int T, int k, int H, int kslices, long long slice,
                               float* __restrict__ y) {
  const int t = blockIdx.y;
  const bool bad = meta[2] != 0;
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < H; r += gridDim.x * blockDim.x) {
    float acc = 0.0f;
    for (int s = 0; s < k; ++s) {
      const int pos = inv[t * k + s];
      if (pos < 0 || bad) continue;
      float o = 0.0f;
      for (int j = 0; j < kslices; ++j) o += O[j * slice + static_cast<size_t>(pos) * H + r];
      acc = fmaf(gate[t * k + s], o, acc);
    }
    y[static_cast<size_t>(t) * H + r] = acc;
  }
}

}  // namespace pw
