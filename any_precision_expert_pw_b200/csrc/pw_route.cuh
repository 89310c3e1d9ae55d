// K1 router GEMV + softmax top-k, K3a substitution, K3b remap.
//
// Routing (LYNX, 1 "Énoncé du Problème"): each token picks its k best experts.  The logits are
// accumulated in float64 (every bf16 x fp32 product is exact there) and rounded once to fp32,
// so the selection -- taken on the fp32 logits, ties to the lower index -- and the softmax
// (float64 over all experts, rounded once) are reproducible.
// Substitution ("Which Expert Misses Are Worth Waiting For?", "Méthodologie") and remap
// (LYNX, 2.1 and 2.2) rewrite the assignments in rank order, one warp per token.
#pragma once
#include "pw_common.cuh"

namespace pw {

constexpr int kRouteExpertsPerCta = 8;   // one warp per expert

__device__ __forceinline__ double bf16lo(uint32_t v) {
  return static_cast<double>(__uint_as_float(v << 16));
}
__device__ __forceinline__ double bf16hi(uint32_t v) {
  return static_cast<double>(__uint_as_float(v & 0xffff0000u));
}

// logits[t][e] = fp32(sum_h x[t][h] * Wr[e][h] + bias[e]) with a float64 accumulator.
// Warp = expert; CTA = 8 experts x TT tokens; each lane takes 8 consecutive h per 256-wide chunk
// (16-byte loads when `vec`), so the router weights are read once per token tile.
template <int TT>
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const float* __restrict__ Wr,
                                                            const float* __restrict__ bias,
                                                            int T, int H, int E, int vec,
                                                            float* __restrict__ logits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kRouteExpertsPerCta + warp;
  if (e >= E) return;
  const int t0 = blockIdx.y * TT;
  const int nt = min(TT, T - t0);
  const float* w = Wr + static_cast<size_t>(e) * H;
  double acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.0;
  int hs = 0;
  if (vec) {
    const int hv = (H / 256) * 256;
#pragma unroll 2
    for (int h0 = lane * 8; h0 < hv; h0 += 256) {
      const float4 wa = __ldg(reinterpret_cast<const float4*>(w + h0));
      const float4 wb = __ldg(reinterpret_cast<const float4*>(w + h0 + 4));
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        if (t < nt) {
          const uint4 xv =
              __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0 + t) * H + h0));
          double a = acc[t];
          a = fma(bf16lo(xv.x), static_cast<double>(wa.x), a);
          a = fma(bf16hi(xv.x), static_cast<double>(wa.y), a);
          a = fma(bf16lo(xv.y), static_cast<double>(wa.z), a);
          a = fma(bf16hi(xv.y), static_cast<double>(wa.w), a);
          a = fma(bf16lo(xv.z), static_cast<double>(wb.x), a);
          a = fma(bf16hi(xv.z), static_cast<double>(wb.y), a);
          a = fma(bf16lo(xv.w), static_cast<double>(wb.z), a);
          a = fma(bf16hi(xv.w), static_cast<double>(wb.w), a);
          acc[t] = a;
        }
      }
    }
    hs = hv;
  }
  for (int h = hs + lane; h < H; h += 32) {
    const double wv = static_cast<double>(w[h]);
#pragma unroll
    for (int t = 0; t < TT; ++t)
      if (t < nt) acc[t] = fma(static_cast<double>(bf16_to_f32(x[static_cast<size_t>(t0 + t) * H + h])), wv, acc[t]);
  }
  const double b = bias ? static_cast<double>(bias[e]) : 0.0;
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    const double v = warp_sum_f64(acc[t]);
    if (lane == 0 && t < nt) logits[static_cast<size_t>(t0 + t) * E + e] = static_cast<float>(v + b);
  }
}

constexpr int kMaxPerLane = PW_MAX_EXPERTS / 32;

// One warp per token: top-k by (logit desc, index asc), softmax over all E in float64.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E,
                                                   int k, int renorm, int32_t* __restrict__ idx,
                                                   float* __restrict__ gate) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* l = logits + static_cast<size_t>(t) * E;
  float v[kMaxPerLane];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? l[e] : -INFINITY;
    mx = fmaxf(mx, v[i]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  double z = 0.0;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i)
    if (lane + 32 * i < E) z += exp(static_cast<double>(v[i]) - static_cast<double>(mx));
  z = warp_sum_f64(z);

  uint32_t taken = 0;  // bit i: element lane+32i already chosen
  double psel[PW_MAX_TOPK];
  int esel[PW_MAX_TOPK];
  double psum = 0.0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (bi < 0 || v[i] > bv)) {
        bv = v[i];
        bi = e;
      }
    }
    warp_argmax(bv, bi);
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    const double p = exp(static_cast<double>(bv) - static_cast<double>(mx)) / z;
    psel[j] = p;
    esel[j] = bi;
    psum += p;
  }
  if (lane == 0) {
    for (int j = 0; j < k; ++j) {
      idx[static_cast<size_t>(t) * k + j] = esel[j];
      gate[static_cast<size_t>(t) * k + j] =
          static_cast<float>(renorm ? psel[j] / psum : psel[j]);
    }
  }
}

// Highest-logit expert e with allowed[e] and e not in cur[0..k) (ties: lower index); -1 if none.
__device__ __forceinline__ int best_candidate(const float* __restrict__ l, const uint8_t* allowed,
                                              int E, const int* cur, int k) {
  const int lane = threadIdx.x & 31;
  float bv = -INFINITY;
  int bi = -1;
  for (int e = lane; e < E; e += 32) {
    if (!allowed[e]) continue;
    bool in_set = false;
    for (int j = 0; j < k; ++j) in_set |= (cur[j] == e);
    if (in_set) continue;
    const float le = l[e];
    if (bi < 0 || le > bv) {
      bv = le;
      bi = e;
    }
  }
  warp_argmax(bv, bi);
  return bi;
}

__global__ void __launch_bounds__(256) substitute_kernel(
    const float* __restrict__ logits, int32_t* __restrict__ idx, const float* __restrict__ gate,
    const uint8_t* __restrict__ resident, int T, int E, int k, int policy, float threshold,
    uint8_t* __restrict__ action, float* __restrict__ mass) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int cur[PW_MAX_TOPK];
  bool bad = false;
  for (int j = 0; j < k; ++j) {
    cur[j] = idx[static_cast<size_t>(t) * k + j];
    bad |= (cur[j] < 0 || cur[j] >= E);
  }
  if (bad) {  // ids out of range: leave the token untouched
    if (lane == 0) set_status(PW_ERR_BAD_EXPERT);
    return;
  }
  const float* l = logits + static_cast<size_t>(t) * E;
  double sub = 0.0, tot = 0.0;
  uint8_t act[PW_MAX_TOPK];
  for (int s = 0; s < k; ++s) {
    const float g = gate[static_cast<size_t>(t) * k + s];
    tot += static_cast<double>(g);
    if (resident[cur[s]]) {
      act[s] = PW_ACT_HIT;
      continue;
    }
    bool fetch;
    if (policy == PW_POLICY_FETCH_ALL) fetch = true;
    else if (policy == PW_POLICY_FIRST_CHOICE) fetch = (s == 0);
    else fetch = (s == 0) || (g >= threshold);
    act[s] = PW_ACT_FETCH;
    if (!fetch) {
      const int c = best_candidate(l, resident, E, cur, k);
      if (c >= 0) {
        cur[s] = c;
        act[s] = PW_ACT_SUBST;
        sub += static_cast<double>(g);
      }
    }
  }
  if (lane == 0) {
    for (int s = 0; s < k; ++s) {
      idx[static_cast<size_t>(t) * k + s] = cur[s];
      if (action) action[static_cast<size_t>(t) * k + s] = act[s];
    }
    if (mass) mass[t] = static_cast<float>(tot > 0.0 ? sub / tot : 0.0);
  }
}

// Single CTA: batch gate sums, critical set, then one warp per token remaps.
__global__ void __launch_bounds__(1024) remap_kernel(const float* __restrict__ logits,
                                                     int32_t* __restrict__ idx,
                                                     const float* __restrict__ gate, int T, int E,
                                                     int k, int critical_n,
                                                     uint8_t* __restrict__ critical) {
  __shared__ double S[PW_MAX_EXPERTS];
  __shared__ uint8_t r0[PW_MAX_EXPERTS];
  __shared__ uint8_t crit[PW_MAX_EXPERTS];
  __shared__ int n_r0;
  __shared__ int bad;
  const int tid = threadIdx.x;
  const int TK = T * k;
  if (tid == 0) {
    n_r0 = 0;
    bad = 0;
  }
  for (int e = tid; e < E; e += blockDim.x) r0[e] = 0;
  __syncthreads();
  for (int a = tid; a < TK; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) atomicExch(&bad, 1);
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_status(PW_ERR_BAD_EXPERT);
    return;
  }
  for (int t = tid; t < T; t += blockDim.x) r0[idx[static_cast<size_t>(t) * k]] = 1;
  // S_e: float64, ascending (token, slot) order -- one thread per expert scans the batch.
  for (int e = tid; e < E; e += blockDim.x) {
    double s = 0.0;
    for (int a = 0; a < TK; ++a)
      if (idx[a] == e) s += static_cast<double>(gate[a]);
    S[e] = s;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x)
    if (r0[e]) atomicAdd(&n_r0, 1);
  __syncthreads();
  const int need = max(critical_n - n_r0, 0);
  for (int e = tid; e < E; e += blockDim.x) {
    bool c = r0[e];
    if (!c) {
      int rank = 0;
      const double se = S[e];
      for (int f = 0; f < E; ++f)
        if (!r0[f] && (S[f] > se || (S[f] == se && f < e))) ++rank;
      c = rank < need;
    }
    crit[e] = c ? 1 : 0;
  }
  __syncthreads();
  if (critical)
    for (int e = tid; e < E; e += blockDim.x) critical[e] = crit[e];
  const int warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  for (int t = warp; t < T; t += nw) {
    int cur[PW_MAX_TOPK];
    for (int j = 0; j < k; ++j) cur[j] = idx[static_cast<size_t>(t) * k + j];
    const float* l = logits + static_cast<size_t>(t) * E;
    for (int s = 1; s < k; ++s) {
      if (crit[cur[s]]) continue;
      const int c = best_candidate(l, crit, E, cur, k);
      if (c >= 0) cur[s] = c;
    }
    __syncwarp();
    if (lane == 0)
      for (int s = 1; s < k; ++s) idx[static_cast<size_t>(t) * k + s] = cur[s];
  }
}

}  // namespace pw
