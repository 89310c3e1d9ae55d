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

constexpr int kRouteExpertsPerCta = 8;
constexpr int kRouteThreads = 256;

__device__ __forceinline__ double bf16lo(uint32_t v) {
  return static_cast<double>(__uint_as_float(v << 16));
}
__device__ __forceinline__ double bf16hi(uint32_t v) {
  return static_cast<double>(__uint_as_float(v & 0xffff0000u));
}

// One warp, one token: top-k by (logit desc, index asc) over l[0..E), softmax over all E in
// float64, gates rounded once (renormalised over the k when asked).  Every exp is taken once
// (float64 exp has a long latency): the selected experts' probabilities are read back from the
// lane that holds them.  PL = elements per lane (E <= 32 * PL), so the code is no larger than
// E needs (a cold kernel fetches every instruction it runs from memory).
// float64 exp behind a call, so the PL exponentials of topk_warp share one copy of its code
// (a cold kernel fetches every instruction it runs from memory).
__device__ __noinline__ double exp_f64(double v) { return exp(v); }

template <int PL>
__device__ __forceinline__ void topk_warp(const float* l, int E, int k, int renorm,
                                          int32_t* __restrict__ idx_out,
                                          float* __restrict__ gate_out) {
  const int lane = threadIdx.x & 31;
  float v[PL];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? l[e] : -INFINITY;
    mx = fmaxf(mx, v[i]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  double ex[PL];
  double z = 0.0;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    ex[i] = 0.0;
    if (lane + 32 * i < E) {
      ex[i] = PL > 2 ? exp_f64(static_cast<double>(v[i]) - static_cast<double>(mx))
                     : exp(static_cast<double>(v[i]) - static_cast<double>(mx));
      z += ex[i];
    }
  }
  z = warp_sum_f64(z);

  uint32_t taken = 0;  // bit i: element lane+32i already chosen
  double psum = 0.0, mine = 0.0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = -1;
    double be = 0.0;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (bi < 0 || v[i] > bv)) {
        bv = v[i];
        bi = e;
        be = ex[i];
      }
    }
    warp_argmax(bv, bi);
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    // the winner's exp, from the lane whose own candidate it was
    const double p = __shfl_sync(0xffffffffu, be, bi & 31) / z;
    psum += p;
    if (lane == j) mine = p;
    if (lane == 0) idx_out[j] = bi;
  }
  if (lane < k) gate_out[lane] = static_cast<float>(renorm ? mine / psum : mine);
}

// logits[t][e] = fp32(sum_h x[t][h] * Wr[e][h] + bias[e]) with float64 accumulation.
// CTA = 8 experts x TT tokens; all 256 threads split H (8 consecutive h per thread per
// 2048-wide chunk, 16-byte loads when `vec`), so every load of a CTA is in flight at once; the
// 256 partial sums of each (expert, token) are added in a fixed order.  With fuse_k > 0 (the
// whole E fits one CTA) the CTA then runs the top-k of its tokens as well.
template <int TT>
__global__ void __launch_bounds__(kRouteThreads) router_logits_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ Wr, const float* __restrict__ bias,
    int T, int H, int E, int vec, float* __restrict__ logits, int fuse_k, int renorm,
    int32_t* __restrict__ idx, float* __restrict__ gate) {
  griddep_launch();  // the next kernel (a rewrite or the forward's setup) may be scheduled now
  __shared__ double part[kRouteThreads / 32][kRouteExpertsPerCta][TT];
  __shared__ float lsm[TT][kRouteExpertsPerCta];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int e0 = blockIdx.x * kRouteExpertsPerCta;
  const int ne = min(kRouteExpertsPerCta, E - e0);
  const int t0 = blockIdx.y * TT;
  const int nt = min(TT, T - t0);
  double acc[kRouteExpertsPerCta][TT];
#pragma unroll
  for (int e = 0; e < kRouteExpertsPerCta; ++e)
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[e][t] = 0.0;
  // Rows past E (or T) are clamped to the last valid one and their sums discarded, so every
  // load of an iteration is unconditional and all of them are in flight together.
  const uint16_t* xr[TT];
  const float* wr[kRouteExpertsPerCta];
#pragma unroll
  for (int t = 0; t < TT; ++t) xr[t] = x + static_cast<size_t>(t0 + min(t, nt - 1)) * H;
#pragma unroll
  for (int e = 0; e < kRouteExpertsPerCta; ++e)
    wr[e] = Wr + static_cast<size_t>(e0 + min(e, ne - 1)) * H;
  if (vec) {
    // CH chunks of 2048 columns per round (two for a single token, so that both rounds of a
    // 4096-wide row are loaded at once); a chunk past H re-reads chunk 0 and is not added
    constexpr int CH = TT == 1 ? 2 : 1;
    for (int hb = tid * 8; hb < H; hb += CH * kRouteThreads * 8) {
      uint4 xv[CH][TT];
      float4 wa[CH][kRouteExpertsPerCta], wb[CH][kRouteExpertsPerCta];
      bool live[CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        live[c] = hb + c * kRouteThreads * 8 < H;
        const int h0 = live[c] ? hb + c * kRouteThreads * 8 : hb;
#pragma unroll
        for (int t = 0; t < TT; ++t) xv[c][t] = __ldg(reinterpret_cast<const uint4*>(xr[t] + h0));
#pragma unroll
        for (int e = 0; e < kRouteExpertsPerCta; ++e) {
          wa[c][e] = __ldg(reinterpret_cast<const float4*>(wr[e] + h0));
          wb[c][e] = __ldg(reinterpret_cast<const float4*>(wr[e] + h0 + 4));
        }
      }
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        if (!live[c]) continue;
#pragma unroll
        for (int e = 0; e < kRouteExpertsPerCta; ++e) {
#pragma unroll
          for (int t = 0; t < TT; ++t) {
            const uint4 xq = xv[c][t];
            const float4 a4 = wa[c][e], b4 = wb[c][e];
            double a = acc[e][t];
            a = fma(bf16lo(xq.x), static_cast<double>(a4.x), a);
            a = fma(bf16hi(xq.x), static_cast<double>(a4.y), a);
            a = fma(bf16lo(xq.y), static_cast<double>(a4.z), a);
            a = fma(bf16hi(xq.y), static_cast<double>(a4.w), a);
            a = fma(bf16lo(xq.z), static_cast<double>(b4.x), a);
            a = fma(bf16hi(xq.z), static_cast<double>(b4.y), a);
            a = fma(bf16lo(xq.w), static_cast<double>(b4.z), a);
            a = fma(bf16hi(xq.w), static_cast<double>(b4.w), a);
            acc[e][t] = a;
          }
        }
      }
    }
  } else {
    for (int h = tid; h < H; h += kRouteThreads) {
      double xv[TT], wv[kRouteExpertsPerCta];
#pragma unroll
      for (int t = 0; t < TT; ++t) xv[t] = static_cast<double>(bf16_to_f32(xr[t][h]));
#pragma unroll
      for (int e = 0; e < kRouteExpertsPerCta; ++e) wv[e] = static_cast<double>(wr[e][h]);
#pragma unroll
      for (int e = 0; e < kRouteExpertsPerCta; ++e)
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[e][t] = fma(xv[t], wv[e], acc[e][t]);
    }
  }
#pragma unroll
  for (int e = 0; e < kRouteExpertsPerCta; ++e)
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const double v = warp_sum_f64(acc[e][t]);
      if (lane == 0) part[warp][e][t] = v;
    }
  __syncthreads();
  if (tid < kRouteExpertsPerCta * TT) {
    const int e = tid / TT, t = tid - e * TT;
    if (e < ne && t < nt) {
      double s = 0.0;
#pragma unroll
      for (int w = 0; w < kRouteThreads / 32; ++w) s += part[w][e][t];
      const double b = bias ? static_cast<double>(bias[e0 + e]) : 0.0;
      const float lv = static_cast<float>(s + b);
      logits[static_cast<size_t>(t0 + t) * E + e0 + e] = lv;
      lsm[t][e] = lv;
    }
  }
  if (fuse_k > 0) {
    __syncthreads();
    for (int t = warp; t < nt; t += kRouteThreads / 32)
      topk_warp<1>(lsm[t], E, fuse_k, renorm, idx + static_cast<size_t>(t0 + t) * fuse_k,
                gate + static_cast<size_t>(t0 + t) * fuse_k);
  }
}

// One warp per token: top-k of a logits row in global memory (E <= 32 * PL).
template <int PL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E,
                                                   int k, int renorm, int32_t* __restrict__ idx,
                                                   float* __restrict__ gate) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  topk_warp<PL>(logits + static_cast<size_t>(t) * E, E, k, renorm, idx + static_cast<size_t>(t) * k,
            gate + static_cast<size_t>(t) * k);
}

// A token's logits row held by one warp: element e = lane + 32 i in v[i] (-inf past E),
// E <= 32 * PL.
template <int PL>
struct WarpRow {
  float v[PL];
};

template <int PL>
__device__ __forceinline__ void load_row(const float* __restrict__ l, int E, WarpRow<PL>& r) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    r.v[i] = (e < E) ? l[e] : -INFINITY;
  }
}

// Bit i of the result: expert lane + 32 i is one of cur[0..k).
__device__ __forceinline__ uint32_t lane_set(const int* cur, int k) {
  const int lane = threadIdx.x & 31;
  uint32_t m = 0;
  for (int j = 0; j < k; ++j)
    if ((cur[j] & 31) == lane) m |= 1u << (cur[j] >> 5);
  return m;
}

// Highest-logit expert e with bit (e >> 5) of this lane's `allowed` set and e not in `chosen`
// (ties: lower index); -1 if none.
template <int PL>
__device__ __forceinline__ int best_candidate(const WarpRow<PL>& r, uint32_t allowed,
                                              uint32_t chosen, int E) {
  const int lane = threadIdx.x & 31;
  float bv = -INFINITY;
  int bi = -1;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    if (e < E && ((allowed >> i) & 1u) && !((chosen >> i) & 1u) && (bi < 0 || r.v[i] > bv)) {
      bv = r.v[i];
      bi = e;
    }
  }
  warp_argmax(bv, bi);
  return bi;
}

// Replace cur[s] by c in the per-lane chosen mask.
__device__ __forceinline__ void swap_chosen(uint32_t& chosen, int old_e, int new_e) {
  const int lane = threadIdx.x & 31;
  if ((old_e & 31) == lane) chosen &= ~(1u << (old_e >> 5));
  if ((new_e & 31) == lane) chosen |= 1u << (new_e >> 5);
}

template <int PL>
__global__ void __launch_bounds__(256) substitute_kernel(
    const float* __restrict__ logits, int32_t* __restrict__ idx, const float* __restrict__ gate,
    const uint8_t* __restrict__ resident, int T, int E, int k, int policy, float threshold,
    uint8_t* __restrict__ action, float* __restrict__ mass) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  // lane j < k reads slot j (id, gate, residency of the routed expert), so the token's slots
  // cost two dependent round trips to memory instead of two per slot
  int my_e = 0;
  float my_g = 0.0f;
  int my_res = 0;
  if (lane < k) {
    my_e = idx[static_cast<size_t>(t) * k + lane];
    my_g = gate[static_cast<size_t>(t) * k + lane];
  }
  const bool bad = __any_sync(0xffffffffu, lane < k && (my_e < 0 || my_e >= E));
  if (bad) {  // ids out of range: leave the token untouched
    if (lane == 0) set_status(PW_ERR_BAD_EXPERT);
    return;
  }
  if (lane < k) my_res = resident[my_e] ? 1 : 0;
  const uint32_t res_slots = __ballot_sync(0xffffffffu, my_res != 0);  // bit s: slot s resident
  int cur[PW_MAX_TOPK];
  for (int j = 0; j < k; ++j) cur[j] = __shfl_sync(0xffffffffu, my_e, j);
  WarpRow<PL> row;
  load_row(logits + static_cast<size_t>(t) * E, E, row);
  uint32_t res = 0;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    if (e < E && resident[e]) res |= 1u << i;
  }
  uint32_t chosen = lane_set(cur, k);
  double sub = 0.0, tot = 0.0;
  uint8_t act[PW_MAX_TOPK];
  for (int s = 0; s < k; ++s) {
    const float g = __shfl_sync(0xffffffffu, my_g, s);
    tot += static_cast<double>(g);
    if ((res_slots >> s) & 1u) {  // the expert routed to slot s (never rewritten before s)
      act[s] = PW_ACT_HIT;
      continue;
    }
    bool fetch;
    if (policy == PW_POLICY_FETCH_ALL) fetch = true;
    else if (policy == PW_POLICY_FIRST_CHOICE) fetch = (s == 0);
    else fetch = (s == 0) || (g >= threshold);
    act[s] = PW_ACT_FETCH;
    if (!fetch) {
      const int c = best_candidate(row, res, chosen, E);
      if (c >= 0) {
        swap_chosen(chosen, cur[s], c);
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

constexpr int kRemapMaxAssign = 8192;  // T * k of the single-CTA batch rewrites
constexpr int kRemapGateSmem = 4096;   // up to this T * k the gates are staged in shared memory

// Number of distinct experts among the TK assignments (idx_s: shared copy, or idx: global,
// read after the CTA's own writes); `flags` [E] and `n` are shared scratch.  CTA-wide: every
// thread calls it, and every thread gets the count.
__device__ __forceinline__ int distinct_experts(const int16_t* idx_s, const int32_t* idx, int TK,
                                                int E, uint8_t* flags, int* n) {
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) flags[e] = 0;
  if (threadIdx.x == 0) *n = 0;
  __syncthreads();
  for (int a = threadIdx.x; a < TK; a += blockDim.x) flags[idx_s ? idx_s[a] : idx[a]] = 1;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (flags[e]) atomicAdd(n, 1);
  __syncthreads();
  return *n;
}

// Single CTA: batch gate sums, critical set, then one warp per token remaps (E <= 32 * PL).
template <int PL>
__global__ void __launch_bounds__(1024) remap_kernel(const float* __restrict__ logits,
                                                     int32_t* __restrict__ idx,
                                                     const float* __restrict__ gate, int T, int E,
                                                     int k, int critical_n,
                                                     uint8_t* __restrict__ critical,
                                                     int32_t* __restrict__ unique) {
  __shared__ double S[PW_MAX_EXPERTS];
  __shared__ uint8_t r0[PW_MAX_EXPERTS];
  __shared__ uint8_t crit[PW_MAX_EXPERTS];
  __shared__ uint8_t used[PW_MAX_EXPERTS];
  __shared__ int16_t idx_s[kRemapMaxAssign];  // the assignments, scanned once per expert
  __shared__ float gate_s[kRemapGateSmem];     // their gates (small batches)
  __shared__ int n_r0;
  __shared__ int n_used;
  __shared__ int bad;
  const int tid = threadIdx.x;
  const int TK = T * k;
  if (tid == 0) {
    n_r0 = 0;
    bad = 0;
  }
  for (int e = tid; e < E; e += blockDim.x) r0[e] = 0;
  __syncthreads();
  const bool stage_gates = TK <= kRemapGateSmem;
  for (int a = tid; a < TK; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) atomicExch(&bad, 1);
    idx_s[a] = static_cast<int16_t>(e);
    if (stage_gates) gate_s[a] = gate[a];
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_status(PW_ERR_BAD_EXPERT);
    return;
  }
  const int before = unique ? distinct_experts(idx_s, nullptr, TK, E, used, &n_used) : 0;
  for (int t = tid; t < T; t += blockDim.x) r0[idx_s[t * k]] = 1;
  // S_e: float64, ascending (token, slot) order -- one thread per expert scans the batch (the
  // gates from shared memory when staged, so the scan waits on no global load)
  const float* gsrc = stage_gates ? gate_s : gate;
  for (int e = tid; e < E; e += blockDim.x) {
    double s = 0.0;
    for (int a = 0; a < TK; ++a)
      if (idx_s[a] == e) s += static_cast<double>(gsrc[a]);
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
  uint32_t crit_bits = 0;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    if (e < E && crit[e]) crit_bits |= 1u << i;
  }
  for (int t = warp; t < T; t += nw) {
    int cur[PW_MAX_TOPK];
    for (int j = 0; j < k; ++j) cur[j] = idx_s[t * k + j];  // the staged copy: no global load
    WarpRow<PL> row;
    load_row(logits + static_cast<size_t>(t) * E, E, row);
    uint32_t chosen = lane_set(cur, k);
    for (int s = 1; s < k; ++s) {
      if (crit[cur[s]]) continue;
      const int c = best_candidate(row, crit_bits, chosen, E);
      if (c >= 0) {
        swap_chosen(chosen, cur[s], c);
        cur[s] = c;
      }
    }
    __syncwarp();
    if (lane == 0)
      for (int s = 1; s < k; ++s) idx[static_cast<size_t>(t) * k + s] = cur[s];
  }
  if (unique) {
    const int after = distinct_experts(nullptr, idx, TK, E, used, &n_used);
    if (tid == 0) {
      unique[0] = before;
      unique[1] = after;
    }
  }
}

// LYNX AffinityBinning (2.1, 2.2): per-token confidence bins from the top-2 logit gap, batch
// expert scores S_e = sum of 2^bin * gate (float64, ascending (token, slot) order), the critical
// set from those scores, then the remap of low-affinity tokens (bin < low) as in remap_kernel.
// One CTA; bins[T] (int32) may be null.
template <int PL>
__global__ void __launch_bounds__(1024) affinity_remap_kernel(
    const float* __restrict__ logits, int32_t* __restrict__ idx, const float* __restrict__ gate,
    int T, int E, int k, int critical_n, int B, double w, int low,
    uint8_t* __restrict__ critical, int32_t* __restrict__ bins_out,
    int32_t* __restrict__ unique) {
  __shared__ double S[PW_MAX_EXPERTS];
  __shared__ uint8_t r0[PW_MAX_EXPERTS];
  __shared__ uint8_t crit[PW_MAX_EXPERTS];
  __shared__ uint8_t used[PW_MAX_EXPERTS];
  __shared__ uint8_t bin_s[PW_MAX_TOKENS];
  __shared__ int16_t idx_s[kRemapMaxAssign];
  __shared__ float gate_s[kRemapGateSmem];  // the gates (small batches)
  __shared__ int n_r0;
  __shared__ int n_used;
  __shared__ int bad;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  const int TK = T * k;
  if (tid == 0) {
    n_r0 = 0;
    bad = 0;
  }
  for (int e = tid; e < E; e += blockDim.x) r0[e] = 0;
  __syncthreads();
  const bool stage_gates = TK <= kRemapGateSmem;
  for (int a = tid; a < TK; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) atomicExch(&bad, 1);
    idx_s[a] = static_cast<int16_t>(e);
    if (stage_gates) gate_s[a] = gate[a];
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_status(PW_ERR_BAD_EXPERT);
    return;
  }
  const int before = unique ? distinct_experts(idx_s, nullptr, TK, E, used, &n_used) : 0;
  // confidence bins: warp per token, gap between the two largest logits (fp32)
  for (int t = warp; t < T; t += nw) {
    WarpRow<PL> row;
    load_row(logits + static_cast<size_t>(t) * E, E, row);
    float v0 = -INFINITY, v1 = -INFINITY;
    int i0 = -1, i1 = -1;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && (i0 < 0 || row.v[i] > v0)) {
        v0 = row.v[i];
        i0 = e;
      }
    }
    warp_argmax(v0, i0);
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && e != i0 && (i1 < 0 || row.v[i] > v1)) {
        v1 = row.v[i];
        i1 = e;
      }
    }
    warp_argmax(v1, i1);
    if (lane == 0) {
      int b = 0;
      if (!isinf(w)) {
        if (i1 < 0) {
          b = B - 1;
        } else {
          const double qd = static_cast<double>(v0 - v1) / w;
          b = qd >= static_cast<double>(B - 1) ? B - 1 : static_cast<int>(floor(qd));
        }
      }
      bin_s[t] = static_cast<uint8_t>(b);
      if (bins_out) bins_out[t] = b;
    }
  }
  for (int t = tid; t < T; t += blockDim.x) r0[idx_s[t * k]] = 1;
  __syncthreads();
  // S_e: one thread per expert scans the batch in (token, slot) order (the gates from shared
  // memory when staged)
  const float* gsrc = stage_gates ? gate_s : gate;
  for (int e = tid; e < E; e += blockDim.x) {
    double sc = 0.0;
    for (int t = 0, a = 0; t < T; ++t) {
      const double wt = ldexp(1.0, bin_s[t]);
      for (int s = 0; s < k; ++s, ++a)
        if (idx_s[a] == e) sc += wt * static_cast<double>(gsrc[a]);
    }
    S[e] = sc;
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
  uint32_t crit_bits = 0;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    if (e < E && crit[e]) crit_bits |= 1u << i;
  }
  for (int t = warp; t < T; t += nw) {
    if (bin_s[t] >= low) continue;  // high-affinity token: its experts stay
    int cur[PW_MAX_TOPK];
    for (int j = 0; j < k; ++j) cur[j] = idx_s[t * k + j];  // the staged copy: no global load
    WarpRow<PL> row;
    load_row(logits + static_cast<size_t>(t) * E, E, row);
    uint32_t chosen = lane_set(cur, k);
    for (int s = 1; s < k; ++s) {
      if (crit[cur[s]]) continue;
      const int c = best_candidate(row, crit_bits, chosen, E);
      if (c >= 0) {
        swap_chosen(chosen, cur[s], c);
        cur[s] = c;
      }
    }
    __syncwarp();
    if (lane == 0)
      for (int s = 1; s < k; ++s) idx[static_cast<size_t>(t) * k + s] = cur[s];
  }
  if (unique) {
    const int after = distinct_experts(nullptr, idx, TK, E, used, &n_used);
    if (tid == 0) {
      unique[0] = before;
      unique[1] = after;
    }
  }
}

}  // namespace pw
