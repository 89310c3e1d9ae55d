// Expert cache policy across decode steps ("Which Expert Misses Are Worth Waiting For?",
// "Méthodologie" and "Contributions Clés" 5): the 0.15 / first-choice substitution against the
// current resident set, frequency-based eviction and background admission of experts whose
// accumulated substituted gate mass reaches beta.  One CTA per step (E <= 1024, T*k <= 4096).
#pragma once
#include "pw_common.cuh"
#include "pw_route.cuh"

namespace pw {

constexpr int kCacheMaxAssign = 4096;

template <int PL>
__global__ void __launch_bounds__(1024) cache_step_kernel(
    const float* __restrict__ logits, int32_t* __restrict__ idx, const float* __restrict__ gate,
    int T, int E, int k, int policy, float threshold, double beta, uint8_t* __restrict__ resident,
    double* __restrict__ mass, uint32_t* __restrict__ freq, int capacity,
    uint8_t* __restrict__ action_out, float* __restrict__ mass_t, int32_t* __restrict__ stats) {
  __shared__ int16_t idx0_s[kCacheMaxAssign];  // the step's routed experts
  __shared__ int16_t idx2_s[kCacheMaxAssign];  // after the rewrite
  __shared__ uint8_t act_s[kCacheMaxAssign];
  __shared__ double mass_s[PW_MAX_EXPERTS];
  __shared__ uint32_t freq_s[PW_MAX_EXPERTS];
  __shared__ uint8_t start[PW_MAX_EXPERTS];  // resident at the start of the step
  __shared__ uint8_t used[PW_MAX_EXPERTS];   // referenced after the rewrite
  __shared__ uint8_t ins[PW_MAX_EXPERTS];    // inserted this step
  __shared__ uint8_t adm[PW_MAX_EXPERTS];    // background admission this step
  __shared__ int16_t flist[PW_MAX_EXPERTS], alist[PW_MAX_EXPERTS];
  __shared__ int bad, n_over, n_f, n_a, n_start;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  const int TK = T * k;
  if (tid == 0) {
    bad = 0;
    n_start = 0;
    n_f = 0;
    n_a = 0;
  }
  for (int e = tid; e < E; e += blockDim.x) {
    start[e] = resident[e] ? 1 : 0;
    mass_s[e] = mass[e];
    freq_s[e] = freq[e];
    used[e] = 0;
    ins[e] = 0;
    adm[e] = 0;
  }
  for (int a = tid; a < TK; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) atomicExch(&bad, 1);
    idx0_s[a] = static_cast<int16_t>(e);
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_status(PW_ERR_BAD_EXPERT);
    return;
  }
  // 1. selections
  for (int a = tid; a < TK; a += blockDim.x) atomicAdd(&freq_s[idx0_s[a]], 1u);
  for (int e = tid; e < E; e += blockDim.x)
    if (start[e]) atomicAdd(&n_start, 1);
  // 2. the substitution rule against the start-of-step resident set, warp per token
  for (int t = warp; t < T; t += nw) {
    int cur[PW_MAX_TOPK];
    for (int j = 0; j < k; ++j) cur[j] = idx0_s[t * k + j];
    WarpRow<PL> row;
    load_row(logits + static_cast<size_t>(t) * E, E, row);
    uint32_t res = 0;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && start[e]) res |= 1u << i;
    }
    uint32_t chosen = lane_set(cur, k);
    double sub = 0.0, tot = 0.0;
    for (int s = 0; s < k; ++s) {
      const float g = gate[static_cast<size_t>(t) * k + s];
      tot += static_cast<double>(g);
      uint8_t act = PW_ACT_HIT;
      if (!start[cur[s]]) {
        bool fetch;
        if (policy == PW_POLICY_FETCH_ALL) fetch = true;
        else if (policy == PW_POLICY_FIRST_CHOICE) fetch = (s == 0);
        else fetch = (s == 0) || (g >= threshold);
        act = PW_ACT_FETCH;
        if (!fetch) {
          const int c = best_candidate(row, res, chosen, E);
          if (c >= 0) {
            swap_chosen(chosen, cur[s], c);
            cur[s] = c;
            act = PW_ACT_SUBST;
            sub += static_cast<double>(g);
          }
        }
      }
      if (lane == 0) act_s[t * k + s] = act;
    }
    if (lane == 0) {
      for (int s = 0; s < k; ++s) {
        idx[static_cast<size_t>(t) * k + s] = cur[s];
        idx2_s[t * k + s] = static_cast<int16_t>(cur[s]);
        used[cur[s]] = 1;
        if (action_out) action_out[static_cast<size_t>(t) * k + s] = act_s[t * k + s];
      }
      if (mass_t) mass_t[t] = static_cast<float>(tot > 0.0 ? sub / tot : 0.0);
    }
  }
  __syncthreads();
  // 3. accumulated substituted mass: one thread per expert adds its own substituted slots in
  //    ascending (token, slot) order (float64); fetched experts are flagged by their slots
  for (int e = tid; e < E; e += blockDim.x) {
    double m = mass_s[e];
    for (int a = 0; a < TK; ++a)
      if (idx0_s[a] == e && act_s[a] == PW_ACT_SUBST) m += static_cast<double>(gate[a]);
    mass_s[e] = m;
  }
  for (int a = tid; a < TK; a += blockDim.x) {
    const int e = idx2_s[a];
    if (act_s[a] == PW_ACT_FETCH && !start[e]) ins[e] = 1;  // every writer stores 1
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    if (ins[e]) atomicAdd(&n_f, 1);
    else if (!start[e] && mass_s[e] >= beta) {
      adm[e] = 1;
      atomicAdd(&n_a, 1);
    }
  }
  __syncthreads();
  if (tid == 0 && n_f + n_a > capacity) {
    // more insertions than the cache holds (rare): keep the most selected fetches, then the
    // heaviest admissions (ties: lower index)
    int nf = 0, na = 0;
    for (int e = 0; e < E; ++e) {
      if (ins[e]) flist[nf++] = static_cast<int16_t>(e);
      if (adm[e]) alist[na++] = static_cast<int16_t>(e);
    }
    for (int i = 0; i < nf; ++i)
      for (int j = i + 1; j < nf; ++j) {
        const int a = flist[i], b = flist[j];
        if (freq_s[b] > freq_s[a] || (freq_s[b] == freq_s[a] && b < a)) {
          flist[i] = static_cast<int16_t>(b);
          flist[j] = static_cast<int16_t>(a);
        }
      }
    for (int i = 0; i < na; ++i)
      for (int j = i + 1; j < na; ++j) {
        const int a = alist[i], b = alist[j];
        if (mass_s[b] > mass_s[a] || (mass_s[b] == mass_s[a] && b < a)) {
          alist[i] = static_cast<int16_t>(b);
          alist[j] = static_cast<int16_t>(a);
        }
      }
    const int kf = min(nf, capacity), ka = min(na, max(capacity - kf, 0));
    for (int i = kf; i < nf; ++i) ins[flist[i]] = 0;
    for (int i = ka; i < na; ++i) adm[alist[i]] = 0;
    n_f = kf;
    n_a = ka;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x)
    if (ins[e] || adm[e]) {
      ins[e] = 1;
      mass_s[e] = 0.0;
    }
  if (tid == 0) n_over = n_start + n_f + n_a - capacity;
  __syncthreads();
  // 4. evictions: start residents ranked by (used, selections, index), the first n_over go
  int n_ev = 0;
  for (int e = tid; e < E; e += blockDim.x) {
    bool victim = false;
    if (start[e] && n_over > 0) {
      int rank = 0;
      for (int f = 0; f < E; ++f) {
        if (!start[f] || f == e) continue;
        const bool before = used[f] < used[e] ||
                            (used[f] == used[e] &&
                             (freq_s[f] < freq_s[e] || (freq_s[f] == freq_s[e] && f < e)));
        rank += before;
      }
      victim = rank < n_over;
    }
    n_ev += victim;
    resident[e] = ((start[e] && !victim) || ins[e]) ? 1 : 0;
    mass[e] = mass_s[e];
    freq[e] = freq_s[e];
  }
  if (stats) {
    n_ev = __reduce_add_sync(0xffffffffu, n_ev);
    if (lane == 0 && n_ev) atomicAdd(&stats[2], n_ev);
    if (tid == 0) {
      atomicAdd(&stats[0], n_f);
      atomicAdd(&stats[1], n_a);
    }
  }
}

}  // namespace pw
