// K2: token -> expert grouping, table check and activation staging for the grouped FFN, and
// the final gate-weighted combine.
// Assignment a = t*k + slot.  Within an expert the assignments are kept in ascending a (the
// set of experts to load grows with the batch -- LYNX, 1 "Énoncé du Problème").
#pragma once
#include "pw_common.cuh"
#include "pw_ffn.cuh"

namespace pw {

constexpr int kGroupThreads = 1024;
constexpr int kMaxAssign = 8192;  // T * k handled by the single-CTA grouping step
constexpr int kPassTokens = 64;   // tokens of one expert per tensor-core pass (MMA N <= 64)
constexpr int kTcChunkCols = 256; // K columns per tensor-core pipeline step (operand chunk)
constexpr int kEarlyDescExperts = 64;  // setup reads every expert's blocks before grouping

// What the tensor-core FFN needs beyond the plain grouping.  Each expert's tokens are split
// into passes of up to kPassTokens; a pass of m tokens is padded to np = m rounded up to 16
// (the MMA's N).  Padded rows: expert e owns rows [pbase[e], pbase[e] + roundup16(count)),
// pass j of it rows pbase[e] + 64j ..; ptok[row] = token of the row (-1 for padding),
// pnn[row] = np << 16 | (row - first row of its pass); pass_tab[i] = a | j << 16 for the i-th
// (active expert a, pass j) in ascending (a, j); meta[5] = number of passes, meta[6] = number
// of padded rows.
struct PassOut {
  int32_t* pbase;     // [E]
  int32_t* ptok;      // [padded rows]
  int32_t* pnn;       // [padded rows]
  int32_t* pass_tab;  // [E + T*k/64 + 1]
};

__host__ __device__ __forceinline__ int pass_np(int count, int j) {
  const int m = min(kPassTokens, count - kPassTokens * j);
  return (m + 15) & ~15;
}

// Exclusive prefix sums of four counters over the threads of the CTA (blockDim.x <= 1024, a
// multiple of 32), in thread order; every thread also gets the totals.  CTA-wide.
__device__ __forceinline__ int4 block_scan4(int4 v, int4& total) {
  __shared__ int4 wsum[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int4 inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, inc.x, off), y = __shfl_up_sync(0xffffffffu, inc.y, off);
    const int z = __shfl_up_sync(0xffffffffu, inc.z, off), w = __shfl_up_sync(0xffffffffu, inc.w, off);
    if (lane >= off) {
      inc.x += x;
      inc.y += y;
      inc.z += z;
      inc.w += w;
    }
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int4 t = lane < nw ? wsum[lane] : make_int4(0, 0, 0, 0);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, t.x, off), y = __shfl_up_sync(0xffffffffu, t.y, off);
      const int z = __shfl_up_sync(0xffffffffu, t.z, off), w = __shfl_up_sync(0xffffffffu, t.w, off);
      if (lane >= off) {
        t.x += x;
        t.y += y;
        t.z += z;
        t.w += w;
      }
    }
    if (lane < nw) wsum[lane] = t;  // inclusive sums of the warp totals
  }
  __syncthreads();
  const int4 before = warp ? wsum[warp - 1] : make_int4(0, 0, 0, 0);
  total = wsum[nw - 1];
  __syncthreads();  // wsum may be reused by the next call
  return make_int4(before.x + inc.x - v.x, before.y + inc.y - v.y, before.z + inc.z - v.z,
                   before.w + inc.w - v.w);
}

// Grouping, run by one CTA.  counts[E], offsets[E+1], perm[T*k] (grouped position ->
// assignment), inv[T*k] (assignment -> grouped position, -1 for an invalid expert id),
// active[E] (experts with work, ascending), meta[0] = number of active experts (0 when the page
// table does not match (layer, E)), meta[1] = number of valid assignments, meta[2] = 1 for a
// mismatched table, meta[4] = 0 (the FFN launch's work counter); and the PassOut arrays.
// Returns, to thread e < E, expert e's exclusive scan values: .x its offset, .y its index in
// the active list (when it has assignments).
__device__ __forceinline__ int4 group_block(const pw_page_table* __restrict__ pt, int layer,
                                            const int32_t* __restrict__ idx, int TK, int k,
                                            int E, const PassOut& po,
                                            int32_t* __restrict__ counts,
                                            int32_t* __restrict__ offsets,
                                            int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                            int32_t* __restrict__ active,
                                            int32_t* __restrict__ meta) {
  __shared__ int cnt[PW_MAX_EXPERTS];
  __shared__ int off[PW_MAX_EXPERTS + 1];
  __shared__ int act_pos[PW_MAX_EXPERTS + 1];
  __shared__ int pb[PW_MAX_EXPERTS];
  __shared__ int16_t eid[kMaxAssign];
  __shared__ int run[PW_MAX_EXPERTS];
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
  // per expert (thread e): assignments, active or not, padded rows and tensor-core passes;
  // their exclusive prefix sums give the offsets, the active index, the padded row base and
  // the first pass of each expert (E <= blockDim.x)
  const bool bad = pt->blocks == nullptr || static_cast<unsigned>(layer) >= pt->num_layers ||
                   static_cast<int>(pt->num_experts) != E ||
                   (reinterpret_cast<uintptr_t>(pt->blocks) & 63) != 0;
  const int c = tid < E ? cnt[tid] : 0;
  const int4 mine = make_int4(c, c > 0 ? 1 : 0, (c + 15) & ~15,
                              bad ? 0 : (c + kPassTokens - 1) / kPassTokens);
  int4 total;
  const int4 ex = block_scan4(mine, total);
  if (tid < E) {
    off[tid] = ex.x;
    act_pos[tid] = ex.y;
    pb[tid] = ex.z;
    for (int j = 0; j < mine.w; ++j) po.pass_tab[ex.w + j] = ex.y | (j << 16);
  }
  if (tid == 0) {
    if (bad) set_status(PW_ERR_INVALID_ARG);
    off[E] = total.x;
    act_pos[E] = total.y;
    meta[0] = bad ? 0 : total.y;
    meta[1] = total.x;
    meta[2] = bad ? 1 : 0;
    meta[4] = 0;  // work counter of the FFN launch
    meta[5] = total.w;
    meta[6] = total.z;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    counts[e] = cnt[e];
    offsets[e] = off[e];
    po.pbase[e] = pb[e];
    if (cnt[e] > 0) active[act_pos[e]] = e;
    for (int r = cnt[e]; r < ((cnt[e] + 15) & ~15); ++r) {  // padding rows of the last pass
      po.ptok[pb[e] + r] = -1;
      po.pnn[pb[e] + r] = (pass_np(cnt[e], r / kPassTokens) << 16) | (r % kPassTokens);
    }
  }
  if (tid == 0) offsets[E] = off[E];
  // rank of each assignment among its expert's (ascending a): chunks of blockDim assignments in
  // order; inside a warp the peers of an expert come from one match, and the warps of a chunk
  // take their bases from run[e] one after the other
  const int lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  for (int e = tid; e < E; e += blockDim.x) run[e] = 0;
  __syncthreads();
  for (int c0 = 0; c0 < TK; c0 += blockDim.x) {
    const int a = c0 + tid;
    const int e = a < TK ? eid[a] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    int base = 0;
    const int nwc = min(nw, (TK - c0 + 31) >> 5);  // warps of this chunk holding assignments
    for (int w = 0; w < nwc; ++w) {
      if (warp == w && e >= 0 && lane == leader) {
        base = run[e];
        run[e] = base + __popc(peers);
      }
      __syncthreads();
    }
    base = __shfl_sync(0xffffffffu, base, leader);
    if (a >= TK) continue;
    if (e < 0) {
      inv[a] = -1;
      continue;
    }
    const int r = base + __popc(peers & ((1u << lane) - 1u));
    const int pos = off[e] + r;
    perm[pos] = a;
    inv[a] = pos;
    po.ptok[pb[e] + r] = a / k;
    po.pnn[pb[e] + r] = (pass_np(cnt[e], r / kPassTokens) << 16) | (r % kPassTokens);
  }
  return ex;
}

// The one launch before the grouped FFN.  CTA 0 checks the page table and groups the
// assignments; CTAs 1.. convert x to the CUDA-core FFN's activation layout: X[t] holds, per
// 512-column stage, the stage's columns as fp16 (bf16 -> fp16 is exact for values in fp16's
// normal range) in the decode's order (k4::xpos, a permutation inside each 32-column group),
// with zeros for H <= c < ldx.  One row per token: the gate_up producer maps a grouped position
// to its token.  `vec`: x is 16-byte aligned (H is a multiple of 128), so a thread converts 8
// columns from one load.  The tensor-core FFN stages its activations with stage_x_kernel
// instead; it launches this kernel with CTA 0 alone.
__global__ void __launch_bounds__(kGroupThreads) setup_kernel(
    const pw_page_table* __restrict__ pt, int layer, const int32_t* __restrict__ idx, int T,
    int k, int E, const uint16_t* __restrict__ x, int H, int I, int ldx, int vec,
    __half* __restrict__ X, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv, int32_t* __restrict__ active,
    int32_t* __restrict__ meta, int32_t* __restrict__ done, PassOut po,
    k4::ExpertDesc* __restrict__ xd) {
  griddep_wait();  // launched as a dependent of whatever precedes it in the stream
  griddep_launch();
  if (blockIdx.x == 0) {
    // the CUDA-core FFN's per-(module, active expert) block descriptors.  With few experts
    // (E <= kEarlyDescExperts), thread e reads both blocks of expert e from the page table
    // before grouping, so those reads overlap it, and files them under e's active index once
    // the grouping has given it; with many, only the active experts' blocks are read, after it.
    const bool early = xd != nullptr && E <= kEarlyDescExperts;
    const bool want_xd = early && static_cast<int>(threadIdx.x) < E;
    const bool table_ok = pt->blocks != nullptr && static_cast<unsigned>(layer) < pt->num_layers &&
                          static_cast<int>(pt->num_experts) == E &&
                          (reinterpret_cast<uintptr_t>(pt->blocks) & 63) == 0;
    k4::ExpertDesc xg, xdn;
    if (want_xd && table_ok) {
      xg = k4::expert_desc(pt, layer, E, threadIdx.x, k4::MODE_GATE_UP, 2 * I, H, 0, 0);
      xdn = k4::expert_desc(pt, layer, E, threadIdx.x, k4::MODE_DOWN, H, I, 0, 0);
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) done[e] = 0;
    const int4 ex = group_block(pt, layer, idx, T * k, k, E, po, counts, offsets, perm, inv,
                                active, meta);
    if (xd != nullptr) {
      __syncthreads();  // the grouping's outputs are written (the whole CTA takes the barrier)
      if (early) {
        const int c = want_xd && table_ok ? counts[threadIdx.x] : 0;
        if (c > 0) {
          xg.te = xdn.te = c;
          xg.pos0 = xdn.pos0 = ex.x;
          xd[k4::MODE_GATE_UP * E + ex.y] = xg;
          xd[k4::MODE_DOWN * E + ex.y] = xdn;
        }
      } else {
        const int na = meta[0];
        for (int i = threadIdx.x; i < 2 * na; i += blockDim.x) {
          const int mode = i / na, a = i - mode * na;
          const int e = active[a];
          const int rows = mode == k4::MODE_GATE_UP ? 2 * I : H;
          const int cols = mode == k4::MODE_GATE_UP ? H : I;
          xd[mode * E + a] =
              k4::expert_desc(pt, layer, E, e, mode, rows, cols, counts[e], offsets[e]);
        }
      }
    }
    return;
  }
  const size_t nthr = static_cast<size_t>(gridDim.x - 1) * blockDim.x;
  const size_t t0 = static_cast<size_t>(blockIdx.x - 1) * blockDim.x + threadIdx.x;
  const int g8 = ldx / 8;  // 8-column groups per row
  for (size_t i = t0; i < static_cast<size_t>(T) * g8; i += nthr) {
    const size_t t = i / g8;
    const int c = static_cast<int>(i - t * g8) * 8;
    float v[8];
    if (c >= H) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.0f;
    } else if (vec) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + t * H + c));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = bf16_to_f32(x[t * H + c + j]);
    }
    __half* row = X + t * ldx;
#pragma unroll
    for (int j = 0; j < 8; ++j) row[k4::xpos(c + j)] = __float2half_rn(v[j]);
  }
}

// The tensor-core FFN's gate_up operand: for every padded row (ptok, pnn as in PassOut) the
// token's activations as fp16, in the MMA's K-major core-matrix order per 256-column chunk:
// element (n, c) of the pass starting at padded row r0 (np rows) sits at
//   r0 * H + (c / 256) * np * 256 + ((c % 256) / 8) * np * 8 + n * 8 + c % 8
// (so one chunk of a pass is np * 512 contiguous bytes, a last chunk of 128 columns half
// that); padding rows are zeros.  bf16 -> fp16
// is exact for values in fp16's normal range.  `vec`: x is 16-byte aligned.
__global__ void __launch_bounds__(256) stage_x_kernel(const uint16_t* __restrict__ x, int H,
                                                      int vec, const int32_t* __restrict__ ptok,
                                                      const int32_t* __restrict__ pnn,
                                                      const int32_t* __restrict__ meta,
                                                      int T, int rows_cap,
                                                      __half* __restrict__ XB) {
  griddep_wait();  // grouping of the launch before
  griddep_launch();
  int rows = meta[6];
  if (!PW_CHECK(rows <= rows_cap)) rows = 0;
  const int g8 = H / 8;
  const size_t n_all = static_cast<size_t>(rows) * g8;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_all;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(i / g8);
    const int c = static_cast<int>(i - static_cast<size_t>(row) * g8) * 8;
    const int tok = ptok[row];
    const int nn = pnn[row];
    const int np = nn >> 16, n = nn & 0xffff;
    if (!PW_CHECK(tok < T && n < np && row - n + np <= rows)) continue;
    __half* dst = XB + static_cast<size_t>(row - n) * H + (c / kTcChunkCols) * np * kTcChunkCols +
                  ((c % kTcChunkCols) / 8) * np * 8 + n * 8;
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (tok >= 0) {
      const uint16_t* src = x + static_cast<size_t>(tok) * H + c;
      uint32_t w[4];
      if (vec) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
        w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          w[j] = static_cast<uint32_t>(src[2 * j]) | (static_cast<uint32_t>(src[2 * j + 1]) << 16);
      }
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 h = __floats2half2_rn(__uint_as_float(w[j] << 16),
                                            __uint_as_float(w[j] & 0xffff0000u));
        o[j] = *reinterpret_cast<const uint32_t*>(&h);
      }
      out = make_uint4(o[0], o[1], o[2], o[3]);
    }
    *reinterpret_cast<uint4*>(dst) = out;
  }
}

// y[t][r] = sum over slots (in slot order) of gate[t][s] * o[t, s][r], where o is the sum of
// the down projection's k-slice partials (in slice order).  fp32.
__global__ void combine_kernel(const float* __restrict__ O, const int32_t* __restrict__ inv,
                               const float* __restrict__ gate, const int32_t* __restrict__ meta,
                               int T, int k, int H, int kslices, long long slice,
                               float* __restrict__ y) {
  griddep_wait();  // O is written by the down projection launched just before
  const int t = blockIdx.y;
  const bool bad = meta[2] != 0;
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < H; r += gridDim.x * blockDim.x) {
    float acc = 0.0f;
    for (int s = 0; s < k; ++s) {
      const int pos = inv[t * k + s];
      if (pos < 0 || bad) continue;
      if (!PW_CHECK(static_cast<long long>(pos) * H < slice)) continue;
      float o = 0.0f;
      for (int j = 0; j < kslices; ++j) o += O[j * slice + static_cast<size_t>(pos) * H + r];
      acc = fmaf(gate[t * k + s], o, acc);
    }
    y[static_cast<size_t>(t) * H + r] = acc;
  }
}

}  // namespace pw
