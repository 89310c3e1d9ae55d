// K4: fused any-precision grouped expert GEMV (PagedWeight, "Composants Clés" 1 and 3: one
// fused kernel reads the bit-planes and LUTs directly, each block at its own bitwidth).
//
// Work item = (active expert, 32-row tile).  A tile is two 16-row segments: for gate_up the
// gate rows [16i, 16i+16) and the matching up rows [I+16i, I+16i+16) (so SiLU(gate)*up is
// formed in the epilogue); for down the rows [32i, 32i+32).  Each decode thread owns one row
// (its lane) and keeps that row's LUT, converted to fp32, in shared memory laid out
// lane-interleaved (entry v of lane L at word 32v+L), so the per-weight gather is free of
// bank conflicts.  A producer warp streams, per 1024-column stage, the top-q bit-planes of
// the 32 rows with 2-D TMA copies (128-byte swizzle) and the matching activation chunk with
// 1-D bulk copies, through a ring of mbarrier-guarded stages.  Four decode warps split each
// stage's columns, rebuild the q-bit indices, gather from the LUT and accumulate in fp32;
// the four partial sums are added in a fixed order.
#pragma once
#include "pw_common.cuh"

namespace pw {
namespace k4 {

constexpr int kRows = 32;
constexpr int kSegRows = 16;
constexpr int kStageWords = 32;                          // words per row per plane per stage
constexpr int kStageCols = kStageWords * 32;             // 1024 columns
constexpr int kStages = 3;
constexpr int kTok = 2;                                  // tokens per pass over a tile
constexpr int kDecodeWarps = 4;
constexpr int kThreads = (kDecodeWarps + 1) * 32;
constexpr int kBoxBytes = kSegRows * kStageWords * 4;    // one 16-row TMA box
constexpr int kPlaneBytes = kRows * kStageWords * 4;     // one plane of a stage
constexpr int kStagePlaneBytes = PW_MAX_BITS * kPlaneBytes;
constexpr int kStageXBytes = kTok * kStageCols * 4;
constexpr int kStageBytes = kStagePlaneBytes + kStageXBytes;
constexpr int kLutBytes = 256 * kRows * 4;
constexpr int kLutStageBytes = kRows * 256 * 2;
constexpr int kRedBytes = kDecodeWarps * kTok * 32 * 4;
constexpr int kBarBytes = (2 * kStages + 4) * 8 + 16;
constexpr int kSmemBytes =
    1024 + kStages * kStageBytes + kLutBytes + 2 * kLutStageBytes + kRedBytes + kBarBytes;
static_assert(kStageBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

struct Params {
  const pw_page_table* pt;
  int layer;
  int E;
  int rows;      // expected block rows (2I or H)
  int cols;      // expected block cols (H or I)
  int half;      // gate_up: I (offset of the up rows); down: 0
  int tiles;     // work items per expert
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* meta;
  const float* act;  // [pos][ld_act] fp32 activations, zero beyond cols
  int ld_act;
  float* out;        // gate_up: h [pos][ld_out]; down: partial [pos][ld_out]
  int ld_out;
};

struct Item {
  const pw_block* blk;
  const uint16_t* lut;
  int q, tile, te, pos0, segA, segB;
  bool valid;
};

template <int MODE>
__device__ __forceinline__ Item resolve(const Params& p, int item) {
  Item it;
  const int a = item / p.tiles;
  it.tile = item - a * p.tiles;
  const int e = p.active[a];
  it.blk = p.pt->blocks + (static_cast<size_t>(p.layer) * p.E + e) * 2 + MODE;
  const pw_block* b = it.blk;
  it.q = b->committed_bits;
  it.te = p.counts[e];
  it.pos0 = p.offsets[e];
  if (MODE == MODE_GATE_UP) {
    it.segA = it.tile * kSegRows;
    it.segB = p.half + it.tile * kSegRows;
  } else {
    it.segA = it.tile * kRows;
    it.segB = it.segA + kSegRows;
  }
  const bool bits_ok = it.q >= b->min_bits && it.q <= b->parent_bits && it.q >= 1 &&
                       it.q <= PW_MAX_BITS && b->lut[it.q] != nullptr && b->planes != nullptr;
  const bool shape_ok = static_cast<int>(b->rows) == p.rows && static_cast<int>(b->cols) == p.cols;
  it.lut = bits_ok ? b->lut[it.q] : nullptr;
  it.valid = bits_ok && shape_ok && b->state == PW_PAGE_GPU;
  return it;
}

template <int MODE>
__device__ __forceinline__ int item_status(const Item& it, const Params& p) {
  const pw_block* b = it.blk;
  if (static_cast<int>(b->rows) != p.rows || static_cast<int>(b->cols) != p.cols)
    return PW_ERR_INVALID_ARG;
  if (b->state != PW_PAGE_GPU) return PW_ERR_NOT_RESIDENT;
  return PW_ERR_BAD_BITS;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (!mbar_wait(bar, parity)) {
    *abort_flag = 1;
    return false;
  }
  return true;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) ffn_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  float* lut_s = reinterpret_cast<float*>(smem + kStages * kStageBytes);
  uint16_t* lut_stage = reinterpret_cast<uint16_t*>(smem + kStages * kStageBytes + kLutBytes);
  float* red = reinterpret_cast<float*>(smem + kStages * kStageBytes + kLutBytes +
                                        2 * kLutStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + kDecodeWarps * kTok * 32);
  uint64_t* empty = full + kStages;
  uint64_t* lut_full = empty + kStages;
  uint64_t* lut_empty = lut_full + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(lut_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecodeWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&lut_full[b], 1);
      mbar_init(&lut_empty[b], kDecodeWarps);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  const int n_items = p.meta[0] * p.tiles;
  const int nst = (p.cols + kStageCols - 1) / kStageCols;

  if (warp == kDecodeWarps) {
    // ---------------- producer: one thread issues every copy ----------------
    if (lane != 0) return;
    uint32_t g = 0, lc = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = resolve<MODE>(p, item);
      if (!it.valid) continue;
      const void* desc = it.blk->tma_desc;
      prefetch_desc(desc);
      const int lb = lc & 1;
      wait_bar(&lut_empty[lb], ((lc >> 1) & 1) ^ 1, abort_flag);
      const uint32_t seg_lut = static_cast<uint32_t>(kSegRows) << it.q << 1;  // bytes
      uint16_t* ls = lut_stage + lb * (kLutStageBytes / 2);
      mbar_arrive_expect_tx(&lut_full[lb], 2 * seg_lut);
      bulk_g2s(ls, it.lut + (static_cast<size_t>(it.segA) << it.q), seg_lut, &lut_full[lb]);
      bulk_g2s(ls + (kSegRows << it.q), it.lut + (static_cast<size_t>(it.segB) << it.q), seg_lut,
               &lut_full[lb]);
      ++lc;
      for (int ch = 0; ch < it.te; ch += kTok) {
        const int ntok = min(kTok, it.te - ch);
        for (int s = 0; s < nst; ++s, ++g) {
          const int slot = g % kStages;
          wait_bar(&empty[slot], ((g / kStages) & 1) ^ 1, abort_flag);
          uint8_t* st = stages + slot * kStageBytes;
          mbar_arrive_expect_tx(&full[slot], it.q * kPlaneBytes + ntok * kStageCols * 4);
          for (int pl = 0; pl < it.q; ++pl) {
            tma_g2s_2d(st + pl * kPlaneBytes, desc, s * kStageWords, pl * p.rows + it.segA,
                       &full[slot]);
            tma_g2s_2d(st + pl * kPlaneBytes + kBoxBytes, desc, s * kStageWords,
                       pl * p.rows + it.segB, &full[slot]);
          }
          for (int t = 0; t < ntok; ++t)
            bulk_g2s(st + kStagePlaneBytes + t * kStageCols * 4,
                     p.act + static_cast<size_t>(it.pos0 + ch + t) * p.ld_act +
                         static_cast<size_t>(s) * kStageCols,
                     kStageCols * 4, &full[slot]);
        }
      }
    }
    // drain: every issued stage has landed before the block exits
    for (uint32_t d = (g > kStages ? g - kStages : 0); d < g; ++d)
      wait_bar(&full[d % kStages], (d / kStages) & 1, abort_flag);
    return;
  }

  // ---------------- decode warps ----------------
  const int tid = threadIdx.x;  // 0..127
  uint32_t g = 0, lc = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const Item it = resolve<MODE>(p, item);
    if (!it.valid) {
      if (tid == 0) set_status(item_status<MODE>(it, p));
      for (int i = tid; i < it.te * kRows; i += kDecodeWarps * 32) {
        const int t = i / kRows, r = i - t * kRows;
        const size_t row = static_cast<size_t>(it.pos0 + t) * p.ld_out;
        if (MODE == MODE_GATE_UP) {
          if (r < kSegRows) p.out[row + it.tile * kSegRows + r] = 0.0f;
        } else {
          p.out[row + it.tile * kRows + r] = 0.0f;
        }
      }
      continue;
    }
    const int q = it.q;
    const int nv = 1 << q;
    named_sync(1, kDecodeWarps * 32);  // previous item's LUT no longer in use
    const int lb = lc & 1;
    wait_bar(&lut_full[lb], (lc >> 1) & 1, abort_flag);
    const uint16_t* ls = lut_stage + lb * (kLutStageBytes / 2);
    for (int i = tid; i < kRows * nv; i += kDecodeWarps * 32) {
      const int r = i & 31, v = i >> 5;
      lut_s[v * 32 + r] = f16_to_f32(ls[(r << q) + v]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&lut_empty[lb]);
    named_sync(1, kDecodeWarps * 32);
    ++lc;

    for (int ch = 0; ch < it.te; ch += kTok) {
      const int ntok = min(kTok, it.te - ch);
      float acc[kTok];
#pragma unroll
      for (int t = 0; t < kTok; ++t) acc[t] = 0.0f;
      for (int s = 0; s < nst; ++s, ++g) {
        const int slot = g % kStages;
        wait_bar(&full[slot], (g / kStages) & 1, abort_flag);
        const uint32_t* st = reinterpret_cast<const uint32_t*>(stages + slot * kStageBytes);
        const float* xs = reinterpret_cast<const float*>(stages + slot * kStageBytes +
                                                         kStagePlaneBytes);
        for (int i = 0; i < 8; ++i) {
          const int word = warp * 8 + i;
          // 128-byte swizzle: 16-byte chunk index XOR (row % 8)
          const int off = lane * kStageWords + (((word >> 2) ^ (lane & 7)) << 2) + (word & 3);
          uint32_t P[PW_MAX_BITS];
          for (int pl = 0; pl < q; ++pl) P[pl] = st[pl * (kPlaneBytes / 4) + off];
          for (int j = 0; j < 32; ++j) {
            uint32_t v = 0;
            for (int pl = 0; pl < q; ++pl) v = (v << 1) | ((P[pl] >> j) & 1u);
            const float w = lut_s[v * 32 + lane];
            const int col = word * 32 + j;
            for (int t = 0; t < ntok; ++t) acc[t] = fmaf(w, xs[t * kStageCols + col], acc[t]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
#pragma unroll
      for (int t = 0; t < kTok; ++t) red[(warp * kTok + t) * 32 + lane] = acc[t];
      named_sync(1, kDecodeWarps * 32);
      if (warp == 0) {
        for (int t = 0; t < ntok; ++t) {
          float tot = 0.0f;
#pragma unroll
          for (int w = 0; w < kDecodeWarps; ++w) tot += red[(w * kTok + t) * 32 + lane];
          const size_t row = static_cast<size_t>(it.pos0 + ch + t) * p.ld_out;
          if (MODE == MODE_GATE_UP) {
            const float u = __shfl_down_sync(0xffffffffu, tot, 16);
            if (lane < kSegRows) {
              const float h = tot / (1.0f + expf(-tot)) * u;
              p.out[row + it.tile * kSegRows + lane] = h;
            }
          } else {
            p.out[row + it.tile * kRows + lane] = tot;
          }
        }
      }
      named_sync(1, kDecodeWarps * 32);
    }
  }
}

}  // namespace k4
}  // namespace pw
