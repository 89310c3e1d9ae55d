// K4: fused any-precision grouped expert GEMV (PagedWeight, "Composants Clés" 1 and 3: one
// fused kernel reads the bit-planes and LUTs directly, each block at its own bitwidth).
//
// Work item = (active expert, 32-row tile, k-slice).  A tile is two 16-row segments: for
// gate_up the gate rows [16i, 16i+16) and the matching up rows [I+16i, I+16i+16), so that
// SiLU(gate) * up is formed in the epilogue (gate_up is never split along k); for down the
// rows [32i, 32i+32), optionally split into k-slices whose partial sums the combine adds.
//
// Each decode thread owns one row (its lane).  The row's q-bit LUT lives in shared memory as
// fp32, lane-interleaved with a 256-byte entry stride (entry v of lane L in buffer u at byte
// 256v + 128u + 4L), so every per-weight gather is bank-conflict free and its address is one
// byte permute of an index byte.  A producer warp streams, per 1024-column stage, the top-q
// bit-planes of the 32 rows with 2-D TMA copies (128-byte swizzle) and the stage's activation
// chunk with 1-D bulk copies, through a ring of mbarrier-guarded stages.  Eight decode warps
// take 128 columns each: one 16-byte shared load per plane, an 8x8 bit-matrix transpose per
// 32 columns turns the q plane words into 32 byte-sized indices, and packed fp32x2 FMAs
// accumulate.  The transpose emits columns in the order 8b+i -> slot 4i+b inside each group of
// 32; activations are stored in that order (see xslot()) so one broadcast 16-byte load feeds
// four weights.  The eight partial sums of a row are added in a fixed order.
#pragma once
#include "pw_common.cuh"

namespace pw {
namespace k4 {

constexpr int kRows = 32;
constexpr int kSegRows = 16;
constexpr int kStageWords = 32;                          // words per row per plane per stage
constexpr int kStageCols = kStageWords * 32;             // 1024 columns
constexpr int kDecodeWarps = 8;
constexpr int kWarpWords = kStageWords / kDecodeWarps;   // 4 words = 128 columns per warp
constexpr int kThreads = (kDecodeWarps + 1) * 32;
constexpr int kBoxBytes = kSegRows * kStageWords * 4;    // one 16-row TMA box
constexpr int kPlaneBytes = kRows * kStageWords * 4;     // one plane of a stage
constexpr int kStagePlaneBytes = PW_MAX_BITS * kPlaneBytes;
constexpr int kLutBytes = 256 * 256;                     // 2^8 entries x 256-byte stride
constexpr int kLutStageBytes = kRows * 256 * 2;          // fp16 staging of one tile's LUT
constexpr int kMaxKSlices = 8;

// slot of column c inside the decode order (a permutation inside each 32-column group)
__host__ __device__ __forceinline__ int xslot(int c) {
  return (c & ~31) | ((c & 7) << 2) | ((c >> 3) & 3);
}

template <int NTP>
struct Layout {
  static constexpr int kStages = NTP >= 4 ? 2 : 3;
  static constexpr int kStageXBytes = NTP * kStageCols * 4;
  static constexpr int kStageBytes = kStagePlaneBytes + kStageXBytes;
  static constexpr int kOffLut = 0;
  static constexpr int kOffStages = kLutBytes;
  static constexpr int kOffLutStage = kOffStages + kStages * kStageBytes;
  static constexpr int kOffRed = kOffLutStage + kLutStageBytes;
  static constexpr int kRedBytes = kDecodeWarps * NTP * 32 * 4;
  static constexpr int kOffBar = kOffRed + kRedBytes;
  static constexpr int kBarBytes = (2 * kStages + 2) * 8 + 16;
  static constexpr int kSmem = kOffBar + kBarBytes;
  static_assert(kStageBytes % 1024 == 0 && kOffStages % 1024 == 0, "swizzle alignment");
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

struct Params {
  const pw_page_table* pt;
  int layer;
  int E;
  int mode;      // MODE_GATE_UP or MODE_DOWN
  int rows;      // expected block rows (2I or H)
  int cols;      // expected block cols (H or I)
  int half;      // gate_up: I (offset of the up rows); down: 0
  int tiles;     // row tiles per expert
  int kslices;   // k-slices per tile (1 for gate_up)
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* meta;
  const float* act;  // [pos][ld_act] fp32 activations in decode order, zero beyond cols
  int ld_act;
  float* out;        // gate_up: h [pos][ld_out] (decode order); down: [kslice][pos][ld_out]
  int ld_out;
  long long out_slice;  // elements between k-slices of `out`
};

struct Item {
  const pw_block* blk;
  const uint16_t* lut;
  int q, tile, ks, te, pos0, segA, segB, s0, s1;
  bool valid;
};

__device__ __forceinline__ Item resolve(const Params& p, int item, int nst) {
  Item it;
  const int per_expert = p.tiles * p.kslices;
  const int a = item / per_expert;
  const int rem = item - a * per_expert;
  it.tile = rem / p.kslices;
  it.ks = rem - it.tile * p.kslices;
  const int e = p.active[a];
  it.blk = p.pt->blocks + (static_cast<size_t>(p.layer) * p.E + e) * 2 + p.mode;
  const pw_block* b = it.blk;
  it.q = b->committed_bits;
  it.te = p.counts[e];
  it.pos0 = p.offsets[e];
  if (p.mode == MODE_GATE_UP) {
    it.segA = it.tile * kSegRows;
    it.segB = p.half + it.tile * kSegRows;
  } else {
    it.segA = it.tile * kRows;
    it.segB = it.segA + kSegRows;
  }
  it.s0 = (nst * it.ks) / p.kslices;
  it.s1 = (nst * (it.ks + 1)) / p.kslices;
  const bool bits_ok = it.q >= b->min_bits && it.q <= b->parent_bits && it.q >= PW_MIN_BITS &&
                       it.q <= PW_MAX_BITS && b->lut[it.q] != nullptr && b->planes != nullptr;
  const bool shape_ok = static_cast<int>(b->rows) == p.rows && static_cast<int>(b->cols) == p.cols;
  it.lut = bits_ok ? b->lut[it.q] : nullptr;
  it.valid = bits_ok && shape_ok && b->state == PW_PAGE_GPU;
  return it;
}

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

// Exchange the bits of a selected by (m << S) with the bits of b selected by m.
template <int S, uint32_t M>
__device__ __forceinline__ void bswap(uint32_t& a, uint32_t& b) {
  constexpr uint32_t MH = M << S;
  const uint32_t an = (a & ~MH) | ((b << S) & MH);
  const uint32_t bn = (b & ~M) | ((a >> S) & M);
  a = an;
  b = bn;
}

// Per byte lane, an 8x8 bit transpose across R[0..7]: afterwards bit j of byte k of R[i] is
// what bit i of byte k of R[j] was.
__device__ __forceinline__ void transpose8(uint32_t (&R)[8]) {
  bswap<4, 0x0F0F0F0Fu>(R[0], R[4]);
  bswap<4, 0x0F0F0F0Fu>(R[1], R[5]);
  bswap<4, 0x0F0F0F0Fu>(R[2], R[6]);
  bswap<4, 0x0F0F0F0Fu>(R[3], R[7]);
  bswap<2, 0x33333333u>(R[0], R[2]);
  bswap<2, 0x33333333u>(R[1], R[3]);
  bswap<2, 0x33333333u>(R[4], R[6]);
  bswap<2, 0x33333333u>(R[5], R[7]);
  bswap<1, 0x55555555u>(R[0], R[1]);
  bswap<1, 0x55555555u>(R[2], R[3]);
  bswap<1, 0x55555555u>(R[4], R[5]);
  bswap<1, 0x55555555u>(R[6], R[7]);
}

__device__ __forceinline__ uint32_t comp(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// One stage, one warp: its 4 words (128 columns) of every plane, NT tokens.
template <int Q, int NT>
__device__ __forceinline__ void decode_stage(const uint8_t* __restrict__ planes,
                                             const float* __restrict__ xs, int x_stride,
                                             const uint8_t* __restrict__ lut,
                                             uint32_t lane_base, int warp, int lane,
                                             float2 (&acc)[NT][2]) {
  const uint32_t chunk = lane * 128 + ((warp ^ (lane & 7)) << 4);  // 128-byte swizzle
  uint4 P[Q];
#pragma unroll
  for (int p = 0; p < Q; ++p)
    P[p] = *reinterpret_cast<const uint4*>(planes + p * kPlaneBytes + chunk);
#pragma unroll
  for (int wi = 0; wi < kWarpWords; ++wi) {
    uint32_t R[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) R[j] = (j < Q) ? comp(P[Q - 1 - j], wi) : 0u;
    transpose8(R);
    const float* xw = xs + (warp * kWarpWords + wi) * 32;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float w[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t addr = __byte_perm(R[i], lane_base, 0x7604u | (b << 4));
        w[b] = *reinterpret_cast<const float*>(lut + addr);
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float4 xv = *reinterpret_cast<const float4*>(xw + t * x_stride + 4 * i);
        acc[t][0] = __ffma2_rn(make_float2(w[0], w[1]), make_float2(xv.x, xv.y), acc[t][0]);
        acc[t][1] = __ffma2_rn(make_float2(w[2], w[3]), make_float2(xv.z, xv.w), acc[t][1]);
      }
    }
  }
}

template <int Q, int NT>
__device__ __noinline__ void run_stages(const Params& p, const Item& it, uint8_t* smem,
                                        uint64_t* full, uint64_t* empty, volatile int* abort_flag,
                                        uint32_t& g, int n_stages, int stage_bytes, int x_stride,
                                        uint32_t lane_base, int words_total, float (&part)[4]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float2 acc[NT][2];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = make_float2(0.f, 0.f);
  for (int s = it.s0; s < it.s1; ++s, ++g) {
    const int slot = g % n_stages;
    wait_bar(&full[slot], (g / n_stages) & 1, abort_flag);
    const uint8_t* st = smem + kLutBytes + slot * stage_bytes;
    const float* xs = reinterpret_cast<const float*>(st + kStagePlaneBytes);
    if ((s * kStageWords + warp * kWarpWords) < words_total)
      decode_stage<Q, NT>(st, xs, x_stride, smem, lane_base, warp, lane, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) part[t] = (acc[t][0].x + acc[t][0].y) + (acc[t][1].x + acc[t][1].y);
}

template <int NT>
__device__ __forceinline__ void run_q(int q, const Params& p, const Item& it, uint8_t* smem,
                                      uint64_t* full, uint64_t* empty, volatile int* abort_flag,
                                      uint32_t& g, int n_stages, int stage_bytes, int x_stride,
                                      uint32_t lane_base, int words_total, float (&part)[4]) {
  switch (q) {
    case 3: run_stages<3, NT>(p, it, smem, full, empty, abort_flag, g, n_stages, stage_bytes, x_stride, lane_base, words_total, part); break;
    case 4: run_stages<4, NT>(p, it, smem, full, empty, abort_flag, g, n_stages, stage_bytes, x_stride, lane_base, words_total, part); break;
    case 5: run_stages<5, NT>(p, it, smem, full, empty, abort_flag, g, n_stages, stage_bytes, x_stride, lane_base, words_total, part); break;
    case 6: run_stages<6, NT>(p, it, smem, full, empty, abort_flag, g, n_stages, stage_bytes, x_stride, lane_base, words_total, part); break;
    case 7: run_stages<7, NT>(p, it, smem, full, empty, abort_flag, g, n_stages, stage_bytes, x_stride, lane_base, words_total, part); break;
    default: run_stages<8, NT>(p, it, smem, full, empty, abort_flag, g, n_stages, stage_bytes, x_stride, lane_base, words_total, part); break;
  }
}

template <int NTP>
__global__ void __launch_bounds__(kThreads, 1) ffn_kernel(const Params p) {
  using LY = Layout<NTP>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* stages = smem + LY::kOffStages;
  uint16_t* lut_stage = reinterpret_cast<uint16_t*>(smem + LY::kOffLutStage);
  float* red = reinterpret_cast<float*>(smem + LY::kOffRed);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::kOffBar);
  uint64_t* empty = full + LY::kStages;
  uint64_t* lut_full = empty + LY::kStages;
  uint64_t* lut_empty = lut_full + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(lut_empty + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {  // the swizzled TMA layout needs 1 KB alignment
    if (threadIdx.x == 0) set_status(PW_ERR_UNSUPPORTED);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < LY::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecodeWarps);
    }
    mbar_init(lut_full, 1);
    mbar_init(lut_empty, kDecodeWarps);
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  const int nst = (p.cols + kStageCols - 1) / kStageCols;
  const int words_total = p.cols / 32;
  const int n_items = p.meta[0] * p.tiles * p.kslices;

  if (warp == kDecodeWarps) {
    // ---------------- producer: one thread issues every copy ----------------
    if (lane != 0) return;
    uint32_t g = 0, lc = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = resolve(p, item, nst);
      if (!it.valid) continue;
      const void* desc = it.blk->tma_desc;
      prefetch_desc(desc);
      wait_bar(lut_empty, (lc & 1) ^ 1, abort_flag);
      const uint32_t seg_lut = static_cast<uint32_t>(kSegRows) << it.q << 1;  // bytes
      mbar_arrive_expect_tx(lut_full, 2 * seg_lut);
      bulk_g2s(lut_stage, it.lut + (static_cast<size_t>(it.segA) << it.q), seg_lut, lut_full);
      bulk_g2s(lut_stage + (kSegRows << it.q), it.lut + (static_cast<size_t>(it.segB) << it.q),
               seg_lut, lut_full);
      ++lc;
      for (int ch = 0; ch < it.te; ch += NTP) {
        const int ntok = min(NTP, it.te - ch);
        for (int s = it.s0; s < it.s1; ++s, ++g) {
          const int slot = g % LY::kStages;
          wait_bar(&empty[slot], ((g / LY::kStages) & 1) ^ 1, abort_flag);
          uint8_t* st = stages + slot * LY::kStageBytes;
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
    for (uint32_t d = (g > LY::kStages ? g - LY::kStages : 0); d < g; ++d)
      wait_bar(&full[d % LY::kStages], (d / LY::kStages) & 1, abort_flag);
    return;
  }

  // ---------------- decode warps ----------------
  const int tid = threadIdx.x;
  const int ndec = kDecodeWarps * 32;
  uint32_t g = 0, lc = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const Item it = resolve(p, item, nst);
    if (!it.valid) {
      if (tid == 0) set_status(item_status(it, p));
      for (int i = tid; i < it.te * kRows; i += ndec) {
        const int t = i / kRows, r = i - t * kRows;
        if (p.mode == MODE_GATE_UP) {
          if (r < kSegRows)
            p.out[static_cast<size_t>(it.pos0 + t) * p.ld_out + xslot(it.tile * kSegRows + r)] = 0.f;
        } else {
          p.out[it.ks * p.out_slice + static_cast<size_t>(it.pos0 + t) * p.ld_out +
                it.tile * kRows + r] = 0.f;
        }
      }
      continue;
    }
    const int q = it.q;
    const int nv = 1 << q;
    const uint32_t u = lc & 1;
    wait_bar(lut_full, lc & 1, abort_flag);
    {  // fp16 [32 rows][2^q] -> fp32 lane-interleaved, rows on lanes, entries on a diagonal
      const int per_warp = nv / kDecodeWarps > 0 ? nv / kDecodeWarps : 1;
      const int it0 = warp * per_warp;
      for (int k = 0; k < per_warp && it0 + k < nv; ++k) {
        const int v = (lane + it0 + k) & (nv - 1);
        const float f = f16_to_f32(lut_stage[(lane << q) + v]);
        *reinterpret_cast<float*>(smem + v * 256 + u * 128 + lane * 4) = f;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(lut_empty);
    named_sync(1, ndec);
    ++lc;
    const uint32_t lane_base = u * 128 + lane * 4;

    for (int ch = 0; ch < it.te; ch += NTP) {
      const int ntok = min(NTP, it.te - ch);
      float part[4] = {0.f, 0.f, 0.f, 0.f};
      const int xstride = kStageCols;
      if (NTP == 1 || ntok == 1)
        run_q<1>(q, p, it, smem, full, empty, abort_flag, g, LY::kStages, LY::kStageBytes,
                 xstride, lane_base, words_total, part);
      else if (NTP >= 2 && ntok == 2)
        run_q<(NTP >= 2 ? 2 : 1)>(q, p, it, smem, full, empty, abort_flag, g, LY::kStages,
                                  LY::kStageBytes, xstride, lane_base, words_total, part);
      else if (NTP >= 4 && ntok == 3)
        run_q<(NTP >= 4 ? 3 : 1)>(q, p, it, smem, full, empty, abort_flag, g, LY::kStages,
                                  LY::kStageBytes, xstride, lane_base, words_total, part);
      else
        run_q<(NTP >= 4 ? 4 : 1)>(q, p, it, smem, full, empty, abort_flag, g, LY::kStages,
                                  LY::kStageBytes, xstride, lane_base, words_total, part);
#pragma unroll
      for (int t = 0; t < NTP; ++t) red[(warp * NTP + t) * 32 + lane] = part[t];
      named_sync(1, ndec);
      if (warp == 0) {
        for (int t = 0; t < ntok; ++t) {
          float tot = 0.f;
#pragma unroll
          for (int w = 0; w < kDecodeWarps; ++w) tot += red[(w * NTP + t) * 32 + lane];
          const size_t row = static_cast<size_t>(it.pos0 + ch + t) * p.ld_out;
          if (p.mode == MODE_GATE_UP) {
            const float up = __shfl_down_sync(0xffffffffu, tot, 16);
            if (lane < kSegRows) {
              const float h = tot / (1.0f + expf(-tot)) * up;
              p.out[row + xslot(it.tile * kSegRows + lane)] = h;
            }
          } else {
            p.out[it.ks * p.out_slice + row + it.tile * kRows + lane] = tot;
          }
        }
      }
      named_sync(1, ndec);
    }
  }
}

}  // namespace k4
}  // namespace pw
