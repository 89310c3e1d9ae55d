// K4: fused any-precision grouped expert GEMV (PagedWeight, "Composants Clés" 1 and 3: one
// fused kernel reads the bit-planes and LUTs directly, each block at its own bitwidth).
//
// Work item = (active expert, 32-row tile, k-slice).  A tile is two 16-row segments: for
// gate_up the gate rows [16i, 16i+16) and the matching up rows [I+16i, I+16i+16), so that
// SiLU(gate) * up is formed in the epilogue (gate_up is never split along k); for down the
// rows [32i, 32i+32), optionally split into k-slices whose partial sums the combine adds.
//
// Warp roles (one CTA per SM, persistent over the items):
//   producer (1 warp)   resolves items from the Weight Page Table into a descriptor ring,
//                       prefetches each item's fp16 LUT one item ahead (1-D bulk copies, two
//                       staging buffers) and streams, per 1024-column stage, the top-q
//                       bit-planes of the 32 rows (2-D TMA, 128-byte swizzle) plus the stage's
//                       activation chunk through a ring of mbarrier-guarded stages;
//   LUT (2 warps)       turn each item's staged LUT into its decode table in one of two table
//                       buffers, then signal it ready; a buffer is rewritten only after every
//                       decode warp has released it, so decode warps never meet a CTA barrier;
//   decode (16 warps)   take 64 columns of each stage; each thread owns one row (its lane).
// Three decode paths, chosen per block by its committed q:
//   q >= 5  an 8x8 bit-matrix transpose of the q plane words (per 32 columns) yields one index
//           byte per weight; the table is fp32, lane-interleaved with a 256-byte entry stride
//           (entry v of lane L in buffer u at byte 256v + 128u + 4L), so a gather is bank
//           conflict free and its address is one byte permute of the index byte;
//   q == 4  a 4x8 transpose yields index nibbles; two nibbles form a byte that indexes a pair
//           table of 256 half2 entries (LUT[a], LUT[b]) laid out the same way; one gather per
//           two weights;
//   q == 3  the 8-entry LUT lives in registers as low-byte and high-byte tables; byte permutes
//           with the nibble indices as selectors look up four weights at a time.
// Packed fp32x2 FMAs accumulate.  The decode emits columns as pairs (8b+i, 8b+4+i);
// activations are stored so every such pair is adjacent (xslot()), two pairs per 16-byte
// broadcast load.  The sixteen per-warp partial sums of a row are added in a fixed order by
// whichever decode warp finishes the pass last.
#pragma once
#include "pw_common.cuh"

namespace pw {
namespace k4 {

constexpr int kRows = 32;
constexpr int kSegRows = 16;
constexpr int kStageWords = 32;                          // words per row per plane per stage
constexpr int kStageCols = kStageWords * 32;             // 1024 columns
constexpr int kDecodeWarps = 16;
constexpr int kLutWarps = 2;
constexpr int kWarpWords = kStageWords / kDecodeWarps;   // 2 words = 64 columns per warp
constexpr int kLutWarp0 = kDecodeWarps;
constexpr int kProducerWarp = kDecodeWarps + kLutWarps;
constexpr int kThreads = (kProducerWarp + 1) * 32;
constexpr int kBoxBytes = kSegRows * kStageWords * 4;    // one 16-row TMA box
constexpr int kPlaneBytes = kRows * kStageWords * 4;     // one plane of a stage
constexpr int kStagePlaneBytes = PW_MAX_BITS * kPlaneBytes;
constexpr int kLutBytes = 256 * 256;                     // 2^8 entries x 256-byte stride
constexpr int kLutStageBytes = kRows * 256 * 2;          // fp16 staging of one tile's LUT
constexpr int kMaxKSlices = 8;
constexpr int kDescRing = 4;

// The kernel's dynamic shared memory, named directly (not through a pointer) wherever the
// decode loop indexes it, so every table gather is one load with a constant base folded in.
extern __shared__ __align__(1024) uint8_t g_smem[];

// Slot of column c in the activation layout the decode reads: inside each 32-column group,
// columns 8b+i and 8b+4+i (i < 4) sit at slots 8i+2b and 8i+2b+1.
__host__ __device__ __forceinline__ int xslot(int c) {
  const int l = c & 31;
  return (c & ~31) | ((l & 3) << 3) | (((l >> 3) & 3) << 1) | ((l >> 2) & 1);
}

// A stage slot holds either one 1024-column stage (all q) or, in the one-token kernel, a
// double-width 2048-column stage for blocks with q <= 4, laid out as two 1024-column halves
// (planes of half h at h*q*kPlaneBytes; activations of half h at kStagePlaneBytes + h*4 KB),
// so that low-bitwidth blocks keep as many bytes in flight as high-bitwidth ones.
template <int NTP>
struct Layout {
  static constexpr int kStages = NTP >= 4 ? 2 : 3;
  static constexpr bool kWide = NTP == 1;
  static constexpr int kStageXBytes = (kWide ? 2 : NTP) * kStageCols * 4;
  static constexpr int kStageBytes = kStagePlaneBytes + kStageXBytes;
  static constexpr int kOffLut = 0;
  static constexpr int kOffStages = kLutBytes;
  static constexpr int kOffLutStage = kOffStages + kStages * kStageBytes;
  static constexpr int kOffRed = kOffLutStage + 2 * kLutStageBytes;
  static constexpr int kRedBytes = 2 * kDecodeWarps * NTP * 32 * 4;
  static constexpr int kOffDesc = kOffRed + kRedBytes;
  static constexpr int kDescBytes = 2 * kDescRing * 48;
  static constexpr int kOffBar = kOffDesc + kDescBytes;
  static constexpr int kBarBytes = (2 * kStages + 8) * 8 + 32;
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
  const float* act;  // [pos][ld_act] fp32 activations in xslot order, zero beyond cols
  int ld_act;
  float* out;        // gate_up: h [pos][ld_out] (xslot order); down: [kslice][pos][ld_out]
  int ld_out;
  long long out_slice;  // elements between k-slices of `out`
};

// What the producer tells the LUT and decode warps about an item (shared-memory rings).
struct Desc {
  int valid, status, q, te, pos0, tile, ks, s0, s1, w, pad1, pad2;
};
static_assert(sizeof(Desc) == 48, "descriptor size");

struct Item {
  const pw_block* blk;
  const uint16_t* lut;
  int q, tile, ks, te, pos0, segA, segB, s0, s1, w, status;
  bool valid;
};

// wide: the kernel uses double-width stages for q <= 4.
__device__ __forceinline__ Item resolve(const Params& p, int item, bool wide) {
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
  it.w = (wide && it.q <= 4) ? 2 : 1;
  const int scols = kStageCols * it.w;
  const int nst = (p.cols + scols - 1) / scols;
  it.s0 = (nst * it.ks) / p.kslices;
  it.s1 = (nst * (it.ks + 1)) / p.kslices;
  const bool bits_ok = it.q >= b->min_bits && it.q <= b->parent_bits && it.q >= PW_MIN_BITS &&
                       it.q <= PW_MAX_BITS && b->lut[it.q] != nullptr && b->planes != nullptr;
  const bool shape_ok = static_cast<int>(b->rows) == p.rows && static_cast<int>(b->cols) == p.cols;
  const bool resident = b->state == PW_PAGE_GPU;
  it.lut = bits_ok ? b->lut[it.q] : nullptr;
  it.valid = bits_ok && shape_ok && resident;
  it.status = !shape_ok ? PW_ERR_INVALID_ARG : (!resident ? PW_ERR_NOT_RESIDENT : PW_ERR_BAD_BITS);
  return it;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (!mbar_wait(bar, parity)) {
    *abort_flag = 1;
    return false;
  }
  return true;
}

// Exchange the bits of a selected by (M << S) with the bits of b selected by M.
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

// Per nibble lane, a 4x4 bit transpose across R[0..3]: afterwards bit j of nibble n of R[i] is
// what bit i of nibble n of R[j] was.
__device__ __forceinline__ void transpose4(uint32_t (&R)[4]) {
  bswap<2, 0x33333333u>(R[0], R[2]);
  bswap<2, 0x33333333u>(R[1], R[3]);
  bswap<1, 0x55555555u>(R[0], R[1]);
  bswap<1, 0x55555555u>(R[2], R[3]);
}

__device__ __forceinline__ float lds_f32(uint32_t off) {
  return *reinterpret_cast<const float*>(g_smem + off);
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(g_smem + off);
}
__device__ __forceinline__ float2 h2f2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}
__device__ __forceinline__ float2 lo2(const float4& v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4& v) { return make_float2(v.z, v.w); }

// One stage, one warp: its 2 words (64 columns) of every plane, NT tokens.
// planes_off / xs_off: byte offsets of the stage's planes and activations in g_smem.
// reg_lut: the q = 3 tables (low bytes of entries 0-3, 4-7, high bytes of 0-3, 4-7).
template <int Q, int NT>
__device__ __forceinline__ void decode_stage(uint32_t planes_off, uint32_t xs_off,
                                             uint32_t lane_base, const uint4& reg_lut, int warp,
                                             int lane, float2 (&acc)[NT][2]) {
  // 128-byte swizzle: 16-byte chunk index XOR (row % 8); this warp owns half a chunk
  const uint32_t off = planes_off + lane * 128 + (((warp >> 1) ^ (lane & 7)) << 4) +
                       ((warp & 1) << 3);
  uint2 P[Q];
#pragma unroll
  for (int p = 0; p < Q; ++p)
    P[p] = *reinterpret_cast<const uint2*>(g_smem + off + p * kPlaneBytes);
  constexpr int x_stride = kStageCols;
#pragma unroll
  for (int wi = 0; wi < kWarpWords; ++wi) {
    const float* xw =
        reinterpret_cast<const float*>(g_smem + xs_off) + (warp * kWarpWords + wi) * 32;
    if constexpr (Q >= 5) {
      uint32_t R[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) R[j] = (j < Q) ? (wi ? P[Q - 1 - j].y : P[Q - 1 - j].x) : 0u;
      transpose8(R);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 w[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const uint32_t sel = 0x7604u | (b << 4);
          w[b].x = lds_f32(__byte_perm(R[i], lane_base, sel));
          w[b].y = lds_f32(__byte_perm(R[i + 4], lane_base, sel));
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float4 xa = *reinterpret_cast<const float4*>(xw + t * x_stride + 8 * i);
          const float4 xb = *reinterpret_cast<const float4*>(xw + t * x_stride + 8 * i + 4);
          acc[t][0] = __ffma2_rn(w[0], lo2(xa), acc[t][0]);
          acc[t][1] = __ffma2_rn(w[1], hi2(xa), acc[t][1]);
          acc[t][0] = __ffma2_rn(w[2], lo2(xb), acc[t][0]);
          acc[t][1] = __ffma2_rn(w[3], hi2(xb), acc[t][1]);
        }
      }
    } else {
      uint32_t R[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) R[j] = (j < Q) ? (wi ? P[Q - 1 - j].y : P[Q - 1 - j].x) : 0u;
      transpose4(R);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 w[4];
        if constexpr (Q == 4) {
#pragma unroll
          for (int b = 0; b < 4; ++b)
            w[b] = h2f2(lds_u32(__byte_perm(R[i], lane_base, 0x7604u | (b << 4))));
        } else {
          const uint32_t r2 = R[i] >> 16;
          const uint32_t la = __byte_perm(reg_lut.x, reg_lut.y, R[i]);
          const uint32_t ha = __byte_perm(reg_lut.z, reg_lut.w, R[i]);
          const uint32_t lb = __byte_perm(reg_lut.x, reg_lut.y, r2);
          const uint32_t hb = __byte_perm(reg_lut.z, reg_lut.w, r2);
          w[0] = h2f2(__byte_perm(la, ha, 0x5140u));
          w[1] = h2f2(__byte_perm(la, ha, 0x7362u));
          w[2] = h2f2(__byte_perm(lb, hb, 0x5140u));
          w[3] = h2f2(__byte_perm(lb, hb, 0x7362u));
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float4 xa = *reinterpret_cast<const float4*>(xw + t * x_stride + 8 * i);
          const float4 xb = *reinterpret_cast<const float4*>(xw + t * x_stride + 8 * i + 4);
          acc[t][0] = __ffma2_rn(w[0], lo2(xa), acc[t][0]);
          acc[t][1] = __ffma2_rn(w[1], hi2(xa), acc[t][1]);
          acc[t][0] = __ffma2_rn(w[2], lo2(xb), acc[t][0]);
          acc[t][1] = __ffma2_rn(w[3], hi2(xb), acc[t][1]);
        }
      }
    }
  }
}

// The stage loop of one pass over an item, one decode warp.  Every argument is a scalar
// passed by value so nothing of it lives in local memory.  Returns the warp's partial sums
// (one per token); the caller advances its stage counter by s1 - s0.
template <int Q, int NT>
__device__ __noinline__ float4 run_stages(uint64_t* full, uint64_t* empty,
                                          volatile int* abort_flag, int n_stages, int stage_bytes,
                                          int words_total, uint32_t lane_base, uint32_t l0,
                                          uint32_t l1, uint32_t l2, uint32_t l3, int s0, int s1,
                                          uint32_t g, int w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4 reg_lut = make_uint4(l0, l1, l2, l3);
  float2 acc[NT][2];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = make_float2(0.f, 0.f);
  for (int s = s0; s < s1; ++s, ++g) {
    const int slot = g % n_stages;
    wait_bar(&full[slot], (g / n_stages) & 1, abort_flag);
    const uint32_t st = kLutBytes + slot * stage_bytes;
    for (int h = 0; h < w; ++h) {
      if (((s * w + h) * kStageWords + warp * kWarpWords) < words_total)
        decode_stage<Q, NT>(st + h * Q * kPlaneBytes, st + kStagePlaneBytes + h * kStageCols * 4,
                            lane_base, reg_lut, warp, lane, acc);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
  float r[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int t = 0; t < NT; ++t) r[t] = (acc[t][0].x + acc[t][1].x) + (acc[t][0].y + acc[t][1].y);
  return make_float4(r[0], r[1], r[2], r[3]);
}

#define PW_RUN_ARGS                                                                          \
  full, empty, abort_flag, LY::kStages, LY::kStageBytes, words_total, lane_base, reg_lut.x,  \
      reg_lut.y, reg_lut.z, reg_lut.w, d.s0, d.s1, g, d.w

template <int NT, int NTP>
__device__ __forceinline__ float4 run_q(const Desc& d, uint64_t* full, uint64_t* empty,
                                        volatile int* abort_flag, int words_total,
                                        uint32_t lane_base, const uint4& reg_lut, uint32_t g) {
  using LY = Layout<NTP>;
  switch (d.q) {
    case 3: return run_stages<3, NT>(PW_RUN_ARGS);
    case 4: return run_stages<4, NT>(PW_RUN_ARGS);
    case 5: return run_stages<5, NT>(PW_RUN_ARGS);
    case 6: return run_stages<6, NT>(PW_RUN_ARGS);
    case 7: return run_stages<7, NT>(PW_RUN_ARGS);
    default: return run_stages<8, NT>(PW_RUN_ARGS);
  }
}
#undef PW_RUN_ARGS

// LUT warp lw (0 or 1), lane = row: staged fp16 [32 rows][2^q] -> decode table in buffer u.
__device__ __forceinline__ void build_table(const uint16_t* __restrict__ ls, int q, uint32_t u,
                                            int lw, int lane) {
  const uint32_t col = u * 128 + lane * 4;
  if (q >= 5) {  // fp32 entries; rows on lanes, entries on a diagonal (conflict-free reads)
    const int nv = 1 << q, half = nv >> 1;
    for (int k = 0; k < half; ++k) {
      const int v = lw * half + ((lane + k) & (half - 1));
      *reinterpret_cast<float*>(g_smem + v * 256 + col) = f16_to_f32(ls[(lane << q) + v]);
    }
  } else if (q == 4) {  // pair entries a + 16b = (LUT[a], LUT[b]); warp lw takes b in [8lw, 8lw+8)
    const uint4* row = reinterpret_cast<const uint4*>(ls + (lane << 4));
    const uint4 v0 = row[0], v1 = row[1];
    const uint32_t lw8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    const uint4 hsrc = lw ? v1 : v0;  // entries 8lw .. 8lw+7
    const uint32_t hw[4] = {hsrc.x, hsrc.y, hsrc.z, hsrc.w};
#pragma unroll
    for (int kb = 0; kb < 8; ++kb) {
      const uint32_t hi = (kb & 1) ? (hw[kb >> 1] >> 16) : (hw[kb >> 1] & 0xffffu);
      const int b = lw * 8 + kb;
#pragma unroll
      for (int a = 0; a < 16; ++a) {
        const uint32_t lo = (a & 1) ? (lw8[a >> 1] >> 16) : (lw8[a >> 1] & 0xffffu);
        *reinterpret_cast<uint32_t*>(g_smem + (a + 16 * b) * 256 + col) = lo | (hi << 16);
      }
    }
  } else if (lw == 0) {  // q == 3: low-byte / high-byte tables for the register lookup
    const uint4 row = *reinterpret_cast<const uint4*>(ls + (lane << 3));
    *reinterpret_cast<uint32_t*>(g_smem + 0 * 256 + col) = __byte_perm(row.x, row.y, 0x6420u);
    *reinterpret_cast<uint32_t*>(g_smem + 1 * 256 + col) = __byte_perm(row.z, row.w, 0x6420u);
    *reinterpret_cast<uint32_t*>(g_smem + 2 * 256 + col) = __byte_perm(row.x, row.y, 0x7531u);
    *reinterpret_cast<uint32_t*>(g_smem + 3 * 256 + col) = __byte_perm(row.z, row.w, 0x7531u);
  }
}

// Bounded wait until a shared counter reaches `target` (decode warps, partial-sum buffers).
__device__ __forceinline__ void wait_count(volatile int* c, int target, volatile int* abort_flag) {
  if (*c >= target || *abort_flag) return;
  const unsigned long long t0 = global_ns();
  while (*c < target) {
    __nanosleep(64);
    if (global_ns() - t0 > kWaitLimitNs) {
      set_status(PW_ERR_TIMEOUT);
      *abort_flag = 1;
      return;
    }
  }
}

template <int NTP>
__global__ void __launch_bounds__(kThreads, 1) ffn_kernel(const Params p) {
  using LY = Layout<NTP>;
  uint8_t* const smem = g_smem;
  uint8_t* stages = smem + LY::kOffStages;
  uint16_t* lut_stage = reinterpret_cast<uint16_t*>(smem + LY::kOffLutStage);
  float* red = reinterpret_cast<float*>(smem + LY::kOffRed);
  Desc* pdesc = reinterpret_cast<Desc*>(smem + LY::kOffDesc);
  Desc* cdesc = pdesc + kDescRing;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::kOffBar);
  uint64_t* empty = full + LY::kStages;
  uint64_t* lut_full = empty + LY::kStages;   // [2] staging landed (producer -> LUT warps)
  uint64_t* lut_empty = lut_full + 2;         // [2] staging consumed (LUT warps -> producer)
  uint64_t* lut_ready = lut_empty + 2;        // [2] table built (LUT warps -> decode)
  uint64_t* lut_free = lut_ready + 2;         // [2] table released (decode -> LUT warps)
  int* counters = reinterpret_cast<int*>(lut_free + 2);
  int* red_arrived = counters;                // [2] monotonic, per pass parity
  int* red_done = counters + 2;               // [2] monotonic, per pass parity
  volatile int* abort_flag = counters + 4;

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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&lut_full[b], 1);
      mbar_init(&lut_empty[b], kLutWarps);
      mbar_init(&lut_ready[b], kLutWarps);
      mbar_init(&lut_free[b], kDecodeWarps);
    }
    for (int i = 0; i < 4; ++i) counters[i] = 0;
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  const int n_items = p.meta[0] * p.tiles * p.kslices;

  if (warp == kProducerWarp) {
    // ---------------- producer: one thread resolves items and issues every copy ----------
    if (lane != 0) return;
    const int nst1k = (p.cols + kStageCols - 1) / kStageCols;
    uint32_t g = 0;
    auto issue_item = [&](const Item& it, uint32_t j) {
      const int b = j & 1;
      wait_bar(&lut_empty[b], ((j >> 1) & 1) ^ 1, abort_flag);
      Desc& d = pdesc[j % kDescRing];
      d.valid = it.valid;
      d.status = it.status;
      d.q = it.q;
      d.te = it.te;
      d.pos0 = it.pos0;
      d.tile = it.tile;
      d.ks = it.ks;
      d.s0 = it.s0;
      d.s1 = it.s1;
      d.w = it.w;
      if (it.valid) {
        const uint32_t seg_lut = static_cast<uint32_t>(kSegRows) << it.q << 1;  // bytes
        uint16_t* ls = lut_stage + b * (kLutStageBytes / 2);
        mbar_arrive_expect_tx(&lut_full[b], 2 * seg_lut);
        bulk_g2s(ls, it.lut + (static_cast<size_t>(it.segA) << it.q), seg_lut, &lut_full[b]);
        bulk_g2s(ls + (kSegRows << it.q), it.lut + (static_cast<size_t>(it.segB) << it.q),
                 seg_lut, &lut_full[b]);
      } else {
        mbar_arrive(&lut_full[b]);
      }
    };
    int item = blockIdx.x;
    uint32_t j = 0;
    Item cur;
    if (item < n_items) {
      cur = resolve(p, item, LY::kWide);
      issue_item(cur, 0);
    }
    for (; item < n_items; item += gridDim.x, ++j) {
      const int next = item + gridDim.x;
      Item nxt;
      if (next < n_items) {  // the next item's LUT lands while this item streams
        nxt = resolve(p, next, LY::kWide);
        issue_item(nxt, j + 1);
      }
      if (cur.valid) {
        const void* desc = cur.blk->tma_desc;
        prefetch_desc(desc);
        for (int ch = 0; ch < cur.te; ch += NTP) {
          const int ntok = min(NTP, cur.te - ch);
          for (int s = cur.s0; s < cur.s1; ++s, ++g) {
            const int slot = g % LY::kStages;
            wait_bar(&empty[slot], ((g / LY::kStages) & 1) ^ 1, abort_flag);
            uint8_t* st = stages + slot * LY::kStageBytes;
            const int chunks = min(cur.w, nst1k - s * cur.w);  // 1024-column chunks present
            mbar_arrive_expect_tx(&full[slot],
                                  chunks * (cur.q * kPlaneBytes + ntok * kStageCols * 4));
            for (int h = 0; h < chunks; ++h) {
              const int c1k = s * cur.w + h;
              uint8_t* sp = st + h * cur.q * kPlaneBytes;
              for (int pl = 0; pl < cur.q; ++pl) {
                tma_g2s_2d(sp + pl * kPlaneBytes, desc, c1k * kStageWords, pl * p.rows + cur.segA,
                           &full[slot]);
                tma_g2s_2d(sp + pl * kPlaneBytes + kBoxBytes, desc, c1k * kStageWords,
                           pl * p.rows + cur.segB, &full[slot]);
              }
              for (int t = 0; t < ntok; ++t)
                bulk_g2s(st + kStagePlaneBytes + (h + t) * kStageCols * 4,
                         p.act + static_cast<size_t>(cur.pos0 + ch + t) * p.ld_act +
                             static_cast<size_t>(c1k) * kStageCols,
                         kStageCols * 4, &full[slot]);
            }
          }
        }
      }
      cur = nxt;
    }
    // drain: every issued copy has landed before the block exits
    for (uint32_t d = (g > LY::kStages ? g - LY::kStages : 0); d < g; ++d)
      wait_bar(&full[d % LY::kStages], (d / LY::kStages) & 1, abort_flag);
    return;
  }

  if (warp >= kLutWarp0) {
    // ---------------- LUT warps: staged fp16 LUT -> decode table ----------------
    const int lw = warp - kLutWarp0;
    uint32_t j = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++j) {
      const int b = j & 1;
      wait_bar(&lut_full[b], (j >> 1) & 1, abort_flag);
      const Desc d = pdesc[j % kDescRing];
      wait_bar(&lut_free[b], ((j >> 1) & 1) ^ 1, abort_flag);  // decode warps left item j-2
      if (d.valid) build_table(lut_stage + b * (kLutStageBytes / 2), d.q, b, lw, lane);
      if (lw == 0 && lane == 0) cdesc[j % kDescRing] = d;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&lut_empty[b]);
        mbar_arrive(&lut_ready[b]);
      }
    }
    return;
  }

  // ---------------- decode warps ----------------
  const int tid = threadIdx.x;
  const int ndec = kDecodeWarps * 32;
  const int words_total = p.cols / 32;
  uint32_t g = 0, j = 0, rc = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++j) {
    const uint32_t u = j & 1;
    wait_bar(&lut_ready[u], (j >> 1) & 1, abort_flag);
    const Desc d = cdesc[j % kDescRing];
    if (!d.valid) {
      if (tid == 0) set_status(d.status);
      for (int i = tid; i < d.te * kRows; i += ndec) {
        const int t = i / kRows, r = i - t * kRows;
        if (p.mode == MODE_GATE_UP) {
          if (r < kSegRows)
            p.out[static_cast<size_t>(d.pos0 + t) * p.ld_out + xslot(d.tile * kSegRows + r)] = 0.f;
        } else {
          p.out[d.ks * p.out_slice + static_cast<size_t>(d.pos0 + t) * p.ld_out +
                d.tile * kRows + r] = 0.f;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&lut_free[u]);
      continue;
    }
    const uint32_t lane_base = u * 128 + lane * 4;
    uint4 reg_lut = make_uint4(0u, 0u, 0u, 0u);
    if (d.q == 3)
      reg_lut = make_uint4(lds_u32(0 * 256 + lane_base), lds_u32(1 * 256 + lane_base),
                           lds_u32(2 * 256 + lane_base), lds_u32(3 * 256 + lane_base));

    for (int ch = 0; ch < d.te; ch += NTP, ++rc) {
      const int ntok = min(NTP, d.te - ch);
      float4 pv;
      if (NTP == 1 || ntok == 1)
        pv = run_q<1, NTP>(d, full, empty, abort_flag, words_total, lane_base, reg_lut, g);
      else if (NTP >= 2 && ntok == 2)
        pv = run_q<(NTP >= 2 ? 2 : 1), NTP>(d, full, empty, abort_flag, words_total, lane_base,
                                            reg_lut, g);
      else if (NTP >= 4 && ntok == 3)
        pv = run_q<(NTP >= 4 ? 3 : 1), NTP>(d, full, empty, abort_flag, words_total, lane_base,
                                            reg_lut, g);
      else
        pv = run_q<(NTP >= 4 ? 4 : 1), NTP>(d, full, empty, abort_flag, words_total, lane_base,
                                            reg_lut, g);
      g += d.s1 - d.s0;
      if (ch + NTP >= d.te) {  // last pass over this item: release the table
        __syncwarp();
        if (lane == 0) mbar_arrive(&lut_free[u]);
      }
      // partial sums: buffer rc & 1 is free once pass rc - 2 has been reduced
      const int par = rc & 1;
      const int k = static_cast<int>(rc >> 1);
      if (lane == 0) wait_count(&red_done[par], k, abort_flag);
      __syncwarp();
      float* rb = red + par * (kDecodeWarps * NTP * 32);
      const float part[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
      for (int t = 0; t < NTP; ++t) rb[(warp * NTP + t) * 32 + lane] = part[t];
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        __threadfence_block();
        last = atomicAdd(&red_arrived[par], 1) == kDecodeWarps * (k + 1) - 1;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {  // the last warp to finish adds the sixteen partials in warp order
        __threadfence_block();
        for (int t = 0; t < ntok; ++t) {
          float tot = 0.f;
#pragma unroll
          for (int w = 0; w < kDecodeWarps; ++w)
            tot += *reinterpret_cast<volatile float*>(&rb[(w * NTP + t) * 32 + lane]);
          const size_t row = static_cast<size_t>(d.pos0 + ch + t) * p.ld_out;
          if (p.mode == MODE_GATE_UP) {
            const float up = __shfl_down_sync(0xffffffffu, tot, 16);
            if (lane < kSegRows) {
              const float h = tot / (1.0f + expf(-tot)) * up;
              p.out[row + xslot(d.tile * kSegRows + lane)] = h;
            }
          } else {
            p.out[d.ks * p.out_slice + row + d.tile * kRows + lane] = tot;
          }
        }
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          atomicAdd(&red_done[par], 1);
        }
      }
    }
  }
}

}  // namespace k4
}  // namespace pw
