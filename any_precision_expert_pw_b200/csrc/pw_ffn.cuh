// K4: fused any-precision grouped expert GEMV (PagedWeight, "Composants Clés" 1 and 3: one
// fused kernel reads the bit-planes and LUTs directly, each block at its own bitwidth).
//
// Work item = (active expert, 32-row tile, k-slice).  A tile is two 16-row segments: for
// gate_up the gate rows [16i, 16i+16) and the matching up rows [I+16i, I+16i+16), so that
// SiLU(gate) * up is formed in the epilogue (gate_up is never split along k); for down the
// rows [32i, 32i+32), optionally split into k-slices whose partial sums the combine adds.
//
// Warp roles (one CTA per SM, persistent over the items):
//   producer (1 warp)   resolves the items from the Weight Page Table and streams, per
//                       1024-column stage, the top-q bit-planes of the 32 rows (one bulk copy:
//                       in the tiled plane layout they are one contiguous run, already in the
//                       order the decode warps read) plus the stage's activation chunk through
//                       a ring of mbarrier-guarded stages;
//   LUT (4 warps)       resolve the items too, read each item's fp16 LUT rows from global memory
//                       (one row per lane) and build its decode table in one of two table
//                       buffers, one item ahead of the decode warps, then signal it ready; a
//                       buffer is rewritten only after every decode warp has released it, so
//                       decode warps never meet a CTA barrier;
//   decode (16 warps)   take 64 columns of each stage; each thread owns one row (its lane);
//   reducer (1 warp)    adds the sixteen per-warp partial sums of every pass in a fixed order
//                       and writes the output (SiLU(gate) * up for gate_up).
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
// broadcast load.
#pragma once
#include "pw_common.cuh"

namespace pw {
namespace k4 {

constexpr int kRows = 32;
constexpr int kSegRows = 16;
constexpr int kStageWords = 32;                          // words per row per plane per stage
constexpr int kStageCols = kStageWords * 32;             // 1024 columns
constexpr int kDecodeWarps = 16;
constexpr int kLutWarps = 4;
constexpr int kWarpWords = kStageWords / kDecodeWarps;   // 2 words = 64 columns per warp
constexpr int kLutWarp0 = kDecodeWarps;
constexpr int kProducerWarp = kDecodeWarps + kLutWarps;
constexpr int kReducerWarp = kProducerWarp + 1;
constexpr int kThreads = (kReducerWarp + 1) * 32;
constexpr int kPlaneBytes = kRows * kStageWords * 4;     // one plane of a full stage
constexpr int kStagePlaneBytes = PW_MAX_BITS * kPlaneBytes;
constexpr int kLutBytes = 256 * 256;                     // 2^8 entries x 256-byte stride
constexpr int kMaxKSlices = 8;
constexpr int kDescRing = 8;    // item descriptors in flight (LUT warps -> every other role)
constexpr int kLutBarrier = 1;  // named barrier of the four LUT warps

// The kernel's dynamic shared memory, named directly (not through a pointer) wherever the
// decode loop indexes it, so every table gather is one load with a constant base folded in.
extern __shared__ __align__(1024) uint8_t g_smem[];

// Slot of column c in the activation layout the decode reads: inside each 32-column group,
// columns 8b+i and 8b+4+i (i < 4) sit at slots 8i+2b and 8i+2b+1.
__host__ __device__ __forceinline__ int xslot(int c) {
  const int l = c & 31;
  return (c & ~31) | ((l & 3) << 3) | (((l >> 3) & 3) << 1) | ((l >> 2) & 1);
}

template <int NTP>
struct Layout {
  static constexpr int kStages = NTP == 1 ? 4 : 3;
  static constexpr int kStageXBytes = NTP * kStageCols * 4;
  static constexpr int kStageBytes = kStagePlaneBytes + kStageXBytes;
  static constexpr int kOffLut = 0;
  static constexpr int kOffStages = kLutBytes;
  static constexpr int kOffRed = kOffStages + kStages * kStageBytes;
  static constexpr int kRedBytes = 2 * kDecodeWarps * NTP * 32 * 4;
  static constexpr int kOffDesc = kOffRed + kRedBytes;
  static constexpr int kDescBytes = kDescRing * 80;
  static constexpr int kOffBar = kOffDesc + kDescBytes;
  static constexpr int kBarBytes = (2 * kStages + 8 + 2 * kDescRing) * 8 + 32;
  static constexpr int kSmem = kOffBar + kBarBytes;
  static_assert(kStageBytes % 128 == 0 && kOffStages % 128 == 0, "stage alignment");
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

// One module's half of the launch.
struct ModeParams {
  int rows;      // expected block rows (2I or H)
  int cols;      // expected block cols (H or I)
  int half;      // gate_up: I (offset of the up rows); down: 0
  int tiles;     // row tiles per expert
  int kslices;   // k-slices per tile (1 for gate_up)
  const float* act;  // [row][ld_act] fp32 activations in xslot order, zero beyond cols
  int ld_act;
  const int32_t* act_map;  // non-null: grouped position pos reads row act_map[pos] / act_div
  int act_div;             // (gate_up: the token of the assignment); null: row = pos
  float* out;        // gate_up: h [pos][ld_out] (xslot order); down: [kslice][pos][ld_out]
  int ld_out;
  long long out_slice;  // elements between k-slices of `out`
};

// The launch covers modes first_mode..last_mode: first every gate_up item (expert-major), then
// every down item.  With both, a down item of active expert a streams h only once done[a]
// counts all gate_up tiles of a (items are claimed in order and only by running CTAs, none of
// which waits on a later item, so the wait always ends).
struct Params {
  const pw_page_table* pt;
  int layer;
  int E;
  int first_mode, last_mode;
  ModeParams m[2];
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* meta;
  int* sched;   // work counter (zero at launch): items after each CTA's first one
  int* done;    // [E] gate_up tiles finished per active expert (zero at launch), both modes
};

// One work item as every warp role sees it: written once by LUT warp 0 into a shared-memory
// ring; item < 0 marks the end of this CTA's work.
struct Desc {
  const uint32_t* planes;  // the tile's run of stages (tiled layout)
  const uint16_t* lut;     // the block's q-bit LUT
  int item, valid, status, q, n, te, pos0, tile, ks, s0, s1, segA, segB, mode, a, pad0;
};
static_assert(sizeof(Desc) == 80, "descriptor size");

struct Item {
  const pw_block* blk;
  const uint16_t* lut;
  const uint32_t* planes;  // the tile's run of stages (tiled layout)
  int q, n, tile, ks, te, pos0, segA, segB, s0, s1, status, mode, a;
  bool valid;
};

__device__ __forceinline__ int items_of(const Params& p, int mode, int n_active) {
  return n_active * p.m[mode].tiles * p.m[mode].kslices;
}

__device__ __forceinline__ Item resolve(const Params& p, int item, int n_active) {
  Item it;
  int mode = p.first_mode;
  if (mode < p.last_mode) {
    const int n0 = items_of(p, mode, n_active);
    if (item >= n0) {
      item -= n0;
      ++mode;
    }
  }
  const ModeParams& mp = p.m[mode];
  it.mode = mode;
  const int per_expert = mp.tiles * mp.kslices;
  const int a = item / per_expert;
  const int rem = item - a * per_expert;
  it.a = a;
  it.tile = rem / mp.kslices;
  it.ks = rem - it.tile * mp.kslices;
  const int e = p.active[a];
  it.blk = p.pt->blocks + (static_cast<size_t>(p.layer) * p.E + e) * 2 + mode;
  const pw_block* b = it.blk;
  it.q = b->committed_bits;
  it.te = p.counts[e];
  it.pos0 = p.offsets[e];
  if (mode == MODE_GATE_UP) {
    it.segA = it.tile * kSegRows;
    it.segB = mp.half + it.tile * kSegRows;
  } else {
    it.segA = it.tile * kRows;
    it.segB = it.segA + kSegRows;
  }
  const int nst = (mp.cols + kStageCols - 1) / kStageCols;
  it.s0 = (nst * it.ks) / mp.kslices;
  it.s1 = (nst * (it.ks + 1)) / mp.kslices;
  // planes held per (tile, stage) run on the device: all parent_bits, or a paged-in prefix
  it.n = b->stored_bits ? b->stored_bits : b->parent_bits;
  const bool bits_ok = it.q >= b->min_bits && it.q <= it.n && it.n <= b->parent_bits &&
                       it.q >= PW_MIN_BITS &&
                       it.q <= PW_MAX_BITS && b->lut[it.q] != nullptr && b->planes != nullptr;
  it.planes = b->planes + static_cast<size_t>(it.tile) * it.n * kRows * (mp.cols / 32);
  const int want_layout = mode == MODE_GATE_UP ? PW_LAYOUT_TILED_GATE_UP : PW_LAYOUT_TILED_DOWN;
  const bool shape_ok = static_cast<int>(b->rows) == mp.rows &&
                        static_cast<int>(b->cols) == mp.cols && b->layout == want_layout;
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

// Bounded wait until *ctr >= target (acquire at GPU scope), then order the async-proxy reads
// that follow after it; false (PW_ERR_TIMEOUT recorded, abort flag set) when the limit ran out.
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ bool wait_count(const int* ctr, int target,
                                           volatile int* abort_flag) {
  if (ld_acquire(ctr) < target) {
    const unsigned long long t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
      __nanosleep(128);
      if (ld_acquire(ctr) >= target) break;
      if (*abort_flag) return false;
      if ((it & 15u) == 0 && global_ns() - t0 > kWaitLimitNs) {
        set_status(PW_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
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
__device__ __forceinline__ void decode_stage(uint32_t planes_off, uint32_t pstride,
                                             uint32_t xs_off, uint32_t lane_base,
                                             const uint4& reg_lut, int warp, int lane,
                                             float2 (&acc)[NT][2]) {
  // tiled layout: a plane of the stage is [word pair][row][2 words]; this warp's pair is 256
  // contiguous bytes, one 8-byte row per lane (conflict free)
  const uint32_t off = planes_off + warp * 256 + lane * 8;
  uint2 P[Q];
#pragma unroll
  for (int p = 0; p < Q; ++p)
    P[p] = *reinterpret_cast<const uint2*>(g_smem + off + p * pstride);
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
template <int Q, int NT, int NS>
__device__ __noinline__ float4 run_stages(uint64_t* full, uint64_t* empty,
                                          volatile int* abort_flag, int stage_bytes,
                                          int words_total, uint32_t lane_base, uint32_t l0,
                                          uint32_t l1, uint32_t l2, uint32_t l3, int s0, int s1,
                                          uint32_t g) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4 reg_lut = make_uint4(l0, l1, l2, l3);
  float2 acc[NT][2];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = make_float2(0.f, 0.f);
  for (int s = s0; s < s1; ++s, ++g) {
    const int slot = g % NS;
    wait_bar(&full[slot], (g / NS) & 1, abort_flag);
    const uint32_t st = kLutBytes + slot * stage_bytes;
    const int ws = min(kStageWords, words_total - s * kStageWords);
    if (warp * kWarpWords < ws)
      decode_stage<Q, NT>(st, ws * kRows * 4, st + kStagePlaneBytes, lane_base, reg_lut, warp,
                          lane, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
  float r[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int t = 0; t < NT; ++t) r[t] = (acc[t][0].x + acc[t][1].x) + (acc[t][0].y + acc[t][1].y);
  return make_float4(r[0], r[1], r[2], r[3]);
}

#define PW_RUN_ARGS                                                                          \
  full, empty, abort_flag, LY::kStageBytes, words_total, lane_base, reg_lut.x,               \
      reg_lut.y, reg_lut.z, reg_lut.w, d.s0, d.s1, g

template <int NT, int NTP>
__device__ __forceinline__ float4 run_q(const Desc& d, uint64_t* full, uint64_t* empty,
                                        volatile int* abort_flag, int words_total,
                                        uint32_t lane_base, const uint4& reg_lut, uint32_t g) {
  using LY = Layout<NTP>;
  switch (d.q) {
    case 3: return run_stages<3, NT, LY::kStages>(PW_RUN_ARGS);
    case 4: return run_stages<4, NT, LY::kStages>(PW_RUN_ARGS);
    case 5: return run_stages<5, NT, LY::kStages>(PW_RUN_ARGS);
    case 6: return run_stages<6, NT, LY::kStages>(PW_RUN_ARGS);
    case 7: return run_stages<7, NT, LY::kStages>(PW_RUN_ARGS);
    default: return run_stages<8, NT, LY::kStages>(PW_RUN_ARGS);
  }
}
#undef PW_RUN_ARGS

// LUT warp lw (0..3), lane = row r of the tile (rows segA.. for lanes 0-15, segB.. for 16-31).
// fetch_table reads the row's share of its fp16 LUT from global memory into registers; it is
// issued before the warp waits for a free table buffer, so the load latency overlaps that wait.
struct LutRegs {
  uint4 v[8];
};

__device__ __forceinline__ void fetch_table(const uint16_t* __restrict__ row, int q, int lw,
                                            LutRegs& r) {
  if (q >= 5) {  // fp32 table; warp lw takes entries [lw * 2^q/4, (lw+1) * 2^q/4)
    const int quarter = 1 << (q - 2);
    const uint4* src = reinterpret_cast<const uint4*>(row + lw * quarter);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < quarter / 8) r.v[k] = __ldg(src + k);
  } else {  // q <= 4: the whole row (16 or 8 entries)
    r.v[0] = __ldg(reinterpret_cast<const uint4*>(row));
    if (q == 4) r.v[1] = __ldg(reinterpret_cast<const uint4*>(row) + 1);
  }
}

// The fetched LUT row -> decode table in buffer u (fp32 entries for q >= 5, half2 pair entries
// for q = 4, low/high byte tables for q = 3).
__device__ __forceinline__ void store_table(const LutRegs& r, int q, uint32_t u, int lw, int lane) {
  const uint32_t col = u * 128 + lane * 4;
  if (q >= 5) {
    const int quarter = 1 << (q - 2);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k >= quarter / 8) break;
      const uint32_t w4[4] = {r.v[k].x, r.v[k].y, r.v[k].z, r.v[k].w};
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int e = lw * quarter + k * 8 + m;
        const uint16_t h = static_cast<uint16_t>((m & 1) ? (w4[m >> 1] >> 16) : (w4[m >> 1] & 0xffffu));
        *reinterpret_cast<float*>(g_smem + e * 256 + col) = f16_to_f32(h);
      }
    }
  } else if (q == 4) {  // pair entries a + 16b = (LUT[a], LUT[b]); warp lw takes b in [4lw, 4lw+4)
    const uint32_t lw8[8] = {r.v[0].x, r.v[0].y, r.v[0].z, r.v[0].w,
                             r.v[1].x, r.v[1].y, r.v[1].z, r.v[1].w};
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      const int b = lw * 4 + kb;
      const uint32_t hw = lw8[b >> 1];
      const uint32_t hi = (b & 1) ? (hw >> 16) : (hw & 0xffffu);
#pragma unroll
      for (int a = 0; a < 16; ++a) {
        const uint32_t lo = (a & 1) ? (lw8[a >> 1] >> 16) : (lw8[a >> 1] & 0xffffu);
        *reinterpret_cast<uint32_t*>(g_smem + (a + 16 * b) * 256 + col) = lo | (hi << 16);
      }
    }
  } else if (lw == 0) {  // q == 3: low-byte / high-byte tables for the register lookup
    const uint4 v = r.v[0];
    *reinterpret_cast<uint32_t*>(g_smem + 0 * 256 + col) = __byte_perm(v.x, v.y, 0x6420u);
    *reinterpret_cast<uint32_t*>(g_smem + 1 * 256 + col) = __byte_perm(v.z, v.w, 0x6420u);
    *reinterpret_cast<uint32_t*>(g_smem + 2 * 256 + col) = __byte_perm(v.x, v.y, 0x7531u);
    *reinterpret_cast<uint32_t*>(g_smem + 3 * 256 + col) = __byte_perm(v.z, v.w, 0x7531u);
  }
}

template <int NTP>
__global__ void __launch_bounds__(kThreads, 1) ffn_kernel(const Params p) {
  using LY = Layout<NTP>;
  uint8_t* const smem = g_smem;
  uint8_t* stages = smem + LY::kOffStages;
  float* red = reinterpret_cast<float*>(smem + LY::kOffRed);
  Desc* cdesc = reinterpret_cast<Desc*>(smem + LY::kOffDesc);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::kOffBar);
  uint64_t* empty = full + LY::kStages;
  uint64_t* lut_ready = empty + LY::kStages;  // [2] table built (LUT warps -> decode)
  uint64_t* lut_free = lut_ready + 2;         // [2] table released (decode -> LUT warps)
  uint64_t* red_full = lut_free + 2;          // [2] partial sums written (decode -> reducer)
  uint64_t* red_free = red_full + 2;          // [2] partial sums consumed (reducer -> decode)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red_free + 2 + 2 * kDescRing);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 127) {  // stage buffers and tables assume 128-byte alignment
    if (threadIdx.x == 0) set_status(PW_ERR_UNSUPPORTED);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < LY::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecodeWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&lut_ready[b], kLutWarps);
      mbar_init(&lut_free[b], kDecodeWarps);
      mbar_init(&red_full[b], kDecodeWarps);
      mbar_init(&red_free[b], 1);
    }
    for (int r = 0; r < kDescRing; ++r) {
      mbar_init(&red_free[2 + r], 1);              // desc_full: written by LUT warp 0
      mbar_init(&red_free[2 + kDescRing + r], 2);  // desc_free: read by producer and reducer
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  // a launch that starts with gate_up reads the grouping written by the launch before it; a
  // down-only launch reads the page table, the grouping (complete before the gate_up launch
  // started) and weights until its producer needs h
  if (p.first_mode == MODE_GATE_UP) griddep_wait();
  griddep_launch();

  const int n_active = p.meta[0];
  int n_items = 0;
  for (int m = p.first_mode; m <= p.last_mode; ++m) n_items += items_of(p, m, n_active);
  const bool fused = p.first_mode == MODE_GATE_UP && p.last_mode == MODE_DOWN;

  uint64_t* const desc_full = red_free + 2;  // [kDescRing] descriptor written (LUT warp 0)
  uint64_t* const desc_free = desc_full + kDescRing;  // [kDescRing] read by producer + reducer

  if (warp == kProducerWarp) {
    // ---------------- producer: one thread streams every stage ----------------
    if (lane != 0) return;
    if (p.first_mode == MODE_DOWN) {
      // while the gate_up grid finishes: this CTA's first item's planes into L2, then wait for h
      if (static_cast<int>(blockIdx.x) < n_items) {
        const Item cur = resolve(p, blockIdx.x, n_active);
        const int wt = p.m[MODE_DOWN].cols / 32;
        if (cur.valid)
          for (int s = cur.s0; s < cur.s1; ++s) {
            const int ws = min(kStageWords, wt - s * kStageWords);
            prefetch_l2(cur.planes + static_cast<size_t>(s) * cur.n * kRows * kStageWords,
                        cur.q * ws * kRows * 4);
          }
      }
      griddep_wait();
    }
    uint32_t g = 0;
    for (uint32_t j = 0;; ++j) {
      wait_bar(&desc_full[j % kDescRing], (j / kDescRing) & 1, abort_flag);
      const Desc cur = cdesc[j % kDescRing];
      mbar_arrive(&desc_free[j % kDescRing]);
      if (cur.item < 0 || *abort_flag) break;
      if (!cur.valid) continue;
      const ModeParams& mp = p.m[cur.mode];
      const int words_total = mp.cols / 32;
      // fused launch: h of this expert is complete once all its gate_up tiles are counted
      if (fused && cur.mode == MODE_DOWN &&
          !wait_count(p.done + cur.a, p.m[MODE_GATE_UP].tiles, abort_flag))
        break;
      for (int ch = 0; ch < cur.te; ch += NTP) {
        const int ntok = min(NTP, cur.te - ch);
        const float* arow[NTP];
        for (int t = 0; t < ntok; ++t) {
          const int pos = cur.pos0 + ch + t;
          const int r = mp.act_map ? mp.act_map[pos] / mp.act_div : pos;
          arow[t] = mp.act + static_cast<size_t>(r) * mp.ld_act;
        }
        for (int s = cur.s0; s < cur.s1; ++s, ++g) {
          const int slot = g % LY::kStages;
          wait_bar(&empty[slot], ((g / LY::kStages) & 1) ^ 1, abort_flag);
          uint8_t* st = stages + slot * LY::kStageBytes;
          const int ws = min(kStageWords, words_total - s * kStageWords);
          const uint32_t pbytes = cur.q * ws * kRows * 4;
          mbar_arrive_expect_tx(&full[slot], pbytes + ntok * kStageCols * 4);
          bulk_g2s(st, cur.planes + static_cast<size_t>(s) * cur.n * kRows * kStageWords, pbytes,
                   &full[slot]);
          for (int t = 0; t < ntok; ++t)
            bulk_g2s(st + kStagePlaneBytes + t * kStageCols * 4,
                     arow[t] + static_cast<size_t>(s) * kStageCols, kStageCols * 4, &full[slot]);
        }
      }
    }
    // drain: every issued copy has landed before the block exits
    for (uint32_t d = (g > LY::kStages ? g - LY::kStages : 0); d < g; ++d)
      wait_bar(&full[d % LY::kStages], (d / LY::kStages) & 1, abort_flag);
    return;
  }

  if (warp == kReducerWarp) {
    // ---------------- reducer: sixteen partial sums per row, in warp order ----------------
    uint32_t rc = 0;
    for (uint32_t j = 0;; ++j) {
      wait_bar(&desc_full[j % kDescRing], (j / kDescRing) & 1, abort_flag);
      const Desc it = cdesc[j % kDescRing];
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_free[j % kDescRing]);
      if (it.item < 0 || *abort_flag) break;
      const ModeParams& mp = p.m[it.mode];
      if (!it.valid) {
        // a block that cannot be read (state, bitwidth or shape): its outputs are zeros
        if (lane == 0) set_status(it.status);
        for (int t = 0; t < it.te; ++t) {
          const size_t row = static_cast<size_t>(it.pos0 + t) * mp.ld_out;
          if (it.mode == MODE_GATE_UP) {
            if (lane < kSegRows) mp.out[row + xslot(it.tile * kSegRows + lane)] = 0.f;
          } else {
            mp.out[it.ks * mp.out_slice + row + it.tile * kRows + lane] = 0.f;
          }
        }
      }
      for (int ch = 0; it.valid && ch < it.te; ch += NTP, ++rc) {
        const int ntok = min(NTP, it.te - ch);
        const int par = rc & 1;
        wait_bar(&red_full[par], (rc >> 1) & 1, abort_flag);
        const float* rb = red + par * (kDecodeWarps * NTP * 32);
        for (int t = 0; t < ntok; ++t) {
          float tot = 0.f;
#pragma unroll
          for (int w = 0; w < kDecodeWarps; ++w) tot += rb[(w * NTP + t) * 32 + lane];
          const size_t row = static_cast<size_t>(it.pos0 + ch + t) * mp.ld_out;
          if (it.mode == MODE_GATE_UP) {
            const float up = __shfl_down_sync(0xffffffffu, tot, 16);
            if (lane < kSegRows) {
              const float h = tot / (1.0f + expf(-tot)) * up;
              mp.out[row + xslot(it.tile * kSegRows + lane)] = h;
            }
          } else {
            mp.out[it.ks * mp.out_slice + row + it.tile * kRows + lane] = tot;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_free[par]);
      }
      if (fused && it.mode == MODE_GATE_UP) {
        // this tile's h rows are written: make them visible, then count the tile
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.done + it.a, 1);
      }
    }
    return;
  }

  if (warp >= kLutWarp0) {
    // ---------------- LUT warps: the item schedule and the decode tables ----------------
    // Item 0 of each CTA is blockIdx.x; every later one is taken from the launch's work counter
    // (gridDim.x + its old value), so CTAs that finish early take more items.  LUT warp 0
    // resolves each item and publishes its descriptor; all four warps then build its table.
    const int lw = warp - kLutWarp0;
    int item = blockIdx.x;
    for (uint32_t j = 0;; ++j) {
      const uint32_t u = j & 1;
      Desc& d = cdesc[j % kDescRing];
      if (lw == 0) {
        if (lane == 0) {
          // the producer and the reducer have read descriptor j - kDescRing from this slot
          wait_bar(&desc_free[j % kDescRing], ((j / kDescRing) & 1) ^ 1, abort_flag);
          if (item < n_items) {
            const Item it = resolve(p, item, n_active);
            d.planes = it.planes;
            d.lut = it.lut;
            d.item = item;
            d.valid = it.valid;
            d.status = it.status;
            d.q = it.q;
            d.n = it.n;
            d.te = it.te;
            d.pos0 = it.pos0;
            d.tile = it.tile;
            d.ks = it.ks;
            d.s0 = it.s0;
            d.s1 = it.s1;
            d.segA = it.segA;
            d.segB = it.segB;
            d.mode = it.mode;
            d.a = it.a;
          } else {
            d.item = -1;
          }
          mbar_arrive(&desc_full[j % kDescRing]);
        }
      }
      named_sync(kLutBarrier, kLutWarps * 32);  // descriptor j visible to the four LUT warps
      const Desc it = d;
      if (it.item < 0 || *abort_flag) {
        // the decode warps read the end marker; like any item it follows their release of
        // buffer u (item j - 2), so no barrier phase runs ahead of a waiter
        wait_bar(&lut_free[u], ((j >> 1) & 1) ^ 1, abort_flag);
        __syncwarp();
        if (lane == 0) mbar_arrive(&lut_ready[u]);
        break;
      }
      LutRegs lr;
      if (it.valid) {
        const int r = lane < kSegRows ? it.segA + lane : it.segB + (lane - kSegRows);
        fetch_table(it.lut + (static_cast<size_t>(r) << it.q), it.q, lw, lr);
      }
      wait_bar(&lut_free[u], ((j >> 1) & 1) ^ 1, abort_flag);  // decode warps left item j-2
      // claim item j + 1 only now, two items ahead of the decode warps: an item claimed earlier
      // would sit in this CTA's queue while other CTAs run dry at the end of the launch
      int next = 0;
      if (lw == 0 && lane == 0) next = gridDim.x + atomicAdd(p.sched, 1);
      if (it.valid) store_table(lr, it.q, u, lw, lane);
      if (lw == 0) item = __shfl_sync(0xffffffffu, next, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(&lut_ready[u]);
    }
    return;
  }

  // ---------------- decode warps ----------------
  uint32_t g = 0, rc = 0;
  for (uint32_t j = 0;; ++j) {
    const uint32_t u = j & 1;
    wait_bar(&lut_ready[u], (j >> 1) & 1, abort_flag);
    const Desc d = cdesc[j % kDescRing];
    if (d.item < 0 || *abort_flag) break;
    if (!d.valid) {  // the reducer writes this item's zeros
      __syncwarp();
      if (lane == 0) mbar_arrive(&lut_free[u]);
      continue;
    }
    const int words_total = p.m[d.mode].cols / 32;
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
      // partial sums into buffer rc & 1 once the reducer has consumed pass rc - 2
      const int par = rc & 1;
      wait_bar(&red_free[par], ((rc >> 1) & 1) ^ 1, abort_flag);
      float* rb = red + par * (kDecodeWarps * NTP * 32);
      const float part[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
      for (int t = 0; t < NTP; ++t) rb[(warp * NTP + t) * 32 + lane] = part[t];
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_full[par]);
    }
  }
}

}  // namespace k4
}  // namespace pw
