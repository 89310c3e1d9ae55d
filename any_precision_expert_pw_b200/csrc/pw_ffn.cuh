// K4: fused any-precision grouped expert GEMV (PagedWeight, "Composants Clés" 1 and 3: one
// fused kernel reads the bit-planes and LUTs directly, each block at its own bitwidth).
//
// Work item = (active expert, pair of 32-row tiles, k-slice).  Lane i of every warp holds row
// i of both tiles ("row a" of tile 2P, "row b" of tile 2P + 1), so each activation value that a
// warp loads serves two rows.  gate_up tiles are 16 gate rows then the 16 matching up rows, so
// lane i < 16 holds gate rows and lane i + 16 the up rows of the same features: SiLU(gate) * up
// is formed in the epilogue (gate_up is never split along k); down is split into k-slices
// whose partial sums the combine adds.
//
// Warp roles (one CTA per SM, persistent over the items):
//   producer (1 warp)   streams, per 512-column stage, the top-q bit-planes of the two tiles
//                       (one bulk copy per tile: in the tiled plane layout a tile's top q planes
//                       of a stage are one contiguous run, already in the order the decode
//                       warps read) plus the stage's activation chunk of every token of the
//                       pass into a ring of fixed slots; a slot holds one stage, or two for
//                       q <= 4 (a stage of a low-bitwidth block is small and decodes fast), so
//                       every item keeps about the same time of work in flight;
//                       It also claims the items from the launch's work counter, one ahead of
//                       the item it streams, and publishes each item's descriptor;
//   LUT (4 warps)       read each item's fp16 LUT rows from global memory (lane i: rows a and
//                       b) and build its decode table in one of two buffers, one item ahead of
//                       the decode warps;
//   decode (16 warps)   warp w takes word w (32 columns) of every stage, both rows of its lane;
//   reducer (1 warp)    adds the sixteen per-warp partial sums of every pass in a fixed order
//                       and writes the output (SiLU(gate) * up for gate_up).
// Activations are fp16 (gate_up: x, bf16 -> fp16, exact in fp16's normal range; down: h as a
// pair hi + lo of fp16 values, hi = fp16(h), lo = fp16(h - hi), so the products keep h to about
// 22 bits -- a single fp16 rounding of h leaves the whole output of some batches at the edge of
// the parity bar) and every product is one fma.rn.f32.f16: the fp16 weight times the fp16
// activation, exact, added in fp32.
// Decode tables hold fp16 LUT values; slot s of lane i sits at byte 256 s + 128 u + 4 i (u =
// table buffer), so a gather of 32 lanes is conflict free and its address is one byte
// permute of the code byte.  After an 8x8 bit transpose of plane words, byte k of register j
// holds the code of column 8k + j of the word; two paths, chosen per block by its committed q:
//   q >= 5  each row's q planes are transposed on their own (code = the q-bit index v); slot
//           v holds (LUT_a[v], LUT_b[v]): one gather per weight, the row picks its half;
//   q <= 4  rows a and b are transposed together (code = v_a + 16 v_b); slot v_a + 16 v_b
//           holds (LUT_a[v_a], LUT_b[v_b]): one gather gives the weights of both rows.
#pragma once
#include "pw_common.cuh"

namespace pw {
namespace k4 {

constexpr int kTiles = 2;                                  // 32-row tiles per item
constexpr int kItemRows = kTiles * kTileRows;              // 64
constexpr int kStageWords = kTileStageWords;               // 16 words per row per stage
constexpr int kStageCols = kTileStageCols;                 // 512 columns
constexpr int kDecodeWarps = kStageWords;                  // one word each
constexpr int kLutWarps = 4;
constexpr int kLutWarp0 = kDecodeWarps;
constexpr int kProducerWarp = kDecodeWarps + kLutWarps;
constexpr int kReducerWarp = kProducerWarp + 1;
constexpr int kThreads = (kReducerWarp + 1) * 32;
constexpr int kTableBytes = 256 * 256;                     // 256 slots x 256-byte stride
constexpr int kXBytes = kStageCols * 2;                    // fp16 x, one stage, one token
constexpr int kXBytesDown = 2 * kXBytes;                   // h: 512 hi then 512 lo
constexpr int kSlotPlaneBytes = kTiles * PW_MAX_BITS * kStageWords * 128;  // 32 KB
constexpr int kMaxKSlices = 8;
constexpr int kDescRing = 8;    // item descriptors in flight (LUT warps -> every other role)

// The kernel's dynamic shared memory, named directly (not through a pointer) wherever the
// decode loop indexes it, so every table gather is one load with a constant base folded in.
extern __shared__ __align__(1024) uint8_t g_smem[];

// Position of column c in the fp16 activation layout the decode reads: inside each 32-column
// group, column 8k + i sits at 8 (i % 4) + 4 (i / 4) + k, so that one 16-byte load holds the
// columns of code registers i and i + 4 (i < 4).
__host__ __device__ __forceinline__ int xpos(int c) {
  const int l = c & 31, i = l & 7, k = l >> 3;
  return (c & ~31) | ((i & 3) << 3) | ((i >> 2) << 2) | k;
}

// What the setup kernel resolves once per (module, active expert) from the Weight Page Table, so
// that an item's descriptor costs one load: the block's planes and q-bit LUT, its bitwidth and
// stored planes per run, whether it can be read (else the status to record), and the expert's
// grouped tokens.
struct ExpertDesc {
  const uint32_t* planes;
  const uint16_t* lut;
  long long tile_words;  // words between the runs of consecutive tiles
  int q, n, valid, status, te, pos0, pad0, pad1;
};
static_assert(sizeof(ExpertDesc) == 56, "expert descriptor size");

// One work item as every warp role sees it: written once by the producer into a shared-memory
// ring; item < 0 marks the end of this CTA's work.
struct Desc {
  const uint32_t* planes;  // tile 2P's run of stages (tiled layout); tile 2P + 1 follows
  const uint16_t* lut;     // the block's q-bit LUT
  long long tile_words;    // words between the runs of consecutive tiles
  int item, valid, status, q, n, te, pos0, pair, ks, s0, s1, mode, a, pad0, pad1, pad2;
};
static_assert(sizeof(Desc) == 88, "descriptor size");

// Stages per slot for a block of committed bitwidth q, at most ms (the layout's).
__host__ __device__ __forceinline__ int sub_stages(int q, int ms) { return q <= 4 ? ms : 1; }

template <int NTP>
struct Layout {
  static constexpr int kStages = NTP == 1 ? 4 : 3;  // slots
  static constexpr int kMaxSub = NTP == 4 ? 1 : 2;   // stages per slot at most (q <= 4)
  static constexpr int kSlotBytes = kSlotPlaneBytes + NTP * kMaxSub * kXBytesDown;
  static constexpr int kRedBytes = 2 * kDecodeWarps * NTP * kTiles * 32 * 4;
  static constexpr int kDescBytes = kDescRing * static_cast<int>(sizeof(Desc));
  static constexpr int kBarBytes = (2 * kStages + 8 + 2 * kDescRing) * 8 + 32;
  // the two modes' parameters and the activation rows of the current pass: producer state
  // kept in shared memory rather than in the (small) L1 cache
  static constexpr int kMiscBytes = 2 * 128 + NTP * 8;
  static constexpr int kOffTable = 0;
  static constexpr int kOffRing = kTableBytes;
  static constexpr int kOffRed = kOffRing + kStages * kSlotBytes;
  static constexpr int kOffDesc = kOffRed + kRedBytes;
  static constexpr int kOffBar = kOffDesc + kDescBytes;
  static constexpr int kOffMisc = kOffBar + kBarBytes;
  static constexpr int kSmem = kOffMisc + kMiscBytes;
  static_assert(kOffRing % 128 == 0 && kSlotBytes % 128 == 0, "slot alignment");
  static_assert(kOffBar % 8 == 0 && kOffMisc % 16 == 0, "alignment");
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

// One module's half of the launch.
struct ModeParams {
  int rows;      // expected block rows (2I or H)
  int cols;      // expected block cols (H or I)
  int half;      // gate_up: I (offset of the up rows); down: 0
  int pairs;     // tile pairs (items per k-slice) per expert
  int kslices;   // k-slices per tile pair (1 for gate_up)
  const __half* act;  // fp16 activations [row][ld_act], xpos order (one 1 KB chunk per stage)
  long long ld_act;   // elements between rows of act
  const int32_t* act_map;  // non-null: grouped position pos reads row act_map[pos] / act_div
  int act_div;             // (gate_up: the token of the assignment); null: row = pos
  int act_rows;            // rows of act (bounds of the debug build)
  int out_rows;            // grouped positions (T * k)
  int ld_out;
  __half* hout;         // gate_up: the down projection's activations [pos][ld_hout], xpos order
  long long ld_hout;
  float* out;           // down: partial sums [kslice][pos][ld_out]
  long long out_slice;  // elements between k-slices of `out`
};

static_assert(sizeof(ModeParams) <= 128, "mode parameters fit their shared-memory copy");

// The launch covers every gate_up item (expert-major), then every down item.  A down item of
// active expert a streams h only once done[a] counts all gate_up items of a.  The wait always
// ends, whatever number of CTAs is resident: items are claimed from one counter in order, only
// by CTAs that are running, and each CTA works through its items in claim order; every gate_up
// item is claimed before any down item and waits on nothing, so each counted item is finished
// by the CTA that claimed it.
struct Params {
  const pw_page_table* pt;
  int layer;
  int E;
  ModeParams m[2];
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* meta;
  const ExpertDesc* xd;  // [2][E]: per module, per active expert (setup kernel)
  int* sched;     // work counter (zero at launch): every item is claimed from it
  int* done;      // [E] gate_up items finished per active expert (zero at launch)
  uint32_t one;   // 1, opaque to the compiler: base of the transpose's shift multipliers
};

__device__ __forceinline__ int items_of(const ModeParams* mps, int mode, int n_active) {
  return n_active * mps[mode].pairs * mps[mode].kslices;
}

__device__ __forceinline__ Desc resolve(const Params& p, const ModeParams* mps, int item,
                                        int n_active) {
  Desc d;
  d.item = item;
  int mode = MODE_GATE_UP;
  const int n0 = items_of(mps, MODE_GATE_UP, n_active);
  if (item >= n0) {
    item -= n0;
    mode = MODE_DOWN;
  }
  const ModeParams& mp = mps[mode];
  d.mode = mode;
  const int per_expert = mp.pairs * mp.kslices;
  const int a = item / per_expert;
  const int rem = item - a * per_expert;
  d.a = a;
  d.pair = rem / mp.kslices;
  d.ks = rem - d.pair * mp.kslices;
  ExpertDesc x = p.xd[mode * p.E + a];
  if (!PW_CHECK(a < p.E && x.pos0 >= 0 && x.te >= 0 && x.pos0 + x.te <= mp.out_rows)) {
    x.valid = 0;  // an inconsistent grouping: nothing of this item is read or written
    x.te = 0;
    x.status = PW_ERR_BOUNDS;
  }
  d.q = x.q;
  d.n = x.n;
  d.te = x.te;
  d.pos0 = x.pos0;
  d.valid = x.valid;
  d.status = x.status;
  d.lut = x.lut;
  d.tile_words = x.tile_words;
  d.planes = x.planes + static_cast<size_t>(d.pair) * kTiles * x.tile_words;
  const int nst = (mp.cols + kStageCols - 1) / kStageCols;
  d.s0 = (nst * d.ks) / mp.kslices;
  d.s1 = (nst * (d.ks + 1)) / mp.kslices;
  d.pad0 = d.pad1 = d.pad2 = 0;
  return d;
}

// The ExpertDesc of (module `mode`, active expert a = expert e) from the Weight Page Table: the
// block must have the module's shape and tiled layout, be resident, and carry a committed
// bitwidth within [min_bits, stored planes] with its LUT.
__device__ __forceinline__ ExpertDesc expert_desc(const pw_page_table* pt, int layer, int E, int e,
                                                  int mode, int rows, int cols, int te, int pos0) {
  ExpertDesc x;
  const pw_block* b = pt->blocks + (static_cast<size_t>(layer) * E + e) * 2 + mode;
  x.q = b->committed_bits;
  // planes held per (tile, stage) run on the device: all parent_bits, or a paged-in prefix
  x.n = b->stored_bits ? b->stored_bits : b->parent_bits;
  // every LUT pointer a committed bitwidth can select, read with the other fields (one round
  // trip to memory rather than a second one that waits for the bitwidth)
  const uint16_t* lq = nullptr;
#pragma unroll
  for (int q = PW_MIN_BITS; q <= PW_MAX_BITS; ++q) {
    const uint16_t* l = b->lut[q];
    if (x.q == q) lq = l;
  }
  const bool bits_ok = x.q >= b->min_bits && x.q <= x.n && x.n <= b->parent_bits &&
                       x.q >= PW_MIN_BITS && x.q <= PW_MAX_BITS && lq != nullptr &&
                       b->planes != nullptr;
  const int want_layout = mode == MODE_GATE_UP ? PW_LAYOUT_TILED_GATE_UP : PW_LAYOUT_TILED_DOWN;
  const bool shape_ok = static_cast<int>(b->rows) == rows && static_cast<int>(b->cols) == cols &&
                        b->layout == want_layout;
  const bool resident = b->state == PW_PAGE_GPU;
  x.planes = b->planes;
  x.lut = bits_ok ? lq : nullptr;
  x.tile_words = static_cast<long long>(x.n) * kTileRows * (cols / 32);
  x.valid = bits_ok && shape_ok && resident;
  x.status = !shape_ok ? PW_ERR_INVALID_ARG : (!resident ? PW_ERR_NOT_RESIDENT : PW_ERR_BAD_BITS);
  x.te = te;
  x.pos0 = pos0;
  x.pad0 = x.pad1 = 0;
  return x;
}

// Block row of lane i's row of tile t (gate_up: 16 gate rows then the 16 matching up rows).
__device__ __forceinline__ int tile_row(int mode, int half, int t, int i) {
  if (mode == MODE_GATE_UP) return i < 16 ? t * 16 + i : half + t * 16 + (i - 16);
  return t * kTileRows + i;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (!mbar_wait(bar, parity, abort_flag)) {
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
  target += *static_cast<volatile int*>(&g_test_hold);
  if (ld_acquire(ctr) < target) {
    const unsigned long long t0 = global_ns();
    const unsigned long long limit = wait_limit_ns();
    for (uint32_t it = 1;; ++it) {
      __nanosleep(128);
      if (ld_acquire(ctr) >= target) break;
      if (*abort_flag) return false;
      if ((it & 15u) == 0 && global_ns() - t0 > limit) {
        set_status(PW_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// Exchange the bits of a selected by (M << S) with the bits of b selected by M; the left shift
// is a multiply by mul = 1 << S.  With mul opaque to the compiler it runs on the FMA pipe and
// leaves the logic pipe to the masks and the right shift.
template <int S, uint32_t M>
__device__ __forceinline__ void bswap(uint32_t& a, uint32_t& b, uint32_t mul) {
  constexpr uint32_t MH = M << S;
  const uint32_t an = (a & ~MH) | ((b * mul) & MH);
  const uint32_t bn = (b & ~M) | ((a >> S) & M);
  a = an;
  b = bn;
}

// Per byte lane, an 8x8 bit transpose across R[0..7]: afterwards bit j of byte k of R[i] is
// what bit i of byte k of R[j] was.  m_S = 1 << S.
__device__ __forceinline__ void transpose8(uint32_t (&R)[8], uint32_t m1, uint32_t m2,
                                           uint32_t m4) {
  bswap<4, 0x0F0F0F0Fu>(R[0], R[4], m4);
  bswap<4, 0x0F0F0F0Fu>(R[1], R[5], m4);
  bswap<4, 0x0F0F0F0Fu>(R[2], R[6], m4);
  bswap<4, 0x0F0F0F0Fu>(R[3], R[7], m4);
  bswap<2, 0x33333333u>(R[0], R[2], m2);
  bswap<2, 0x33333333u>(R[1], R[3], m2);
  bswap<2, 0x33333333u>(R[4], R[6], m2);
  bswap<2, 0x33333333u>(R[5], R[7], m2);
  bswap<1, 0x55555555u>(R[0], R[1], m1);
  bswap<1, 0x55555555u>(R[2], R[3], m1);
  bswap<1, 0x55555555u>(R[4], R[5], m1);
  bswap<1, 0x55555555u>(R[6], R[7], m1);
}
__device__ __forceinline__ void transpose8(uint32_t (&R)[8]) { transpose8(R, 2u, 4u, 16u); }

__device__ __forceinline__ uint32_t lds_u32(uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(g_smem + off);
}
__device__ __forceinline__ uint4 lds_u128(uint32_t off) {
  return *reinterpret_cast<const uint4*>(g_smem + off);
}

// acc + (half WH of w) * (half XH of x): fp16 operands, exact product, one fp32 rounding.
template <int WH, int XH>
__device__ __forceinline__ float hfma(uint32_t w, uint32_t x, float acc) {
  float d;
  if constexpr (WH == 0 && XH == 0)
    asm("{.reg .b16 a,b,c,e; mov.b32 {a,b},%1; mov.b32 {c,e},%2; fma.rn.f32.f16 %0,a,c,%3;}"
        : "=f"(d) : "r"(w), "r"(x), "f"(acc));
  else if constexpr (WH == 0 && XH == 1)
    asm("{.reg .b16 a,b,c,e; mov.b32 {a,b},%1; mov.b32 {c,e},%2; fma.rn.f32.f16 %0,a,e,%3;}"
        : "=f"(d) : "r"(w), "r"(x), "f"(acc));
  else if constexpr (WH == 1 && XH == 0)
    asm("{.reg .b16 a,b,c,e; mov.b32 {a,b},%1; mov.b32 {c,e},%2; fma.rn.f32.f16 %0,b,c,%3;}"
        : "=f"(d) : "r"(w), "r"(x), "f"(acc));
  else
    asm("{.reg .b16 a,b,c,e; mov.b32 {a,b},%1; mov.b32 {c,e},%2; fma.rn.f32.f16 %0,b,e,%3;}"
        : "=f"(d) : "r"(w), "r"(x), "f"(acc));
  return d;
}

// Products for code byte k of registers i (weights w0 / wb0, activation x0) and i + 4 (w1 /
// wb1, x1) into acc = {row a of 8k+i, row b of 8k+i, row a of 8k+i+4, row b of 8k+i+4}.
// PAIR: w0 holds (row a, row b) of one column; otherwise row a's weight is the low half of w0
// and row b's the high half of wb0.
template <bool PAIR, int XH>
__device__ __forceinline__ void fma4(uint32_t w0, uint32_t w1, uint32_t wb0, uint32_t wb1,
                                     uint32_t x0, uint32_t x1, float (&acc)[4]) {
  acc[0] = hfma<0, XH>(w0, x0, acc[0]);
  acc[1] = hfma<1, XH>(PAIR ? w0 : wb0, x0, acc[1]);
  acc[2] = hfma<0, XH>(w1, x1, acc[2]);
  acc[3] = hfma<1, XH>(PAIR ? w1 : wb1, x1, acc[3]);
}

// One word (32 columns) of rows a and b of this lane, NT tokens.  pa / pb: byte offsets of the
// word's most significant plane in the two tiles (planes pstride apart); xs: the word's fp16
// activations of token 0 (xstride bytes between tokens; DOWN: the lo parts 1024 bytes on).
template <int Q, int NT, bool DOWN>
__device__ __forceinline__ void decode_word(uint32_t pa, uint32_t pb, uint32_t pstride,
                                            uint32_t xs, uint32_t xstride, uint32_t lane_base,
                                            uint32_t m1, uint32_t m2, uint32_t m4,
                                            float (&acc)[NT][4]) {
  constexpr bool PAIR = Q <= 4;
  uint32_t A[8], Bq[8];
  if constexpr (PAIR) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      A[j] = j < Q ? lds_u32(pa + (Q - 1 - j) * pstride) : 0u;
      A[4 + j] = j < Q ? lds_u32(pb + (Q - 1 - j) * pstride) : 0u;
    }
    transpose8(A, m1, m2, m4);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      A[j] = j < Q ? lds_u32(pa + (Q - 1 - j) * pstride) : 0u;
      Bq[j] = j < Q ? lds_u32(pb + (Q - 1 - j) * pstride) : 0u;
    }
    transpose8(A, m1, m2, m4);
    transpose8(Bq, m1, m2, m4);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t sel = 0x7604u | (k << 4);
      const uint32_t w0 = lds_u32(__byte_perm(A[i], lane_base, sel));
      const uint32_t w1 = lds_u32(__byte_perm(A[i + 4], lane_base, sel));
      uint32_t wb0 = 0u, wb1 = 0u;
      if constexpr (!PAIR) {
        wb0 = lds_u32(__byte_perm(Bq[i], lane_base, sel));
        wb1 = lds_u32(__byte_perm(Bq[i + 4], lane_base, sel));
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        // 8 fp16 activations: words .x/.y = columns 8k+i (k = 0..3), .z/.w = 8k+i+4
        const uint4 xv = lds_u128(xs + t * xstride + i * 16);
        const uint32_t x0 = (k >> 1) ? xv.y : xv.x, x1 = (k >> 1) ? xv.w : xv.z;
        if (k & 1)
          fma4<PAIR, 1>(w0, w1, wb0, wb1, x0, x1, acc[t]);
        else
          fma4<PAIR, 0>(w0, w1, wb0, wb1, x0, x1, acc[t]);
        if constexpr (DOWN) {
          const uint4 xl = lds_u128(xs + 1024 + t * xstride + i * 16);
          const uint32_t y0 = (k >> 1) ? xl.y : xl.x, y1 = (k >> 1) ? xl.w : xl.z;
          if (k & 1)
            fma4<PAIR, 1>(w0, w1, wb0, wb1, y0, y1, acc[t]);
          else
            fma4<PAIR, 0>(w0, w1, wb0, wb1, y0, y1, acc[t]);
        }
      }
    }
  }
}

// Byte offsets inside a slot holding stages s, s + 1 (m of them) of an item at bitwidth q: tile
// 2P's planes of sub-stage j at j q 2 KB, tile 2P + 1's m q 2 KB further on, then the
// activation chunk of token t and sub-stage j at 2 m q 2 KB + (t m + j) xunit (xunit: 1 KB of
// x for gate_up, 2 KB of h hi and lo for down).
__host__ __device__ __forceinline__ uint32_t slot_tile_b(int q, int m) {
  return static_cast<uint32_t>(m * q * kStageWords * 128);
}
__host__ __device__ __forceinline__ uint32_t slot_x(int q, int m) { return 2 * slot_tile_b(q, m); }

// The stage loop of one pass over an item, one decode warp.  Every argument is a scalar
// passed by value so nothing of it lives in local memory.  Slot unit g of the launch sits in
// ring slot g % NS and holds M = sub_stages(Q) consecutive stages.  At the end it waits until
// the reducer has freed the partial-sum buffer (rfree, phase rphase) and writes the warp's sums
// of rows a and b per token there; the caller advances its slot counter by the item's units.
template <int Q, int NT, int NS, int MS, bool DOWN>
__device__ __noinline__ void run_stages(uint64_t* full, uint64_t* empty,
                                        volatile int* abort_flag, uint32_t slot_bytes,
                                        int words_total, uint32_t lane_base, int s0, int s1,
                                        uint32_t g, uint32_t one, float* part, uint64_t* rfree,
                                        uint32_t rphase) {
  constexpr int M = Q <= 4 ? MS : 1;
  constexpr int XU = DOWN ? kXBytesDown : kXBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t m1 = one << 1, m2 = one << 2, m4 = one << 4;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  for (int s = s0; s < s1; s += M, ++g) {
    const int slot = g % NS;
    wait_bar(&full[slot], (g / NS) & 1, abort_flag);
    const uint32_t st = kTableBytes + slot * slot_bytes;
#pragma unroll
    for (int j = 0; j < M; ++j) {
      if (s + j >= s1) break;
      const int ws = min(kStageWords, words_total - (s + j) * kStageWords);
      if (warp < ws) {
        const uint32_t pa = st + j * Q * kStageWords * 128 + warp * 128 + lane * 4;
        decode_word<Q, NT, DOWN>(pa, pa + M * Q * kStageWords * 128, ws * 128,
                                 st + 2 * M * Q * kStageWords * 128 + j * XU + warp * 64,
                                 M * XU, lane_base, m1, m2, m4, acc);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
  wait_bar(rfree, rphase, abort_flag);
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    part[(2 * t) * 32] = acc[t][0] + acc[t][2];
    part[(2 * t + 1) * 32] = acc[t][1] + acc[t][3];
  }
}

#define PW_RUN_ARGS                                                                          \
  full, empty, abort_flag, LY::kSlotBytes, words_total, lane_base, d.s0, d.s1, g, one, part,  \
      rfree, rphase

template <int NT, int NTP, bool DOWN>
__device__ __forceinline__ void run_qm(const Desc& d, uint64_t* full, uint64_t* empty,
                                       volatile int* abort_flag, int words_total,
                                       uint32_t lane_base, uint32_t g, uint32_t one, float* part,
                                       uint64_t* rfree, uint32_t rphase) {
  using LY = Layout<NTP>;
  constexpr int NS = LY::kStages, MS = LY::kMaxSub;
  switch (d.q) {
    case 3: run_stages<3, NT, NS, MS, DOWN>(PW_RUN_ARGS); break;
    case 4: run_stages<4, NT, NS, MS, DOWN>(PW_RUN_ARGS); break;
    case 5: run_stages<5, NT, NS, MS, DOWN>(PW_RUN_ARGS); break;
    case 6: run_stages<6, NT, NS, MS, DOWN>(PW_RUN_ARGS); break;
    case 7: run_stages<7, NT, NS, MS, DOWN>(PW_RUN_ARGS); break;
    default: run_stages<8, NT, NS, MS, DOWN>(PW_RUN_ARGS); break;
  }
}

template <int NT, int NTP>
__device__ __forceinline__ void run_q(const Desc& d, uint64_t* full, uint64_t* empty,
                                      volatile int* abort_flag, int words_total,
                                      uint32_t lane_base, uint32_t g, uint32_t one, float* part,
                                      uint64_t* rfree, uint32_t rphase) {
  if (d.mode == MODE_DOWN)
    run_qm<NT, NTP, true>(d, full, empty, abort_flag, words_total, lane_base, g, one, part,
                          rfree, rphase);
  else
    run_qm<NT, NTP, false>(d, full, empty, abort_flag, words_total, lane_base, g, one, part,
                           rfree, rphase);
}
#undef PW_RUN_ARGS

// LUT warp lw (0..3), lane i (rows a and b of lane i).  fetch_table reads one round of the
// lane's share of the two fp16 LUT rows into registers (q >= 5: round h = entries
// [lw 2^q/4 + 32h, +32) of each row; q = 8 takes two rounds, q <= 7 one); round 0 is issued
// before the warp waits for a free table buffer, so its load latency overlaps that wait.
struct LutRegs {
  uint4 a[4], b[4];  // q >= 5: up to 32 entries of rows a and b; q <= 4: a[0..1] = row a
  uint2 bq;          // q <= 4: entries [lw 2^q/4, (lw+1) 2^q/4) of row b
};

// 16 / 8 / 4 bytes of read-only global data (the LUT rows: the four LUT warps read the same
// rows for q <= 4, so they go through L1).
__device__ __forceinline__ uint4 ldg16(const void* p) { return __ldg(static_cast<const uint4*>(p)); }
__device__ __forceinline__ uint2 ldg8(const void* p) { return __ldg(static_cast<const uint2*>(p)); }
__device__ __forceinline__ uint32_t ldg4(const void* p) {
  return __ldg(static_cast<const uint32_t*>(p));
}

__device__ __forceinline__ void fetch_table(const uint16_t* __restrict__ ra,
                                            const uint16_t* __restrict__ rb, int q, int lw,
                                            int round, LutRegs& r) {
  if (q >= 5) {
    const int quarter = 1 << (q - 2);
    const int n8 = min(quarter, 32) / 8;  // uint4 per row this round
    const uint4* sa = reinterpret_cast<const uint4*>(ra + lw * quarter + 32 * round);
    const uint4* sb = reinterpret_cast<const uint4*>(rb + lw * quarter + 32 * round);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < n8) {
        r.a[k] = ldg16(sa + k);
        r.b[k] = ldg16(sb + k);
      }
  } else {
    r.a[0] = ldg16(ra);
    if (q == 4) {
      r.a[1] = ldg16(ra + 8);
      r.bq = ldg8(rb + 4 * lw);                  // 4 entries
    } else {
      r.bq = make_uint2(ldg4(rb + 2 * lw), 0u);  // 2 entries
    }
  }
}

// Entry e (static) of 16 fp16 values held in two uint4.
__device__ __forceinline__ uint32_t entry16(const uint4 (&v)[4], int e) {
  const uint4 u = v[e >> 3];
  const int w = (e >> 1) & 3;
  const uint32_t x = w == 0 ? u.x : w == 1 ? u.y : w == 2 ? u.z : u.w;
  return (e & 1) ? (x >> 16) : (x & 0xffffu);
}

// One fetched round of the LUT rows -> its slots of the decode table in buffer u.
__device__ __forceinline__ void store_table(const LutRegs& r, int q, uint32_t u, int lw,
                                            int round, int lane) {
  const uint32_t col = u * 128 + lane * 4;
  if (q >= 5) {  // slot v = (LUT_a[v], LUT_b[v]), v in this warp's quarter
    const int quarter = 1 << (q - 2);
    const int n8 = min(quarter, 32) / 8;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k >= n8) break;
      const uint32_t wa[4] = {r.a[k].x, r.a[k].y, r.a[k].z, r.a[k].w};
      const uint32_t wb[4] = {r.b[k].x, r.b[k].y, r.b[k].z, r.b[k].w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int v = lw * quarter + 32 * round + k * 8 + 2 * m;
        *reinterpret_cast<uint32_t*>(g_smem + v * 256 + col) = __byte_perm(wa[m], wb[m], 0x5410u);
        *reinterpret_cast<uint32_t*>(g_smem + (v + 1) * 256 + col) =
            __byte_perm(wa[m], wb[m], 0x7632u);
      }
    }
  } else {  // slot va + 16 vb = (LUT_a[va], LUT_b[vb]), vb in this warp's quarter
    const int nv = 1 << q, qv = nv >> 2;
    const uint32_t bw[4] = {r.bq.x & 0xffffu, r.bq.x >> 16, r.bq.y & 0xffffu, r.bq.y >> 16};
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      if (kb >= qv) break;
      const int vb = lw * qv + kb;
      const uint32_t hb = bw[kb] << 16;
#pragma unroll
      for (int va = 0; va < 16; ++va) {
        if (va >= nv) break;
        *reinterpret_cast<uint32_t*>(g_smem + (va + 16 * vb) * 256 + col) = entry16(r.a, va) | hb;
      }
    }
  }
}

// h of feature f at its place in the down projection's activations: per 512-column stage,
// 512 hi values then 512 lo values (hi = fp16(h), lo = fp16(h - hi)), xpos order inside.
__device__ __forceinline__ void store_h(__half* hrow, int f, float h) {
  const __half hi = __float2half_rn(h);
  __half* c = hrow + (f / kStageCols) * (2 * kStageCols) + xpos(f % kStageCols);
  c[0] = hi;
  c[kStageCols] = __float2half_rn(h - __half2float(hi));
}

template <int NTP>
__global__ void __launch_bounds__(kThreads, 1) ffn_kernel(const Params p) {
  using LY = Layout<NTP>;
  uint8_t* const smem = g_smem;
  uint8_t* ring = smem + LY::kOffRing;  // LY::kStages slots
  float* red = reinterpret_cast<float*>(smem + LY::kOffRed);
  Desc* cdesc = reinterpret_cast<Desc*>(smem + LY::kOffDesc);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::kOffBar);
  uint64_t* empty = full + LY::kStages;
  uint64_t* lut_ready = empty + LY::kStages;  // [2] table built (LUT warps -> decode)
  uint64_t* lut_free = lut_ready + 2;         // [2] table released (decode -> LUT warps)
  uint64_t* red_full = lut_free + 2;          // [2] partial sums written (decode -> reducer)
  uint64_t* red_free = red_full + 2;          // [2] partial sums consumed (reducer -> decode)
  uint64_t* const desc_full = red_free + 2;   // [kDescRing] descriptor written (producer)
  uint64_t* const desc_free = desc_full + kDescRing;  // [kDescRing] read by all other warps
  volatile int* abort_flag = reinterpret_cast<volatile int*>(desc_free + kDescRing);
  ModeParams* mps = reinterpret_cast<ModeParams*>(smem + LY::kOffMisc);
  const uint8_t** arow = reinterpret_cast<const uint8_t**>(smem + LY::kOffMisc + 2 * 128);

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
      mbar_init(&desc_full[r], 1);  // written by the producer
      mbar_init(&desc_free[r], kLutWarps + 1 + kDecodeWarps);  // read by every other warp
    }
    *abort_flag = 0;
    mps[0] = p.m[0];
    mps[1] = p.m[1];
    mbar_fence_init();
  }
  __syncthreads();
  griddep_wait();  // the grouping and the activations come from the launch before
  griddep_launch();

  const int n_active = p.meta[0];
  const int n_items = items_of(mps, MODE_GATE_UP, n_active) + items_of(mps, MODE_DOWN, n_active);

  if (warp == kProducerWarp) {
    // ---------------- producer: one thread streams every stage ----------------
    if (lane != 0) return;
    uint32_t g = 0;  // slot units issued
    int ready_a = -1;  // active expert whose h was last seen complete
    int arow_mode = -1, arow_a = -1;  // whose activation rows arow holds
    // Descriptor j + 1 is published before item j is streamed, so the LUT warps build its
    // table while the stages before it are still being fetched; the item for descriptor j + 2
    // is claimed right after, and the counter's reply is only needed one item later, so the
    // atomic's round trip overlaps the streaming of item j.
    auto publish = [&](uint32_t jj, int item) -> Desc {
      Desc d;
      d.item = -1;
      if (item < n_items) d = resolve(p, mps, item, n_active);
      // every other warp has read descriptor jj - kDescRing from this slot
      wait_bar(&desc_free[jj % kDescRing], ((jj / kDescRing) & 1) ^ 1, abort_flag);
      cdesc[jj % kDescRing] = d;
      mbar_arrive(&desc_full[jj % kDescRing]);
      return d;
    };
    Desc nxt = publish(0, atomicAdd(p.sched, 1));
    int claimed = nxt.item >= 0 ? atomicAdd(p.sched, 1) : n_items;
    for (uint32_t j = 0;; ++j) {
      const Desc cur = nxt;
      if (cur.item < 0 || *abort_flag) break;
      nxt = publish(j + 1, claimed);
      claimed = nxt.item >= 0 ? atomicAdd(p.sched, 1) : n_items;
      if (!cur.valid) continue;
      const ModeParams& mp = mps[cur.mode];
      const int words_total = mp.cols / 32;
      // h of this expert is complete once all its gate_up items are counted.  The count only
      // grows, so once seen complete it is not read again for the expert's later items (they
      // are claimed one after the other): the acquire and its fence already order every later
      // copy of h.
      if (cur.mode == MODE_DOWN && cur.a != ready_a) {
        if (!wait_count(p.done + cur.a, mps[MODE_GATE_UP].pairs, abort_flag)) break;
        ready_a = cur.a;
      }
      const uint32_t* pa = cur.planes;
      const uint32_t* pb = cur.planes + cur.tile_words;
      for (int ch = 0; ch < cur.te; ch += NTP) {
        const int ntok = min(NTP, cur.te - ch);
        // the activation rows of the pass (a gate_up row comes from the grouping, one global
        // load each): an item whose tokens fit one pass reuses the rows of the item before it
        // when both are of the same module and expert
        const bool reuse = cur.te <= NTP && cur.mode == arow_mode && cur.a == arow_a;
        if (!reuse) {
          for (int t = 0; t < ntok; ++t) {
            const int pos = cur.pos0 + ch + t;
            int r = mp.act_map ? mp.act_map[pos] / mp.act_div : pos;
            if (!PW_CHECK(r >= 0 && r < mp.act_rows)) r = 0;  // (debug build) read row 0
            arow[t] =
                reinterpret_cast<const uint8_t*>(mp.act + static_cast<size_t>(r) * mp.ld_act);
          }
          arow_mode = cur.te <= NTP ? cur.mode : -1;
          arow_a = cur.a;
        }
        const int m = sub_stages(cur.q, LY::kMaxSub);
        const uint32_t tb = slot_tile_b(cur.q, m), xo = slot_x(cur.q, m);
        const uint32_t xu = cur.mode == MODE_DOWN ? kXBytesDown : kXBytes;
        for (int s = cur.s0; s < cur.s1; s += m, ++g) {
          const int slot = g % LY::kStages;
          wait_bar(&empty[slot], ((g / LY::kStages) & 1) ^ 1, abort_flag);
          uint8_t* st = ring + slot * LY::kSlotBytes;
          const int nsub = min(m, cur.s1 - s);
          uint32_t bytes = ntok * nsub * xu;
          for (int j = 0; j < nsub; ++j)
            bytes += 2 * cur.q * min(kStageWords, words_total - (s + j) * kStageWords) * 128;
          mbar_arrive_expect_tx(&full[slot], bytes);
          for (int j = 0; j < nsub; ++j) {
            const int ws = min(kStageWords, words_total - (s + j) * kStageWords);
            const uint32_t pbytes = cur.q * ws * kTileRows * 4;
            const size_t soff = static_cast<size_t>(s + j) * cur.n * kTileRows * kStageWords;
            const uint32_t sub = j * cur.q * kStageWords * 128;
            bulk_g2s(st + sub, pa + soff, pbytes, &full[slot]);
            bulk_g2s(st + tb + sub, pb + soff, pbytes, &full[slot]);
            for (int t = 0; t < ntok; ++t)
              bulk_g2s(st + xo + (t * m + j) * xu, arow[t] + static_cast<size_t>(s + j) * xu, xu,
                       &full[slot]);
          }
        }
        if (*abort_flag) break;
      }
      if (*abort_flag) break;
    }
    // drain: every issued copy has landed before the block exits (abort or not)
    for (uint32_t d = (g > LY::kStages ? g - LY::kStages : 0); d < g; ++d)
      mbar_wait(&full[d % LY::kStages], (d / LY::kStages) & 1);
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
      const ModeParams& mp = mps[it.mode];
      if (!it.valid) {
        // a block that cannot be read (state, bitwidth or shape): its outputs are zeros
        if (lane == 0) set_status(it.status);
        for (int t = 0; t < it.te; ++t) {
          const size_t pos = static_cast<size_t>(it.pos0 + t);
          if (it.mode == MODE_GATE_UP) {
            store_h(mp.hout + pos * mp.ld_hout, it.pair * 32 + lane, 0.f);
          } else if (PW_CHECK(pos < static_cast<size_t>(mp.out_rows) &&
                              it.pair * kItemRows + 64 <= mp.ld_out)) {
            float* o = mp.out + it.ks * mp.out_slice + pos * mp.ld_out + it.pair * kItemRows;
            o[lane] = 0.f;
            o[32 + lane] = 0.f;
          }
        }
      }
      for (int ch = 0; it.valid && ch < it.te; ch += NTP, ++rc) {
        const int ntok = min(NTP, it.te - ch);
        const int par = rc & 1;
        wait_bar(&red_full[par], (rc >> 1) & 1, abort_flag);
        const float* rb = red + par * (kDecodeWarps * NTP * kTiles * 32);
        for (int t = 0; t < ntok; ++t) {
          float ta = 0.f, tb = 0.f;
#pragma unroll
          for (int w = 0; w < kDecodeWarps; ++w) {
            ta += rb[((w * NTP + t) * 2) * 32 + lane];
            tb += rb[((w * NTP + t) * 2 + 1) * 32 + lane];
          }
          const size_t pos = static_cast<size_t>(it.pos0 + ch + t);
          if (!PW_CHECK(pos < static_cast<size_t>(mp.out_rows))) continue;
          if (it.mode == MODE_GATE_UP) {
            // lane i < 16: gate rows of features 32P + i (row a) and 32P + 16 + i (row b);
            // lane i + 16: the matching up rows
            const float ua = __shfl_down_sync(0xffffffffu, ta, 16);
            const float ub = __shfl_down_sync(0xffffffffu, tb, 16);
            if (lane < 16) {
              __half* hrow = mp.hout + pos * mp.ld_hout;
              store_h(hrow, it.pair * 32 + lane, ta / (1.0f + expf(-ta)) * ua);
              store_h(hrow, it.pair * 32 + 16 + lane, tb / (1.0f + expf(-tb)) * ub);
            }
          } else {
            float* o = mp.out + it.ks * mp.out_slice + pos * mp.ld_out + it.pair * kItemRows;
            o[lane] = ta;
            o[32 + lane] = tb;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_free[par]);
      }
      if (it.mode == MODE_GATE_UP) {
        // this item's h rows are written: make them visible, then count the item
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.done + it.a, 1);
      }
    }
    return;
  }

  if (warp >= kLutWarp0) {
    // ---------------- LUT warps: the decode tables ----------------
    const int lw = warp - kLutWarp0;
    for (uint32_t j = 0;; ++j) {
      const uint32_t u = j & 1;
      wait_bar(&desc_full[j % kDescRing], (j / kDescRing) & 1, abort_flag);
      const Desc it = cdesc[j % kDescRing];
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_free[j % kDescRing]);
      if (it.item < 0 || *abort_flag) {
        // the decode warps learn of the end through lut_ready like any item; it follows their
        // release of buffer u (item j - 2), so no barrier phase runs ahead of a waiter
        wait_bar(&lut_free[u], ((j >> 1) & 1) ^ 1, abort_flag);
        __syncwarp();
        if (lane == 0) mbar_arrive(&lut_ready[u]);
        break;
      }
      LutRegs lr;
      const uint16_t* lra = nullptr;
      const uint16_t* lrb = nullptr;
      if (it.valid) {
        const int half = mps[it.mode].half;
        lra = it.lut + (static_cast<size_t>(tile_row(it.mode, half, 2 * it.pair, lane)) << it.q);
        lrb = it.lut +
              (static_cast<size_t>(tile_row(it.mode, half, 2 * it.pair + 1, lane)) << it.q);
        fetch_table(lra, lrb, it.q, lw, 0, lr);
      }
      wait_bar(&lut_free[u], ((j >> 1) & 1) ^ 1, abort_flag);  // decode warps left item j-2
      if (it.valid) {
        store_table(lr, it.q, u, lw, 0, lane);
        if (it.q == 8) {  // the second round of 32 entries
          fetch_table(lra, lrb, it.q, lw, 1, lr);
          store_table(lr, it.q, u, lw, 1, lane);
        }
      }
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
    __syncwarp();
    if (lane == 0) mbar_arrive(&desc_free[j % kDescRing]);
    if (d.item < 0 || *abort_flag) break;
    if (!d.valid) {  // the reducer writes this item's zeros
      __syncwarp();
      if (lane == 0) mbar_arrive(&lut_free[u]);
      continue;
    }
    const ModeParams& mp = mps[d.mode];
    const int words_total = mp.cols / 32;
    const uint32_t lane_base = u * 128 + lane * 4;
    for (int ch = 0; ch < d.te; ch += NTP, ++rc) {
      const int ntok = min(NTP, d.te - ch);
      // partial sums into buffer rc & 1 once the reducer has consumed pass rc - 2
      const int par = rc & 1;
      float* part = red + par * (kDecodeWarps * NTP * kTiles * 32) + warp * NTP * kTiles * 32 +
                    lane;
      uint64_t* rfree = &red_free[par];
      const uint32_t rphase = ((rc >> 1) & 1) ^ 1;
      const uint32_t one = p.one;
      if (NTP == 1 || ntok == 1)
        run_q<1, NTP>(d, full, empty, abort_flag, words_total, lane_base, g, one, part, rfree,
                      rphase);
      else if (NTP >= 2 && ntok == 2)
        run_q<(NTP >= 2 ? 2 : 1), NTP>(d, full, empty, abort_flag, words_total, lane_base, g,
                                       one, part, rfree, rphase);
      else if (NTP >= 4 && ntok == 3)
        run_q<(NTP >= 4 ? 3 : 1), NTP>(d, full, empty, abort_flag, words_total, lane_base, g,
                                       one, part, rfree, rphase);
      else
        run_q<(NTP >= 4 ? 4 : 1), NTP>(d, full, empty, abort_flag, words_total, lane_base, g,
                                       one, part, rfree, rphase);
      {
        const int m = sub_stages(d.q, LY::kMaxSub);
        g += (d.s1 - d.s0 + m - 1) / m;
      }
      if (ch + NTP >= d.te) {  // last pass over this item: release the table
        __syncwarp();
        if (lane == 0) mbar_arrive(&lut_free[u]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_full[par]);
    }
  }
}

}  // namespace k4
}  // namespace pw
