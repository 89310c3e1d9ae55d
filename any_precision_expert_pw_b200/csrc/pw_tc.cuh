// K5: the grouped expert FFN for larger batches, on the tensor cores (PagedWeight, "Composants
// Clés" 1 and 3: one fused kernel reads the bit-planes and LUTs directly, each block at its own
// bitwidth).  With many tokens per expert the bit-plane GEMV of K4, which decodes every weight
// once per four tokens, becomes a GEMM: here each weight is decoded once per pass of up to 64
// tokens and the products run on tcgen05.
//
// Work item = (active expert, pass of up to 64 of its tokens, 128-row block = four 32-row
// tiles, k-slice).  A block whose columns are not a multiple of 256 ends in a 128-column chunk.  D[128 rows][np tokens] (fp32, in tensor memory) += A[128][K] * B[np][K]^T,
// with A the decoded weights (fp16 LUT values, exact; in tensor memory) and B the pass's
// activations (fp16, in shared memory).
//
// Warp roles (one CTA per SM, persistent over the items):
//   decode (16 warps)      warp w takes tile w % 4 of the block and words 2(w / 4), 2(w / 4) + 1
//                          (64 columns) of each 256-column chunk; lane = row.  An 8x8 bit
//                          transpose of its q plane words gives one code byte per weight, a
//                          gather from the row's table gives the fp16 value, and each word's
//                          32 values go to the chunk's A buffer in tensor memory (the warp's
//                          own lane quarter, two fp16 per column) with one tcgen05.st;
//                          At each item's start the sixteen warps first build its decode table
//                          together (warp w: tile w % 4, a quarter of the slots);
//   epilogue (4)           warp 16 + j reads rows 32j.. of the accumulator back (tensor-memory
//                          lane quarter j): SiLU(gate) * up as fp16 into the down projection's
//                          operand, or the down rows into the k-slice partials; warp 16 also
//                          takes the items from a work counter (the first one included, so
//                          only running CTAs own items), one ahead,
//                          and prefetches the next item's LUT rows and first planes into L2;
//   plane producer (1)     bulk-copies each chunk's top-q planes of the four tiles (4q runs of
//                          1 KB in the tiled layout) into a ring of three stages;
//   operand producer (1)   bulk-copies each chunk's activations (np * 512 contiguous bytes;
//                          for down, h as hi + lo fp16 parts, one block per 32-token sub-pass);
//                          a down item first waits until every gate_up item of its expert is
//                          counted;
//   MMA (1)                one thread issues 16 tcgen05.mma (K = 16 each) per chunk and operand
//                          part into one of two accumulators and commits each operand block's
//                          completion to the barrier that frees its B buffer, each chunk's to the
//                          one that frees its A buffer.
// The down projection's activations h are fp32 results of the gate_up epilogue; they are held as
// hi = fp16(h) and lo = fp16(h - hi), so the products keep h to about 22 bits (a single fp16
// rounding of h, 2^-11 relative, leaves the whole output of a large batch at the edge of the
// parity bar).  A down operand block stacks, per 8-column K group, the nps hi rows and then the
// nps lo rows: one MMA of N = 2 nps per K step writes the hi products to accumulator columns
// [0, nps) and the lo products to [nps, 2 nps), and the epilogue adds the two.  A pass of more
// than 32 tokens is split into two sub-passes of 32 + the rest (accumulator columns 64 sp ..),
// so that a sub-pass's block of a chunk fits one B buffer.
// The decode table pairs rows r and r + 64 of the item: the 32-bit slot at byte 256v + 4r
// (r < 64) holds (LUT_r[v], LUT_{r+64}[v]).  A warp's 32 rows are 32 consecutive r mod 64, so
// its gathers hit 32 different banks, the slot address is one byte permute of the code byte,
// and which half a warp takes is fixed (tiles 0-1 low, 2-3 high): one more byte permute packs
// two weights.
#pragma once
#include "pw_common.cuh"
#include "pw_ffn.cuh"
#include "pw_group.cuh"

namespace pw {
namespace k5 {

constexpr int kRows = 128;        // MMA M
constexpr int kTiles = 4;         // 32-row tiles per item
constexpr int kChunkCols = kTcChunkCols;  // K columns per pipeline step (256)
constexpr int kChunkWords = kChunkCols / 32;
constexpr int kPass = kPassTokens;
constexpr int kDecodeWarps = 16;
constexpr int kEpiWarp0 = 16;
constexpr int kEpiWarps = 4;
constexpr int kPlaneWarp = 20;
constexpr int kOperandWarp = 21;
constexpr int kMmaWarp = 22;
constexpr int kThreads = 23 * 32;
// tensor memory: two accumulators of 128 fp32 columns (a gate_up pass uses np of them, a down
// pass 2 np: the products with h's hi parts and with its lo parts side by side), then two A
// buffers of 128 columns (128 rows x 256 fp16): 512 columns
constexpr int kTmemCols = 512;
constexpr int kAccCols = 2 * kPass;
constexpr int kTmemA = 2 * kAccCols;
constexpr int kACols = kChunkCols / 2;
constexpr int kPlaneStages = 3;
constexpr int kDescRing = 8;
constexpr int kDescReaders = 3 + kDecodeWarps + 3;

constexpr int kOffTable = 0;
constexpr int kTableBytes = 256 * 64 * 4;               // 2^8 entries x 64 row pairs x 4 bytes
constexpr int kOffB = kOffTable + kTableBytes;
constexpr int kBBytes = (kChunkCols / 8) * kPass * 16;  // [32 k-groups][np rows][16 bytes]
constexpr int kOffPlanes = kOffB + 2 * kBBytes;
constexpr int kPieceBytes = kChunkWords * 32 * 4;       // one plane of one tile for one chunk
constexpr int kPlaneStageBytes = kTiles * PW_MAX_BITS * kPieceBytes;
constexpr int kOffDesc = kOffPlanes + kPlaneStages * kPlaneStageBytes;

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

struct ModeParams {
  int rows;      // expected block rows (2I or H)
  int cols;      // expected block cols (H or I)
  int half;      // gate_up: I (offset of the up rows); down: 0
  int mblocks;   // 128-row blocks per expert
  int kslices;   // k-slices per block (1 for gate_up)
  const __half* bsrc;  // operand staging [padded rows][cols], chunk order (stage_x_kernel)
  __half* hout;        // gate_up: the down projection's operand staging, 2 I per padded row
  float* out;          // down: [kslice][pos][ld_out]
  int ld_out;
  long long out_slice;
};

// gate_up items: passes x gate_up blocks; then down items: passes x down blocks x k-slices.
struct Params {
  const pw_page_table* pt;
  int layer;
  int E;
  ModeParams m[2];
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* meta;
  const int32_t* pbase;
  const int32_t* pass_tab;
  int* sched;  // work counter (zero at launch)
  int* done;   // [E] per active expert: gate_up items finished x 4 epilogue warps (zero at launch)
};

struct Desc {
  const uint32_t* planes;  // tile 0 of the block (tiled layout); tiles follow at tile_words
  const uint16_t* lut;     // the block's q-bit LUT
  const __half* bsrc;      // chunk 0 of this pass's operand
  long long tile_words;
  int item, valid, status, q, n, mode, a, mb, ks, c0, c1, np, te, pos0, prow0, target;
};
static_assert(sizeof(Desc) == 96, "descriptor size");

constexpr int kOffBar = kOffDesc + kDescRing * static_cast<int>(sizeof(Desc));
// barriers: pl_full[3] pl_empty[3] b_full[2] ab_empty[2] a_full[2] acc_full[2] acc_empty[2]
// b_empty[2] table_ready table_free desc_full[8] desc_free[8] mma_done; then the TMEM address
// and the abort flag
constexpr int kNumBars = 2 * kPlaneStages + 12 + 2 + 2 * kDescRing + 1;
constexpr int kSmem = kOffBar + kNumBars * 8 + 16;
static_assert(kSmem <= 227 * 1024, "shared memory budget");
static_assert(kOffB % 1024 == 0 && kOffPlanes % 1024 == 0, "alignment");

__device__ __forceinline__ int items_of(const Params& p, int mode, int npass) {
  return npass * p.m[mode].mblocks * p.m[mode].kslices;
}

__device__ __forceinline__ Desc resolve(const Params& p, int item, int npass) {
  Desc d;
  int mode = MODE_GATE_UP;
  const int n0 = items_of(p, MODE_GATE_UP, npass);
  if (item >= n0) {
    item -= n0;
    mode = MODE_DOWN;
  }
  const ModeParams& mp = p.m[mode];
  const int per_pass = mp.mblocks * mp.kslices;
  const int pi = item / per_pass;
  const int rem = item - pi * per_pass;
  d.mb = rem / mp.kslices;
  d.ks = rem - d.mb * mp.kslices;
  const int pt_ent = p.pass_tab[pi];
  const int a = pt_ent & 0xffff, j = pt_ent >> 16;
  const int e = p.active[a];
  const int cnt = p.counts[e];
  d.mode = mode;
  d.a = a;
  d.te = min(kPass, cnt - kPass * j);
  d.np = pass_np(cnt, j);
  d.pos0 = p.offsets[e] + kPass * j;
  d.prow0 = p.pbase[e] + kPass * j;
  // each of the four epilogue warps counts every gate_up item of the expert once
  d.target = kEpiWarps * p.m[MODE_GATE_UP].mblocks * ((cnt + kPass - 1) / kPass);
  const int nch = (mp.cols + kChunkCols - 1) / kChunkCols;  // a last chunk may hold 128 columns
  d.c0 = (nch * d.ks) / mp.kslices;
  d.c1 = (nch * (d.ks + 1)) / mp.kslices;
  // gate_up operand: cols fp16 per padded row; down: hi and lo, 2 cols per padded row
  d.bsrc = mp.bsrc + static_cast<size_t>(d.prow0) * mp.cols * (mode == MODE_DOWN ? 2 : 1);
  const pw_block* b = p.pt->blocks + (static_cast<size_t>(p.layer) * p.E + e) * 2 + mode;
  d.q = b->committed_bits;
  d.n = b->stored_bits ? b->stored_bits : b->parent_bits;
  const bool bits_ok = d.q >= b->min_bits && d.q <= d.n && d.n <= b->parent_bits &&
                       d.q >= PW_MIN_BITS && d.q <= PW_MAX_BITS && b->lut[d.q] != nullptr &&
                       b->planes != nullptr;
  const int want_layout = mode == MODE_GATE_UP ? PW_LAYOUT_TILED_GATE_UP : PW_LAYOUT_TILED_DOWN;
  const bool shape_ok = static_cast<int>(b->rows) == mp.rows &&
                        static_cast<int>(b->cols) == mp.cols && b->layout == want_layout;
  const bool resident = b->state == PW_PAGE_GPU;
  d.tile_words = static_cast<long long>(d.n) * 32 * (mp.cols / 32);
  // gate_up tiles are 16 gate + 16 up rows (tile index = 16-row group); down tiles 32 rows
  d.planes = b->planes + static_cast<size_t>(d.mb) * kTiles * d.tile_words;
  d.lut = bits_ok ? b->lut[d.q] : nullptr;
  d.valid = bits_ok && shape_ok && resident;
  d.status = !shape_ok ? PW_ERR_INVALID_ARG : (!resident ? PW_ERR_NOT_RESIDENT : PW_ERR_BAD_BITS);
  // (debug build) the pass lies inside the grouping: positions and padded rows
  if (!PW_CHECK(a < p.E && d.pos0 >= 0 && d.pos0 + d.te <= p.meta[1] &&
                d.prow0 + d.np <= p.meta[6])) {
    d.valid = 0;
    d.te = 0;
    d.status = PW_ERR_BOUNDS;
  }
  return d;
}

// ---- tcgen05 wrappers ----
// Shared-memory matrix descriptor, no swizzle, K-major: start address, leading byte offset
// (between core matrices adjacent in K), stride byte offset (between 8-row groups), version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3fffu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3fffu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::f16: fp16 A and B (both K-major), fp32 D, M = 128, N = n.
__device__ __forceinline__ uint32_t instr_desc(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(kRows >> 4) << 24);
}

// D (tensor memory) = or += A (tensor memory; a_tmem: lane 0, first column of the 128 x 16
// slice, two fp16 per column) x B (shared-memory descriptor) for one K = 16 step.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on `bar` when every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                   "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive fp32 columns of this warp's tensor-memory lane quarter, one row per lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (!mbar_wait(bar, parity, abort_flag)) {
    *abort_flag = 1;
    return false;
  }
  return true;
}

// Every lane of the warp waits (a wait by lane 0 alone, the others held at a warp barrier,
// measured about twice as slow for the decode warps); the result is the same in all lanes
// (false if any lane's wait failed), so no later warp-wide step meets a split warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag));
}

using k4::g_smem;

__device__ __forceinline__ uint32_t lds_u32(uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(g_smem + off);
}

// One decode warp, one chunk: words 2jj and 2jj + 1 (64 columns) of tile t's rows at q planes
// -> 2 x 32 fp16 weights, stored to tensor memory at a_taddr and a_taddr + 16 (lane = row;
// column j holds columns 2j, 2j + 1 of the pair).
template <int Q>
__device__ __forceinline__ void decode_pair(uint32_t planes_off, uint32_t a_taddr, int t, int jj,
                                            int lane) {
  const int r = t * 32 + lane;  // row of the item's 128
  // piece (t, p) = [word][row]: words 2jj and 2jj + 1 of this lane's row, 4 bytes each (a
  // warp's load is 128 contiguous bytes: conflict free)
  const uint32_t off = planes_off + jj * 256 + lane * 4;
  uint2 P[Q];
#pragma unroll
  for (int p = 0; p < Q; ++p) {
    P[p].x = *reinterpret_cast<const uint32_t*>(g_smem + off + (t * Q + p) * kPieceBytes);
    P[p].y = *reinterpret_cast<const uint32_t*>(g_smem + off + 128 + (t * Q + p) * kPieceBytes);
  }
  // slot address of code v: 256v + 4 (r mod 64); the byte permute puts v in byte 1
  const uint32_t lbase = static_cast<uint32_t>((r & 63) * 4);
  const uint32_t psel = (t >> 1) ? 0x7632u : 0x5410u;  // high or low halves
#pragma unroll
  for (int wi = 0; wi < 2; ++wi) {
    uint32_t R[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) R[j] = j < Q ? (wi ? P[Q - 1 - j].y : P[Q - 1 - j].x) : 0u;
    k4::transpose8(R);  // byte b of R[i] = code of column 8b + i
    uint32_t w[16];     // w[4b + m] = columns 8b + 2m, 8b + 2m + 1
#pragma unroll
    for (int b = 0; b < 4; ++b) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t sel = 0x7604u | (b << 4);
        const uint32_t s0 = lds_u32(kOffTable + __byte_perm(R[2 * m], lbase, sel));
        const uint32_t s1 = lds_u32(kOffTable + __byte_perm(R[2 * m + 1], lbase, sel));
        w[4 * b + m] = __byte_perm(s0, s1, psel);
      }
    }
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(
            a_taddr + 16 * wi),
        "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
        "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]),
        "r"(w[15])
        : "memory");
  }
}

// The chunks c0..c1 of one item, one decode warp; returns the chunk counter after them.
// words_total = the block's columns / 32 (a last chunk may hold only 4 words: warps whose pair
// lies beyond it only take part in the hand-offs).
template <int Q>
__device__ __noinline__ uint32_t decode_item(int c0, int c1, int words_total, uint64_t* pl_full,
                                             uint64_t* pl_empty, uint64_t* a_full,
                                             uint64_t* ab_empty, volatile int* abort_flag,
                                             uint32_t g, uint32_t tmem_base) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = warp & 3, jj = warp >> 2;
  // this warp's lane quarter (rows 32t..) and its 32 columns of each A buffer
  const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(t * 32) << 16) + kTmemA + 32 * jj;
  for (int c = c0; c < c1; ++c, ++g) {
    const int ps = g % kPlaneStages, ab = g & 1;
    if (!warp_wait(&pl_full[ps], (g / kPlaneStages) & 1, abort_flag)) return g;
    if (!warp_wait(&ab_empty[ab], ((g >> 1) & 1) ^ 1, abort_flag)) return g;
    tc_fence_after();  // the MMA that read this A buffer has completed
    if (2 * jj < words_total - kChunkWords * c)
      decode_pair<Q>(kOffPlanes + ps * kPlaneStageBytes, a_lane + ab * kACols, t, jj, lane);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&a_full[ab]);
      mbar_arrive(&pl_empty[ps]);
    }
  }
  return g;
}

// LUT row of the block behind row r of the item's 128 (gate_up: rows 16 * tile .. of the gate
// half for tile rows 0-15, the matching up rows for 16-31).
__device__ __forceinline__ int block_row(const Desc& d, const ModeParams& mp, int r) {
  const int tile = d.mb * kTiles + (r >> 5), i = r & 31;
  if (d.mode == MODE_GATE_UP) return i < 16 ? tile * 16 + i : mp.half + tile * 16 + (i - 16);
  return tile * 32 + i;
}

// Decode warp w's share of the item's table: row pair (r, r + 64) with r = 32 (w % 2) + lane,
// entries [(w / 2) * 2^q / 8, (w / 2 + 1) * 2^q / 8).
__device__ __forceinline__ void build_part(const Desc& d, const ModeParams& mp, int w, int lane) {
  const int r = 32 * (w & 1) + lane;
  const int ne = 1 << (d.q - 3);  // entries of this share
  const int v0 = (w >> 1) * ne;
  const uint16_t* lo = d.lut + (static_cast<size_t>(block_row(d, mp, r)) << d.q) + v0;
  const uint16_t* hi = d.lut + (static_cast<size_t>(block_row(d, mp, r + 64)) << d.q) + v0;
  uint8_t* dst = g_smem + kOffTable + v0 * 256 + r * 4;
  if (ne >= 8) {  // 16-byte loads, 8 entries each
    uint4 a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (8 * i < ne) {
        a[i] = __ldg(reinterpret_cast<const uint4*>(lo) + i);
        b[i] = __ldg(reinterpret_cast<const uint4*>(hi) + i);
      }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (8 * i >= ne) break;
      const uint32_t aw[4] = {a[i].x, a[i].y, a[i].z, a[i].w};
      const uint32_t bw[4] = {b[i].x, b[i].y, b[i].z, b[i].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        *reinterpret_cast<uint32_t*>(dst + (8 * i + 2 * k) * 256) = __byte_perm(aw[k], bw[k], 0x5410u);
        *reinterpret_cast<uint32_t*>(dst + (8 * i + 2 * k + 1) * 256) = __byte_perm(aw[k], bw[k], 0x7632u);
      }
    }
  } else {
    for (int v = 0; v < ne; ++v)
      *reinterpret_cast<uint32_t*>(dst + v * 256) =
          static_cast<uint32_t>(__ldg(lo + v)) | (static_cast<uint32_t>(__ldg(hi + v)) << 16);
  }
}

// L2 prefetch of what an item reads first: the LUT rows of its 128 rows and, for each of its
// four tiles, the top q planes of its first 512-column stage.
__device__ __forceinline__ void prefetch_item(const Params& p, const Desc& d) {
  if (!d.valid) return;
  const ModeParams& mp = p.m[d.mode];
  const uint32_t row_bytes = 2u << d.q;
  if (d.mode == MODE_GATE_UP) {
    prefetch_l2(d.lut + (static_cast<size_t>(d.mb * 64) << d.q), 64 * row_bytes);
    prefetch_l2(d.lut + (static_cast<size_t>(mp.half + d.mb * 64) << d.q), 64 * row_bytes);
  } else {
    prefetch_l2(d.lut + (static_cast<size_t>(d.mb * kRows) << d.q), kRows * row_bytes);
  }
  const int W = mp.cols / 32, s = d.c0 * kChunkCols / kTileStageCols;
  const int ws = min(kTileStageWords, W - kTileStageWords * s);
  for (int t = 0; t < kTiles; ++t)
    prefetch_l2(d.planes + t * d.tile_words +
                    static_cast<size_t>(s) * d.n * kTileRows * kTileStageWords,
                d.q * 32 * ws * 4);
}

// Place of h element (token n of the pass, feature f) in the down operand staging, relative to
// the pass's first padded row (2 I fp16 per padded row): sub-pass sp = n / 32 of a pass of
// more than 32 tokens (sub-pass 0 then holds 32 rows), then per 256-column chunk one block of
// 2 np_s rows in the MMA's K-major core-matrix order: rows [0, np_s) the hi parts of the
// sub-pass's tokens, rows [np_s, 2 np_s) their lo parts.
struct HPlace {
  size_t hi, lo;
};
__device__ __forceinline__ HPlace h_place(int np, int I, int n, int f) {
  const int sp = (np > 32 && n >= 32) ? 1 : 0;
  const int nps = np > 32 ? (sp ? np - 32 : 32) : np;
  const int nn = n - 32 * sp;
  const int c = f / kChunkCols, cc = min(kChunkCols, I - c * kChunkCols);
  const size_t blk = static_cast<size_t>(sp) * 64 * I + static_cast<size_t>(c) * 2 * nps * kChunkCols;
  const size_t in = static_cast<size_t>((f % kChunkCols) / 8) * 2 * nps * 8 + nn * 8 + (f % 8);
  (void)cc;
  return {blk + in, blk + in + static_cast<size_t>(nps) * 8};
}

// Epilogue of one item, warp j (rows 32j.. of the accumulator).  gate_up: lanes 0-15 hold the
// gate rows and lanes 16-31 the matching up rows of features 16 * tile + lane; h = SiLU(gate)
// * up goes to the down operand staging as fp16, padding tokens included (they are zeros).
// down: the partial sums of rows 32 * tile + lane for the pass's real tokens.
__device__ __forceinline__ void epilogue(const Desc& d, const ModeParams& mp, int j, int lane,
                                         uint32_t tmem_acc) {
  const int tile = d.mb * kTiles + j;
  const uint32_t lane_addr = tmem_acc + (static_cast<uint32_t>(j * 32) << 16);
  for (int c0 = 0; c0 < d.np; c0 += 16) {
    if (d.mode == MODE_GATE_UP) {
      float v[16];
      tmem_ld16(lane_addr + c0, v);
      const int f = tile * 16 + (lane & 15);
      // the down operand has I = mp.half columns
      __half* base = mp.hout + static_cast<size_t>(d.prow0) * 2 * mp.half;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const float up = __shfl_down_sync(0xffffffffu, v[n], 16);
        if (lane < 16) {
          const float g = v[n];
          const float h = g / (1.0f + expf(-g)) * up;
          const __half hi = __float2half_rn(h);
          const HPlace pl = h_place(d.np, mp.half, c0 + n, f);
          base[pl.hi] = hi;
          base[pl.lo] = __float2half_rn(h - __half2float(hi));
        }
      }
    } else {
      // tokens c0 .. c0 + 15 lie in one sub-pass sp: their hi products at accumulator columns
      // 64 sp + (c0 - 32 sp) .., their lo products nps columns further
      const int sp = (d.np > 32 && c0 >= 32) ? 1 : 0;
      const int nps = d.np > 32 ? (sp ? d.np - 32 : 32) : d.np;
      float* base = mp.out + d.ks * mp.out_slice + static_cast<size_t>(d.pos0) * mp.ld_out +
                    tile * 32 + lane;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t col = 64 * sp + (c0 - 32 * sp) + 8 * h;
        float a[8], b[8];
        tmem_ld8(lane_addr + col, a);
        tmem_ld8(lane_addr + col + nps, b);
#pragma unroll
        for (int n = 0; n < 8; ++n)
          if (c0 + 8 * h + n < d.te)
            base[static_cast<size_t>(c0 + 8 * h + n) * mp.ld_out] = a[n] + b[n];
      }
    }
  }
}

// Zeros for an item whose block cannot be read (state, bitwidth or shape), warp j.
__device__ __forceinline__ void zero_outputs(const Desc& d, const ModeParams& mp, int j,
                                             int lane) {
  const int tile = d.mb * kTiles + j;
  if (d.mode == MODE_GATE_UP) {
    if (lane >= 16) return;
    const int f = tile * 16 + lane;
    __half* base = mp.hout + static_cast<size_t>(d.prow0) * 2 * mp.half;
    for (int n = 0; n < d.np; ++n) {
      const HPlace pl = h_place(d.np, mp.half, n, f);
      base[pl.hi] = __float2half_rn(0.0f);
      base[pl.lo] = __float2half_rn(0.0f);
    }
  } else {
    float* base = mp.out + d.ks * mp.out_slice + static_cast<size_t>(d.pos0) * mp.ld_out +
                  tile * 32 + lane;
    for (int n = 0; n < d.te; ++n) base[static_cast<size_t>(n) * mp.ld_out] = 0.0f;
  }
}

__global__ void __launch_bounds__(kThreads, 1) tc_ffn_kernel(const Params p) {
  uint8_t* const smem = g_smem;
  Desc* cdesc = reinterpret_cast<Desc*>(smem + kOffDesc);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* pl_full = bars;
  uint64_t* pl_empty = pl_full + kPlaneStages;
  uint64_t* b_full = pl_empty + kPlaneStages;
  uint64_t* ab_empty = b_full + 2;
  uint64_t* a_full = ab_empty + 2;
  uint64_t* acc_full = a_full + 2;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* b_empty = acc_empty + 2;  // [2] B buffer read by its MMAs (MMA -> operand producer)
  uint64_t* table_ready = b_empty + 2;
  uint64_t* table_free = table_ready + 1;
  uint64_t* desc_full = table_free + 1;
  uint64_t* desc_free = desc_full + kDescRing;
  uint64_t* mma_done = desc_free + kDescRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {  // descriptors and buffers assume 1024-byte alignment
    if (threadIdx.x == 0) set_status(PW_ERR_UNSUPPORTED);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPlaneStages; ++s) {
      mbar_init(&pl_full[s], 1);
      mbar_init(&pl_empty[s], kDecodeWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&b_full[b], 1);
      mbar_init(&ab_empty[b], 1);
      mbar_init(&b_empty[b], 1);
      mbar_init(&a_full[b], kDecodeWarps);
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(table_ready, kDecodeWarps);
    mbar_init(table_free, kDecodeWarps);
    for (int r = 0; r < kDescRing; ++r) {
      mbar_init(&desc_full[r], 1);
      // read by: plane and operand producers, MMA issuer, 16 decode warps, epilogue warps 1-3
      mbar_init(&desc_free[r], kDescReaders);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  griddep_wait();  // grouping and operand staging of the launches before
  griddep_launch();
  const int npass = p.meta[5];
  const int n_items = items_of(p, MODE_GATE_UP, npass) + items_of(p, MODE_DOWN, npass);

  if (warp == kPlaneWarp) {
    // ---------------- plane producer ----------------
    uint32_t g = 0;
    for (uint32_t j = 0;; ++j) {
      int stop = 0;
      if (lane == 0) stop = !wait_bar(&desc_full[j % kDescRing], (j / kDescRing) & 1, abort_flag);
      stop = __shfl_sync(0xffffffffu, stop, 0);
      if (stop) break;
      __syncwarp();  // lane 0's acquire of the descriptor orders the other lanes' reads
      const Desc d = cdesc[j % kDescRing];
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_free[j % kDescRing]);
      if (d.item < 0) break;
      if (!d.valid) continue;
      const int W = p.m[d.mode].cols / 32;
      for (int c = d.c0; c < d.c1; ++c, ++g) {
        const int ps = g % kPlaneStages;
        int ok = 1;
        if (lane == 0) {
          ok = wait_bar(&pl_empty[ps], ((g / kPlaneStages) & 1) ^ 1, abort_flag);
          if (ok)
            mbar_arrive_expect_tx(&pl_full[ps],
                                  kTiles * d.q * min(kChunkWords, W - kChunkWords * c) * 128);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        constexpr int kChunksPerStage = kTileStageWords / kChunkWords;
        const int s = c / kChunksPerStage;  // 512-column stage of the tiled layout
        const int ws = min(kTileStageWords, W - kTileStageWords * s);
        if (lane < kTiles * d.q) {
          const int t = lane / d.q, pl = lane - t * d.q;
          const uint32_t* src = d.planes + t * d.tile_words +
                                static_cast<size_t>(s) * d.n * kTileRows * kTileStageWords +
                                pl * kTileRows * ws + (c % kChunksPerStage) * kChunkWords * 32;
          bulk_g2s(smem + kOffPlanes + ps * kPlaneStageBytes + (t * d.q + pl) * kPieceBytes, src,
                   min(kChunkWords, W - kChunkWords * c) * 128, &pl_full[ps]);
        }
        __syncwarp();
      }
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
    }
    if (lane == 0)  // every issued copy has landed before the block exits
      for (uint32_t x = (g > kPlaneStages ? g - kPlaneStages : 0); x < g; ++x)
        mbar_wait(&pl_full[x % kPlaneStages], (x / kPlaneStages) & 1);
  } else if (warp == kOperandWarp) {
    // ---------------- operand producer ----------------
    if (lane == 0) {
      uint32_t g = 0;
      for (uint32_t j = 0;; ++j) {
        if (!wait_bar(&desc_full[j % kDescRing], (j / kDescRing) & 1, abort_flag)) break;
        const Desc d = cdesc[j % kDescRing];
        mbar_arrive(&desc_free[j % kDescRing]);
        if (d.item < 0) break;
        if (!d.valid) continue;
        // the down operand (h) of this expert is complete once all its gate_up items count
        if (d.mode == MODE_DOWN && !k4::wait_count(p.done + d.a, d.target, abort_flag)) break;
        const int W = p.m[d.mode].cols / 32, I2 = 2 * p.m[d.mode].cols;
        const bool down = d.mode == MODE_DOWN;
        const int nsp = down && d.np > 32 ? 2 : 1;
        bool ok = true;
        for (int c = d.c0; ok && c < d.c1; ++c) {
          const int cc = min(kChunkWords, W - kChunkWords * c) * 32;  // the chunk's columns
          for (int sp = 0; sp < nsp; ++sp, ++g) {
            const int b = g & 1;
            const int nps = nsp == 2 ? (sp ? d.np - 32 : 32) : d.np;
            // gate_up: np rows x cc columns of fp16 x; down: the hi and lo blocks of a sub-pass
            const uint32_t bytes = (down ? 2 : 1) * nps * cc * 2;
            const __half* src =
                down ? d.bsrc + static_cast<size_t>(sp) * 32 * I2 + static_cast<size_t>(c) * 2 * nps * kChunkCols
                     : d.bsrc + static_cast<size_t>(c) * d.np * kChunkCols;
            if (!(ok = wait_bar(&b_empty[b], ((g >> 1) & 1) ^ 1, abort_flag))) break;
            mbar_arrive_expect_tx(&b_full[b], bytes);
            bulk_g2s(smem + kOffB + b * kBBytes, src, bytes, &b_full[b]);
          }
        }
        if (!ok) break;
      }
      for (uint32_t x = (g > 2 ? g - 2 : 0); x < g; ++x) mbar_wait(&b_full[x & 1], (x >> 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t g = 0, va = 0, ga = 0;  // B blocks, valid items, chunks (A buffers)
      for (uint32_t j = 0;; ++j) {
        if (!wait_bar(&desc_full[j % kDescRing], (j / kDescRing) & 1, abort_flag)) break;
        const Desc d = cdesc[j % kDescRing];
        mbar_arrive(&desc_free[j % kDescRing]);
        if (d.item < 0) break;
        if (!d.valid) continue;
        const uint32_t acc = va & 1;
        if (!wait_bar(&acc_empty[acc], ((va >> 1) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        const int W = p.m[d.mode].cols / 32;
        const bool down = d.mode == MODE_DOWN;
        const int nsp = down && d.np > 32 ? 2 : 1;
        bool ok = true;
        for (int c = d.c0; ok && c < d.c1; ++c, ++ga) {
          const int ab = ga & 1;
          if (!(ok = wait_bar(&a_full[ab], (ga >> 1) & 1, abort_flag))) break;
          const uint32_t a_tmem = tmem_base + kTmemA + ab * kACols;
          const int ksteps = 2 * min(kChunkWords, W - kChunkWords * c);  // K = 16 each
          const int cc = ksteps * 16;
          for (int sp = 0; sp < nsp; ++sp, ++g) {
            const int b = g & 1;
            if (!(ok = wait_bar(&b_full[b], (g >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            const uint32_t b_addr = smem_u32(smem + kOffB + b * kBBytes);
            // the rows of B this block multiplies (gate_up: the pass's np tokens; down: sub-pass
            // sp's nps tokens, hi rows then lo rows) and where they accumulate (down: columns
            // 64 sp .., hi products then lo products)
            const int nps = down ? (nsp == 2 ? (sp ? d.np - 32 : 32) : d.np) : d.np;
            const int nb = down ? 2 * nps : d.np;
            const uint32_t idesc = instr_desc(nb);
            const uint32_t dt = d_tmem + (down ? 64 * sp : 0);
            // descriptor of K step 0; step s starts 2 K groups (2 nb 16 bytes) further on, a
            // plain add to the address field (shared-memory addresses stay below 2^18)
            const uint64_t bd0 = smem_desc(b_addr, nb * 16, 128);
            const uint64_t bstep = static_cast<uint64_t>((2 * nb * 16) >> 4);
            mma_f16_ts(dt, a_tmem, bd0, idesc, c > d.c0 ? 1u : 0u);
            for (int s = 1; s < ksteps; ++s)  // 8 columns of A per step
              mma_f16_ts(dt, a_tmem + 8 * s, bd0 + s * bstep, idesc, 1u);
            (void)cc;
            mma_commit(&b_empty[b]);
          }
          if (ok) mma_commit(&ab_empty[ab]);  // the chunk's A buffer is read
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
        ++va;
      }
      // every issued MMA has completed before the accumulators are released
      mma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------- item schedule, epilogue ----------------
    // The four warps never meet a CTA or named barrier: they follow the descriptors through
    // their mbarriers, and each counts its own share of a finished gate_up item.
    const int ew = warp - kEpiWarp0;
    Desc next;  // warp 16, lane 0: the item claimed for the next descriptor
    if (ew == 0 && lane == 0) {
      next.item = -1;
      const int it0 = atomicAdd(p.sched, 1);  // every item comes from the counter
      if (it0 < n_items) {
        next = resolve(p, it0, npass);
        next.item = it0;
        prefetch_item(p, next);
      }
    }
    Desc prev;
    bool have_prev = false;
    uint32_t va = 0;  // valid items (each fills one accumulator)
    for (uint32_t j = 0;; ++j) {
      Desc& slot = cdesc[j % kDescRing];
      if (ew == 0) {
        if (lane == 0) {
          // every reader has read descriptor j - kDescRing from this slot
          wait_bar(&desc_free[j % kDescRing], ((j / kDescRing) & 1) ^ 1, abort_flag);
          if (*abort_flag) next.item = -1;
          slot = next;
          mbar_arrive(&desc_full[j % kDescRing]);
          if (next.item >= 0) {
            const int it2 = atomicAdd(p.sched, 1);
            next.item = -1;
            if (it2 < n_items) {
              next = resolve(p, it2, npass);
              next.item = it2;
              prefetch_item(p, next);
            }
          }
        }
        __syncwarp();
      } else {
        warp_wait(&desc_full[j % kDescRing], (j / kDescRing) & 1, abort_flag);
      }
      const Desc it = slot;
      if (ew != 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&desc_free[j % kDescRing]);
      }
      if (__any_sync(0xffffffffu, it.item < 0 || *abort_flag)) break;
      if (!it.valid) {
        if (ew == 0 && lane == 0) set_status(it.status);
        zero_outputs(it, p.m[it.mode], ew, lane);
        if (it.mode == MODE_GATE_UP) {
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(p.done + it.a, 1);
        }
        continue;
      }
      if (have_prev) {
        // epilogue of the previous valid item while the decode warps work on this one
        const uint32_t acc = (va - 1) & 1;
        if (!warp_wait(&acc_full[acc], ((va - 1) >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        epilogue(prev, p.m[prev.mode], ew, lane, tmem_base + acc * kAccCols);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        if (prev.mode == MODE_GATE_UP) {
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(p.done + prev.a, 1);
        }
      }
      prev = it;
      have_prev = true;
      ++va;
    }
    if (have_prev) {
      const uint32_t acc = (va - 1) & 1;
      if (warp_wait(&acc_full[acc], ((va - 1) >> 1) & 1, abort_flag)) {
        tc_fence_after();
        epilogue(prev, p.m[prev.mode], ew, lane, tmem_base + acc * kAccCols);
        tc_fence_before();
        if (prev.mode == MODE_GATE_UP) {
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(p.done + prev.a, 1);
        }
      }
    }
  } else {
    // ---------------- decode warps ----------------
    uint32_t g = 0, vt = 0;
    for (uint32_t j = 0;; ++j) {
      if (!warp_wait(&desc_full[j % kDescRing], (j / kDescRing) & 1, abort_flag)) break;
      const Desc d = cdesc[j % kDescRing];
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_free[j % kDescRing]);
      if (__any_sync(0xffffffffu, d.item < 0 || *abort_flag)) break;
      if (!d.valid) continue;
      // the table is rewritten once every decode warp has left the previous item; all sixteen
      // build it, and decode once all shares are in
      if (!warp_wait(table_free, (vt & 1) ^ 1, abort_flag)) break;
      build_part(d, p.m[d.mode], warp, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(table_ready);
      if (!warp_wait(table_ready, vt & 1, abort_flag)) break;
#define PW_DECODE(Q) \
  decode_item<Q>(d.c0, d.c1, p.m[d.mode].cols / 32, pl_full, pl_empty, a_full, ab_empty, \
                 abort_flag, g, tmem_base)
      switch (d.q) {
        case 3: g = PW_DECODE(3); break;
        case 4: g = PW_DECODE(4); break;
        case 5: g = PW_DECODE(5); break;
        case 6: g = PW_DECODE(6); break;
        case 7: g = PW_DECODE(7); break;
        default: g = PW_DECODE(8); break;
      }
#undef PW_DECODE
      __syncwarp();
      if (lane == 0) mbar_arrive(table_free);
      ++vt;
    }
    // an item left early (abort) may have a store in flight: it lands before the release
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace k5
}  // namespace pw
