/*
 * pw.h -- C ABI of libpw, a B200 (sm_100a) any-precision MoE decode layer.
 *
 * The layer (one MoE layer, decode phase) is:
 *   router GEMV -> softmax top-k -> substitution (residency rule) or batch remap
 *   -> fused grouped expert FFN over Any-Precision bit-planes + per-row LUTs
 *   -> gate-weighted combine.
 *
 * Sources, by page and section:
 *   [PW1]  PagedWeight, "Composants Clés" 1 (Paged Weight Representation): per-(layer, expert,
 *          module) linear blocks, stacked bit-plane weights with look-up tables, and a Weight
 *          Page Table holding the desired bitwidth d_i, the committed bitwidth q_i and the page
 *          state (GPU-resident, CPU-resident, in transfer) of each block.
 *   [PW3]  PagedWeight, "Composants Clés" 3: one fused mixed-precision kernel reads the
 *          bit-planes and LUTs directly, each block at its own bitwidth; bitwidth commits only
 *          happen at safe boundaries.
 *   [SUB]  "Which Expert Misses Are Worth Waiting For?", "Méthodologie": fetch-every-miss,
 *          the 0.15 rule, the first-choice rule and the substituted gate mass m.
 *   [LX1]  LYNX, 1 "Énoncé du Problème": each token independently picks its top-k experts.
 *   [LX2]  LYNX, 2.1 and 2.2: rank-0 dominates; batch-wide expert scores pick a critical set;
 *          low-affinity assignments are remapped to it and every token keeps exactly k experts.
 *
 * Conventions for every function below:
 *   - Pointers named *_dev, and every array argument of a compute call, are DEVICE pointers.
 *     The caller owns and allocates every buffer (inputs, outputs, workspace, page table,
 *     planes, LUTs).  libpw allocates no device or host memory and keeps no state besides one
 *     device status word per GPU.
 *   - Every compute call other than pw_moe_anyprec_forward_static is asynchronous on `stream`
 *     (0 = legacy default stream) and may be captured in a CUDA graph.  Argument and shape
 *     errors return immediately with PW_ERR_INVALID_ARG (or PW_ERR_UNSUPPORTED) and launch
 *     nothing.
 *   - Errors found on the device (a block that is not GPU-resident, a committed bitwidth out
 *     of range, an expert id out of range, a bounded wait that ran out) never trap: the first
 *     one is recorded in the device status word and the affected work is skipped (its outputs
 *     are written as zeros).  pw_get_status() reads and clears it.
 *   - Floating-point data: bf16 and fp16 are passed as uint16_t bit patterns.
 */
#ifndef PW_H_
#define PW_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* pw_stream_t; /* same object as cudaStream_t */

typedef enum {
  PW_OK = 0,
  PW_ERR_INVALID_ARG = 1,  /* bad pointer, size, shape or config; nothing launched       */
  PW_ERR_UNSUPPORTED = 2,  /* valid request outside what the library implements        */
  PW_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, sync, symbol copy)    */
  PW_ERR_NOT_RESIDENT = 4, /* device: a used block's page state is not PW_PAGE_GPU      */
  PW_ERR_TIMEOUT = 5,      /* device: a bounded wait gave up                            */
  PW_ERR_BAD_EXPERT = 6,   /* device: an expert id outside [0, E)                        */
  PW_ERR_BAD_BITS = 7,     /* device: committed bitwidth outside [min_bits, parent_bits]
                              or its LUT missing                                        */
  PW_ERR_BOUNDS = 8        /* device, debug build (libpw_debug.so) only: an address derived
                              from runtime data fell outside its buffer; the access was
                              skipped                                                   */
} pw_status;

enum { PW_MOD_GATE_UP = 0, PW_MOD_DOWN = 1 };

/* Bit-plane layouts written by pw_pack_bitplanes (see pw_block for their definitions). */
enum {
  PW_LAYOUT_ROWS = 0,          /* [n][rows][cols/32]: the bit-plane format of [PW1]          */
  PW_LAYOUT_TILED_GATE_UP = 1, /* the FFN kernel's layout for a gate_up block               */
  PW_LAYOUT_TILED_DOWN = 2     /* the FFN kernel's layout for a down block                  */
};

/* Page states of a Weight Page Table entry [PW1]. */
enum { PW_PAGE_GPU = 0, PW_PAGE_CPU = 1, PW_PAGE_XFER = 2 };

/* Assignment rewrite policies [SUB], [LX2]. */
enum {
  PW_POLICY_FETCH_ALL = 0,    /* every missing expert is fetched (the rule is the identity)  */
  PW_POLICY_THRESHOLD = 1,    /* fetch if first choice or gate >= threshold, else substitute */
  PW_POLICY_FIRST_CHOICE = 2  /* fetch only a missing first choice, substitute the rest      */
};

/* Substitution actions, one per (token, slot). */
enum { PW_ACT_HIT = 0, PW_ACT_FETCH = 1, PW_ACT_SUBST = 2 };

#define PW_MIN_BITS 3
#define PW_MAX_BITS 8
#define PW_MAX_EXPERTS 1024
#define PW_MAX_TOPK 16
#define PW_MAX_TOKENS 4096

/*
 * One Weight Page Table entry: one linear block (layer, expert, module) [PW1].
 *   gate_up: rows = 2I, cols = H (rows 0..I-1 gate, rows I..2I-1 up); down: rows = H, cols = I.
 *   rows % 32 == 0, cols % 128 == 0.
 *   Bit-planes: plane p holds bit (parent_bits-1-p) of every parent index (plane 0 = most
 *   significant), so the top q planes give the q-bit index = top q bits of the parent index.
 *   In PW_LAYOUT_ROWS a plane is uint32 [rows][cols/32] and column 32w+j sits at bit j of
 *   word w.  The FFN reads the same words rearranged so that everything one CTA needs for a
 *   32-row tile and a 512-column stage is one contiguous run, most significant plane first:
 *     tile t, row i of the tile:  PW_LAYOUT_TILED_DOWN    -> block row 32t + i;
 *                                 PW_LAYOUT_TILED_GATE_UP -> gate row 16t + i for i < 16,
 *                                                            up row I + 16t + (i - 16) otherwise;
 *     stage s = words 16s .. 16s + ws - 1 of each row, ws = min(16, cols/32 - 16s);
 *     word w = 16s + u of plane p, row i of tile t sits at uint32 index
 *       t * (n * 32 * cols/32) + s * (n * 32 * 16) + p * (32 * ws) + u * 32 + i
 *     (n = parent_bits).  Reading the top q planes of (t, s) reads the first q * 32 * ws words
 *     of that run; inside it a plane is [word][row], so one word of 32 consecutive rows is 128
 *     contiguous bytes.  `layout` holds PW_LAYOUT_TILED_GATE_UP or PW_LAYOUT_TILED_DOWN; the
 *     forward checks it against the module.  `planes` is 16-byte aligned.
 *   stored_bits: how many planes each (tile, stage) run holds in `planes` (0 = parent_bits):
 *     a block paged in at bitwidth q (pw_page_copy) keeps only its top q planes on the device,
 *     runs packed with that stride, so committed_bits may not exceed it.
 *   lut[b]: fp16 [rows][1<<b] for every b in [min_bits, parent_bits] (NULL otherwise);
 *           weight(r, c) at bitwidth q = lut[q][r][top q bits of idx(r, c)].
 *   committed_bits (q_i) is read once per forward call; desired_bits (d_i) is stored for a
 *   planner and ignored by the kernels.
 *   The entry must sit at a 64-byte aligned address on the device.
 * sizeof(pw_block) == 256.
 */
typedef struct pw_block {
  uint32_t rows;
  uint32_t cols;
  uint8_t parent_bits;
  uint8_t min_bits;
  uint8_t desired_bits;
  uint8_t committed_bits;
  uint8_t state;
  uint8_t layout;
  uint8_t stored_bits;
  uint8_t reserved0[1];
  const uint32_t* planes;
  const uint16_t* lut[9];
  uint8_t reserved1[160];
} pw_block;

/* The Weight Page Table: device-resident; blocks[(layer * num_experts + e) * 2 + module]. */
typedef struct pw_page_table {
  uint32_t num_layers;
  uint32_t num_experts;
  pw_block* blocks; /* device pointer, 64-byte aligned */
} pw_page_table;

/* Routing configuration. */
typedef struct pw_route_cfg {
  int32_t k;          /* experts per token, 1..min(E, PW_MAX_TOPK)                      */
  int32_t renorm;     /* 1: gates = p_sel / sum(p_sel); 0: gates = p_sel                */
  int32_t policy;     /* PW_POLICY_* (pw_substitute only)                                */
  float threshold;    /* gate threshold of PW_POLICY_THRESHOLD (0.15 in [SUB])           */
  int32_t critical_n; /* target size of the critical set (pw_remap; 32 for the LYNX case) */
} pw_route_cfg;

/* ---------------------------------------------------------------------------------------
 * pw_block_prepare (host only, no GPU work): validates a host copy of a block entry before
 * it is copied to the device.  Returns PW_ERR_INVALID_ARG for a bad shape, bitwidth range,
 * layout, missing LUT or misaligned pointer, PW_ERR_UNSUPPORTED for a block too large for
 * 32-bit row indexing.
 * ------------------------------------------------------------------------------------- */
pw_status pw_block_prepare(pw_block* blk_host);

/* ---------------------------------------------------------------------------------------
 * pw_pack_bitplanes [PW1]: uint8 parent indices idx[rows][cols] (values < 2^n) into n
 * bit-planes in `layout` (PW_LAYOUT_*, defined with pw_block).  cols % 32 == 0 for
 * PW_LAYOUT_ROWS; rows % 32 == 0 and cols % 128 == 0 for the tiled layouts; 1 <= n <= 8.
 * Bits of idx above n are ignored.  planes holds n * rows * cols / 32 uint32 words, 16-byte
 * aligned.  Offline (untimed) step.
 * ------------------------------------------------------------------------------------- */
pw_status pw_pack_bitplanes(const uint8_t* idx, int rows, int cols, int n, int layout,
                            uint32_t* planes, pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_route_topk [LX1]: logits = x W_r^T + bias, then per token the k largest logits in
 * descending order (equal logits: lower expert index first), and their softmax gates over
 * all E experts (renormalised over the k when cfg->renorm).
 *   x_bf16 [T][H] bf16, Wr [E][H] fp32, bias [E] fp32 or NULL.
 *   logits [T][E] fp32: the float64 dot product plus bias, rounded once to fp32.
 *   idx [T][k] int32, gate [T][k] fp32 (computed in float64 from the fp32 logits, rounded
 *   once).  1 <= T <= PW_MAX_TOKENS, 1 <= E <= PW_MAX_EXPERTS, H >= 1.
 * ------------------------------------------------------------------------------------- */
pw_status pw_route_topk(const uint16_t* x_bf16, const float* Wr, const float* bias, int T,
                        int H, int E, const pw_route_cfg* cfg, float* logits, int32_t* idx,
                        float* gate, pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_topk [LX1]: the selection half of pw_route_topk on logits the caller already has:
 * logits [T][E] fp32 -> idx [T][k] int32, gate [T][k] fp32, same rules.
 * ------------------------------------------------------------------------------------- */
pw_status pw_topk(const float* logits, int T, int E, const pw_route_cfg* cfg, int32_t* idx,
                  float* gate, pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_substitute [SUB]: residency-aware rewrite of the routed assignments, in place.
 * For each token, slots in rank order: a resident expert is a hit; a missing one is fetched
 * (kept, counted) when the policy says so (rank 0, or gate >= threshold for
 * PW_POLICY_THRESHOLD; always for PW_POLICY_FETCH_ALL); otherwise it is replaced by the
 * highest-logit resident expert not in the token's current set (ties: lower index), keeping
 * its gate.  With no resident candidate left the miss is fetched.
 *   logits [T][E] fp32, idx [T][k] int32 (in/out), gate [T][k] fp32, resident [E] uint8.
 *   action [T][k] uint8 (PW_ACT_*), mass [T] fp32 = substituted gates / all gates of the
 *   token (float64 sums, rounded once).  action and mass may be NULL.
 * ------------------------------------------------------------------------------------- */
pw_status pw_substitute(const float* logits, int32_t* idx, const float* gate,
                        const uint8_t* resident, int T, int E, const pw_route_cfg* cfg,
                        uint8_t* action, float* mass, pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_remap [LX2]: batch-aware remap to a critical expert set, in place.
 * S_e = sum of the gates routed to e (float64, ascending (token, slot) order).  The critical
 * set C is every rank-0 expert plus experts outside it by S_e descending (ties: lower index)
 * until |C| = cfg->critical_n.  Each slot of rank > 0 whose expert is not in C is replaced,
 * in rank order, by the highest-logit expert of C not in the token's current set (ties: lower
 * index), keeping its gate; with none left the slot is kept.  Every token keeps exactly k
 * distinct experts.
 *   logits [T][E] fp32, idx [T][k] int32 (in/out), gate [T][k] fp32, critical [E] uint8
 *   (may be NULL), unique int32[2] (may be NULL): the number of distinct experts the batch
 *   routes to before and after the remap -- the experts whose weights the FFN reads.
 *   Runs as one thread block: T * k <= 8192.
 * ------------------------------------------------------------------------------------- */
pw_status pw_remap(const float* logits, int32_t* idx, const float* gate, int T, int E,
                   const pw_route_cfg* cfg, uint8_t* critical, int32_t* unique,
                   pw_stream_t stream);

/* AffinityBinning configuration (pw_affinity_remap). */
typedef struct pw_affinity_cfg {
  int32_t num_bins;  /* B >= 1 (<= 256)                                                   */
  int32_t low_bins;  /* tokens whose bin is < low_bins are low-affinity (remapped)          */
  double bin_width;  /* w > 0, +inf allowed (every token in bin 0)                          */
} pw_affinity_cfg;

/* ---------------------------------------------------------------------------------------
 * pw_affinity_default [LX2] (host only): the bins from the sparsity ratio k/N alone:
 * B = ceil(E/k), w = ln(E/k) / B, low_bins = ceil(B/2); E/k <= 1 gives one bin of width +inf.
 * ------------------------------------------------------------------------------------- */
pw_status pw_affinity_default(int E, int k, pw_affinity_cfg* out);

/* ---------------------------------------------------------------------------------------
 * pw_affinity_remap [LX1][LX2]: LYNX AffinityBinning, in place.  The pages give the
 * structure (confidence from the gap between the top-ranked logits, binned with widths set by
 * k/N; batch expert scores with exponential weights of the bins; a critical set; low-affinity
 * assignments remapped, k experts kept) but no formula; this is one reading of it:
 *   d_t = fp32 gap between token t's two largest logits (ties: lower index ranks first);
 *   bin_t = min(floor(d_t / w), B - 1) in float64 (B - 1 when E = 1, 0 when w = +inf);
 *   S_e = sum over assignments (t, s) with idx = e of 2^bin_t * gate[t][s], float64 in
 *         ascending (token, slot) order;
 *   critical set C and the remap as in pw_remap with S_e in place of the gate sums, applied
 *   only to tokens with bin_t < low_bins.  With w = +inf this is exactly pw_remap.
 *   logits [T][E] fp32, idx [T][k] int32 (in/out), gate [T][k] fp32, critical [E] uint8,
 *   bins [T] int32 and unique int32[2] (distinct experts before / after, as in pw_remap)
 *   outputs (each may be NULL).  One thread block: T * k <= 8192.
 * ------------------------------------------------------------------------------------- */
pw_status pw_affinity_remap(const float* logits, int32_t* idx, const float* gate, int T, int E,
                            const pw_route_cfg* cfg, const pw_affinity_cfg* acfg,
                            uint8_t* critical, int32_t* bins, int32_t* unique,
                            pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_cache_step [SUB]: one decode step of an expert cache (Quality-First = PW_POLICY_THRESHOLD
 * with threshold 0.15, Speed-First = PW_POLICY_FIRST_CHOICE; both with frequency-based
 * eviction and background admission at beta = 0.5).  The pages list the components, not
 * their order; this call does, on device state the caller owns:
 *   1. freq[e] += 1 for every routed assignment (idx as given);
 *   2. idx is rewritten in place by the rule of pw_substitute against resident[] as it is at
 *      the start of the step (action, mass_t as in pw_substitute; either may be NULL);
 *   3. mass[e] += gate of every substituted slot, e = the expert it replaced (float64,
 *      ascending (token, slot) order);
 *   4. inserted: the experts fetched this step (first occurrence order), then every other
 *      non-resident expert with mass[e] >= beta; an inserted expert's mass becomes 0; if the
 *      insertions alone exceed `capacity`, the most selected fetches and then the heaviest
 *      admissions are kept (ties: lower index);
 *   5. evicted: start-of-step residents, ordered by (used after the rewrite, freq, index),
 *      until at most `capacity` experts are resident.
 *   resident [E] uint8, mass [E] double, freq [E] uint32: in/out.  stats [3] int32 (may be
 *   NULL): fetched, admitted, evicted.  One thread block: T * k <= 4096.
 * ------------------------------------------------------------------------------------- */
pw_status pw_cache_step(const float* logits, int32_t* idx, const float* gate, int T, int E,
                        const pw_route_cfg* cfg, double beta, uint8_t* resident, double* mass,
                        uint32_t* freq, int capacity, uint8_t* action, float* mass_t,
                        int32_t* stats, pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_moe_workspace_bytes: device workspace needed by pw_moe_anyprec_forward (0 on bad args).
 * After a forward the workspace begins with the grouping it ran on, each region at a 256-byte
 * boundary: counts int32[E] (assignments per expert), offsets int32[E+1] (exclusive prefix
 * sums), perm int32[T*k] (grouped position -> assignment t*k + slot, ascending within an
 * expert), inv int32[T*k] (assignment -> grouped position, -1 for an invalid expert id),
 * active int32[E] (experts with work, ascending; the first meta[0] are valid), meta int32[8]
 * (meta[0] = active experts).  The rest is scratch of no fixed layout.
 * ------------------------------------------------------------------------------------- */
size_t pw_moe_workspace_bytes(int T, int k, int E, int H, int I);

/* ---------------------------------------------------------------------------------------
 * pw_moe_anyprec_forward [PW1][PW3]: grouped expert FFN of one layer, each (expert, module)
 * block read at its committed bitwidth q straight from its top-q bit-planes and its q-bit
 * LUT, then the gate-weighted combine.
 *   for each token t and slot s, e = idx[t][s]:
 *     g = W_gate(e) x_t, u = W_up(e) x_t, h = SiLU(g) * u, o = W_down(e) h
 *   y[t] = sum over s (in slot order) of gate[t][s] * o      (fp32 accumulation)
 *   pt_dev: device page table; layer < num_layers; E must equal its num_experts (checked on
 *   the device: a mismatch records PW_ERR_INVALID_ARG and the call produces zeros).
 *   x_bf16 [T][H] bf16, idx [T][k] int32 in [0, E), gate [T][k] fp32, y [T][H] fp32.
 *   workspace: >= pw_moe_workspace_bytes(T, k, E, H, I) bytes, 256-byte aligned; its
 *   contents need no initialisation and are overwritten.
 *   Blocks must be GPU-resident (else PW_ERR_NOT_RESIDENT on the device, that expert's
 *   contribution is zero).  H % 128 == 0, I % 128 == 0.
 *   Two FFN paths give the same result within the tolerance of the arithmetic (the choice
 *   never changes routing): while T*k < m * min(E, T*k) (m = pw_set_tc_min_tokens, default
 *   4) a CUDA-core bit-plane GEMV (each weight decoded once per four tokens); otherwise the
 *   tensor-core GEMM (tcgen05; each weight decoded once per 64 tokens of its expert).  Both
 *   multiply the fp16 LUT values by fp16 activations with fp32 accumulation: x is rounded bf16
 *   -> fp16 (exact for values within fp16's normal range), h = SiLU(g) * u (computed in fp32)
 *   is carried as two fp16 parts hi = fp16(h), lo = fp16(h - hi), both multiplied (about 22
 *   bits of h); values beyond fp16's range (|v| > 65504) become infinities.
 * ------------------------------------------------------------------------------------- */
pw_status pw_moe_anyprec_forward(const pw_page_table* pt_dev, int layer, int E,
                                 const uint16_t* x_bf16, int T, int H, int I, int k,
                                 const int32_t* idx, const float* gate, float* y, void* workspace,
                                 size_t ws_bytes, pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_moe_anyprec_forward_static: pw_moe_anyprec_forward without a caller-provided workspace.
 * The pages have no counterpart to this call; it exists for callers that cannot allocate
 * device memory for scratch -- for instance a host program that only receives device
 * pointers from a serving engine which owns and budgets every GPU allocation (weights, KV
 * cache), or a plain C caller with no device allocator of its own.
 *   Same arguments and results as pw_moe_anyprec_forward, minus workspace and ws_bytes.
 *   Scratch: one array of PW_STATIC_WORKSPACE_BYTES inside libpw, present on every GPU that
 *   loads the library until the process exits.  Shapes whose pw_moe_workspace_bytes(T, k, E,
 *   H, I) exceeds it return PW_ERR_UNSUPPORTED and launch nothing.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *   with that device current; make that first call before any stream capture.
 *   Every call on a device shares the one array and it keeps the last call's contents (the
 *   forward overwrites every scratch word it reads, so nothing needs clearing); calls that
 *   overlap on the GPU -- different streams, or different host threads -- race on it and
 *   must be serialised by the caller.  It allocates no memory (no cudaMalloc or cudaFree).
 * ------------------------------------------------------------------------------------- */
#define PW_STATIC_WORKSPACE_BYTES (16u << 20)

pw_status pw_moe_anyprec_forward_static(const pw_page_table* pt_dev, int layer, int E,
                                        const uint16_t* x_bf16, int T, int H, int I, int k,
                                        const int32_t* idx, const float* gate, float* y,
                                        pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_set_tc_min_tokens: process-wide switch between the two FFN paths of
 * pw_moe_anyprec_forward: the tensor-core path is taken when the batch routes on average at
 * least `tokens_per_expert` tokens to each active expert (T*k >= m * min(E, T*k)); 0 selects
 * it always, a value above PW_MAX_TOKENS * PW_MAX_TOPK never.  Default 4.  Affects calls
 * made (or graphs captured) after it returns.  PW_ERR_INVALID_ARG for a negative value.
 * ------------------------------------------------------------------------------------- */
pw_status pw_set_tc_min_tokens(int tokens_per_expert);

/* ---------------------------------------------------------------------------------------
 * Test hooks (no counterpart on the pages).  They exist so that the tests can reach paths that
 * a healthy run never takes; production code leaves them at their defaults.
 *
 * pw_set_ffn_grid: number of CTAs of the FFN launch of pw_moe_anyprec_forward (both paths);
 *   0 (default) = one per SM (capped by the work items on the CUDA-core path).  A grid larger
 *   than the GPU can hold at once (more than one CTA per SM never fits) checks that the
 *   gate_up -> down dependency does not assume every CTA to be resident.  Process-wide, host
 *   state only; takes effect on later calls.  Negative -> PW_ERR_INVALID_ARG.
 *
 * pw_set_wait_limit_ns: bound of every spin wait in libpw's kernels on the current device
 *   (a wait that has not completed within it records PW_ERR_TIMEOUT and gives up, and the
 *   work it guarded writes zeros).  0 restores the default of 2 s.  Synchronous (a copy to a
 *   device variable); call it between launches, not during stream capture.
 *
 * pw_test_hold_down_items: every down item of the fused FFN launch on the current device waits
 *   for `extra` more gate_up completions than exist, so its bounded wait runs out and the
 *   forward ends with PW_ERR_TIMEOUT (the failure path of a gate_up tile that never finishes).
 *   0 (default) restores normal behaviour.  Synchronous, like pw_set_wait_limit_ns.
 * ------------------------------------------------------------------------------------- */
pw_status pw_set_ffn_grid(int ctas);
pw_status pw_set_wait_limit_ns(unsigned long long ns);
pw_status pw_test_hold_down_items(int extra);

/* ---------------------------------------------------------------------------------------
 * pw_commit_bits [PW1][PW3]: set committed_bits of `count` blocks (device arrays block_ids
 * [count] int32 and q [count] uint8), stream-ordered, so that a commit takes effect exactly
 * between two forward calls on the stream (a safe boundary).  A block id out of range or a q
 * outside [min_bits, parent_bits] (or without a LUT) leaves that block unchanged and records
 * PW_ERR_BAD_BITS.  num_blocks is the table's entry count (num_layers * num_experts * 2).
 * ------------------------------------------------------------------------------------- */
pw_status pw_commit_bits(pw_page_table* pt_dev, int num_blocks, const int32_t* block_ids,
                         const uint8_t* q, int count, pw_stream_t stream);

/* One page-table edit for pw_page_update: block id (layer*E + e)*2 + module; each other field
 * 0 / NULL = leave unchanged.  state holds PW_PAGE_* + 1. */
typedef struct pw_page_update_t {
  int32_t block;
  uint8_t state;          /* PW_PAGE_GPU + 1, PW_PAGE_CPU + 1, PW_PAGE_XFER + 1, or 0 */
  uint8_t stored_bits;    /* planes per run now held by `planes` (min_bits..parent_bits) */
  uint8_t committed_bits; /* q_i (min_bits..stored bits)                                 */
  uint8_t reserved;
  const uint32_t* planes; /* new device plane buffer (16-byte aligned), or NULL            */
} pw_page_update_t;

/* ---------------------------------------------------------------------------------------
 * pw_page_copy [PW1][PW3]: page movement of Any-Precision planes.  Copies the top q planes of
 * every (tile, stage) run between two buffers of the same block in the tiled layout holding
 * src_bits and dst_bits planes per run (q <= both): host -> device (page in at bitwidth q,
 * the device copy keeping only q planes per run), device -> host, device -> device.  Host
 * buffers must be pinned for the copy to be asynchronous.  One pitched copy per 512-column
 * stage, on `stream`.  rows % 32 == 0, cols % 128 == 0, both pointers 16-byte aligned.
 * ------------------------------------------------------------------------------------- */
pw_status pw_page_copy(const uint32_t* src, int src_bits, uint32_t* dst, int dst_bits, int rows,
                       int cols, int q, pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_page_update [PW1][PW3]: applies `count` page-table edits (device array of
 * pw_page_update_t) in stream order, e.g. state XFER before a pw_page_copy and
 * {GPU, stored_bits = q, committed_bits = q, planes = new buffer} after it, so a forward
 * ordered after the update sees a consistent entry, and one racing the transfer sees XFER
 * (PW_ERR_NOT_RESIDENT, zeros).  Inconsistent edits are skipped with PW_ERR_BAD_BITS.
 * ------------------------------------------------------------------------------------- */
pw_status pw_page_update(pw_page_table* pt_dev, int num_blocks, const pw_page_update_t* updates,
                         int count, pw_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * pw_plan_bitwidths [PW1] (host only): the damage-greedy bitwidth planner.  For nblocks
 * blocks, damage[i][q] and bytes[i][q] (row-major [nblocks][PW_MAX_BITS + 1], read for q in
 * [qmin[i], qmax[i]]): start every block at qmax, then, while the total bytes exceed `budget`,
 * lower by one bit the block whose step adds the least damage per byte saved
 * ((damage[i][q-1] - damage[i][q]) / (bytes[i][q] - bytes[i][q-1]), float64; ties: lower
 * block index; a step that saves no bytes ranks last).  q_out[i] gets the plan, to be
 * committed with pw_commit_bits at a safe boundary.  Returns PW_ERR_UNSUPPORTED when even
 * every block at qmin exceeds the budget (q_out then holds qmin).
 * ------------------------------------------------------------------------------------- */
pw_status pw_plan_bitwidths(int nblocks, const double* damage, const uint64_t* bytes,
                            const uint8_t* qmin, const uint8_t* qmax, uint64_t budget,
                            uint8_t* q_out);

/* ---------------------------------------------------------------------------------------
 * pw_get_status: synchronises `stream`, then returns and clears the device status word of
 * the current device (PW_OK if no device-side error was recorded).  Not capturable.
 * ------------------------------------------------------------------------------------- */
pw_status pw_get_status(pw_stream_t stream);

/* Human-readable name of a status code (static string). */
const char* pw_status_string(pw_status s);

/* Library version string (static). */
const char* pw_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PW_H_ */
