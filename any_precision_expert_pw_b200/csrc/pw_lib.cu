// libpw: host side of the C ABI declared in include/pw.h.  One translation unit: the step
// kernels live in the pw_*.cuh headers included below.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <mutex>
#include <queue>
#include <vector>

#include "pw.h"
#include "pw_cache.cuh"
#include "pw_common.cuh"
#include "pw_ffn.cuh"
#include "pw_group.cuh"
#include "pw_pack.cuh"
#include "pw_route.cuh"
#include "pw_table.cuh"
#include "pw_tc.cuh"

static_assert(sizeof(pw_block) == 256, "pw_block layout");
static_assert(offsetof(pw_block, planes) == 16, "pw_block layout");
static_assert(offsetof(pw_block, lut) == 24, "pw_block layout");
static_assert(offsetof(pw_block, layout) == 13, "pw_block layout");
static_assert(sizeof(pw_page_table) == 16, "pw_page_table layout");
static_assert(sizeof(pw_route_cfg) == 20, "pw_route_cfg layout");
static_assert(sizeof(pw_affinity_cfg) == 16, "pw_affinity_cfg layout");
static_assert(sizeof(pw_page_update_t) == 16, "pw_page_update_t layout");
static_assert(offsetof(pw_block, stored_bits) == 14, "pw_block layout");

namespace {

constexpr int kMaxDevices = 64;

inline cudaStream_t as_cuda(pw_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

inline pw_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? PW_OK : PW_ERR_CUDA;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct DeviceInfo {
  int sms = 0;
  bool ffn_attr_set = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Per-device, once: SM count and the large dynamic shared memory opt-in of the FFN kernels.
pw_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PW_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.sms == 0) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return PW_ERR_CUDA;
  }
  if (!d.ffn_attr_set) {
    if (cudaFuncSetAttribute(pw::k4::ffn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pw::k4::Layout<1>::kSmem) != cudaSuccess ||
        cudaFuncSetAttribute(pw::k4::ffn_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pw::k4::Layout<2>::kSmem) != cudaSuccess ||
        cudaFuncSetAttribute(pw::k4::ffn_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pw::k4::Layout<4>::kSmem) != cudaSuccess ||
        cudaFuncSetAttribute(pw::k5::tc_ffn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pw::k5::kSmem) != cudaSuccess)
      return PW_ERR_CUDA;
    d.ffn_attr_set = true;
  }
  *out = &d;
  return PW_OK;
}

// Workspace layout of pw_moe_anyprec_forward.
struct Workspace {
  size_t counts, offsets, perm, inv, active, meta, done, X, Hbuf, O;
  size_t xd;                                         // CUDA-core path block descriptors
  size_t pbase, ptok, pnn, pass_tab, XB, HB, total;  // tensor-core path
  int ldx, ldh;
};

// Most k-slices either FFN path splits a down projection of I columns into (the CUDA-core
// path's rule and choose_kslices both stay within it): at most kMaxKSlices, at least two
// 512-column stages per slice.
int max_kslices(int I) {
  const int nst = (I + pw::k4::kStageCols - 1) / pw::k4::kStageCols;
  return std::min(pw::k4::kMaxKSlices, std::max(1, nst / 2));
}

Workspace ws_layout(int T, int k, int E, int H, int I) {
  Workspace w;
  const size_t TK = static_cast<size_t>(T) * k;
  // CUDA-core path activations (fp16, decode order): x per token, h (hi and lo parts) per
  // grouped position, rows padded to whole 512-column stages
  w.ldx = static_cast<int>(align_up(H, pw::k4::kStageCols));
  w.ldh = static_cast<int>(2 * align_up(I, pw::k4::kStageCols));
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  w.counts = take(4 * static_cast<size_t>(E));
  w.offsets = take(4 * static_cast<size_t>(E + 1));
  w.perm = take(4 * TK);
  w.inv = take(4 * TK);
  w.active = take(4 * static_cast<size_t>(E));
  w.meta = take(32);  // [0] active experts, [1] valid assignments, [2] bad table, [4] work counter
  w.done = take(4 * static_cast<size_t>(E));  // gate_up tiles finished per active expert
  w.X = take(2 * static_cast<size_t>(T) * w.ldx);
  w.Hbuf = take(2 * TK * w.ldh);
  w.O = take(4 * TK * H * static_cast<size_t>(max_kslices(I)));
  w.xd = take(sizeof(pw::k4::ExpertDesc) * 2 * static_cast<size_t>(E));
  // tensor-core path: each active expert's rows padded to a multiple of 16
  const size_t rows_pad = TK + 15 * std::min<size_t>(E, TK);
  w.pbase = take(4 * static_cast<size_t>(E));
  w.ptok = take(4 * rows_pad);
  w.pnn = take(4 * rows_pad);
  w.pass_tab = take(4 * (std::min<size_t>(E, TK) + TK / pw::kPassTokens + 1));
  w.XB = take(2 * rows_pad * H);
  w.HB = take(2 * 2 * rows_pad * I);  // h as hi and lo fp16 parts
  w.total = o;
  return w;
}

// Scratch of pw_moe_anyprec_forward_static: one fixed array per GPU that loads the library.
// Host code must not hand this symbol to a kernel: on the host it only names the array.  The
// device address is looked up once per device (g_static_ws_addr) and passed as a pointer.
static __device__ __align__(256) uint8_t g_static_ws[PW_STATIC_WORKSPACE_BYTES];
void* g_static_ws_addr[kMaxDevices] = {};
std::mutex g_static_ws_mu;


// Average routed tokens per active expert from which the tensor-core FFN is used.
std::atomic<int> g_tc_min_tokens{4};
// FFN launch grid override (test hook; 0 = one CTA per SM).
std::atomic<int> g_ffn_grid{0};

// k-slices for the down projection: fill the GPU in whole waves of work items, with at least
// two stages of the tiled layout (512 columns each) per slice.
int choose_kslices(int items, int nst, int sms) {
  int best = 1;
  double best_eff = 0.0;
  const int kmax = std::min(pw::k4::kMaxKSlices, std::max(1, nst / 2));
  for (int ks = 1; ks <= kmax; ++ks) {
    const double n = static_cast<double>(items) * ks;
    const double waves = std::ceil(n / sms);
    const double eff = n / (waves * sms) - 0.01 * ks;
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = ks;
    }
  }
  return best;
}

// Launch with programmatic dependent launch allowed: the kernel may be scheduled while the one
// before it in the stream is still running, and orders itself with griddepcontrol.wait.
template <typename... KArgs, typename... Args>
pw_status launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? PW_OK : PW_ERR_CUDA;
}

pw_status launch_ffn(const pw::k4::Params& p, int max_active, int ntp, int sms,
                     cudaStream_t st) {
  long long items = 0;
  for (int m = pw::k4::MODE_GATE_UP; m <= pw::k4::MODE_DOWN; ++m)
    items += static_cast<long long>(max_active) * p.m[m].pairs * p.m[m].kslices;
  const int over = g_ffn_grid.load();
  const int grid = over > 0 ? over : static_cast<int>(items < sms ? items : sms);
  if (ntp == 1)
    return launch_dependent(pw::k4::ffn_kernel<1>, dim3(grid), dim3(pw::k4::kThreads),
                            pw::k4::Layout<1>::kSmem, st, p);
  if (ntp == 2)
    return launch_dependent(pw::k4::ffn_kernel<2>, dim3(grid), dim3(pw::k4::kThreads),
                            pw::k4::Layout<2>::kSmem, st, p);
  return launch_dependent(pw::k4::ffn_kernel<4>, dim3(grid), dim3(pw::k4::kThreads),
                          pw::k4::Layout<4>::kSmem, st, p);
}

// Argument and shape checks shared by both forward entry points (the workspace is checked by
// the caller): the same arguments give the same status from either.
pw_status forward_args_status(const pw_page_table* pt_dev, int layer, int E,
                              const uint16_t* x_bf16, int T, int H, int I, int k,
                              const int32_t* idx, const float* gate, float* y) {
  if (!pt_dev || !x_bf16 || !idx || !gate || !y) return PW_ERR_INVALID_ARG;
  if (T < 1 || T > PW_MAX_TOKENS || k < 1 || k > PW_MAX_TOPK || layer < 0) return PW_ERR_INVALID_ARG;
  if (E < 1 || E > PW_MAX_EXPERTS || k > E) return PW_ERR_INVALID_ARG;
  if (H < 128 || I < 128 || H % 128 || I % 128) return PW_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * k > pw::kMaxAssign) return PW_ERR_UNSUPPORTED;
  return PW_OK;
}

}  // namespace

extern "C" {

#ifdef PW_DEBUG
const char* pw_version(void) { return "libpw 0.2 (sm_100a, debug: device bounds checks)"; }
#else
const char* pw_version(void) { return "libpw 0.2 (sm_100a)"; }
#endif

const char* pw_status_string(pw_status s) {
  switch (s) {
    case PW_OK: return "PW_OK";
    case PW_ERR_INVALID_ARG: return "PW_ERR_INVALID_ARG";
    case PW_ERR_UNSUPPORTED: return "PW_ERR_UNSUPPORTED";
    case PW_ERR_CUDA: return "PW_ERR_CUDA";
    case PW_ERR_NOT_RESIDENT: return "PW_ERR_NOT_RESIDENT";
    case PW_ERR_TIMEOUT: return "PW_ERR_TIMEOUT";
    case PW_ERR_BAD_EXPERT: return "PW_ERR_BAD_EXPERT";
    case PW_ERR_BAD_BITS: return "PW_ERR_BAD_BITS";
    case PW_ERR_BOUNDS: return "PW_ERR_BOUNDS";
  }
  return "PW_ERR_UNKNOWN";
}

pw_status pw_block_prepare(pw_block* blk) {
  if (!blk || !blk->planes) return PW_ERR_INVALID_ARG;
  const uint32_t rows = blk->rows, cols = blk->cols;
  const int n = blk->parent_bits, mn = blk->min_bits;
  if (rows == 0 || cols == 0 || rows % 32 || cols % 128) return PW_ERR_INVALID_ARG;
  if (n < 1 || n > PW_MAX_BITS || mn < 1 || mn > n) return PW_ERR_INVALID_ARG;
  if (static_cast<uint64_t>(rows) * n > 0x7fffffffull) return PW_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(blk->planes) % 16) return PW_ERR_INVALID_ARG;
  for (int b = 0; b <= PW_MAX_BITS; ++b) {
    const bool want = (b >= mn && b <= n);
    if (want && (!blk->lut[b] || reinterpret_cast<uintptr_t>(blk->lut[b]) % 16))
      return PW_ERR_INVALID_ARG;
  }
  const int stored = blk->stored_bits ? blk->stored_bits : n;
  if (stored < mn || stored > n) return PW_ERR_INVALID_ARG;
  if (blk->committed_bits < mn || blk->committed_bits > stored) return PW_ERR_INVALID_ARG;
  if (blk->layout != PW_LAYOUT_TILED_GATE_UP && blk->layout != PW_LAYOUT_TILED_DOWN)
    return PW_ERR_INVALID_ARG;
  return PW_OK;
}

size_t pw_moe_workspace_bytes(int T, int k, int E, int H, int I) {
  if (T < 1 || k < 1 || E < 1 || H < 1 || I < 1) return 0;
  return ws_layout(T, k, E, H, I).total;
}

pw_status pw_moe_anyprec_forward(const pw_page_table* pt_dev, int layer, int E,
                                 const uint16_t* x_bf16, int T, int H, int I, int k,
                                 const int32_t* idx, const float* gate, float* y, void* workspace,
                                 size_t ws_bytes, pw_stream_t stream) {
  const pw_status v = forward_args_status(pt_dev, layer, E, x_bf16, T, H, I, k, idx, gate, y);
  if (v != PW_OK) return v;
  if (!workspace) return PW_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return PW_ERR_INVALID_ARG;
  const Workspace w = ws_layout(T, k, E, H, I);
  if (ws_bytes < w.total) return PW_ERR_INVALID_ARG;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != PW_OK) return PW_ERR_CUDA;
  cudaStream_t st = as_cuda(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  int32_t* counts = reinterpret_cast<int32_t*>(base + w.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(base + w.offsets);
  int32_t* perm = reinterpret_cast<int32_t*>(base + w.perm);
  int32_t* inv = reinterpret_cast<int32_t*>(base + w.inv);
  int32_t* active = reinterpret_cast<int32_t*>(base + w.active);
  int32_t* meta = reinterpret_cast<int32_t*>(base + w.meta);
  int32_t* done = reinterpret_cast<int32_t*>(base + w.done);
  __half* X = reinterpret_cast<__half*>(base + w.X);
  pw::k4::ExpertDesc* xd = reinterpret_cast<pw::k4::ExpertDesc*>(base + w.xd);
  __half* Hb = reinterpret_cast<__half*>(base + w.Hbuf);
  float* O = reinterpret_cast<float*>(base + w.O);
  const int TK = T * k;
  const int max_active = E < TK ? E : TK;
  // tensor-core FFN once the batch routes enough tokens to each expert
  const bool use_tc = static_cast<long long>(TK) >=
                      static_cast<long long>(g_tc_min_tokens.load()) * max_active;
  pw::PassOut po;
  po.pbase = reinterpret_cast<int32_t*>(base + w.pbase);
  po.ptok = reinterpret_cast<int32_t*>(base + w.ptok);
  po.pnn = reinterpret_cast<int32_t*>(base + w.pnn);
  po.pass_tab = reinterpret_cast<int32_t*>(base + w.pass_tab);
  const int vec = (reinterpret_cast<uintptr_t>(x_bf16) % 16) == 0;

  {
    // CTA 0 groups; the others convert x (8 columns per thread) for the CUDA-core FFN
    const long long groups = static_cast<long long>(T) * (w.ldx / 8);
    const long long conv = (groups + pw::kGroupThreads - 1) / pw::kGroupThreads;
    const int grid =
        use_tc ? 1 : 1 + static_cast<int>(std::min<long long>(std::max(conv, 1LL), 2LL * di->sms));
    if (launch_dependent(pw::setup_kernel, dim3(grid), dim3(pw::kGroupThreads), 0, st, pt_dev,
                         layer, idx, T, k, E, x_bf16, H, I, w.ldx, vec, X, counts,
                         offsets, perm, inv, active, meta, done, po,
                         use_tc ? static_cast<pw::k4::ExpertDesc*>(nullptr) : xd) != PW_OK)
      return PW_ERR_CUDA;
  }
  if (use_tc) {
    __half* XB = reinterpret_cast<__half*>(base + w.XB);
    __half* HB = reinterpret_cast<__half*>(base + w.HB);
    {
      const long long rows_pad = TK + 15LL * max_active;
      const long long n = rows_pad * (H / 8);
      const int grid = static_cast<int>(std::min<long long>((n + 255) / 256, 4LL * di->sms));
      if (launch_dependent(pw::stage_x_kernel, dim3(grid), dim3(256), 0, st, x_bf16, H, vec,
                           static_cast<const int32_t*>(po.ptok),
                           static_cast<const int32_t*>(po.pnn),
                           static_cast<const int32_t*>(meta), T,
                           static_cast<int>(rows_pad), XB) != PW_OK)
        return PW_ERR_CUDA;
    }
    pw::k5::Params q;
    q.pt = pt_dev;
    q.layer = layer;
    q.E = E;
    q.counts = counts;
    q.offsets = offsets;
    q.active = active;
    q.meta = meta;
    q.pbase = po.pbase;
    q.pass_tab = po.pass_tab;
    q.sched = meta + 4;
    q.done = done;
    pw::k5::ModeParams& gu = q.m[pw::k5::MODE_GATE_UP];
    gu.rows = 2 * I;
    gu.cols = H;
    gu.half = I;
    gu.mblocks = I / 64;  // four 16-row gate/up tile pairs per block
    gu.kslices = 1;
    gu.bsrc = XB;
    gu.hout = HB;
    gu.out = nullptr;
    gu.ld_out = 0;
    gu.out_slice = 0;
    pw::k5::ModeParams& dn = q.m[pw::k5::MODE_DOWN];
    dn.rows = H;
    dn.cols = I;
    dn.half = 0;
    dn.mblocks = H / pw::k5::kRows;
    dn.kslices = choose_kslices(max_active * dn.mblocks,
                                (I + pw::k4::kStageCols - 1) / pw::k4::kStageCols, di->sms);
    dn.bsrc = HB;
    dn.hout = nullptr;
    dn.out = O;
    dn.ld_out = H;
    dn.out_slice = static_cast<long long>(TK) * H;
    const int over = g_ffn_grid.load();
    if (launch_dependent(pw::k5::tc_ffn_kernel, dim3(over > 0 ? over : di->sms),
                         dim3(pw::k5::kThreads),
                         pw::k5::kSmem, st, q) != PW_OK)
      return PW_ERR_CUDA;
    const dim3 g((H + 255) / 256, T);
    return launch_dependent(pw::combine_kernel, g, dim3(256), 0, st,
                            static_cast<const float*>(O), static_cast<const int32_t*>(inv), gate,
                            static_cast<const int32_t*>(meta), T, k, H, dn.kslices,
                            static_cast<long long>(TK) * H, y);
  }
  pw::k4::Params p;
  p.pt = pt_dev;
  p.layer = layer;
  p.E = E;
  p.counts = counts;
  p.offsets = offsets;
  p.active = active;
  p.meta = meta;
  p.sched = meta + 4;
  p.done = done;
  p.one = 1;
  p.xd = xd;
  // one launch: every gate_up item (h = SiLU(W_gate x) * (W_up x)), then every down item
  // (o = W_down h, split along k so that the work items fill the GPU); a down item streams h
  // once all gate_up items of its expert are counted
  pw::k4::ModeParams& gu = p.m[pw::k4::MODE_GATE_UP];
  gu.rows = 2 * I;
  gu.cols = H;
  gu.half = I;
  gu.pairs = I / 32;  // tile pairs: 32 gate rows and the 32 matching up rows
  gu.kslices = 1;
  gu.act = X;
  gu.ld_act = w.ldx;
  gu.act_map = perm;  // grouped position -> assignment t*k+slot -> token row of X
  gu.act_div = k;
  gu.act_rows = T;
  gu.out_rows = TK;
  gu.hout = Hb;
  gu.ld_hout = w.ldh;
  gu.out = nullptr;
  gu.ld_out = 0;
  gu.out_slice = 0;
  pw::k4::ModeParams& dn = p.m[pw::k4::MODE_DOWN];
  dn.rows = H;
  dn.cols = I;
  dn.half = 0;
  dn.pairs = H / pw::k4::kItemRows;
  // down items split along k to about the size of a gate_up item (64 rows x H columns): each
  // item carries a fixed cost (its decode table, the first slot of its pipeline), so slicing
  // finer than that costs more than the shorter end of the launch saves (measured)
  dn.kslices = std::max(1, std::min({pw::k4::kMaxKSlices, (I + H / 2) / H,
                                     (I + pw::k4::kStageCols - 1) / pw::k4::kStageCols / 2}));
  dn.act = Hb;
  dn.ld_act = w.ldh;
  dn.act_map = nullptr;
  dn.act_div = 1;
  dn.act_rows = TK;
  dn.out_rows = TK;
  dn.hout = nullptr;
  dn.ld_hout = 0;
  dn.out = O;
  dn.ld_out = H;
  dn.out_slice = static_cast<long long>(TK) * H;
  const int ntp = T == 1 ? 1 : (T == 2 ? 2 : 4);
  if (launch_ffn(p, max_active, ntp, di->sms, st) != PW_OK) return PW_ERR_CUDA;
  {
    const dim3 g((H + 255) / 256, T);
    return launch_dependent(pw::combine_kernel, g, dim3(256), 0, st,
                            static_cast<const float*>(O), static_cast<const int32_t*>(inv), gate,
                            static_cast<const int32_t*>(meta), T, k, H, dn.kslices,
                            static_cast<long long>(TK) * H, y);
  }
}

pw_status pw_moe_anyprec_forward_static(const pw_page_table* pt_dev, int layer, int E,
                                        const uint16_t* x_bf16, int T, int H, int I, int k,
                                        const int32_t* idx, const float* gate, float* y,
                                        pw_stream_t stream) {
  const pw_status v = forward_args_status(pt_dev, layer, E, x_bf16, T, H, I, k, idx, gate, y);
  if (v != PW_OK) return v;
  const size_t need = pw_moe_workspace_bytes(T, k, E, H, I);
  if (need == 0) return PW_ERR_INVALID_ARG;
  if (need > PW_STATIC_WORKSPACE_BYTES) return PW_ERR_UNSUPPORTED;  // shape too large for it
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PW_ERR_CUDA;
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_static_ws_mu);
    ws = g_static_ws_addr[dev];
    if (!ws) {  // first call on this device: look up the array's device address
      if (cudaGetSymbolAddress(&ws, g_static_ws) != cudaSuccess || !ws) return PW_ERR_CUDA;
      g_static_ws_addr[dev] = ws;
    }
  }
  return pw_moe_anyprec_forward(pt_dev, layer, E, x_bf16, T, H, I, k, idx, gate, y, ws, need,
                                stream);
}

pw_status pw_set_tc_min_tokens(int tokens_per_expert) {
  if (tokens_per_expert < 0) return PW_ERR_INVALID_ARG;
  g_tc_min_tokens.store(tokens_per_expert);
  return PW_OK;
}

pw_status pw_set_ffn_grid(int ctas) {
  if (ctas < 0) return PW_ERR_INVALID_ARG;
  g_ffn_grid.store(ctas);
  return PW_OK;
}

pw_status pw_set_wait_limit_ns(unsigned long long ns) {
  const unsigned long long v = ns ? ns : pw::kWaitLimitNs;
  return cudaMemcpyToSymbol(pw::g_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? PW_OK
                                                                               : PW_ERR_CUDA;
}

pw_status pw_test_hold_down_items(int extra) {
  if (extra < 0) return PW_ERR_INVALID_ARG;
  return cudaMemcpyToSymbol(pw::g_test_hold, &extra, sizeof(extra)) == cudaSuccess ? PW_OK
                                                                                   : PW_ERR_CUDA;
}

pw_status pw_commit_bits(pw_page_table* pt_dev, int num_blocks, const int32_t* block_ids,
                         const uint8_t* q, int count, pw_stream_t stream) {
  if (!pt_dev || !block_ids || !q || count < 0 || num_blocks < 1) return PW_ERR_INVALID_ARG;
  if (count == 0) return PW_OK;
  pw::commit_bits_kernel<<<(count + 255) / 256, 256, 0, as_cuda(stream)>>>(pt_dev, num_blocks,
                                                                           block_ids, q, count);
  return launch_status();
}

pw_status pw_get_status(pw_stream_t stream) {
  if (cudaStreamSynchronize(as_cuda(stream)) != cudaSuccess) return PW_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, pw::g_status, sizeof(int)) != cudaSuccess) return PW_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(pw::g_status, &zero, sizeof(int)) != cudaSuccess) return PW_ERR_CUDA;
  return static_cast<pw_status>(v);
}

}  // extern "C"

// Routing-side entry points (pw_route_topk, pw_topk, pw_substitute, pw_remap, AffinityBinning,
// the expert cache) and page movement / planning: same translation unit.
#include "pw_route_api.cuh"
#include "pw_page_api.cuh"
