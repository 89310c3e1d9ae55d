// Shared device helpers for libpw: the device status word, bounded mbarrier waits, TMA
// (cp.async.bulk / cp.async.bulk.tensor) wrappers and small warp utilities.  sm_100a only.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pw.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libpw targets sm_100a (B200) only"
#endif

namespace pw {

// The tiled plane layout (pw.h, pw_block): 32-row tiles, stages of kTileStageWords words
// (512 columns); inside a (tile, stage) run [plane][word][row], most significant plane first.
constexpr int kTileRows = 32;
constexpr int kTileStageWords = 16;
constexpr int kTileStageCols = kTileStageWords * 32;

// uint32 offset of (tile t, stage s, plane p, word u of the stage, row i) in a block of W
// words per row holding n planes per run.
__host__ __device__ __forceinline__ long long tiled_word(long long t, int s, int p, int u, int i,
                                                         int n, int W) {
  const int ws = (W - kTileStageWords * s) < kTileStageWords ? (W - kTileStageWords * s)
                                                             : kTileStageWords;
  return t * n * kTileRows * W + static_cast<long long>(s) * n * kTileRows * kTileStageWords +
         static_cast<long long>(p) * kTileRows * ws + u * kTileRows + i;
}

// First device-side error wins; read and cleared by pw_get_status().
__device__ int g_status = 0;

__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

// Device bounds checks of the debug build (compiled with PW_DEBUG, libpw_debug.so): a global
// address derived from runtime data (expert ids, counts, offsets, positions, block descriptors)
// is checked against its buffer before the access; a failed check records PW_ERR_BOUNDS and the
// access is skipped -- the kernel never traps.  In the normal build the checks compile away.
#ifdef PW_DEBUG
__device__ __forceinline__ bool pw_check(bool ok) {
  if (!ok) set_status(PW_ERR_BOUNDS);
  return ok;
}
#define PW_CHECK(cond) (::pw::pw_check(static_cast<bool>(cond)))
#else
#define PW_CHECK(cond) true
#endif

// Bound on every spin wait: a wait that has not completed after g_wait_limit_ns nanoseconds of
// global time records PW_ERR_TIMEOUT and gives up.  Normal waits finish in microseconds; the
// default is 2 s, and pw_set_wait_limit_ns() (a test hook) shortens it.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
__device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;

// Test hook (pw_test_hold_down_items): extra gate_up completions a down item waits for, so that
// its bounded wait runs out.  Zero in normal use.
__device__ int g_test_hold = 0;

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One bounded try: the thread may be suspended (up to kSuspendHintNs) until the phase of the
// given parity completes, instead of spinning.
constexpr uint32_t kSuspendHintNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long wait_limit_ns() {
  return *static_cast<volatile unsigned long long*>(&g_wait_limit_ns);
}

// Bounded wait for the phase of the given parity; false (and PW_ERR_TIMEOUT recorded) when
// the limit ran out.  With `abort_flag`, also gives up (false, nothing recorded) once another
// thread of the CTA has set it.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort_flag = nullptr) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  const unsigned long long limit = wait_limit_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (abort_flag && *abort_flag) return false;
      if (global_ns() - t0 > limit) {
        set_status(PW_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// 1-D bulk copy global -> shared, completion counted on `bar` (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 prefetch of `bytes` (multiple of 16) at a 16-byte aligned global address.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Programmatic dependent launch.  griddep_wait: the calling thread waits until the grids this
// one depends on have completed and their writes are visible (returns at once for a plain
// launch).  griddep_launch: this CTA allows the next grid in the stream to be scheduled.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Named barrier over a subset of warps (id 1..15).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float f16_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// Warp arg-max of (value, index): larger value wins, equal values -> lower index.
// Lanes with index < 0 hold no candidate.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, off);
    const int oi = __shfl_xor_sync(0xffffffffu, i, off);
    const bool take = (oi >= 0) && (i < 0 || ov > v || (ov == v && oi < i));
    if (take) {
      v = ov;
      i = oi;
    }
  }
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

}  // namespace pw
