// decode_ceiling: the rate of the CUDA-core FFN's decode loop (k4::decode_word, the shipped
// code) on data already in shared memory, per committed bitwidth, and the same loop while a
// bulk-copy stream fills another part of shared memory on the same SM -- the two numbers that
// bound the fused any-precision GEMV (PagedWeight, "Composants Clés" 3) on this GPU.
//
//   decode only   16 warps per SM run decode_word over resident planes, LUT tables and
//                 activations: weights per clock per SM (all SMs busy).
//   with stream   the same plus one warp streaming 16 KB bulk copies (global -> shared, a ring
//                 of 4 slots, no consumer) from a 600 MB buffer: the decode rate, and the bytes
//                 per clock per SM the copies still deliver.
//
// Build and run (one GPU):  python any_precision_expert_pw_b200/csrc/build.py --ceiling
//                           any_precision_expert_pw_b200/decode_ceiling
// Every index is bounded by construction: plane reads stay in [kPl, kX), table gathers in
// [0, kPl) (code byte x 256 + lane offset < 64 KB), activation reads in [kX, kRing), copies in
// [kRing, kBar); the stream warp waits for each copy it issued before the CTA exits.
#include <cstdint>
#include <cstdio>
#include <cuda_runtime.h>

#include "pw_ffn.cuh"

namespace {

using namespace pw;
using namespace pw::k4;

constexpr int kPl = 65536;                 // decode tables occupy [0, 64 KB)
constexpr int kX = kPl + 32768;            // planes of two tiles, 16 KB each
constexpr int kRing = kX + 8192;           // activations (hi and lo, room for two tokens)
constexpr int kSlot = 16384, kNS = 4;      // stream ring
constexpr int kBar = kRing + kNS * kSlot;
constexpr int kSmem = kBar + 128;
constexpr int kWarps = 16;

template <int Q, bool DOWN, bool STREAM>
__global__ void __launch_bounds__((kWarps + 1) * 32, 1)
    ceiling_kernel(int iters, uint32_t one, const uint8_t* src, size_t per_cta, float* out,
                   long long* cyc, unsigned long long* bytes) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* full = reinterpret_cast<uint64_t*>(g_smem + kBar);
  volatile int* stop = reinterpret_cast<volatile int*>(g_smem + kBar + 64);
  volatile int* ndone = reinterpret_cast<volatile int*>(g_smem + kBar + 68);
  // planes: random bits; tables and activations: small finite fp16 values
  for (int i = threadIdx.x; i < kRing / 4; i += blockDim.x) {
    uint32_t h = static_cast<uint32_t>(i) * 2654435761u;
    h ^= h >> 13;
    h *= 0x5bd1e995u;
    h ^= h >> 15;
    uint32_t v = h;
    if (i < kPl / 4) v = (0x2000u | (h & 0x3ffu)) | ((0x2000u | ((h >> 10) & 0x3ffu)) << 16);
    else if (i >= kX / 4) v = (0x3c00u | (h & 0x3ffu)) | ((0x3c00u | ((h >> 16) & 0x3ffu)) << 16);
    reinterpret_cast<uint32_t*>(g_smem)[i] = v;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) mbar_init(&full[s], 1);
    *stop = 0;
    *ndone = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == kWarps) {  // the stream warp
    if (STREAM && lane == 0) {
      const uint8_t* base = src + blockIdx.x * per_cta;
      const size_t nsl = per_cta / kSlot;
      unsigned long long got = 0;
      for (uint32_t g = 0;; ++g) {
        const int s = g % kNS;
        if (g >= kNS) {
          mbar_wait(&full[s], ((g / kNS) - 1) & 1);
          got += kSlot;
        }
        if (*stop) {
          for (uint32_t d = g >= kNS ? g - kNS + 1 : 0; d < g; ++d)
            mbar_wait(&full[d % kNS], (d / kNS) & 1);
          break;
        }
        mbar_arrive_expect_tx(&full[s], kSlot);
        bulk_g2s(g_smem + kRing + s * kSlot, base + (g % nsl) * kSlot, kSlot, &full[s]);
      }
      bytes[blockIdx.x] = got;
    }
    return;
  }
  float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
  const uint32_t m1 = one << 1, m2 = one << 2, m4 = one << 4;
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
    const int ww = (warp + it) & 15;
    const uint32_t pa = kPl + ww * 128 + lane * 4;
    decode_word<Q, 1, DOWN>(pa, pa + 16384, 2048, kX + ww * 64, 2048,
                            (lane * 4) ^ ((it & 1) << 7), m1, m2, m4, acc);
  }
  const long long t1 = clock64();
  __syncwarp();
  if (lane == 0 && atomicAdd(const_cast<int*>(ndone), 1) == kWarps - 1) *stop = 1;
  out[blockIdx.x * blockDim.x + threadIdx.x] = acc[0][0] + acc[0][1] + acc[0][2] + acc[0][3];
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

struct Result {
  double wpc, bpc;
  bool ok;
};

template <int Q, bool DOWN, bool STREAM>
Result run(const uint8_t* src, size_t per_cta, int sms, float* out, long long* cyc,
           unsigned long long* by) {
  auto kern = ceiling_kernel<Q, DOWN, STREAM>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  cudaMemset(by, 0, sms * sizeof(unsigned long long));
  const int iters = 4096;
  kern<<<sms, (kWarps + 1) * 32, kSmem>>>(8, 1u, src, per_cta, out, cyc, by);
  kern<<<sms, (kWarps + 1) * 32, kSmem>>>(iters, 1u, src, per_cta, out, cyc, by);
  const bool ok = cudaDeviceSynchronize() == cudaSuccess;
  long long h[1024];
  unsigned long long b[1024];
  cudaMemcpy(h, cyc, sms * sizeof(long long), cudaMemcpyDeviceToHost);
  cudaMemcpy(b, by, sms * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  double c = 0, bb = 0;
  for (int i = 0; i < sms; ++i) {
    c += static_cast<double>(h[i]);
    bb += static_cast<double>(b[i]);
  }
  c /= sms;
  bb /= sms;
  return {static_cast<double>(kWarps) * iters * 2048 / c, bb / c, ok};
}

template <int Q, bool DOWN>
bool row(const char* name, const uint8_t* src, size_t per_cta, int sms, float* out,
         long long* cyc, unsigned long long* by) {
  const Result a = run<Q, DOWN, false>(src, per_cta, sms, out, cyc, by);
  const Result b = run<Q, DOWN, true>(src, per_cta, sms, out, cyc, by);
  std::printf("| %-8s | %d | %6.2f | %6.2f | %6.2f | %6.2f |\n", name, Q, a.wpc, b.wpc, b.bpc,
              b.wpc * Q / 8.0);
  return a.ok && b.ok;
}

}  // namespace

int main() {
  int dev = 0, sms = 0, clk = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&clk, cudaDevAttrClockRate, dev);
  if (sms > 1024) return 2;
  const size_t per_cta = 4u << 20;
  uint8_t* src = nullptr;
  float* out = nullptr;
  long long* cyc = nullptr;
  unsigned long long* by = nullptr;
  if (cudaMalloc(&src, per_cta * sms) != cudaSuccess ||
      cudaMalloc(&out, static_cast<size_t>(sms) * (kWarps + 1) * 32 * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&cyc, sms * sizeof(long long)) != cudaSuccess ||
      cudaMalloc(&by, sms * sizeof(unsigned long long)) != cudaSuccess)
    return 3;
  cudaMemset(src, 1, per_cta * sms);
  std::printf("SMs %d, max SM clock %d MHz; weights per clock per SM (w/clk), stream bytes "
              "per clock per SM (B/clk)\n\n", sms, clk / 1000);
  std::printf("| module   | q | decode only w/clk | with stream w/clk | stream B/clk | planes needed B/clk |\n");
  std::printf("|---|---|---|---|---|---|\n");
  bool ok = true;
  ok &= row<3, false>("gate_up", src, per_cta, sms, out, cyc, by);
  ok &= row<4, false>("gate_up", src, per_cta, sms, out, cyc, by);
  ok &= row<5, false>("gate_up", src, per_cta, sms, out, cyc, by);
  ok &= row<6, false>("gate_up", src, per_cta, sms, out, cyc, by);
  ok &= row<8, false>("gate_up", src, per_cta, sms, out, cyc, by);
  ok &= row<3, true>("down", src, per_cta, sms, out, cyc, by);
  ok &= row<4, true>("down", src, per_cta, sms, out, cyc, by);
  ok &= row<5, true>("down", src, per_cta, sms, out, cyc, by);
  ok &= row<8, true>("down", src, per_cta, sms, out, cyc, by);
  cudaFree(src);
  cudaFree(out);
  cudaFree(cyc);
  cudaFree(by);
  return ok ? 0 : 1;
}
