// Host side of the routing calls of include/pw.h (pw_route_topk, pw_substitute, pw_remap).
// Included once, by pw_lib.cu, after its launch helpers: the library is one translation unit
// so that every kernel shares one device status word.
#pragma once

namespace {

bool cfg_ok(const pw_route_cfg* cfg, int E) {
  return cfg && cfg->k >= 1 && cfg->k <= PW_MAX_TOPK && cfg->k <= E;
}

}  // namespace

extern "C" {

pw_status pw_route_topk(const uint16_t* x_bf16, const float* Wr, const float* bias, int T, int H,
                        int E, const pw_route_cfg* cfg, float* logits, int32_t* idx, float* gate,
                        pw_stream_t stream) {
  if (!x_bf16 || !Wr || !logits || !idx || !gate) return PW_ERR_INVALID_ARG;
  if (T < 1 || T > PW_MAX_TOKENS || E < 1 || E > PW_MAX_EXPERTS || H < 1 || !cfg_ok(cfg, E))
    return PW_ERR_INVALID_ARG;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != PW_OK) return PW_ERR_CUDA;
  const int e_tiles = (E + pw::kRouteExpertsPerCta - 1) / pw::kRouteExpertsPerCta;
  const int t_tiles_target = std::max(1, (2 * di->sms + e_tiles - 1) / e_tiles);
  int tt = (T + t_tiles_target - 1) / t_tiles_target;
  tt = tt <= 1 ? 1 : tt <= 2 ? 2 : 4;
  const int vec = (H % 8 == 0) && (reinterpret_cast<uintptr_t>(x_bf16) % 16 == 0) &&
                  (reinterpret_cast<uintptr_t>(Wr) % 16 == 0);
  const dim3 g1(e_tiles, (T + tt - 1) / tt);
  const int fuse_k = (e_tiles == 1) ? cfg->k : 0;  // the whole E in one CTA: top-k fused
  cudaStream_t st = as_cuda(stream);
  switch (tt) {
    case 1: pw::router_logits_kernel<1><<<g1, pw::kRouteThreads, 0, st>>>(x_bf16, Wr, bias, T, H, E, vec, logits, fuse_k, cfg->renorm, idx, gate); break;
    case 2: pw::router_logits_kernel<2><<<g1, pw::kRouteThreads, 0, st>>>(x_bf16, Wr, bias, T, H, E, vec, logits, fuse_k, cfg->renorm, idx, gate); break;
    default: pw::router_logits_kernel<4><<<g1, pw::kRouteThreads, 0, st>>>(x_bf16, Wr, bias, T, H, E, vec, logits, fuse_k, cfg->renorm, idx, gate); break;
  }
  if (launch_status() != PW_OK) return PW_ERR_CUDA;
  if (fuse_k) return PW_OK;
  return pw_topk(logits, T, E, cfg, idx, gate, stream);
}

pw_status pw_substitute(const float* logits, int32_t* idx, const float* gate,
                        const uint8_t* resident, int T, int E, const pw_route_cfg* cfg,
                        uint8_t* action, float* mass, pw_stream_t stream) {
  if (!logits || !idx || !gate || !resident) return PW_ERR_INVALID_ARG;
  if (T < 1 || T > PW_MAX_TOKENS || E < 1 || E > PW_MAX_EXPERTS || !cfg_ok(cfg, E))
    return PW_ERR_INVALID_ARG;
  if (cfg->policy != PW_POLICY_FETCH_ALL && cfg->policy != PW_POLICY_THRESHOLD &&
      cfg->policy != PW_POLICY_FIRST_CHOICE)
    return PW_ERR_INVALID_ARG;
  if (cfg->threshold != cfg->threshold) return PW_ERR_INVALID_ARG;  // NaN
  const dim3 g((T + 7) / 8), b(256);
  cudaStream_t st = as_cuda(stream);
#define PW_SUBST(PL)                                                                          \
  pw::substitute_kernel<PL><<<g, b, 0, st>>>(logits, idx, gate, resident, T, E, cfg->k,      \
                                             cfg->policy, cfg->threshold, action, mass)
  if (E <= 32) PW_SUBST(1);
  else if (E <= 64) PW_SUBST(2);
  else if (E <= 128) PW_SUBST(4);
  else if (E <= 256) PW_SUBST(8);
  else if (E <= 512) PW_SUBST(16);
  else PW_SUBST(32);
#undef PW_SUBST
  return launch_status();
}

pw_status pw_remap(const float* logits, int32_t* idx, const float* gate, int T, int E,
                   const pw_route_cfg* cfg, uint8_t* critical, int32_t* unique,
                   pw_stream_t stream) {
  if (!logits || !idx || !gate) return PW_ERR_INVALID_ARG;
  if (T < 1 || T > PW_MAX_TOKENS || E < 1 || E > PW_MAX_EXPERTS || !cfg_ok(cfg, E))
    return PW_ERR_INVALID_ARG;
  if (cfg->critical_n < 0 || static_cast<long long>(T) * cfg->k > 8192) return PW_ERR_INVALID_ARG;
  cudaStream_t st = as_cuda(stream);
#define PW_REMAP(PL)                                                                          \
  pw::remap_kernel<PL><<<1, 1024, 0, st>>>(logits, idx, gate, T, E, cfg->k, cfg->critical_n, \
                                           critical, unique)
  if (E <= 32) PW_REMAP(1);
  else if (E <= 64) PW_REMAP(2);
  else if (E <= 128) PW_REMAP(4);
  else if (E <= 256) PW_REMAP(8);
  else if (E <= 512) PW_REMAP(16);
  else PW_REMAP(32);
#undef PW_REMAP
  return launch_status();
}

pw_status pw_topk(const float* logits, int T, int E, const pw_route_cfg* cfg, int32_t* idx,
                  float* gate, pw_stream_t stream) {
  if (!logits || !idx || !gate) return PW_ERR_INVALID_ARG;
  if (T < 1 || T > PW_MAX_TOKENS || E < 1 || E > PW_MAX_EXPERTS || !cfg_ok(cfg, E))
    return PW_ERR_INVALID_ARG;
  const int tg = (T + 7) / 8;
  cudaStream_t st = as_cuda(stream);
#define PW_TOPK(PL)                                                                           \
  pw::topk_kernel<PL><<<tg, 256, 0, st>>>(logits, T, E, cfg->k, cfg->renorm, idx, gate)
  if (E <= 32) PW_TOPK(1);
  else if (E <= 64) PW_TOPK(2);
  else if (E <= 128) PW_TOPK(4);
  else if (E <= 256) PW_TOPK(8);
  else if (E <= 512) PW_TOPK(16);
  else PW_TOPK(32);
#undef PW_TOPK
  return launch_status();
}

pw_status pw_affinity_default(int E, int k, pw_affinity_cfg* out) {
  if (!out || E < 1 || k < 1 || k > E) return PW_ERR_INVALID_ARG;
  const double ratio = static_cast<double>(E) / k;
  if (ratio <= 1.0) {
    out->num_bins = 1;
    out->low_bins = 1;
    out->bin_width = INFINITY;
    return PW_OK;
  }
  const int B = static_cast<int>(std::ceil(ratio));
  out->num_bins = B;
  out->low_bins = (B + 1) / 2;
  out->bin_width = std::log(ratio) / B;
  return PW_OK;
}

pw_status pw_affinity_remap(const float* logits, int32_t* idx, const float* gate, int T, int E,
                            const pw_route_cfg* cfg, const pw_affinity_cfg* acfg,
                            uint8_t* critical, int32_t* bins, int32_t* unique,
                            pw_stream_t stream) {
  if (!logits || !idx || !gate || !acfg) return PW_ERR_INVALID_ARG;
  if (T < 1 || T > PW_MAX_TOKENS || E < 1 || E > PW_MAX_EXPERTS || !cfg_ok(cfg, E))
    return PW_ERR_INVALID_ARG;
  if (cfg->critical_n < 0 || static_cast<long long>(T) * cfg->k > 8192) return PW_ERR_INVALID_ARG;
  const double w = acfg->bin_width;
  if (acfg->num_bins < 1 || acfg->num_bins > 256 || acfg->low_bins < 0 || !(w > 0.0))
    return PW_ERR_INVALID_ARG;  // also rejects a NaN width
  cudaStream_t st = as_cuda(stream);
#define PW_AFF(PL)                                                                            \
  pw::affinity_remap_kernel<PL><<<1, 1024, 0, st>>>(logits, idx, gate, T, E, cfg->k,          \
                                                    cfg->critical_n, acfg->num_bins, w,        \
                                                    acfg->low_bins, critical, bins, unique)
  if (E <= 32) PW_AFF(1);
  else if (E <= 64) PW_AFF(2);
  else if (E <= 128) PW_AFF(4);
  else if (E <= 256) PW_AFF(8);
  else if (E <= 512) PW_AFF(16);
  else PW_AFF(32);
#undef PW_AFF
  return launch_status();
}

pw_status pw_cache_step(const float* logits, int32_t* idx, const float* gate, int T, int E,
                        const pw_route_cfg* cfg, double beta, uint8_t* resident, double* mass,
                        uint32_t* freq, int capacity, uint8_t* action, float* mass_t,
                        int32_t* stats, pw_stream_t stream) {
  if (!logits || !idx || !gate || !resident || !mass || !freq) return PW_ERR_INVALID_ARG;
  if (T < 1 || T > PW_MAX_TOKENS || E < 1 || E > PW_MAX_EXPERTS || !cfg_ok(cfg, E))
    return PW_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * cfg->k > pw::kCacheMaxAssign) return PW_ERR_INVALID_ARG;
  if (cfg->policy != PW_POLICY_FETCH_ALL && cfg->policy != PW_POLICY_THRESHOLD &&
      cfg->policy != PW_POLICY_FIRST_CHOICE)
    return PW_ERR_INVALID_ARG;
  if (cfg->threshold != cfg->threshold || beta != beta || capacity < 0 || capacity > E)
    return PW_ERR_INVALID_ARG;
  cudaStream_t st = as_cuda(stream);
  if (stats && cudaMemsetAsync(stats, 0, 3 * sizeof(int32_t), st) != cudaSuccess)
    return PW_ERR_CUDA;
#define PW_CACHE(PL)                                                                          \
  pw::cache_step_kernel<PL><<<1, 1024, 0, st>>>(logits, idx, gate, T, E, cfg->k, cfg->policy,  \
                                                cfg->threshold, beta, resident, mass, freq,    \
                                                capacity, action, mass_t, stats)
  if (E <= 32) PW_CACHE(1);
  else if (E <= 64) PW_CACHE(2);
  else if (E <= 128) PW_CACHE(4);
  else if (E <= 256) PW_CACHE(8);
  else if (E <= 512) PW_CACHE(16);
  else PW_CACHE(32);
#undef PW_CACHE
  return launch_status();
}

}  // extern "C"
