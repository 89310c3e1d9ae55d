#!/usr/bin/env python
"""Benchmark of the any-precision MoE decode layer (one JSON line on rank 0).

Default workload: the Mixtral-8x7B-shaped layer (H 4096, 8 experts, I 14336, top-2 renormalised,
parent 8-bit, per-block bitwidth uniform in 3..8, Zipf(1.2) router bias) at batch 1, synthetic
seeded data.  A step is one whole layer call: router GEMV + softmax top-k (+ the config's
substitution or remap) + grouping + fused any-precision FFN + combine, replayed from a CUDA
graph.  L2 is flushed (a memset of 2.5x the L2 size) before every timed step, outside that
step's CUDA events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pw|reference]

N > 1 runs N independent replicas (one per GPU, launched by torchrun); value = N * T / (max over
ranks of the per-step device time).  --impl reference times the CPU oracle on rank 0 instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE decode layer tokens/s and effective weight HBM GB/s (fraction of peak)"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0          # B200 HBM3e data-sheet figure, for the spec fraction
WORKLOAD = ("mixtral_8x7b", 1)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=("pw", "reference"), default="pw")
    ap.add_argument("--workload", default=f"{WORKLOAD[0]}:{WORKLOAD[1]}",
                    help="config name:T (default mixtral_8x7b:1)")
    ap.add_argument("--tc-min-tokens", type=int, default=None, metavar="M",
                    help="switch of the forward call's FFN paths (pw_set_tc_min_tokens): the "
                         "tensor-core FFN from an average of M routed tokens per active expert "
                         "(library default 4; 0 = always)")
    ap.add_argument("--no-rewrite", action="store_true",
                    help="plain top-k routing: leave out the config's substitution or remap")
    ap.add_argument("--affinity", action="store_true",
                    help="rewrite the assignments with LYNX AffinityBinning (pw_affinity_remap) "
                         "in place of the config's own rewrite")
    ap.add_argument("--cache-stream", choices=("quality", "speed", "fetch-all"), default=None,
                    help="instead of the layer step: drive pw_topk + pw_cache_step over a "
                         "synthetic multi-step logit stream of the workload's router shape")
    ap.add_argument("--page-in", type=int, default=None, metavar="Q",
                    help="instead of the layer step: page one expert of the workload in at "
                         "bitwidth Q (top-Q planes of both blocks, pinned host -> device)")
    ap.add_argument("--skip-cpu-baseline", action="store_true",
                    help="leave out the CPU oracle timing (profiling runs)")
    ap.add_argument("--cpu-sample-rows", type=float, default=None,
                    help="fraction of FFN rows the CPU oracle sample computes")
    return ap.parse_args()


def workload(args):
    import dataclasses
    from any_precision_expert_pw_b200.inputs import CONFIGS, POLICY_AFFINITY, POLICY_NONE
    name, T = args.workload.split(":")
    cfg = CONFIGS[name]
    if getattr(args, "affinity", False):
        cfg = dataclasses.replace(cfg, policy=POLICY_AFFINITY)
    if getattr(args, "no_rewrite", False):
        cfg = dataclasses.replace(cfg, policy=POLICY_NONE, resident_frac=None)
    return cfg, int(T)


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the sources of the kernels pw_moe_anyprec_forward launches (and their launch logic)
FORWARD_SOURCES = ("pw_common.cuh", "pw_ffn.cuh", "pw_group.cuh", "pw_lib.cu", "pw_tc.cuh")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "any_precision_expert_pw_b200", "csrc")
    for f in FORWARD_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_key: str):
    """DRAM traffic per FFN call from the committed ncu summary, if it was taken on this
    workload (`name:T`, default routing) with these sources."""
    p = os.path.join(ROOT, "profiles", "ffn_traffic.txt")
    try:
        kv = {}
        for line in open(p):
            if "=" in line and not line.startswith("#"):
                k, v = line.strip().split("=", 1)
                kv[k.strip()] = v.strip()
        if kv.get("source_sha") == kernel_source_hash() and kv.get("workload") == workload_key:
            return float(kv["traffic_bytes_per_call"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms around the timed region.  The
    timed region of a short run can be shorter than one sampling interval, so the caller keeps
    the GPU on the same step (untimed) until samples() has grown by `min_samples` since the
    timed region began; only those samples are reported."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None
        self.skip = 0

    def start(self, first_sample_timeout_s: float = 5.0):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.gpu_id], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        t0 = time.time()   # nvidia-smi takes a moment to print its first line
        while self.samples() == 0 and time.time() - t0 < first_sample_timeout_s:
            if self.proc.poll() is not None:
                break
            time.sleep(0.05)

    def samples(self) -> int:
        if self.proc is None or self.path is None:
            return 0
        try:
            self.fh.flush()
            with open(self.path) as f:
                return sum(1 for line in f if line.count(",") >= 8)
        except Exception:
            return 0

    def mark(self):
        """Only samples written after this call are reported."""
        self.skip = self.samples()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sms, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        lines = [line for line in open(self.path) if line.count(",") >= 8][self.skip:]
        for line in lines:
            f = [x.strip() for x in line.split(",")]
            try:
                sms.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sms)}


class Replicas:
    """N independent replicas of the layer, one process per GPU (torchrun's RANK / WORLD_SIZE /
    LOCAL_RANK / MASTER_* environment).  The process group carries no layer data: only the
    barriers around the timed region and the max over ranks of the measured times.  backend
    "nccl" on GPUs; "gloo" runs the same bookkeeping on CPU processes."""

    def __init__(self, backend="nccl", timeout_s=120):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.device = torch.device(f"cuda:{self.local}") if backend == "nccl" else torch.device("cpu")
        if self.world > 1:
            import torch.distributed as dist
            kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = self.device
            dist.init_process_group(backend, **kw)

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_over_ranks(self, v):
        if self.world == 1:
            return v
        import torch
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


def replica_value(world, tokens_per_replica, step_ms):
    """Whole-job tokens/s: every replica processes its own batch in the (max) step time."""
    return world * tokens_per_replica / (step_ms * 1e-3)


def oracle_step(L, frac):
    """One bounded oracle sample: full routing, FFN on a fraction of every block's rows.
    Returns the seconds a full step would take (FFN time scaled by 1/frac)."""
    import numpy as np
    from oracle import ffn as offn
    from oracle import layer as olayer
    from oracle.group import group_by_expert
    from oracle.router import bf16_bits_to_f64
    cfg = L.cfg
    if frac >= 1.0:                       # the whole layer, exactly as the oracle computes it
        t0 = time.perf_counter()
        olayer.moe_layer(L)
        return time.perf_counter() - t0
    t0 = time.perf_counter()
    res = olayer.route(L)
    t1 = time.perf_counter()
    idx = res["idx"]
    X = bf16_bits_to_f64(L.x_bf16)
    _, offsets, perm, active = group_by_expert(idx, cfg.E)
    rg = max(1, int(round(2 * cfg.I * frac)))
    rd = max(1, int(round(cfg.H * frac)))
    for e in active:
        a = perm[offsets[e]:offsets[e + 1]]
        Xe = X[a // cfg.k]
        qg, qd = int(L.q[e, 0]), int(L.q[e, 1])
        gu = offn.block_matvec(L.idx[e][0][:rg], L.lut[e][0][qg][:rg], cfg.n, qg, Xe.T)
        h = np.zeros((cfg.I, len(a)))
        h[: min(rg, cfg.I)] = gu[: min(rg, cfg.I)]
        offn.block_matvec(L.idx[e][1][:rd], L.lut[e][1][qd][:rd], cfg.n, qd, h)
    t2 = time.perf_counter()
    return (t1 - t0) + (t2 - t1) / frac


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(L, T, frac, reps=1):
    secs = [oracle_step(L, frac) for _ in range(reps)]
    s = statistics.median(secs)
    return {"value": T / s, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": (f"float64 NumPy oracle, whole layer (routing + FFN + combine) on the "
                       f"bench inputs; median of {reps}" if frac >= 1.0 else
                       f"float64 NumPy oracle: full routing + FFN over {frac:.3f} of every used "
                       f"block's rows, time scaled to the whole layer; median of {reps}")}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from any_precision_expert_pw_b200.inputs import make_layer
    cfg, T = workload(args)
    L = make_layer(cfg, T)
    frac = args.cpu_sample_rows or 1.0
    steps = max(1, min(args.steps, 10))
    warm = max(0, min(args.warmup, 1))
    for _ in range(warm):
        oracle_step(L, frac)
    secs = [oracle_step(L, frac) for _ in range(steps)]
    s = sum(secs) / len(secs)
    v = T / s
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
           "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": s * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic",
           "config": {"workload": f"{cfg.name}-shaped MoE decode layer, T={T}", "H": cfg.H,
                      "E": cfg.E, "I": cfg.I, "k": cfg.k, "parent_bits": cfg.n},
           "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas_threads(),
                            "kind": "oracle",
                            "sample": f"FFN over {frac:.3f} of every used block's rows per step, "
                                      "time scaled to the whole layer"},
           "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_pw(args):
    import numpy as np
    import torch

    from any_precision_expert_pw_b200 import binding as B
    from any_precision_expert_pw_b200.accounting import ffn_bytes, layer_bytes, plane_bytes
    from any_precision_expert_pw_b200.device_layer import DeviceLayer
    from any_precision_expert_pw_b200.inputs import (POLICY_AFFINITY, POLICY_NONE, POLICY_REMAP,
                                                     make_layer)

    rep = Replicas("nccl")
    world, rank, local = rep.world, rep.rank, rep.local
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    cfg, T = workload(args)
    tc_min = 4 if args.tc_min_tokens is None else args.tc_min_tokens
    B.check(B.pw_set_tc_min_tokens(tc_min))
    L = make_layer(cfg, T)
    D = DeviceLayer(L, device=str(dev))
    stream = torch.cuda.Stream(device=dev)
    D.stream = stream.cuda_stream
    with torch.cuda.stream(stream):
        D.forward()
    stream.synchronize()
    st = D.status()
    if st != B.PW_OK:
        raise RuntimeError(f"device status after warm-up: {B.pw_status_string(st)}")

    # parity of this run's routing against the oracle (cheap part of the check)
    if rank == 0:
        from oracle.layer import route as oracle_route
        ref = oracle_route(L)
        if not np.array_equal(D.idx.cpu().numpy(), ref["idx"]):
            raise RuntimeError("routing of the bench inputs differs from the oracle")

    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        D.forward()
    g_ffn = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ffn, stream=stream):
        D.ffn()
    # router (+ separate top-k for E > 8), the assignment rewrite if any, setup, the FFN
    # (gate_up and down in one launch) and combine; the tensor-core FFN adds its operand staging
    tc_path = T * cfg.k >= tc_min * min(cfg.E, T * cfg.k)
    launches_step = ((1 if cfg.E <= 8 else 2) + (0 if cfg.policy == POLICY_NONE else 1) + 3 +
                     (1 if tc_path else 0))

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(int(2.5 * l2), dtype=torch.uint8, device=dev)

    def timed(graph, n, record=True):
        evs = []
        with torch.cuda.stream(stream):
            for _ in range(n):
                flush.fill_(1)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                evs.append((e0, e1))
        return evs

    def mean_ms(evs):
        return sum(a.elapsed_time(b) for a, b in evs) / len(evs)

    def median_ms(evs):
        return statistics.median(a.elapsed_time(b) for a, b in evs)

    barrier = rep.barrier
    max_over_ranks = rep.max_over_ranks

    timed(g_step, args.warmup)
    torch.cuda.synchronize(dev)
    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", local))
    gpu_id = uuid if uuid.startswith("GPU-") else (f"GPU-{uuid}" if len(uuid) > 30 else str(local))
    clocks = ClockSampler(gpu_id)
    clocks.start()
    barrier()
    torch.cuda.synchronize(dev)
    clocks.mark()
    t_wall0 = time.perf_counter()
    evs = timed(g_step, args.steps)
    torch.cuda.synchronize(dev)
    barrier()
    t_wall1 = time.perf_counter()
    # a short timed region sees no sample: keep the GPU on the same step (untimed) until three
    # samples cover the region and what follows it, at most 3 s
    t_keep = time.perf_counter()
    extra_steps = 0
    while clocks.samples() - clocks.skip < 3 and time.perf_counter() - t_keep < 3.0:
        timed(g_step, 20)
        torch.cuda.synchronize(dev)
        extra_steps += 20
    clk = clocks.stop()
    clk["window"] = ("timed region" if extra_steps == 0 else
                     f"timed region + {extra_steps} untimed replays of the same step")
    step_ms = max_over_ranks(mean_ms(evs))
    step_med_ms = max_over_ranks(median_ms(evs))

    # FFN call alone (the dominant kernels): roofline numerator
    timed(g_ffn, args.warmup)
    ffn_evs = timed(g_ffn, args.steps)
    torch.cuda.synchronize(dev)
    ffn_ms = max_over_ranks(mean_ms(ffn_evs))

    # end to end through the public API: pinned x in, forward, y out, every step
    x_host = torch.from_numpy(L.x_bf16.view(np.int16).copy()).pin_memory()
    y_host = torch.empty((T, cfg.H), dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, 1000))
    e2e_evs = []
    with torch.cuda.stream(stream):
        for i in range(e2e_steps + 5):
            flush.fill_(1)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            D.x.copy_(x_host, non_blocking=True)
            D.forward()
            y_host.copy_(D.y, non_blocking=True)
            e1.record(stream)
            if i >= 5:
                e2e_evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(mean_ms(e2e_evs))
    st = D.status()
    if st != B.PW_OK:
        raise RuntimeError(f"device status after timing: {B.pw_status_string(st)}")

    used = np.unique(D.idx.cpu().numpy())
    b_layer = layer_bytes(cfg.H, cfg.I, cfg.E, L.q, used, T, bool(np.any(L.bias != 0)))
    b_ffn = ffn_bytes(cfg.H, cfg.I, L.q, used, T)
    b_planes = plane_bytes(cfg.H, cfg.I, L.q, used)
    peak, peak_kind = read_peaks()
    achieved = b_ffn / (ffn_ms * 1e-3) / 1e9
    plain = not (getattr(args, "affinity", False) or getattr(args, "no_rewrite", False))
    traffic = recorded_traffic(f"{cfg.name}:{T}") if plain else None
    value = replica_value(world, T, step_ms)
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": f"{cfg.name}-shaped MoE decode layer, T={T}", "H": cfg.H,
                   "E": cfg.E, "I": cfg.I, "k": cfg.k, "parent_bits": cfg.n,
                   "bits": L.q.tolist(), "experts_used": used.tolist(),
                   **({"distinct_experts_before_after_rewrite": D.unique.cpu().tolist()}
                      if cfg.policy in (POLICY_REMAP, POLICY_AFFINITY) else {}),
                   "ffn_path": "tensor-core (tcgen05)" if tc_path else "cuda-core",
                   "rewrite": {-1: "none", 0: "fetch-all", 1: "0.15 rule", 2: "first choice",
                               3: "batch remap", 4: "AffinityBinning remap"}[cfg.policy],
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "flushed before every step (memset of 2.5x L2, outside the step events)",
                   "timing": "CUDA-graph replay per step, CUDA events on the launching stream"},
        "ms_per_step_median": step_med_ms,
        "effective_gbs": b_layer / (step_ms * 1e-3) / 1e9,
        "hbm_frac": b_layer / (step_ms * 1e-3) / 1e9 / peak,
        "hbm_frac_of_spec": b_layer / (step_ms * 1e-3) / 1e9 / SPEC_HBM_GBS,
        "plane_gbs": b_planes / (step_ms * 1e-3) / 1e9,
        "bytes_per_step": b_layer,
        "ffn_ms": ffn_ms,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "pw_moe_anyprec_forward (grouping + gate_up + down + combine)",
                     "peak_kind": f"{peak_kind} copy bandwidth (burst)"},
        "e2e": {"value": replica_value(world, T, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": int(T * cfg.H * 2), "d2h_bytes_per_step": int(T * cfg.H * 4),
                "ms_per_step": e2e_ms, "path": "pinned x -> pw_route_topk -> "
                "pw_moe_anyprec_forward -> pinned y, direct calls (no graph)"},
        "gpu_launches": launches_step * args.steps,
        "clocks": clk,
        "wall_s_timed_region": t_wall1 - t_wall0,
    }
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        frac = args.cpu_sample_rows or 1.0
        out["cpu_baseline"] = cpu_baseline(L, T, frac, reps=3)
    if rank == 0:
        print(json.dumps(out), flush=True)
    del g_step, g_ffn
    rep.close()


def run_cache_stream(args):
    """Expert cache across decode steps: one step = pw_topk + pw_cache_step on the next logits
    of a seeded stream (topic changes every 32 steps); device time per step from CUDA events,
    and what the policy did per token (fetches, admissions, evictions, substitutions)."""
    import numpy as np
    import torch

    from any_precision_expert_pw_b200 import binding as B
    from any_precision_expert_pw_b200.inputs import logit_stream

    rep = Replicas("nccl")
    dev = torch.device(f"cuda:{rep.local}")
    torch.cuda.set_device(dev)
    cfg, T = workload(args)
    E, k = cfg.E, cfg.k
    policy = {"quality": 1, "speed": 2, "fetch-all": 0}[args.cache_stream]
    frac = cfg.resident_frac if cfg.resident_frac else 0.25
    cap = int(frac * E)
    steps, warm = args.steps, args.warmup
    lo = torch.from_numpy(logit_stream(E, T, warm + steps, seed=1 + rep.rank, topic_len=32)).to(dev)
    res0 = np.zeros(E, np.uint8)
    res0[np.random.default_rng(np.random.SeedSequence([11, E, rep.rank])).choice(
        E, cap, replace=False)] = 1
    d_res = torch.from_numpy(res0).to(dev)
    d_mass = torch.zeros(E, dtype=torch.float64, device=dev)
    d_freq = torch.zeros(E, dtype=torch.int32, device=dev)
    d_idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    d_gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    d_act = torch.empty((warm + steps, T, k), dtype=torch.uint8, device=dev)
    d_m = torch.empty((warm + steps, T), dtype=torch.float32, device=dev)
    d_stats = torch.zeros((warm + steps, 3), dtype=torch.int32, device=dev)
    rcfg = B.pw_route_cfg(k=k, renorm=int(cfg.renorm), policy=policy, threshold=0.15,
                          critical_n=0)
    stream = torch.cuda.Stream(device=dev)
    cs = stream.cuda_stream
    evs = []
    rep.barrier()
    with torch.cuda.stream(stream):
        for s in range(warm + steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            B.check(B.pw_topk(lo[s].data_ptr(), T, E, rcfg, d_idx.data_ptr(), d_gate.data_ptr(),
                              cs), "pw_topk")
            B.check(B.pw_cache_step(lo[s].data_ptr(), d_idx.data_ptr(), d_gate.data_ptr(), T, E,
                                    rcfg, 0.5, d_res.data_ptr(), d_mass.data_ptr(),
                                    d_freq.data_ptr(), cap, d_act[s].data_ptr(),
                                    d_m[s].data_ptr(), d_stats[s].data_ptr(), cs),
                    "pw_cache_step")
            e1.record(stream)
            if s >= warm:
                evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    rep.barrier()
    st = B.pw_get_status(cs)
    if st != B.PW_OK:
        raise RuntimeError(f"device status: {B.pw_status_string(st)}")
    ms = rep.max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / len(evs))
    stats = d_stats[warm:].sum(0).cpu().numpy()
    tokens = steps * T
    out = {"metric": "expert-cache decode step (pw_topk + pw_cache_step)",
           "value": rep.world * 1e3 / ms, "unit": "steps/s", "n_gpus": rep.world,
           "steps": steps, "warmup": warm, "ms_per_step": ms, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64", "data": "synthetic",
           "config": {"workload": f"{cfg.name}-shaped router stream, T={T}",
                      "policy": {1: "Quality-First (0.15 rule)", 2: "Speed-First (first choice)",
                                 0: "fetch every miss"}[policy] +
                      " + frequency eviction + background admission (beta 0.5)",
                      "E": E, "k": k, "capacity": cap, "topic_len": 32},
           "fetched_per_token": float(stats[0]) / tokens,
           "admitted_per_token": float(stats[1]) / tokens,
           "evicted_per_token": float(stats[2]) / tokens,
           "substituted_per_token": float((d_act[warm:] == 2).sum().item()) / tokens,
           "mean_substituted_mass": float(d_m[warm:].mean().item()),
           "gpu_launches": 2 * steps}
    if rep.rank == 0:
        print(json.dumps(out), flush=True)
    rep.close()


def run_page_in(args):
    """Page movement: one expert's two blocks move from pinned host memory (all n planes per
    run) to compact device buffers holding the top q planes per run (pw_page_copy), then the
    table entries are switched over (pw_page_update).  Device time per expert from CUDA events;
    plane bytes moved per second."""
    import numpy as np
    import torch

    from any_precision_expert_pw_b200 import binding as B
    from any_precision_expert_pw_b200.device_layer import DeviceLayer
    from any_precision_expert_pw_b200.inputs import MOD_DOWN, MOD_GATE_UP, make_layer

    rep = Replicas("nccl")
    dev = torch.device(f"cuda:{rep.local}")
    torch.cuda.set_device(dev)
    cfg, T = workload(args)
    q = int(args.page_in)
    n = cfg.n
    if not (3 <= q <= n):
        raise SystemExit(f"--page-in needs 3 <= Q <= {n}")
    L = make_layer(cfg, T)
    D = DeviceLayer(L, device=str(dev))
    stream = torch.cuda.Stream(device=dev)
    D.stream = stream.cuda_stream
    e = 0
    blocks = []
    for m in (MOD_GATE_UP, MOD_DOWN):
        R, C = L.block_shape(m)
        host = torch.empty((n * R * C // 32,), dtype=torch.int32).pin_memory()
        host.copy_(D.planes[(e, m)].cpu())
        comp = torch.empty((q * R * C // 32,), dtype=torch.int32, device=dev)
        blocks.append((m, R, C, host, comp))
    moved = sum(q * R * C // 8 for _, R, C, _, _ in blocks)
    ups = (B.pw_page_update_t * 2)()
    for i, (m, R, C, host, comp) in enumerate(blocks):
        ups[i].block = e * 2 + m
        ups[i].state = B.PW_PAGE_GPU + 1
        ups[i].stored_bits = q
        ups[i].committed_bits = q
        ups[i].planes = comp.data_ptr()
    ups_d = torch.frombuffer(bytearray(bytes(ups)), dtype=torch.uint8).to(dev)
    cs = stream.cuda_stream
    evs = []
    rep.barrier()
    with torch.cuda.stream(stream):
        for s in range(args.warmup + args.steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for m, R, C, host, comp in blocks:
                B.check(B.pw_page_copy(host.data_ptr(), n, comp.data_ptr(), q, R, C, q, cs),
                        "pw_page_copy")
            B.check(B.pw_page_update(D.pt_dev.data_ptr(), D.num_blocks, ups_d.data_ptr(), 2, cs),
                    "pw_page_update")
            e1.record(stream)
            if s >= args.warmup:
                evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    rep.barrier()
    st = B.pw_get_status(cs)
    if st != B.PW_OK:
        raise RuntimeError(f"device status: {B.pw_status_string(st)}")
    ms = rep.max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / len(evs))
    full = sum(n * R * C // 8 for _, R, C, _, _ in blocks)
    out = {"metric": "expert page-in (top-q planes, pinned host -> device)",
           "value": rep.world * moved / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": rep.world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32",
           "data": "synthetic",
           "config": {"workload": f"{cfg.name}-shaped expert (gate_up + down), q={q} of n={n}",
                      "bytes_moved": moved, "bytes_all_planes": full,
                      "copies_per_step": sum((C // 32 + 31) // 32 for _, _, C, _, _ in blocks)},
           "gpu_launches": args.steps}
    if rep.rank == 0:
        print(json.dumps(out), flush=True)
    rep.close()


def main():
    args = parse_args()
    if args.page_in is not None:
        run_page_in(args)
        return
    if args.cache_stream:
        run_cache_stream(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_pw(args)


if __name__ == "__main__":
    main()
