"""Benchmark of the routed MoE FFN layer (Gemma-4-26B-A4B shape) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode] [--impl reference]

A step is one moe_forward over one batch (router, dispatch, GEMM-1 + GEGLU, GEMM-2,
combine) with inputs resident in HBM.  L2 is flushed before every step, untimed: a 256 MB
write, then a 256 MB read, so that the dirty lines the write leaves are written back before
the step rather than during it; each step is timed with CUDA events on the launching
stream.  Rank 0 prints
one JSON line.  With N > 1 (torchrun) every rank runs its own batch on its own GPU (weak
scaling, no collective on the data path) and the reported time is the max over ranks.

--impl reference times the fp64 CPU oracle instead (the only baseline this layer has),
on rank 0 only, on the same config.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from expert_routed_ffn_softmax_b200 import workloads as wl  # noqa: E402

METRIC = "MoE-layer tokens/s; HBM GB/s (decode) & BF16 TFLOP/s (prefill) vs peak"
UNIT = "tokens/s"
PER_EXPERT_BYTES = 11_894_784   # 3 * 2816 * 704 * 2: weights one active expert reads
L2_FLUSH_BYTES = 256 << 20


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every millisecond while the
    timed region runs (reads only; nothing is set)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device: torch.device, period_s: float = 0.001):
        self.period = period_s
        self.samples: list[tuple[float, int, int]] = []
        self.h = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            p = torch.cuda.get_device_properties(device)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception:   # no NVML: the line carries "clocks": null
            self.h = None

    def _reasons(self) -> int:
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(fn(self.h))

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def _sample(self):
        nv = self.nv
        try:
            self.samples.append((time.perf_counter(),
                                 nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                 self._reasons()))
        except Exception:
            pass

    def start(self):
        if self.h is None:
            return
        self._sample()          # one sample as the timed region starts, whatever its length
        self._stop = threading.Event()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def stop(self) -> dict | None:
        if self.h is None:
            return None
        self._stop.set()
        self.t.join()
        self._sample()          # and one as it ends (the GPU has just finished its last step)
        if not self.samples:
            return None
        sm = [s[1] for s in self.samples]
        reasons = set()
        for _, _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvml"}


# ----------------------------------------------------------------------------- accounting
def algorithmic(cfg: wl.MoEConfig, counts: np.ndarray, has_bias: bool) -> dict:
    """Bytes/FLOPs the layer itself must move/compute (not Xp/Hbuf/O traffic)."""
    active = int((counts > 0).sum())
    P = cfg.T * cfg.k
    ew = 3 * cfg.H * cfg.I * 2
    step_bytes = (active * ew + cfg.H * cfg.E * 2 + 2 * cfg.T * cfg.H * 2
                  + (cfg.E * 4 if has_bias else 0))
    step_flops = cfg.T * 2 * cfg.H * cfg.E + P * (2 * cfg.H * 2 * cfg.I + 2 * cfg.I * cfg.H)
    return {
        "active_experts": active,
        "step_bytes": step_bytes,
        "step_flops": step_flops,
        "gemm1_bytes": active * 2 * cfg.H * cfg.I * 2,
        "gemm1_flops": P * 2 * cfg.H * 2 * cfg.I,
        "gemm2_bytes": active * cfg.H * cfg.I * 2,
        "gemm2_flops": P * 2 * cfg.I * cfg.H,
    }


def ffn_kernel_name(T: int, tiles: str) -> str:
    """The expert-FFN kernel(s) the library launches for T tokens and a tile family."""
    from expert_routed_ffn_softmax_b200 import _abi
    return _abi.ffn_kernel_name(T, tiles)


# The sources each expert-FFN kernel is built from (a capture stays valid while they do).
KERNEL_SOURCES = {
    "bf16": ("grouped_gemm.cuh", "gemm_persistent.cuh", "ffn_dynamic.cuh", "ffn_pair.cuh",
             "gemm_decode.cuh", "ptx.cuh"),
    "nvfp4": ("grouped_gemm.cuh", "gemm_persistent.cuh", "gemm_decode.cuh", "ptx.cuh",
              "nvfp4.cuh", "nvfp4_mma.cuh"),
}


def kernel_source_sha(family: str = "bf16") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[family]:
        h.update(open(os.path.join(ROOT, "expert_routed_ffn_softmax_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str) -> float | None:
    """DRAM bytes per launch recorded by ncu for this kernel source, else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        rows = json.load(open(p))
    except ValueError:
        return None
    sha = kernel_source_sha("nvfp4" if kernel.startswith("nvfp4") else "bf16")
    for r in rows:
        if r.get("kernel") == kernel and r.get("workload") == workload and r.get("source_sha") == sha:
            return float(r["dram_bytes_per_launch"])
    return None


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(values: list[float], dist=None, device=None) -> list[float]:
    """Element-wise max of per-rank timings (every rank gets the result).  With one rank
    (dist None or world size 1) the values come back unchanged."""
    if dist is None or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world: int, tokens_per_rank: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return world * tokens_per_rank / (max_ms * 1e-3)


TENSOR_BOUND_CONFIGS = ("skewed", "sweep_T32768")


def time_layer(moe, cfg, args, g, x_cpu, dev, stream, flush_l2, dist, e2e: bool) -> dict:
    """Time args.steps graph replays of one moe_forward over cfg's batch (L2 flushed, untimed,
    before every step); per-stage device times from a second graph with the library's stage
    events; optionally the end-to-end time with pinned host buffers.  Device times are the
    max over ranks."""
    x = x_cpu.to(dev)
    y0, aux = moe.forward(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], cfg.k,
                          bias=g["bias"], aux=True, tiles=args.tiles)
    if moe.sync_status() != 0:
        raise SystemExit(f"device status not OK after the first forward ({cfg.name})")
    counts = aux["expert_counts"].cpu().numpy()
    acc = algorithmic(cfg, counts, g["bias"] is not None)
    rstats = moe.router_stats(aux)
    del aux

    # The step as a serving loop runs it: one captured moe_forward per batch (graph replay).
    graph = moe.ForwardGraph(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], cfg.k,
                             bias=g["bias"], tiles=args.tiles)
    for _ in range(args.warmup):
        flush_l2()
        graph.replay()
    torch.cuda.synchronize()
    if not torch.equal(graph.y, y0):
        raise SystemExit(f"graph replay differs from the direct call ({cfg.name})")
    del y0

    # ---- timed region: K steps, L2 flushed (untimed) before each
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2()
        ev[i][0].record(stream)
        graph.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms = sum(step_ms) / len(step_ms)
    if moe.sync_status() != 0:
        raise SystemExit(f"device status not OK after the timed steps ({cfg.name})")

    # ---- per-stage device times: a graph of the same call with the library's stage events
    pgraph = moe.ForwardGraph(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], cfg.k,
                              bias=g["bias"], profile=True, tiles=args.tiles)
    stage_acc: dict[str, list[float]] = {}
    try:
        for _ in range(max(3, min(args.steps, 20))):
            flush_l2()
            pgraph.replay()
            for k, v in moe.last_stage_times().items():
                stage_acc.setdefault(k, []).append(v)
    except RuntimeError as exc:
        print(f"stage timing unavailable: {exc}", file=sys.stderr)
    stages = {k: sum(v) / len(v) for k, v in stage_acc.items()}
    del pgraph

    e2e_ms = None
    if e2e:
        # ---- end to end through the public API with host buffers (pinned), L2 flushed
        x_host = x_cpu.pin_memory()
        y_host = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
        e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
        for i in range(args.warmup + args.steps):
            flush_l2()
            if i >= args.warmup:
                e2e_ev[i - args.warmup][0].record(stream)
            graph.x.copy_(x_host, non_blocking=True)
            graph.replay()
            y_host.copy_(graph.y, non_blocking=True)
            if i >= args.warmup:
                e2e_ev[i - args.warmup][1].record(stream)
        torch.cuda.synchronize()
        e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev) / args.steps
    kernels = graph.kernels_per_replay
    del graph
    vals = [ms, stages.get("expert_ffn", 0.0)] + ([e2e_ms] if e2e else [])
    vals = max_over_ranks(vals, dist, dev)
    ms, ffn_ms = vals[0], vals[1]
    if e2e:
        e2e_ms = vals[2]
    if "expert_ffn" in stages:
        stages["expert_ffn"] = ffn_ms
    return {"ms": ms, "e2e_ms": e2e_ms, "acc": acc, "rstats": rstats, "stages": stages,
            "clocks": clk, "kernels": kernels, "step_ms": step_ms}


FP4_EXPERT_BYTES = 3 * 2816 * 704 // 2 + 3 * 2816 * 704 // 16 + 3 * 4   # codes, scales, ts


def time_nvfp4(moe, cfg, args, g, x_cpu, dev, stream, flush_l2, dist) -> dict:
    """The layer with NVFP4 experts (weights quantised by the library from the bf16 set) on
    cfg's batch: graph replays of moe_forward_nvfp4, L2 flushed before every step, stage
    events from a second graph; device times are the max over ranks."""
    from expert_routed_ffn_softmax_b200 import _abi
    wq = _abi.nvfp4_quantize_layer(g["w_gate"], g["w_up"], g["w_down"])
    x = x_cpu.to(dev)
    y0, aux = _abi.forward_nvfp4(x, g["w_router"], wq, cfg.k, bias=g["bias"], aux=True)
    if moe.sync_status() != 0:
        raise SystemExit("device status not OK after the first NVFP4 forward")
    counts = aux["expert_counts"].cpu().numpy()
    active = int((counts > 0).sum())
    E, I, H = cfg.E, cfg.I, cfg.H
    flags = 0
    nbytes = _abi.load().moe_nvfp4_workspace_size(cfg.T, H, E, I, cfg.k, flags)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    ws_p = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    y = torch.empty_like(y0)

    def capture(profile, buf):
        _abi.forward_nvfp4(x, g["w_router"], wq, cfg.k, bias=g["bias"], out=y, profile=profile,
                           workspace_buf=buf)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            _abi.forward_nvfp4(x, g["w_router"], wq, cfg.k, bias=g["bias"], out=y,
                               profile=profile, workspace_buf=buf)
        return gr, _abi.last_kernel_count()

    graph, kernels = capture(False, ws)
    for _ in range(args.warmup):
        flush_l2()
        graph.replay()
    torch.cuda.synchronize()
    if not torch.equal(y, y0):
        raise SystemExit("NVFP4 graph replay differs from the direct call")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2()
        ev[i][0].record(stream)
        graph.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    pgraph, _ = capture(True, ws_p)
    acc: dict[str, list[float]] = {}
    for _ in range(max(3, min(args.steps, 20))):
        flush_l2()
        pgraph.replay()
        for k2, v in _abi.last_stage_times().items():
            acc.setdefault(k2, []).append(v)
    stages = {k2: sum(v) / len(v) for k2, v in acc.items()}
    del pgraph, graph
    ms, ffn_ms = max_over_ranks([ms, stages.get("expert_ffn", 0.0)], dist, dev)
    return {"ms": ms, "ffn_ms": ffn_ms, "stages": stages, "active": active, "clocks": clk,
            "kernels": kernels}


def nvfp4_entry(cfg, m: dict, world: int, pk: dict) -> dict:
    ffn_bytes = m["active"] * FP4_EXPERT_BYTES
    step_bytes = ffn_bytes + cfg.H * cfg.E * 2 + 2 * cfg.T * cfg.H * 2
    ach = ffn_bytes / (m["ffn_ms"] * 1e-3) / 1e9 if m["ffn_ms"] > 0 else None
    return {
        "workload": f"{cfg.name}: T={cfg.T} H={cfg.H} E={cfg.E} k={cfg.k} I={cfg.I}, expert "
                    "weights and activations NVFP4 (E2M1, E4M3 scale per 16, fp32 per tensor), "
                    "weights quantised from the bf16 set",
        "value": job_throughput(world, cfg.T, m["ms"]), "unit": UNIT, "ms_per_step": m["ms"],
        "expert_ffn": {"kernels": "nvfp4_rows_sorted_kernel + nvfp4_ffn_kernel (tcgen05 kind::mxf4nvf4)", "ms": m["ffn_ms"],
                       "algorithmic_bytes": ffn_bytes, "achieved_gbs": ach,
                       "frac_of_hbm": None if ach is None else ach / pk["hbm_gbs"],
                       "traffic": ncu_traffic("nvfp4_ffn_kernel", f"{cfg.name}_nvfp4")},
        "step_hbm_frac": step_bytes / (m["ms"] * 1e-3) / (pk["hbm_gbs"] * 1e9),
        "active_experts": m["active"], "stages_ms": m["stages"], "clocks": m["clocks"],
        "gpu_launches": m["kernels"] * m["_steps"],
        "note": "reduced-precision variant of the layer (the checkpoint's format), reported "
                "beside the bf16 line, not in place of it",
    }


def tensor_bound_entry(cfg, m: dict, world: int, pk: dict) -> dict:
    """Summary of one large-batch config: tokens/s, the expert FFN's tensor throughput
    against the measured burst and sustained bf16 peaks, and the whole step's."""
    acc = m["acc"]
    kf = acc["gemm1_flops"] + acc["gemm2_flops"]
    ffn_ms = m["stages"].get("expert_ffn", 0.0)
    ffn_tf = kf / (ffn_ms * 1e-3) / 1e12 if ffn_ms > 0 else None
    step_tf = acc["step_flops"] / (m["ms"] * 1e-3) / 1e12
    return {
        "workload": f"{cfg.name}: T={cfg.T} H={cfg.H} E={cfg.E} k={cfg.k} I={cfg.I}"
                    + (" (router bias b_e = 2 ln(1/(e+1)))" if cfg.skew_bias else ""),
        "value": job_throughput(world, cfg.T, m["ms"]), "unit": UNIT,
        "ms_per_step": m["ms"],
        "expert_ffn": {"kernel": ffn_kernel_name(cfg.T, m["_tiles"]), "ms": ffn_ms,
                       "achieved_tflops": ffn_tf,
                       "frac_of_burst": None if ffn_tf is None else ffn_tf / pk["bf16_tflops"],
                       "frac_of_sustained": None if ffn_tf is None
                       else ffn_tf / pk["bf16_tflops_sustained"],
                       "algorithmic_flops": kf},
        "step_tensor_frac": step_tf * 1e12 / (pk["bf16_tflops"] * 1e12),
        "active_experts": acc["active_experts"],
        "stages_ms": m["stages"],
        "router_stats": m["rstats"],
        "clocks": m["clocks"],
        "gpu_launches": m["kernels"] * m["_steps"],
    }



# ----------------------------------------------------------------------------- arms
def run_reference(args, cfg) -> None:
    import oracle
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    d = wl.make_inputs(cfg)
    T_s = min(cfg.T, args.ref_tokens)
    x = d["x"][:T_s].contiguous()

    def step():
        oracle.forward(x, d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k, bias=d["bias"])

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    v = T_s / sec
    sample = f"{T_s} of the {cfg.T} tokens of the {cfg.name} batch per step, fp64, all experts selected"
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{cfg.name}: T={cfg.T} H={cfg.H} E={cfg.E} k={cfg.k} I={cfg.I}",
                   "global_batch": cfg.T, "parallelism": "cpu"},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": oracle.get_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(cfg, d, x_all, budget_s: float) -> dict:
    import oracle
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    T_s = min(cfg.T, 64)
    x = x_all[:T_s].contiguous()
    n, t_total = 0, 0.0
    while t_total < budget_s or n == 0:
        t0 = time.perf_counter()
        oracle.forward(x, d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k, bias=d["bias"])
        t_total += time.perf_counter() - t0
        n += 1
    return {"value": n * T_s / t_total, "unit": UNIT, "cores": oracle.get_threads(),
            "kind": "oracle",
            "sample": f"{n} x forward of the first {T_s} tokens of the {cfg.name} batch "
                      f"({t_total:.1f} s of fp64 CPU work)"}


def run_native(args, cfg) -> None:
    import expert_routed_ffn_softmax_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    d = wl.make_weights(cfg)
    x_cpu = wl.make_x(cfg, seed=rank)
    g = {k: (v.to(dev) if v is not None else None) for k, v in d.items()}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        # write more than L2 holds, then read more than it holds: L2 ends cold and clean
        flush.zero_()
        flush_rd.max()

    m = time_layer(moe, cfg, args, g, x_cpu, dev, stream, flush_l2, dist, e2e=True)
    ms, e2e_ms = m["ms"], m["e2e_ms"]
    acc, rstats, stages, clk, graph_kernels, step_ms = (m["acc"], m["rstats"], m["stages"],
                                                       m["clocks"], m["kernels"], m["step_ms"])
    # the layer with NVFP4 experts at decode, same timing rules, reported beside the line
    fp4 = None
    if not args.no_nvfp4 and cfg.T <= 16 and (cfg.H, cfg.E, cfg.I) == (2816, 128, 704):
        fp4 = time_nvfp4(moe, cfg, args, g, x_cpu, dev, stream, flush_l2, dist)
    # the tensor-bound configs (large batches), same timing rules, reported beside the line
    tensor_bound = []
    if not args.no_tensor_bound:
        for name in TENSOR_BOUND_CONFIGS:
            c2 = wl.CONFIGS[name]
            g2 = dict(g, bias=(wl.skew_bias(c2.E).to(dev) if c2.skew_bias else None))
            m2 = time_layer(moe, c2, args, g2, wl.make_x(c2, seed=rank), dev, stream, flush_l2,
                            dist, e2e=False)
            tensor_bound.append((c2, m2))
    if rank == 0:
        pk = peaks()
        # the dominant kernel: the expert FFN (GEMM-1 + GEGLU and GEMM-2; one launch unless
        # the tiles ask for two)
        dom_ms = stages.get("expert_ffn", 0.0)
        kb = acc["gemm1_bytes"] + acc["gemm2_bytes"]
        kf = acc["gemm1_flops"] + acc["gemm2_flops"]
        ridge = pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)
        kname = ffn_kernel_name(cfg.T, args.tiles)
        traffic = ncu_traffic(kname, cfg.name)
        if kf / kb < ridge:
            achieved = kb / (dom_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                    "kernel": kname, "peak_source": pk["source"] + " hbm_gbs"}
        else:
            achieved = kf / (dom_ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"], "traffic": traffic,
                    "kernel": kname, "peak_source": pk["source"] + " bf16_tflops (burst)",
                    "frac_of_sustained": achieved / pk["bf16_tflops_sustained"]}
        step_s = ms * 1e-3
        line = {
            "metric": METRIC,
            "value": job_throughput(world, cfg.T, ms),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"{cfg.name}: T={cfg.T} H={cfg.H} E={cfg.E} k={cfg.k} "
                                   f"I={cfg.I} (routed MoE FFN layer, Gemma-4-26B-A4B shape)",
                       "global_batch": world * cfg.T, "tokens_per_gpu": cfg.T,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "flushed before every step (256 MB write then 256 MB read, untimed)"},
            "roofline": roof,
            "step_roofline": {
                "hbm_frac": acc["step_bytes"] / step_s / (pk["hbm_gbs"] * 1e9),
                "tensor_frac": acc["step_flops"] / step_s / (pk["bf16_tflops"] * 1e12),
                "algorithmic_bytes": acc["step_bytes"], "algorithmic_flops": acc["step_flops"],
                "active_experts": acc["active_experts"]},
            "stages_ms": stages,
            "router_stats": rstats,
            "e2e": {"value": job_throughput(world, cfg.T, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": cfg.T * cfg.H * 2,
                    "d2h_bytes_per_step": cfg.T * cfg.H * 2},
            "gpu_launches": graph_kernels * args.steps,
            "clocks": clk,
            "step_ms_p10_p50_p90": [float(np.percentile(step_ms, q)) for q in (10, 50, 90)],
        }
        if fp4 is not None:
            fp4["_steps"] = args.steps
            line["nvfp4_decode"] = nvfp4_entry(cfg, fp4, world, pk)
        if tensor_bound:
            line["tensor_bound"] = []
            for c2, m2 in tensor_bound:
                m2["_steps"] = args.steps
                m2["_tiles"] = args.tiles
                line["tensor_bound"].append(tensor_bound_entry(c2, m2, world, pk))
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(cfg, d, x_cpu, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_dense(args, cfg) -> None:
    """--dense: the dense GEGLU MLP beside the MoE (intermediate workloads.DENSE_I) on the
    config's x, one GPU; same timing rules as the layer (clean L2 before every step)."""
    import expert_routed_ffn_softmax_b200 as moe
    if int(os.environ.get("WORLD_SIZE", "1")) != 1 or args.gpus != 1:
        raise SystemExit("--dense runs on one GPU")
    dev = torch.device("cuda", 0)
    I = wl.DENSE_I if cfg.H == 2816 else 2 * cfg.I
    w = wl.make_dense_weights(cfg.H, I)
    g = {k: v.to(dev) for k, v in w.items()}
    x_cpu = wl.make_x(cfg)
    x = x_cpu.to(dev)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        flush.zero_()
        flush_rd.max()

    def step():
        moe.dense_ffn(x, g["w_gate"], g["w_up"], g["w_down"], out=y)

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    if moe.sync_status() != 0:
        raise SystemExit("device status not OK after the warm-up")
    launches = moe.last_kernel_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    clocks.start()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    # end to end: pinned x in, y out, every step
    x_host = x_cpu.pin_memory()
    y_host = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    for i in range(args.warmup + args.steps):
        flush_l2()
        if i >= args.warmup:
            e2e_ev[i - args.warmup][0].record(stream)
        x.copy_(x_host, non_blocking=True)
        step()
        y_host.copy_(y, non_blocking=True)
        if i >= args.warmup:
            e2e_ev[i - args.warmup][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev) / args.steps
    pk = peaks()
    wbytes = 3 * cfg.H * I * 2
    kb = wbytes + 2 * cfg.T * cfg.H * 2
    kf = cfg.T * (2 * cfg.H * 2 * I + 2 * I * cfg.H)
    ridge = pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)
    rname = next(r for r in (8, 16, 32, 64, 128) if cfg.T <= r or r == 128)
    if kf / kb < ridge:
        a = kb / (ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": a, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": a / pk["hbm_gbs"], "traffic": None,
                "kernel": f"expert_ffn_dynamic_kernel<{rname}> (one expert, all rows)",
                "peak_source": pk["source"] + " hbm_gbs"}
    else:
        a = kf / (ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": a, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": a / pk["bf16_tflops"], "traffic": None,
                "kernel": f"expert_ffn_dynamic_kernel<{rname}> (one expert, all rows)",
                "peak_source": pk["source"] + " bf16_tflops (burst)",
                "frac_of_sustained": a / pk["bf16_tflops_sustained"]}
    line = {
        "metric": "dense GEGLU MLP tokens/s (the MLP beside the MoE)", "value": cfg.T / (ms * 1e-3),
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"dense MLP: T={cfg.T} H={cfg.H} I={I} (x of the {cfg.name} config)",
                   "global_batch": cfg.T, "parallelism": "single GPU",
                   "l2": "flushed before every step (256 MB write then 256 MB read, untimed)"},
        "roofline": roof, "gpu_launches": launches * args.steps, "clocks": clk,
        "e2e": {"value": cfg.T / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": cfg.T * cfg.H * 2, "d2h_bytes_per_step": cfg.T * cfg.H * 2},
    }
    if not args.no_cpu_baseline:
        import oracle
        cores = len(os.sched_getaffinity(0))
        oracle.set_threads(cores)
        rows = list(range(min(cfg.T, 8)))
        n, t_total = 0, 0.0
        while t_total < args.cpu_seconds or n == 0:
            t0 = time.perf_counter()
            oracle.dense_ffn(x_cpu, w["w_gate"], w["w_up"], w["w_down"], rows=rows)
            t_total += time.perf_counter() - t0
            n += 1
        line["cpu_baseline"] = {"value": n * len(rows) / t_total, "unit": UNIT,
                                "cores": oracle.get_threads(), "kind": "oracle",
                                "sample": f"{n} x the dense MLP of the first {len(rows)} tokens "
                                          f"({t_total:.1f} s of fp64 CPU work)"}
    print(json.dumps(line), flush=True)


def run_ep(args, cfg) -> None:
    """--ep: the expert-parallel layer (expert_routed_ffn_softmax_b200.ep) with E / N experts on
    each of N ranks (NCCL), every rank bringing its own batch of cfg's shape; the AllToAll
    form above 64 tokens per rank, the AllGather (decode) form at or below.  Same timing
    rules as the default run (untimed L2 flush before every step, CUDA events on the launching
    stream, max over ranks)."""
    import datetime
    import torch.distributed as dist
    from expert_routed_ffn_softmax_b200 import ep
    import expert_routed_ffn_softmax_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29731")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        w = wl.make_weights(cfg)
        lo, hi = ep.expert_range(cfg.E, world, rank)
        g = {"w_router": w["w_router"].to(dev),
             "w_gate": w["w_gate"][lo:hi].contiguous().to(dev),
             "w_up": w["w_up"][lo:hi].contiguous().to(dev),
             "w_down": w["w_down"][lo:hi].contiguous().to(dev)}
        bias = w["bias"].to(dev) if w["bias"] is not None else None
        layer = ep.ExpertParallelMoE(g["w_router"], g["w_gate"], g["w_up"], g["w_down"], cfg.E,
                                     cfg.k, ep.TorchComm(), bias=bias)
        mode = "allgather" if cfg.T <= 64 else "alltoall"
        x = wl.make_x(cfg, seed=rank).to(dev)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        flush_rd = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
        stream = torch.cuda.current_stream()
        for _ in range(args.warmup):
            flush.zero_()
            flush_rd.max()
            layer.forward(x, mode)
        torch.cuda.synchronize()
        if moe.sync_status() != 0:
            raise SystemExit("device status not OK after the warm-up")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        clocks = ClockSampler(dev)
        clocks.start()
        dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()
            flush_rd.max()
            ev[i][0].record(stream)
            layer.forward(x, mode)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        clk = clocks.stop()
        ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
        ms = max_over_ranks([ms], dist, dev)[0]
        if rank == 0:
            line = {
                "metric": METRIC, "value": job_throughput(world, cfg.T, ms), "unit": UNIT,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": {"workload": f"{cfg.name}: T={cfg.T} per rank, H={cfg.H} E={cfg.E} "
                                       f"k={cfg.k} I={cfg.I}, experts split over the ranks",
                           "global_batch": world * cfg.T, "tokens_per_gpu": cfg.T,
                           "parallelism": f"ep{world} ({mode})",
                           "l2": "flushed before every step (256 MB write then 256 MB read, untimed)"},
                "clocks": clk,
                "note": "host-synchronising split-size exchange per step (counts to the host)",
            }
            print(json.dumps(line), flush=True)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="decode", choices=sorted(wl.CONFIGS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tiles", default="auto",
                    choices=["auto", "decode", "prefill", "pairs", "single", "fused", "unfused"],
                    help="expert-GEMM tile family (default: the library's choice)")
    ap.add_argument("--no-nvfp4", action="store_true",
                    help="skip the NVFP4-expert variant reported beside the decode line")
    ap.add_argument("--no-tensor-bound", action="store_true",
                    help="skip the large-batch (tensor-bound) configs reported beside the line")
    ap.add_argument("--ep", action="store_true",
                    help="time the expert-parallel layer (experts split over the ranks, NCCL)")
    ap.add_argument("--dense", action="store_true",
                    help="time the dense GEGLU MLP beside the MoE instead of the MoE layer")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)     # at least 3 untimed warm-up steps
    cfg = wl.CONFIGS[args.config]
    if args.dense:
        run_dense(args, cfg)
    elif args.ep and args.impl != "reference":
        run_ep(args, cfg)
    elif args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_native(args, cfg)


if __name__ == "__main__":
    main()
