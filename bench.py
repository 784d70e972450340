#!/usr/bin/env python
"""Benchmark of the MoE-layer forward pass on B200 (one JSON line on rank 0).

Metric: MoE-layer tokens/s at 1 B200; grouped-GEMM % bf16 peak; route+permute % HBM.

One step = one whole forward of the layer (route -> permute -> grouped expert
FFN -> combine) over one batch of seeded synthetic tokens already resident in
HBM.  The default workload is the Mixtral-shaped layer (x[1024,4096],
expert_weight[8,4096,14336], SwiGLU experts, top-2, no capacity limit): the
configuration the grouped-GEMM and HBM targets are stated on.

  python bench.py [--gpus N --steps K --warmup W] [--config NAME|1..5] [--impl reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own replica on its
own tokens (token data-parallel: the layer needs no collective); the reported
value is the tokens of all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from routing_grouped_expert_moe_b200 import synth  # noqa: E402

METRIC = "MoE-layer tokens/s at 1 B200; grouped-GEMM % bf16 peak; route+permute % HBM"
DEFAULT_CONFIG = "mixtral_e8"
L2_FLUSH_BYTES = 256 << 20
SPEC_HBM_GBS = 8000.0       # ~8 TB/s (spec wording of the targets)
SPEC_BF16_TFLOPS = 2250.0   # dense bf16
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per launch of the grouped GEMM kernels from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the kernel
# source they were taken on; None until captured.
NCU_TRAFFIC = {"source_sha": "82c78a976bf07d0f", "workload": "mixtral_e8",
               "bytes_per_forward": 2.9972e9}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=["layer", "expert_matmul", "route_stats", "ep", "ep_one_rank"],
                    default="layer",
                    help="layer: the MoE layer (default, the headline); expert_matmul: the k=1\n"
                         "up-projection op on x[1024,4096] x W[8,4096,14336]; route_stats: the\n"
                         "router with its load statistics on the e32_long router shape;\n"
                         "ep: the expert-parallel forward, one rank per GPU (torchrun), each\n"
                         "rank owning E/N experts and its own tokens of the --config workload\n"
                         "(on one GPU also timed against the fused forward); ep_one_rank: the\n"
                         "same as ep on one GPU")
    ap.add_argument("--hbm-copy-sweep", action="store_true",
                    help="time plain device copies at the memory stages' sizes and exit")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU seconds for the oracle baseline sample")
    ap.add_argument("--tokens", type=int, default=None,
                    help="token count T in place of the workload's (a sweep over batch x\n"
                         "sequence length; the workload is then named <name>_T<T>)")
    return ap.parse_args(argv)


def resolve_config(name: str, tokens=None) -> synth.MoEConfig:
    if name.isdigit():
        name = synth.NUMBERED[int(name) - 1]
    cfg = synth.CONFIGS[name]
    if tokens is not None:
        if tokens < 1:
            raise ValueError("--tokens must be at least 1")
        from dataclasses import replace
        cfg = replace(cfg, T=int(tokens), name=f"{cfg.name}_T{int(tokens)}",
                      description=f"{cfg.description}; T set to {int(tokens)} tokens")
    return cfg


def workload_desc(cfg: synth.MoEConfig) -> dict:
    return {"workload": cfg.name, "description": cfg.description, "T": cfg.T, "H": cfg.H,
            "F": cfg.F, "E": cfg.E, "top_k": cfg.top_k, "act": cfg.act,
            "capacity_factor": cfg.capacity_factor, "storage": cfg.dtype, "seed": cfg.seed}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def gemm_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("gemm_tokn.cu", "gemm_tcgen05.cu", "gemm_tcgen05_pair.cu", "gemm_common.cuh",
              "common.cuh"):
        with open(os.path.join(ROOT, "routing_grouped_expert_moe_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------- work model

def algorithmic_work(cfg: synth.MoEConfig, counts) -> dict:
    """Algorithmic FLOPs / bytes of one forward, from the pre-drop expert counts."""
    s = cfg.elem_bytes
    T, H, F, E, k = cfg.T, cfg.H, cfg.F, cfg.E, cfg.top_k
    if cfg.capacity_factor > 0:
        import math
        cap = math.ceil(float(torch.tensor(cfg.capacity_factor, dtype=torch.float32)) * T * k / E)
        kept = [min(c, cap) for c in counts]
    else:
        kept = list(counts)
    R = sum(kept)
    active = sum(1 for c in kept if c > 0)
    mats = 3 if cfg.act == "swiglu" else 2
    gemm_flops = 2.0 * R * H * F * mats
    weight_bytes = active * H * F * mats * s
    gemm1_flops = 2.0 * R * H * F * (mats - 1)
    gemm2_flops = 2.0 * R * H * F
    # GEMM bytes: weights once + A rows in + h out (GEMM-1) + h in + y out (GEMM-2)
    gemm1_bytes = active * H * F * (mats - 1) * s + R * H * s + R * F * s
    gemm2_bytes = active * H * F * s + R * F * s + R * H * s
    route_bytes = T * H * s + H * E * s + T * k * 8 + (E * 4 if cfg.bias != "none" else 0)
    scan_bytes = 2 * (E + 1) * 4
    # ids in, row_token and row_map out, x read once, x_perm written (a token's
    # second kept row re-reads the same x row, which the count does not repeat)
    scatter_bytes = T * k * 4 + R * 4 + T * k * 4 + T * H * s + R * H * s
    combine_bytes = R * H * s + T * k * 8 + T * H * s
    return {"R": R, "active_experts": active, "gemm_flops": gemm_flops, "gemm1_flops": gemm1_flops,
            "gemm2_flops": gemm2_flops, "weight_bytes": weight_bytes, "gemm1_bytes": gemm1_bytes,
            "gemm2_bytes": gemm2_bytes, "route_bytes": route_bytes, "scan_bytes": scan_bytes,
            "scatter_bytes": scatter_bytes, "combine_bytes": combine_bytes}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # pragma: no cover
            self.error = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                mhz = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
                rs = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((time.time(), mhz, rs))
            except Exception:
                pass
            time.sleep(self._period)

    def start(self):
        if self._ok:
            self._t.start()
        return self

    def stop(self, t0=None, t1=None):
        self._stop.set()
        if self._ok:
            self._t.join(timeout=2)
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "source": "unavailable"}
        sel = [s for s in self.samples if (t0 is None or s[0] >= t0) and (t1 is None or s[0] <= t1)]
        if not sel:
            sel = self.samples
        mhz = [s[1] for s in sel]
        bits = 0
        for s in sel:
            bits |= int(s[2])
        reasons = [v for k, v in self.REASONS.items() if bits & k and v != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sel), "source": "nvml"}


# ----------------------------------------------------------------------------- oracle timing

def oracle_sample(cfg: synth.MoEConfig, d: dict, n_tokens: int) -> float:
    """Seconds the C++ CPU oracle (plain float64 loops, OpenMP over rows) takes for
    the whole layer on the first n_tokens tokens."""
    from oracle import moe_oracle_cpp as O
    f = lambda t: None if t is None else t.float().numpy()  # noqa: E731
    x = f(d["x"][:n_tokens])
    t0 = time.perf_counter()
    O.moe_forward(x, d["_wg"], d["_b"], d["_w1"], d["_w3"], d["_w2"], cfg.top_k,
                  cfg.capacity_factor, cfg.act, cfg.dtype)
    return time.perf_counter() - t0


def _oracle_inputs(cfg, d):
    f = lambda t: None if t is None else t.float().numpy()  # noqa: E731
    d["_wg"], d["_b"] = f(d["w_gate"]), f(d["gate_bias"])
    d["_w1"], d["_w3"], d["_w2"] = f(d["w1"]), f(d["w3"]), f(d["w2"])


def oracle_threads() -> int:
    """Threads the C++ oracle's OpenMP loops run on."""
    from oracle import moe_oracle_cpp as O
    return O.num_threads()


def calibrate_tokens(cfg, d, target_s: float) -> tuple[int, float]:
    """A token count whose oracle run takes about target_s (capped at the workload's T)."""
    n = min(cfg.T, 64)
    dt = oracle_sample(cfg, d, n)
    while dt < 0.8 * target_s and n < cfg.T:
        n = min(cfg.T, max(n * 2, int(n * target_s / max(dt, 1e-3))))
        dt = oracle_sample(cfg, d, n)
    return n, dt


def cpu_baseline(cfg, d, target_s: float) -> dict:
    _oracle_inputs(cfg, d)
    n, dt = calibrate_tokens(cfg, d, target_s)
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"whole layer (C++ float64 oracle, plain loops, OpenMP) on the first {n} "
                      f"of {cfg.T} tokens of {cfg.name}, {dt:.1f} s"}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    d = synth.make_inputs(cfg)
    _oracle_inputs(cfg, d)
    # each step: the oracle on a bounded sample sized so K+W steps take ~2 minutes
    per_step = max(0.5, 120.0 / max(1, args.steps + args.warmup))
    n, _ = calibrate_tokens(cfg, d, per_step)
    for _ in range(args.warmup):
        oracle_sample(cfg, d, n)
    times = [oracle_sample(cfg, d, n) for _ in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**workload_desc(cfg), "sample_tokens_per_step": n},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle_threads(),
                             "kind": "oracle",
                             "sample": f"{n} of {cfg.T} tokens per step, whole layer, C++ "
                                       f"float64 oracle (plain loops, OpenMP)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- ranks

def rank_inputs(cfg: synth.MoEConfig, rank: int) -> dict:
    """Inputs of one rank: the weights are the same on every rank (same seed, as a
    replicated layer has), the tokens are the rank's own (a seed offset per rank)."""
    d = synth.make_inputs(cfg)
    if rank > 0:
        d["x"] = synth.normal(cfg.seed + 7919 * rank, synth.STREAM_X, (cfg.T, cfg.H), cfg.x_std,
                              cfg.torch_dtype)
    return d


def max_over_ranks(x: float, dist, device) -> float:
    """The largest of every rank's x (the job is as slow as its slowest rank)."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: the tokens all ranks processed over the slowest rank's time."""
    return tokens_per_rank * world * steps / (total_ms / 1000.0)


# ----------------------------------------------------------------------------- main arm

def hbm_copy_sweep() -> int:
    """What a plain device copy achieves at the sizes the memory-bound stages
    move (L2 cold before each copy), one JSON line per size."""
    dev = torch.device("cuda", 0)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for mb in (4, 8, 16, 33, 67, 134, 268, 1024):
        n = mb * (1 << 20) // 2
        a = torch.empty(n, dtype=torch.bfloat16, device=dev)
        b = torch.empty_like(a)
        ts = []
        for i in range(13):
            flush.zero_()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            b.copy_(a)
            s1.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(s0.elapsed_time(s1) * 1000.0)
        us = statistics.median(ts)
        print(json.dumps({"copy_mb_read": mb, "us": us, "gbs_read_plus_write": 2 * n * 2 / us / 1e3}),
              flush=True)
        del a, b
    return 0


def copy_us(nbytes: int, flush, dev, reps: int = 10) -> float:
    """Median CUDA-event microseconds of one plain device copy that moves nbytes in
    all (nbytes/2 read, nbytes/2 written), L2 flushed before each copy."""
    n = max(1, nbytes // 4)
    a = torch.empty(n, dtype=torch.bfloat16, device=dev)
    b = torch.empty_like(a)
    ts = []
    for i in range(reps + 3):
        flush.zero_()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        b.copy_(a)
        s1.record()
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(s0.elapsed_time(s1) * 1000.0)
    return statistics.median(ts)


def kernels_per_call(fn) -> int | None:
    """Kernel launches one call of fn makes, counted as the kernel nodes of a CUDA
    graph captured from it (None when the graph cannot be inspected)."""
    try:
        from cuda.bindings import runtime as rt
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, stream=s):
            fn()
        graph = rt.cudaGraph_t(init_value=int(g.raw_cuda_graph()))
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        count = 0
        for node in nodes[:n]:
            err, typ = rt.cudaGraphNodeGetType(node)
            if typ == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                count += 1
        del g
        torch.cuda.synchronize()
        return count
    except Exception as e:  # pragma: no cover - inspection is best effort
        print(f"kernels_per_call: {e!r}", file=sys.stderr)
        return None


def _time_steps(fn, steps: int, warmup: int, flush) -> list:
    """CUDA-event milliseconds of each of `steps` calls (L2 flushed before each)."""
    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush.zero_()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        fn()
        s1.record()
        ms.append((s0, s1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ms]


def _run_ep(args, B, flush, steps, warmup) -> int:
    """The expert-parallel forward (expert_parallel.ep_forward), one rank per GPU:
    rank r of N owns experts [r*E/N, (r+1)*E/N) and routes its own tokens; every
    step is timed with CUDA events between barriers, and the job's time per step
    is the slowest rank's.  On one rank every exchange is a local copy, and the
    fused forward is timed beside it for the cost of the exchanges' host reads,
    the regroup and the separate launches."""
    import torch.distributed as tdist
    from routing_grouped_expert_moe_b200 import expert_parallel as EP
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dev = torch.device("cuda", torch.cuda.current_device())
    if world > 1:
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
    else:
        tdist.init_process_group("nccl", store=tdist.HashStore(), rank=0, world_size=1)
    try:
        cfg = resolve_config(args.config, args.tokens)
        if cfg.E % world:
            if rank == 0:
                print(json.dumps({"metric": "expert-parallel layer tokens/s", "unavailable":
                                  f"{cfg.E} experts do not split over {world} ranks"}), flush=True)
            return 0
        el = cfg.E // world
        d = rank_inputs(cfg, rank)
        sl = slice(rank * el, (rank + 1) * el)
        local = lambda w: None if w is None else w[sl].contiguous().to(dev)  # noqa: E731
        x, wg = d["x"].to(dev), d["w_gate"].to(dev)
        b = None if d["gate_bias"] is None else d["gate_bias"].to(dev)
        w1, w3, w2 = local(d["w1"]), local(d["w3"]), local(d["w2"])
        ep_args = (x, wg, b, w1, w3, w2, cfg.top_k, cfg.capacity_factor, cfg.act, cfg.E)

        def timed(fn):
            for _ in range(warmup):
                flush.zero_()
                fn()
            torch.cuda.synchronize()
            tdist.barrier()
            ms = []
            for _ in range(steps):
                flush.zero_()
                s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s0.record()
                fn()
                s1.record()
                ms.append((s0, s1))
            torch.cuda.synchronize()
            tdist.barrier()
            mean_ms = statistics.mean(a.elapsed_time(z) for a, z in ms)
            return max_over_ranks(mean_ms, tdist, dev)

        e_ms = timed(lambda: EP.ep_forward(*ep_args))
        o_ms = timed(lambda: EP.ep_forward(*ep_args, overlap=True))
        f_ms = None
        if world == 1:
            ws = B.alloc_workspace(B.workspace_bytes(cfg.T, cfg.H, cfg.F, cfg.E, cfg.top_k,
                                                     cfg.act, cfg.torch_dtype), dev)
            out = torch.empty(cfg.T, cfg.H, dtype=cfg.torch_dtype, device=dev)
            f_ms = timed(lambda: B.forward(x, wg, b, w1, w3, w2, cfg.top_k, cfg.capacity_factor,
                                           cfg.act, out=out, ws=ws))
    finally:
        tdist.destroy_process_group()
    if rank != 0:
        return 0
    line = {"metric": "expert-parallel layer tokens/s", "value": cfg.T * world / (e_ms / 1e3),
            "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": warmup,
            "ms_per_step": e_ms, "higher_is_better": True, "scaling": "weak", "dtype": cfg.dtype,
            "data": "synthetic (seeded Philox normal inputs, random-init weights)",
            "config": {**workload_desc(cfg), "l2": "flushed before every step",
                       "parallelism": (f"ep{world} (rank r owns experts r*E/{world} .. "
                                       f"(r+1)*E/{world}-1, every rank its own tokens)"
                                       if world > 1 else
                                       "ep1 (one NCCL rank: every exchange is a local copy)")},
            "ep_ms": e_ms, "ep_overlap_ms": o_ms, "fused_forward_ms": f_ms,
            "note": "CUDA events around each call on the current stream, slowest rank; the "
                    "expert-parallel path reads its split sizes on the host once per forward"}
    print(json.dumps(line), flush=True)
    return 0


def run_op(args) -> int:
    """One JSON line for a single-op row (not the layer headline)."""
    from routing_grouped_expert_moe_b200 import binding as B
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peaks, peak_src = load_peaks()
    steps, warmup = min(args.steps, 100), max(args.warmup, 3)
    if args.op in ("ep", "ep_one_rank"):
        return _run_ep(args, B, flush, steps, warmup)
    if args.op == "expert_matmul":
        T, H, I, E, seed = 1024, 4096, 14336, 8, 5001
        x = synth.normal(seed, synth.STREAM_X, (T, H), 1.0, torch.bfloat16).to(dev)
        w = synth.normal(seed, synth.STREAM_W1, (E, H, I), H ** -0.5, torch.bfloat16).to(dev)
        ids = synth.random_expert_ids(seed, T, E, 1)[:, 0].contiguous().to(dev)
        out = torch.empty(T, I, dtype=torch.bfloat16, device=dev)
        ws = B.alloc_workspace(B._lib.moe_expert_matmul_workspace_bytes(T, H, I, E, B.BF16), dev)
        ms = _time_steps(lambda: B.expert_matmul(x, w, ids, out=out, ws=ws), steps, warmup, flush)
        if B.device_status(ws) != B.OK:
            raise RuntimeError("expert_matmul device status")
        t_ms = statistics.mean(ms)
        flops = 2.0 * T * H * I
        tflops = flops / (t_ms / 1e3) / 1e12
        tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        # weights of the experts that received tokens, read once, plus x in and out
        used = int(torch.unique(ids).numel())
        nbytes = used * H * I * 2 + T * H * 2 + T * I * 2
        gbs = nbytes / (t_ms / 1e3) / 1e9
        # ~T/E rows per expert: below the ridge point the op is bound by the weight stream
        hbm_bound = flops / nbytes < tc * 1e12 / (hbm * 1e9)
        line = {"metric": "expert_matmul tokens/s (k=1 up-projection)", "value": T / (t_ms / 1e3),
                "unit": "tokens/s", "n_gpus": 1, "steps": steps, "warmup": warmup,
                "ms_per_step": t_ms, "higher_is_better": True, "dtype": "bf16",
                "data": "synthetic (seeded normal x and weights, uniform expert ids)",
                "config": {"workload": "expert_matmul_p4", "T": T, "H": H, "I": I, "E": E,
                           "l2": "flushed before every step"},
                "roofline": ({"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                              "frac": gbs / hbm, "peak_source": peak_src, "algorithmic_bytes": nbytes,
                              "tflops": tflops, "frac_of_bf16_peak": tflops / tc}
                             if hbm_bound else
                             {"bound": "tensor", "achieved": tflops, "peak": tc, "unit": "TFLOP/s",
                              "frac": tflops / tc, "peak_source": f"{peak_src} burst bf16"}),
                "note": "whole op (permute + grouped GEMM + unpermute) time"}
    else:
        cfg = synth.CONFIGS["e32_long"]
        d = synth.make_inputs(cfg, with_weights=False)
        x, wg = d["x"].to(dev), d["w_gate"].to(dev)
        b = None if d["gate_bias"] is None else d["gate_bias"].to(dev)
        ws = B.alloc_workspace(B._lib.moe_route_stats_workspace_bytes(cfg.T, cfg.E), dev)
        ms = _time_steps(lambda: B.route_stats(x, wg, b, cfg.top_k, ws=ws), steps, warmup, flush)
        if B.device_status(ws) != B.OK:
            raise RuntimeError("route_stats device status")
        t_ms = statistics.mean(ms)
        T, H, E, k = cfg.T, cfg.H, cfg.E, cfg.top_k
        nbytes = T * H * 2 + H * E * 2 + T * k * 8 + 2 * T * E * 4   # x, W_gate, idx+gate, logits w+r
        gbs = nbytes / (t_ms / 1e3) / 1e9
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        line = {"metric": "route_stats tokens/s (router + load statistics)", "value": T / (t_ms / 1e3),
                "unit": "tokens/s", "n_gpus": 1, "steps": steps, "warmup": warmup,
                "ms_per_step": t_ms, "higher_is_better": True, "dtype": "bf16",
                "data": "synthetic (seeded Philox normal inputs)",
                "config": {"workload": "e32_long router", "T": T, "H": H, "E": E, "top_k": k,
                           "l2": "flushed before every step"},
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                             "frac": gbs / hbm, "peak_source": peak_src, "algorithmic_bytes": nbytes}}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    cfg = resolve_config(args.config, args.tokens)
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.hbm_copy_sweep:
        return hbm_copy_sweep()
    if args.op != "layer":
        return run_op(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    from routing_grouped_expert_moe_b200 import binding as B

    d = rank_inputs(cfg, rank)
    g = {k: (None if v is None else v.to(dev)) for k, v in d.items()}
    T, H, F, E, k = cfg.T, cfg.H, cfg.F, cfg.E, cfg.top_k
    ws = B.alloc_workspace(B.workspace_bytes(T, H, F, E, k, cfg.act, cfg.torch_dtype), dev)
    out = torch.empty(T, H, dtype=cfg.torch_dtype, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def fwd(out_counts=None):
        B.forward(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"], k,
                  cfg.capacity_factor, cfg.act, out=out, ws=ws, expert_counts_out=out_counts)

    # warm-up
    fwd(counts)
    torch.cuda.synchronize()
    st = B.device_status(ws)
    if st != B.OK:
        raise RuntimeError(f"device status {B.status_string(st)}")
    for _ in range(args.warmup):
        flush.zero_()
        fwd()
    torch.cuda.synchronize()
    work = algorithmic_work(cfg, counts.cpu().tolist())

    # ---- headline: K fused forwards, L2 flushed before each, CUDA events per step.
    # Each timed forward also records an event before GEMM-1 and one after GEMM-2
    # (moe_forward_timed with the other boundaries left out), so the expert GEMMs'
    # roofline comes from the same timed steps as the headline; an event between two
    # kernels ends their programmatic-launch overlap, so only these two are recorded.
    sampler = ClockSampler(dev.index).start()
    time.sleep(0.05)
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    starts, ends = [mk() for _ in range(args.steps)], [mk() for _ in range(args.steps)]
    g_in, g_out = [mk() for _ in range(args.steps)], [mk() for _ in range(args.steps)]
    for e in g_in + g_out:      # create the CUDA events before the timed region
        e.record()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record()
        B.forward_timed(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"], k,
                        cfg.capacity_factor, cfg.act, out, ws,
                        [None, None, None, g_in[i], None, g_out[i], None])
        ends[i].record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if dist:
        dist.barrier()
    clocks = sampler.stop(t_wall0, t_wall1)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    q = sorted(step_ms)
    n10 = max(1, len(step_ms) // 10)
    step_stats = {"p10": q[len(q) // 10], "p50": q[len(q) // 2], "p90": q[(9 * len(q)) // 10],
                  "first_tenth_mean": statistics.mean(step_ms[:n10]),
                  "last_tenth_mean": statistics.mean(step_ms[-n10:])}
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    ms_per_step = total_ms / args.steps
    value = job_tokens_per_s(T, world, args.steps, total_ms)

    # the timed steps in three parts: status clear + route + scatter, the two expert
    # GEMMs, the combine
    mean_ms = lambda a, b: statistics.mean(x.elapsed_time(y) for x, y in zip(a, b))  # noqa: E731
    part_ms = {"route_permute": mean_ms(starts, g_in), "gemms": mean_ms(g_in, g_out),
               "combine": mean_ms(g_out, ends)}

    # ---- detail: every kernel of the fused path apart, in a separate loop after the
    # timed region (events at all stage boundaries)
    n_stage = min(args.steps, 50)
    ev = [[mk() for _ in range(7)] for _ in range(n_stage)]
    for i in range(n_stage):
        flush.zero_()
        B.forward_timed(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"], k,
                        cfg.capacity_factor, cfg.act, out, ws, ev[i])
    torch.cuda.synchronize()
    names = ["route", "scan", "scatter", "gemm1", "gemm2", "combine"]
    stage_ms = {n: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(n_stage))
                for j, n in enumerate(names)}

    # ---- the library's kernel launches per forward (kernel nodes of a captured graph)
    per_fwd = kernels_per_call(fwd)
    gpu_launches = (per_fwd if per_fwd is not None else 6) * args.steps

    # ---- a plain device copy of each memory stage's algorithmic bytes (the rate
    # the stage could reach at its size: launch and ramp dominate small copies)
    same_copy_us = {"route": copy_us(work["route_bytes"], flush, dev),
                    "scatter": copy_us(work["scatter_bytes"], flush, dev),
                    "combine": copy_us(work["combine_bytes"], flush, dev)}

    # ---- end to end through the host-buffer entry point (H2D + layer + D2H)
    n_e2e = min(args.steps, 50)
    x_host = d["x"].pin_memory()
    out_host = torch.empty_like(x_host).pin_memory()
    ws_h = B.alloc_workspace(B.forward_host_workspace_bytes(T, H, F, E, k, cfg.act,
                                                            cfg.torch_dtype), dev)
    e2e_ms = []
    for i in range(n_e2e + 2):
        flush.zero_()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record()
        B.forward_host(x_host, g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"], k,
                       cfg.capacity_factor, cfg.act, out_host=out_host, ws=ws_h)
        s1.record()
        torch.cuda.synchronize()
        if i >= 2:
            e2e_ms.append(s0.elapsed_time(s1))
    serial_step_ms = max_over_ranks(statistics.mean(e2e_ms), dist, dev)
    serial_value = job_tokens_per_s(T, world, 1, serial_step_ms)
    io_bytes = T * H * cfg.elem_bytes
    del ws_h

    # ---- end to end over a run of batches: batch i+1's copy-in and batch i-1's
    # copy-out overlap batch i's layer (moe_forward_host_batches, three streams)
    n_pipe = min(args.steps, 50)
    x_ring = [x_host, x_host.clone().pin_memory()]
    out_ring = [out_host, torch.empty_like(x_host).pin_memory()]
    ws_b = B.alloc_workspace(B.forward_host_batches_workspace_bytes(T, H, F, E, k, cfg.act,
                                                                    cfg.torch_dtype), dev)
    copy_streams = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))

    def run_batches(n):
        B.forward_host_batches([x_ring[i % 2] for i in range(n)], g["w_gate"], g["gate_bias"],
                               g["w1"], g["w3"], g["w2"], k, cfg.capacity_factor, cfg.act,
                               out_hosts=[out_ring[i % 2] for i in range(n)], ws=ws_b,
                               copy_streams=copy_streams)

    run_batches(4)                                   # warm-up
    torch.cuda.synchronize()
    flush.zero_()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record()
    run_batches(n_pipe)
    s1.record()
    torch.cuda.synchronize()
    e2e_step_ms = max_over_ranks(s0.elapsed_time(s1) / n_pipe, dist, dev)
    e2e_value = job_tokens_per_s(T, world, 1, e2e_step_ms)
    if B.device_status(ws_b) != B.OK:
        raise RuntimeError("moe_forward_host_batches reported a device error")
    del ws_b

    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tc_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    # roofline and the memory-stage rates from the timed steps themselves
    gemm_ms = max_over_ranks(part_ms["gemms"], dist, dev)
    gemm_tflops = work["gemm_flops"] / (gemm_ms / 1e3) / 1e12
    rp_bytes = work["route_bytes"] + work["scan_bytes"] + work["scatter_bytes"]
    rp_ms = part_ms["route_permute"]          # includes the 4-byte status clear
    rp_gbs = rp_bytes / (rp_ms / 1e3) / 1e9
    comb_gbs = work["combine_bytes"] / (part_ms["combine"] / 1e3) / 1e9
    traffic = None
    if NCU_TRAFFIC["source_sha"] == gemm_source_sha() and NCU_TRAFFIC["workload"] == cfg.name:
        traffic = NCU_TRAFFIC["bytes_per_forward"]
    # The GEMMs are timed inside every forward of a long loop: when that loop ran
    # into the power cap (sw_power_cap in the clock record of the timed region) the
    # denominator is the sustained bf16 figure (a seconds-long GEMM loop under the
    # same cap); otherwise the burst figure (a GEMM timed alone).
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    tc_used = tc_sus if capped else tc
    tc_src = (f"{peak_src} sustained bf16 (sw_power_cap active in the timed region)" if capped
              else f"{peak_src} burst bf16")

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "step_ms_stats": step_stats,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": cfg.dtype, "data": "synthetic (seeded Philox normal inputs, random-init weights)",
        "config": {**workload_desc(cfg),
                   "l2": "flushed before every step (256 MiB write outside the timed events)",
                   "parallelism": f"replicas x{world} (token data-parallel, no collective)"},
        "clocks": clocks,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": io_bytes,
                "d2h_bytes_per_step": io_bytes, "ms_per_step": e2e_step_ms,
                "entry_point": "moe_forward_host_batches",
                "mode": (f"{n_pipe} batches from page-locked host memory; batch i+1's copy-in and "
                         "batch i-1's copy-out overlap batch i's layer (three streams, two "
                         "device stages); L2 flushed once before the run, weights "
                         f"({work['weight_bytes'] / 1e6:.0f} MB) streamed every batch"),
                "serial": {"value": serial_value, "ms_per_step": serial_step_ms,
                           "entry_point": "moe_forward_host",
                           "mode": "one call per step: copy-in, layer, copy-out in turn on one "
                                   "stream, L2 flushed before each step"}},
        "gpu_launches": gpu_launches,
        "gpu_launches_source": ("kernel nodes of one captured forward x steps" if per_fwd
                                is not None else "plan: 6 kernels per forward x steps"),
        "roofline": {"kernel": "k_gemm_tokn (expert GEMM-1 + GEMM-2)", "bound": "tensor",
                     "achieved": gemm_tflops, "peak": tc_used, "unit": "TFLOP/s",
                     "frac": gemm_tflops / tc_used, "peak_source": tc_src,
                     "frac_of_burst": gemm_tflops / tc,
                     "timed": "events before GEMM-1 and after GEMM-2 of every timed step",
                     "gemm_us_per_step": 1000.0 * gemm_ms,
                     "frac_of_sustained": gemm_tflops / tc_sus,
                     "frac_of_spec": gemm_tflops / SPEC_BF16_TFLOPS,
                     "algorithmic_flops": work["gemm_flops"], "traffic": traffic},
        "grouped_gemm": {"tflops": gemm_tflops, "frac_measured_peak": gemm_tflops / tc_used,
                         "frac_spec_peak": gemm_tflops / SPEC_BF16_TFLOPS,
                         "gemm1_tflops_detail": work["gemm1_flops"] / (stage_ms["gemm1"] / 1e3)
                         / 1e12,
                         "gemm2_tflops_detail": work["gemm2_flops"] / (stage_ms["gemm2"] / 1e3)
                         / 1e12},
        "route_permute": {"gbs": rp_gbs, "frac_measured_hbm": rp_gbs / hbm,
                          "frac_spec_hbm": rp_gbs / SPEC_HBM_GBS, "bytes": rp_bytes,
                          "route_gbs_detail": work["route_bytes"] / (stage_ms["route"] / 1e3)
                          / 1e9},
        "combine": {"gbs": comb_gbs, "frac_measured_hbm": comb_gbs / hbm},
        "memory_stages_vs_same_size_copy": {
            n: {"stage_us": 1000.0 * stage_ms[n], "copy_us": same_copy_us[n],
                "bytes": work[f"{n}_bytes"],
                "frac_of_same_size_copy": same_copy_us[n] / (1000.0 * stage_ms[n])}
            for n in ("route", "scatter", "combine")},
        "timed_parts_us": {n: 1000.0 * v for n, v in part_ms.items()},
        "stage_us_detail": {n: 1000.0 * v for n, v in stage_ms.items()},
        "stage_detail": f"every kernel apart: {n_stage} forwards with events at all stage "
                        "boundaries, in a loop after the timed region",
        "kept_rows": work["R"],
        "page_figures_context": {
            "MoE-32E seq=1024 FP16, Ascend 910": "standard 1850 ms, ops-transformer 620 ms",
            "routing stage, Ascend 910B": "original 8.2 ms, page's method 1.7 ms"},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, d, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
