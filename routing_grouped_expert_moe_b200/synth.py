"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws random numbers: it holds none of the layer's arithmetic
(no logits, no routing, no expert math).  Both the CUDA path (tests, bench) and
the CPU oracle (tests) consume what it produces, so it imports neither.

Every tensor comes from its own counter-based Philox stream, keyed by
(workload seed, stream id), so a tensor can be regenerated alone and the draw
does not depend on the order in which tensors are requested.

Workloads (the shapes of the pages' own examples):
  tiny_f32      T=64 H=128 F=256 E=4 k=2, fp32, SwiGLU, no capacity limit
  page1_gelu    T=4096 H=2048 F=8192 E=8 k=2, bf16, GELU, capacity factor 1.2
                ("FFN(2048, 8192) x 8 experts, top_k=2, capacity_factor=1.2" in
                the hnwysp.cn ops-transformer MoE article, §3.2 call example)
  mixtral_e8    T=1024 H=4096 F=14336 E=8 k=2, bf16, SwiGLU, no limit
                (x[1024,4096], expert_weight[8,4096,14336] in the lshu.cn
                torch_npu fused-operator article, §3 minimal example)
  e32_long      T=32768 H=4096 F=1376 E=32 k=2, bf16, SwiGLU, capacity 1.25
                (MoE-32E, --seq_len 4096 --batch_size 8 in "ops-transformer
                仓库 - MoE 算子优化实战", Step 4)
  e128_skew     T=16384 H=2048 F=768 E=128 k=2, bf16, SwiGLU, no limit, Zipf-like
                router bias (128 experts, top-2, same page, opening paragraph)
  drop_cf05     T=512 H=256 F=512 E=8 k=2, bf16, SwiGLU, capacity factor 0.5:
                a test-only workload in which about half the assignments drop.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field

import numpy as np
import torch

# Philox stream ids, one per tensor.
STREAM_X, STREAM_WG, STREAM_W1, STREAM_W3, STREAM_W2, STREAM_REDRAW = 0, 1, 2, 3, 4, 5


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                 # tokens
    H: int                 # hidden size
    F: int                 # expert intermediate (ffn) size
    E: int                 # experts
    top_k: int
    dtype: str             # "f32" or "bf16": storage type of x, weights, h, y, out
    act: str               # "swiglu" or "gelu"
    capacity_factor: float # <= 0: no per-expert capacity limit
    seed: int
    x_std: float = 1.0
    wg_std: float = 0.0    # router weight std
    w1_std: float = 0.0    # W1 / W3 std (fan_in = H)
    w2_std: float = 0.0    # W2 std (fan_in = F)
    bias: str = "none"     # "none" | "uniform" | "zipf"
    description: str = ""

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


def _fan_in_std(fan_in: int, kaiming: bool = False) -> float:
    return math.sqrt((2.0 if kaiming else 1.0) / fan_in)


def _cfg(name, T, H, F, E, k, dtype, act, cf, seed, kaiming=False, bias="none", wg_std=None,
         description=""):
    return MoEConfig(
        name=name, T=T, H=H, F=F, E=E, top_k=k, dtype=dtype, act=act, capacity_factor=cf,
        seed=seed, x_std=1.0,
        wg_std=wg_std if wg_std is not None else _fan_in_std(H, kaiming),
        w1_std=_fan_in_std(H, kaiming), w2_std=_fan_in_std(F, kaiming), bias=bias,
        description=description)


CONFIGS: dict[str, MoEConfig] = {
    c.name: c for c in [
        _cfg("tiny_f32", 64, 128, 256, 4, 2, "f32", "swiglu", 0.0, 1001,
             description="tiny fp32 layer, SwiGLU, no capacity limit"),
        _cfg("page1_gelu", 4096, 2048, 8192, 8, 2, "bf16", "gelu", 1.2, 1002, kaiming=True,
             description="batch 8 x seq 512, FFN(2048,8192) GELU experts, capacity factor 1.2"),
        _cfg("mixtral_e8", 1024, 4096, 14336, 8, 2, "bf16", "swiglu", 0.0, 1003,
             description="Mixtral-shaped: x[1024,4096], 8 SwiGLU experts [4096,14336]"),
        _cfg("e32_long", 32768, 4096, 1376, 32, 2, "bf16", "swiglu", 1.25, 1004, bias="uniform",
             description="batch 8 x seq 4096, 32 SwiGLU experts, capacity factor 1.25"),
        _cfg("e128_skew", 16384, 2048, 768, 128, 2, "bf16", "swiglu", 0.0, 1005, bias="zipf",
             description="128 SwiGLU experts, Zipf-like router bias (skewed load)"),
        _cfg("drop_cf05", 512, 256, 512, 8, 2, "bf16", "swiglu", 0.5, 1006,
             description="capacity factor 0.5: about half of the assignments overflow"),
    ]
}

# The bench workload order used by the numbered --config flag (1..5) and tests.
NUMBERED = ["tiny_f32", "page1_gelu", "mixtral_e8", "e32_long", "e128_skew"]

# Constant router bias used by the "uniform" workload: every expert gets the same value,
# which leaves the load balanced but exercises the bias input.
UNIFORM_BIAS = 0.5


def _generator(seed: int, stream: int, attempt: int = 0, chunk: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([seed, stream, attempt, chunk])
    return np.random.Generator(np.random.Philox(ss))


_CHUNK = 1 << 24


def normal(seed: int, stream: int, shape, std: float, dtype: torch.dtype,
           attempt: int = 0) -> torch.Tensor:
    """N(0, std^2) draws stored (round-to-nearest-even) in dtype.

    Element i comes from Philox sub-stream (seed, stream, attempt, i // 2**24),
    so chunks are drawn in parallel and the result does not depend on threads.
    """
    from concurrent.futures import ThreadPoolExecutor
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=dtype)

    def fill(ci):
        s = ci * _CHUNK
        e = min(n, s + _CHUNK)
        a = _generator(seed, stream, attempt, ci).standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            a *= np.float32(std)
        out[s:e] = torch.from_numpy(a).to(dtype)

    nchunks = (n + _CHUNK - 1) // _CHUNK
    if nchunks <= 1:
        for ci in range(nchunks):
            fill(ci)
    else:
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.view(*shape)


def router_bias(cfg: MoEConfig) -> torch.Tensor | None:
    """fp32 router bias [E] (None when the workload has none)."""
    if cfg.bias == "none":
        return None
    if cfg.bias == "uniform":
        return torch.full((cfg.E,), UNIFORM_BIAS, dtype=torch.float32)
    if cfg.bias == "zipf":
        # b_e = 1.5 * ln(1 / (e + 1)): expert 0 is favoured, the tail is near-empty.
        e = np.arange(cfg.E, dtype=np.float64)
        return torch.from_numpy((1.5 * np.log(1.0 / (e + 1.0))).astype(np.float32))
    raise ValueError(cfg.bias)


def make_inputs(cfg: MoEConfig, with_weights: bool = True) -> dict:
    """All inputs of one workload as CPU tensors in the workload's storage dtype.

    Layouts: x[T,H], w_gate[H,E], gate_bias[E] fp32 (or None), w1/w3[E,H,F], w2[E,F,H].
    w3 is None for GELU experts.
    """
    dt = cfg.torch_dtype
    d = {
        "x": normal(cfg.seed, STREAM_X, (cfg.T, cfg.H), cfg.x_std, dt),
        "w_gate": normal(cfg.seed, STREAM_WG, (cfg.H, cfg.E), cfg.wg_std, dt),
        "gate_bias": router_bias(cfg),
    }
    if with_weights:
        d["w1"] = normal(cfg.seed, STREAM_W1, (cfg.E, cfg.H, cfg.F), cfg.w1_std, dt)
        d["w3"] = (normal(cfg.seed, STREAM_W3, (cfg.E, cfg.H, cfg.F), cfg.w1_std, dt)
                   if cfg.act == "swiglu" else None)
        d["w2"] = normal(cfg.seed, STREAM_W2, (cfg.E, cfg.F, cfg.H), cfg.w2_std, dt)
    return d


def redraw_rows(cfg: MoEConfig, n_rows: int, attempt: int) -> torch.Tensor:
    """Fresh x rows [n_rows, H] from the redraw stream (attempt numbers the round)."""
    return normal(cfg.seed, STREAM_REDRAW, (n_rows, cfg.H), cfg.x_std, cfg.torch_dtype,
                  attempt=attempt)


def random_logits(seed: int, T: int, E: int, scale: float = 1.0) -> torch.Tensor:
    """fp32 logits [T,E] for the route-from-logits parity hook."""
    return normal(seed, STREAM_X, (T, E), scale, torch.float32)


def random_expert_ids(seed: int, T: int, E: int, k: int, skew: float = 0.0) -> torch.Tensor:
    """int32 [T,k] expert ids, distinct within a token; skew>0 favours low ids."""
    g = _generator(seed, STREAM_X)
    w = np.exp(-skew * np.arange(E)) if skew > 0 else np.ones(E)
    w = w / w.sum()
    ids = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        ids[t] = g.choice(E, size=k, replace=False, p=w)
    return torch.from_numpy(ids)
