"""Test-side helpers: gap-enforced workload inputs and error metrics.

The router-logit gap rule (every consecutive gap among a token's top k+1
logits >= 1e-3, so selection has no near-ties) needs the layer's own logits;
it therefore lives here, on the test side, and uses the oracle's logits.
Violating tokens' x rows are redrawn from the generator's redraw stream.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O
from routing_grouped_expert_moe_b200 import synth

MIN_GAP = 1e-3
TOL = {"f32": 1e-4, "bf16": 2e-2}   # max|gpu - oracle| / max|oracle|


def as_np(t: torch.Tensor) -> np.ndarray:
    """Exact float64 (or int) numpy copy of a CPU/GPU tensor."""
    t = t.detach().cpu()
    if t.is_floating_point():
        return t.to(torch.float64).numpy()
    return t.numpy()


def gap_violations(logits: np.ndarray, k: int, min_gap: float = MIN_GAP) -> np.ndarray:
    E = logits.shape[1]
    m = min(k + 1, E)
    srt = -np.sort(-logits.astype(np.float64), axis=1)[:, :m]
    gaps = srt[:, :-1] - srt[:, 1:]
    return np.nonzero(np.any(gaps < min_gap, axis=1))[0]


def gapped_inputs(cfg: synth.MoEConfig, with_weights: bool = True, max_rounds: int = 50) -> dict:
    d = synth.make_inputs(cfg, with_weights=with_weights)
    x = d["x"]
    wg = as_np(d["w_gate"])
    b = None if d["gate_bias"] is None else as_np(d["gate_bias"])
    bad = np.arange(cfg.T)
    for attempt in range(max_rounds):
        lg = O.router_logits(as_np(x[torch.from_numpy(bad)]) if attempt else as_np(x), wg, b)
        viol = gap_violations(lg, cfg.top_k)
        bad = bad[viol] if attempt else viol
        if len(bad) == 0:
            break
        x[torch.from_numpy(bad)] = synth.redraw_rows(cfg, len(bad), attempt)
    else:
        raise RuntimeError("gap enforcement did not converge")
    d["x"] = x
    return d


def threshold_margin_violations(logits: np.ndarray, delta: float, rel: float = 1e-3) -> np.ndarray:
    """Tokens with an expert whose softmax probability lies within rel * delta of
    delta: there a float32 and a float64 evaluation could decide differently."""
    lg = logits.astype(np.float64)
    z = np.exp(lg - lg.max(axis=1, keepdims=True))
    p = z / z.sum(axis=1, keepdims=True)
    return np.nonzero(np.any(np.abs(p - delta) < rel * delta, axis=1))[0]


def threshold_inputs(cfg: synth.MoEConfig, delta: float, k_max: int, max_rounds: int = 50) -> dict:
    """gapped_inputs whose tokens also keep every probability away from delta and
    a 1e-3 gap between each of their k_max + 1 largest logits."""
    d = gapped_inputs(cfg)
    x = d["x"]
    wg = as_np(d["w_gate"])
    b = None if d["gate_bias"] is None else as_np(d["gate_bias"])
    for attempt in range(max_rounds):
        lg = O.router_logits(as_np(x), wg, b)
        bad = np.union1d(threshold_margin_violations(lg, delta), gap_violations(lg, k_max))
        if len(bad) == 0:
            d["x"] = x
            return d
        x[torch.from_numpy(bad)] = synth.redraw_rows(cfg, len(bad), 100 + attempt)
    raise RuntimeError("threshold margin enforcement did not converge")


def rel_err(gpu, ref) -> float:
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    denom = np.max(np.abs(r)) if r.size else 0.0
    if denom == 0.0:
        return float(np.max(np.abs(g))) if g.size else 0.0
    return float(np.max(np.abs(g - r)) / denom)


# ---------------------------------------------------------------- canary guards
# compute-sanitizer is not available on the GPU pool, so device buffers handed to
# the library are surrounded by sentinel bytes; a kernel that writes past an
# output (or into a part of the workspace it must not touch) changes them.
CANARY = 0xA5
MARGIN = 4096  # bytes before and after every guarded buffer


class Guarded:
    """A device tensor of `shape`/`dtype` inside a uint8 allocation whose MARGIN
    bytes on either side (and, optionally, the tensor itself) hold CANARY."""

    def __init__(self, shape, dtype, device="cuda", fill_canary=True):
        n = 1
        for s in shape:
            n *= int(s)
        self.nbytes = n * torch.empty(0, dtype=dtype).element_size()
        self.raw = torch.full((self.nbytes + 2 * MARGIN,), CANARY, dtype=torch.uint8,
                              device=device)
        self.bytes = self.raw[MARGIN:MARGIN + self.nbytes]
        self.t = self.bytes.view(dtype).view(*shape)
        if not fill_canary:
            self.t.zero_()

    def check(self, what="buffer"):
        torch.cuda.synchronize()
        lo = self.raw[:MARGIN]
        hi = self.raw[MARGIN + self.nbytes:]
        bad_lo = int((lo != CANARY).sum())
        bad_hi = int((hi != CANARY).sum())
        assert bad_lo == 0 and bad_hi == 0, \
            f"{what}: {bad_lo} bytes changed before it, {bad_hi} after it"

    def untouched(self, start_byte, end_byte, what="region"):
        """Asserts bytes [start, end) of the tensor still hold CANARY."""
        torch.cuda.synchronize()
        seg = self.bytes[start_byte:end_byte]
        bad = int((seg != CANARY).sum())
        assert bad == 0, f"{what}: {bad} of {end_byte - start_byte} bytes written"


def guarded_workspace(nbytes, device="cuda") -> Guarded:
    """A 256-byte-aligned workspace (MARGIN is a multiple of 256) filled with CANARY."""
    return Guarded((int(nbytes),), torch.uint8, device)


def check_forward_workspace(ws: Guarded, B, cfg, R: int, act=None, what=""):
    """After a fused forward: the workspace's margins are intact, and the rows
    past the R kept rows of x_perm, h and y, and the row_token entries past R,
    were never written (the permute writes R rows, the GEMMs write only rows of
    their experts' segments)."""
    act = act or cfg.act
    ws.check(f"{what} workspace")
    T, k = cfg.T, cfg.top_k
    eb = 2 if cfg.dtype == "bf16" else 4
    for name, width, esize in (("row_token", 1, 4), ("x_perm", cfg.H, eb), ("h", cfg.F, eb),
                               ("y", cfg.H, eb)):
        if name == "x_perm" and cfg.dtype != "bf16":
            continue
        if name == "h" and act == "identity":
            continue
        sec = B.workspace_section(ws.t, name, T, cfg.H, cfg.F, cfg.E, k, act, cfg.torch_dtype)
        off = sec.data_ptr() - ws.t.data_ptr()
        ws.untouched(off + R * width * esize, off + T * k * width * esize,
                     f"{what} {name} past row {R}")
