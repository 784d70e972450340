"""Whole-layer parity over seeded random shapes: token counts from 1 up, hidden
and intermediate sizes down to 8 (ragged against every tile size), 1 to 256
experts, top-1 to top-8, both activations, both storage types, capacity limits
and router biases — each case against the oracle, indices bit-exact."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from routing_grouped_expert_moe_b200 import synth
from tests.helpers import (TOL, Guarded, as_np, check_forward_workspace, gapped_inputs,
                           guarded_workspace, rel_err)

pytestmark = pytest.mark.gpu


def _cases(n=36, seed=777):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        E = int(rng.choice([1, 2, 3, 4, 5, 8, 12, 16, 24, 32, 64, 96, 128, 256]))
        k = int(rng.integers(1, min(8, E) + 1))
        H = 8 * int(rng.integers(1, 65))
        F = 8 * int(rng.integers(1, 49))
        dtype = "f32" if rng.random() < 0.25 else "bf16"
        act = str(rng.choice(["gelu", "swiglu"]))
        cfg = synth.MoEConfig(
            name=f"fuzz{i}", T=int(rng.integers(1, 700)), H=H, F=F, E=E, top_k=k, dtype=dtype,
            act=act, capacity_factor=float(rng.choice([0.0, 0.0, 0.5, 0.8, 1.0, 1.25])),
            seed=9000 + i, x_std=1.0, wg_std=H ** -0.5, w1_std=H ** -0.5, w2_std=F ** -0.5,
            bias=str(rng.choice(["none", "uniform", "zipf"])))
        out.append(cfg)
    return out


CASES = _cases()


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: f"{c.name}-T{c.T}-H{c.H}-F{c.F}-E{c.E}-k{c.top_k}"
                                                      f"-{c.act}-{c.dtype}-cf{c.capacity_factor}")
def test_forward_fuzz(cfg, gemm_variant):
    """Each case on one of the three bf16 GEMM kernels in turn; outputs and the
    workspace sentinel-guarded, rows past R untouched."""
    from routing_grouped_expert_moe_b200 import binding as B
    gemm_variant(["tokens_pair", "rows128", "rows256_pair", "tokens_pair_nosplit"]
                 [int(cfg.name[4:]) % 4])
    d = gapped_inputs(cfg)
    g = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    ig = Guarded((cfg.T, cfg.top_k), torch.int32)
    cg = Guarded((cfg.E,), torch.int32)
    og = Guarded((cfg.T, cfg.H), cfg.torch_dtype)
    wsg = guarded_workspace(B.workspace_bytes(cfg.T, cfg.H, cfg.F, cfg.E, cfg.top_k, cfg.act,
                                              cfg.torch_dtype))
    idx, cnt = ig.t, cg.t
    out = B.forward(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"], cfg.top_k,
                    cfg.capacity_factor, cfg.act, out=og.t, ws=wsg.t, topk_idx_out=idx,
                    expert_counts_out=cnt)
    assert B.device_status(wsg.t) == B.OK
    for buf, name in ((ig, "topk_idx"), (cg, "counts"), (og, "out")):
        buf.check(name)
    f = lambda t: None if t is None else as_np(t)  # noqa: E731
    ref = O.moe_forward(f(d["x"]), f(d["w_gate"]), f(d["gate_bias"]), f(d["w1"]), f(d["w3"]),
                        f(d["w2"]), cfg.top_k, cfg.capacity_factor, cfg.act, cfg.dtype)
    np.testing.assert_array_equal(as_np(idx), ref["topk_idx"])
    np.testing.assert_array_equal(as_np(cnt), ref["counts"])
    err = rel_err(as_np(out), ref["out"])
    assert err <= TOL[cfg.dtype], err
    check_forward_workspace(wsg, B, cfg, int(ref["R"]), what=cfg.name)


def _thr_cases(n=12, seed=778):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        E = int(rng.choice([2, 4, 8, 16, 32, 64, 128]))
        H = 8 * int(rng.integers(2, 49))
        F = 8 * int(rng.integers(2, 33))
        cfg = synth.MoEConfig(
            name=f"thr{i}", T=int(rng.integers(1, 500)), H=H, F=F, E=E, top_k=2,
            dtype="bf16", act=str(rng.choice(["gelu", "swiglu"])),
            capacity_factor=float(rng.choice([0.0, 0.0, 0.8, 1.25])), seed=9500 + i, x_std=1.0,
            wg_std=3 * H ** -0.5, w1_std=H ** -0.5, w2_std=F ** -0.5, bias="none")
        out.append((cfg, int(rng.integers(1, min(8, E) + 1))))
    return out


@pytest.mark.parametrize("case", _thr_cases(), ids=lambda c: f"{c[0].name}-T{c[0].T}-E{c[0].E}-kmax{c[1]}")
def test_forward_threshold_fuzz(case):
    from routing_grouped_expert_moe_b200 import binding as B
    from tests.helpers import threshold_inputs
    cfg, k_max = case
    d = threshold_inputs(cfg, float(np.float32(1.0 / cfg.E)), k_max)
    g = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    idx = torch.empty(cfg.T, k_max, dtype=torch.int32, device="cuda")
    n = torch.empty(cfg.T, dtype=torch.int32, device="cuda")
    out, ws = B.forward_threshold(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"],
                                  k_max, 0.0, cfg.capacity_factor, cfg.act, topk_idx_out=idx,
                                  n_selected_out=n)
    assert B.device_status(ws) == B.OK
    f = lambda t: None if t is None else as_np(t)  # noqa: E731
    ref = O.moe_forward_threshold(f(d["x"]), f(d["w_gate"]), None, f(d["w1"]), f(d["w3"]),
                                  f(d["w2"]), k_max, None, cfg.capacity_factor, cfg.act, cfg.dtype)
    np.testing.assert_array_equal(as_np(idx), ref["topk_idx"])
    np.testing.assert_array_equal(as_np(n), ref["n_sel"])
    assert rel_err(as_np(out), ref["out"]) <= TOL[cfg.dtype]


def _mm_cases(n=12, seed=779):
    rng = np.random.default_rng(seed)
    return [(int(rng.integers(1, 900)), 8 * int(rng.integers(1, 65)), 8 * int(rng.integers(1, 65)),
             int(rng.choice([1, 2, 3, 8, 16, 64, 256])), str(rng.choice(["bf16", "bf16", "f32"])),
             9700 + i) for i in range(n)]


@pytest.mark.parametrize("case", _mm_cases(), ids=lambda c: "mm-" + "x".join(map(str, c[:4])) + c[4])
def test_expert_matmul_fuzz(case):
    from routing_grouped_expert_moe_b200 import binding as B
    T, H, I, E, dtype, seed = case
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = synth.normal(seed, synth.STREAM_X, (T, H), 1.0, td)
    w = synth.normal(seed, synth.STREAM_W1, (E, H, I), H ** -0.5, td)
    ids = synth.random_expert_ids(seed, T, E, 1, skew=0.5)[:, 0].contiguous()
    out, ws = B.expert_matmul(x.cuda(), w.cuda(), ids.cuda())
    assert B.device_status(ws) == B.OK
    ref = O.expert_matmul(as_np(x), as_np(w), ids.numpy(), dtype)
    assert rel_err(as_np(out), ref) <= TOL[dtype]
