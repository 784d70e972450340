"""Whole-layer parity of moe_forward (the call bench.py times) against the oracle.

Small workloads run every grouped-GEMM kernel and are compared on every
element.  The five workloads at full size run in exactly the launch
configuration the bench times and are compared with the C++ oracle on every
token: indices, pre-drop counts, offsets, row_token and row_map bit for bit
(read from the forward's workspace), gates and outputs within tolerance.
Every buffer the library writes is surrounded by sentinel bytes, and the
workspace rows past the R kept rows must stay untouched.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from oracle import moe_oracle_cpp as OC
from routing_grouped_expert_moe_b200 import synth
from tests.helpers import (TOL, Guarded, as_np, check_forward_workspace, gapped_inputs,
                           guarded_workspace, rel_err)

pytestmark = pytest.mark.gpu


def B():
    from routing_grouped_expert_moe_b200 import binding
    return binding


def _cuda(d):
    return {k: (None if v is None else v.cuda()) for k, v in d.items()}


def _run(cfg, d, act=None, guard=False):
    """One fused forward.  With guard, the output and the workspace are
    sentinel-guarded (returned as Guarded objects) and routing stays in the
    workspace, where the tests read it."""
    g = _cuda(d)
    T, E, k = cfg.T, cfg.E, cfg.top_k
    nbytes = B().workspace_bytes(T, cfg.H, cfg.F, E, k, act or cfg.act, cfg.torch_dtype)
    if guard:
        ws = guarded_workspace(nbytes)
        out = Guarded((T, cfg.H), cfg.torch_dtype)
        B().forward(g["x"], g["w_gate"], g["gate_bias"], g.get("w1"), g.get("w3"), g.get("w2"),
                    k, cfg.capacity_factor, act or cfg.act, out=out.t, ws=ws.t)
        assert B().device_status(ws.t) == B().OK
        return out, ws
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(E, dtype=torch.int32, device="cuda")
    ws = B().alloc_workspace(nbytes)
    out = B().forward(g["x"], g["w_gate"], g["gate_bias"], g.get("w1"), g.get("w3"), g.get("w2"),
                      k, cfg.capacity_factor, act or cfg.act, ws=ws, topk_idx_out=idx,
                      expert_counts_out=cnt)
    assert B().device_status(ws) == B().OK
    return out, idx, cnt, ws


def _section(ws, cfg, name, dtype, shape, act=None):
    sec = B().workspace_section(ws.t, name, cfg.T, cfg.H, cfg.F, cfg.E, cfg.top_k,
                                act or cfg.act, cfg.torch_dtype)
    return sec.view(dtype).view(*shape)


def _check_routing_and_permutation(ws, cfg, ref, act=None):
    """Indices, counts, offsets and the permutation bit for bit; gates to fp32
    rounding; the rows past R untouched."""
    T, E, k = cfg.T, cfg.E, cfg.top_k
    idx = as_np(_section(ws, cfg, "topk_idx", torch.int32, (T, k), act))
    np.testing.assert_array_equal(idx, ref["topk_idx"])
    np.testing.assert_array_equal(as_np(_section(ws, cfg, "counts", torch.int32, (E,), act)),
                                  ref["counts"])
    offs = as_np(_section(ws, cfg, "offsets", torch.int32, (E + 1,), act))
    np.testing.assert_array_equal(offs, ref["offsets"])
    R = int(ref["R"])
    assert offs[E] == R
    rt = as_np(_section(ws, cfg, "row_token", torch.int32, (T * k,), act))
    np.testing.assert_array_equal(rt[:R], ref["row_token"])
    np.testing.assert_array_equal(as_np(_section(ws, cfg, "row_map", torch.int32, (T, k), act)),
                                  ref["row_map"])
    gate = as_np(_section(ws, cfg, "topk_gate", torch.float32, (T, k), act))
    # gates are fp32 outputs of fp32 logits accumulated in another order: the
    # fp32 output tolerance
    assert rel_err(gate, ref["topk_gate"]) <= TOL["f32"]
    check_forward_workspace(ws, B(), cfg, R, act, cfg.name)


def _small_cfg(base_name, **kw):
    base = synth.CONFIGS[base_name]
    from dataclasses import replace
    return replace(base, **kw)


SMALL = [
    synth.CONFIGS["tiny_f32"],
    synth.CONFIGS["drop_cf05"],
    _small_cfg("page1_gelu", name="gelu_small", T=700, H=256, F=512, seed=2001),
    _small_cfg("mixtral_e8", name="swiglu_small", T=333, H=512, F=384, seed=2002),
    _small_cfg("e128_skew", name="skew_small", T=1500, H=256, F=128, seed=2003),
    _small_cfg("e32_long", name="e32_small", T=2049, H=128, F=1376, capacity_factor=1.0,
               seed=2004),
]


@pytest.mark.parametrize("oracle", ["numpy", "cpp"])
@pytest.mark.parametrize("variant", ["rows128", "rows256_pair", "tokens_pair",
                                     "tokens_pair_nosplit"])
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_forward_small_full_compare(cfg, variant, oracle, gemm_variant):
    if cfg.dtype == "f32" and variant != "rows128":
        pytest.skip("the fp32 path has a single CUDA-core kernel")
    gemm_variant(variant)
    d = gapped_inputs(cfg)
    out, ws = _run(cfg, d, guard=True)
    ref = (O if oracle == "numpy" else OC).moe_forward(as_np(d["x"]), as_np(d["w_gate"]),
                        None if d["gate_bias"] is None else as_np(d["gate_bias"]),
                        as_np(d["w1"]), None if d["w3"] is None else as_np(d["w3"]),
                        as_np(d["w2"]), cfg.top_k, cfg.capacity_factor, cfg.act, cfg.dtype)
    _check_routing_and_permutation(ws, cfg, ref)
    err = rel_err(as_np(out.t), ref["out"])
    assert err <= TOL[cfg.dtype], err
    out.check("out")
    if cfg.name == "drop_cf05":
        assert ref["dropped"] > 0


def _f32_np(t):
    return None if t is None else t.float().numpy()


@pytest.mark.slow
@pytest.mark.parametrize("name", ["tiny_f32", "page1_gelu", "mixtral_e8", "e32_long",
                                  "e128_skew"])
def test_forward_full_size_every_token(name):
    """The five workloads at full size, in the bench's launch configuration,
    against the C++ oracle's whole layer: every index, count, offset and
    permutation entry bit for bit and every output element within tolerance."""
    cfg = synth.CONFIGS[name]
    d = gapped_inputs(cfg)
    out, ws = _run(cfg, d, guard=True)
    ref = OC.moe_forward(_f32_np(d["x"]), _f32_np(d["w_gate"]), _f32_np(d["gate_bias"]),
                         _f32_np(d["w1"]), _f32_np(d["w3"]), _f32_np(d["w2"]), cfg.top_k,
                         cfg.capacity_factor, cfg.act, cfg.dtype)
    _check_routing_and_permutation(ws, cfg, ref)
    got = as_np(out.t)
    assert np.all(np.isfinite(got))
    err = rel_err(got, ref["out"])
    assert err <= TOL[cfg.dtype], err
    out.check("out")


def test_forward_identity_experts_give_x_times_gate_sum():
    cfg = _small_cfg("drop_cf05", name="identity", T=900, H=128, F=8)
    d = gapped_inputs(cfg, with_weights=False)
    out, idx, cnt, _ = _run(cfg, {**d, "w1": None, "w3": None, "w2": None}, act="identity")
    lg = O.router_logits(as_np(d["x"]), as_np(d["w_gate"]), None)
    ref = O.moe_forward(as_np(d["x"]), None, None, None, None, None, cfg.top_k,
                        cfg.capacity_factor, "identity", cfg.dtype, logits=lg)
    assert ref["dropped"] > 0
    g = ref["topk_gate"].astype(np.float64) * (ref["row_map"] >= 0)
    np.testing.assert_allclose(as_np(out), as_np(d["x"]) * g.sum(1, keepdims=True), rtol=8e-3,
                               atol=1e-2)
    assert rel_err(as_np(out), ref["out"]) <= TOL["bf16"]


def test_forward_single_expert_is_dense_ffn():
    cfg = _small_cfg("mixtral_e8", name="dense", T=300, H=256, F=512, E=1, top_k=1, seed=2010)
    d = synth.make_inputs(cfg)
    out, *_ = _run(cfg, d)
    xt = d["x"].double()
    h = torch.nn.functional.silu(xt @ d["w1"][0].double()) * (xt @ d["w3"][0].double())
    ref = h.to(torch.bfloat16).double() @ d["w2"][0].double()
    assert rel_err(as_np(out), ref.numpy()) <= TOL["bf16"]


def test_forward_deterministic_and_host_entry_point():
    cfg = _small_cfg("page1_gelu", name="det", T=1024, H=512, F=1024, seed=2020)
    d = synth.make_inputs(cfg)
    o1, *_ = _run(cfg, d)
    o2, *_ = _run(cfg, d)
    assert torch.equal(o1, o2)
    g = _cuda(d)
    xh = d["x"].pin_memory()
    oh = B().forward_host(xh, g["w_gate"], g["gate_bias"], g["w1"], None, g["w2"], cfg.top_k,
                          cfg.capacity_factor, cfg.act)
    torch.cuda.synchronize()
    assert torch.equal(oh, o1.cpu())


@pytest.mark.parametrize("overlap", [True, False], ids=["three_streams", "one_stream"])
def test_host_batches_equal_one_forward_per_batch(overlap):
    """Pipelined host batches (two device stages reused in turn) give, for every
    batch, exactly what one moe_forward of that batch gives; batches 5 and 6
    repeat the host buffers of batches 0 and 1."""
    cfg = _small_cfg("page1_gelu", name="batches", T=4096, H=1024, F=2048, seed=2025)
    d = synth.make_inputs(cfg)
    g = _cuda(d)
    xs = [synth.normal(2025 + i, synth.STREAM_X, (cfg.T, cfg.H), 1.0, torch.bfloat16).pin_memory()
          for i in range(5)]
    xs += xs[:2]
    outs = [torch.empty_like(x, pin_memory=True) for x in xs]
    got = B().forward_host_batches(xs, g["w_gate"], g["gate_bias"], g["w1"], None, g["w2"],
                                   cfg.top_k, cfg.capacity_factor, cfg.act, out_hosts=outs,
                                   copy_streams="new" if overlap else None)
    torch.cuda.synchronize()
    ws = B().alloc_workspace(B().workspace_bytes(cfg.T, cfg.H, cfg.F, cfg.E, cfg.top_k, cfg.act,
                                                 cfg.torch_dtype))
    for i, x in enumerate(xs):
        ref = B().forward(x.cuda(), g["w_gate"], g["gate_bias"], g["w1"], None, g["w2"],
                          cfg.top_k, cfg.capacity_factor, cfg.act, ws=ws)
        assert torch.equal(got[i], ref.cpu()), i
    assert B().device_status(ws) == B().OK
    assert torch.equal(got[5], got[0]) and not torch.equal(got[0], got[1])


def test_forward_empty_and_one_token():
    cfg = _small_cfg("mixtral_e8", name="one", T=1, H=256, F=256, seed=2030)
    d = synth.make_inputs(cfg)
    out, idx, cnt, _ = _run(cfg, d)
    ref = O.moe_forward(as_np(d["x"]), as_np(d["w_gate"]), None, as_np(d["w1"]), as_np(d["w3"]),
                        as_np(d["w2"]), cfg.top_k, 0.0, cfg.act, cfg.dtype)
    assert rel_err(as_np(out), ref["out"]) <= TOL["bf16"]
    g = _cuda(d)
    empty = torch.empty(0, cfg.H, dtype=torch.bfloat16, device="cuda")
    o = B().forward(empty, g["w_gate"], None, g["w1"], g["w3"], g["w2"], 2, 0.0, "swiglu")
    assert o.shape == (0, cfg.H)
