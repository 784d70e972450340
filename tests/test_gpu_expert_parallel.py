"""Expert-parallel forward on the GPU with one NCCL rank: every exchange runs
(counts, rows out, rows back) through NCCL, and every compute step through the
C ABI's kernels: the one-round form with its k = 1 regroup and inverse (the
combine with no gates), and the two-group (overlapped) form, whose per-expert
blocks land in expert order.  More ranks need more GPUs than these tests get; the exchange logic
over several ranks is checked on CPU ranks (test_expert_parallel.py)."""
import numpy as np
import pytest
import torch
import torch.distributed as dist

from oracle import moe_oracle as O
from routing_grouped_expert_moe_b200 import expert_parallel as EP
from routing_grouped_expert_moe_b200 import synth
from tests.helpers import TOL, as_np, gapped_inputs, rel_err

pytestmark = pytest.mark.gpu


def B():
    from routing_grouped_expert_moe_b200 import binding
    return binding


@pytest.fixture(scope="module")
def one_rank():
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1)
    yield
    dist.destroy_process_group()


def test_combine_without_gates_is_a_row_gather():
    y = synth.normal(5100, synth.STREAM_X, (300, 136), 1.0, torch.bfloat16).cuda()
    perm = torch.randperm(300, generator=torch.Generator().manual_seed(5))
    row_map = perm[:257].to(torch.int32).reshape(257, 1).cuda()
    row_map[7, 0] = -1
    out = B().unpermute_combine(y, None, row_map)
    ref = y[row_map[:, 0].clamp(min=0).long()].clone()
    ref[7] = 0
    assert torch.equal(out, ref)


@pytest.mark.parametrize("name,kw", [
    ("gelu_nodrop", dict(base="page1_gelu", T=1500, H=256, F=512, capacity_factor=0.0)),
    ("swiglu_drops", dict(base="mixtral_e8", T=777, H=512, F=384, capacity_factor=0.6)),
    ("skew_e128", dict(base="e128_skew", T=1200, H=256, F=128, capacity_factor=0.0)),
])
def test_expert_parallel_one_rank(one_rank, name, kw):
    from dataclasses import replace
    kw = dict(kw)
    base = kw.pop("base")
    cfg = replace(synth.CONFIGS[base], name=f"ep_{name}", seed=5200 + len(name), **kw)
    d = gapped_inputs(cfg)
    g = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    out = EP.ep_forward(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"],
                        cfg.top_k, cfg.capacity_factor, cfg.act, cfg.E)
    torch.cuda.synchronize()
    f = lambda t: None if t is None else as_np(t)  # noqa: E731
    ref = O.moe_forward(f(d["x"]), f(d["w_gate"]), f(d["gate_bias"]), f(d["w1"]), f(d["w3"]),
                        f(d["w2"]), cfg.top_k, cfg.capacity_factor, cfg.act, cfg.dtype)
    assert rel_err(as_np(out), ref["out"]) <= TOL[cfg.dtype]
    # the same kernels called stage by stage on one device give the same bits
    idx, gate = B().route(g["x"], g["w_gate"], g["gate_bias"], cfg.top_k)
    np.testing.assert_array_equal(as_np(idx), ref["topk_idx"])
    p = B().permute(idx, cfg.E, cfg.capacity_factor, x=g["x"])
    R = int(p["offsets"][-1])
    y = B().grouped_ffn(p["offsets"], g["w1"], g["w3"], g["w2"], cfg.act, x_perm=p["x_perm"][:R])
    staged = B().unpermute_combine(y, gate, p["row_map"])
    assert torch.equal(out, staged)
    # two expert groups (the overlapped exchange; on one rank every block is a local copy):
    # the experts run as two grouped GEMMs, whose tile variant may differ from one GEMM's
    ov = EP.ep_forward(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"],
                       cfg.top_k, cfg.capacity_factor, cfg.act, cfg.E, overlap=True)
    torch.cuda.synchronize()
    assert rel_err(as_np(ov), ref["out"]) <= TOL[cfg.dtype]
    assert float((ov == out).float().mean()) >= 0.999
