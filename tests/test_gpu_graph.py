"""The fused forward is stream-ordered and host-sync-free, so it runs on a
side stream and captures into a CUDA graph; replays give the eager result bit
for bit."""
from dataclasses import replace

import pytest
import torch

from routing_grouped_expert_moe_b200 import synth

pytestmark = pytest.mark.gpu


def _setup():
    from routing_grouped_expert_moe_b200 import binding as B
    cfg = replace(synth.CONFIGS["page1_gelu"], name="graph", T=1024, H=512, F=1024, seed=2040)
    d = synth.make_inputs(cfg)
    g = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    ws = B.alloc_workspace(B.workspace_bytes(cfg.T, cfg.H, cfg.F, cfg.E, cfg.top_k, cfg.act,
                                             cfg.torch_dtype))
    out = torch.empty(cfg.T, cfg.H, dtype=cfg.torch_dtype, device="cuda")
    run = lambda: B.forward(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"],  # noqa: E731
                            cfg.top_k, cfg.capacity_factor, cfg.act, out=out, ws=ws)
    return B, cfg, g, ws, out, run


def test_forward_on_a_side_stream():
    B, cfg, g, ws, out, run = _setup()
    run()
    torch.cuda.synchronize()
    ref = out.clone()
    out.zero_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert B.device_status(ws) == B.OK


def test_forward_captures_into_a_cuda_graph():
    B, cfg, g, ws, out, run = _setup()
    run()                                   # eager: also warms up the launch path
    torch.cuda.synchronize()
    ref = out.clone()
    out.zero_()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            run()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    # new inputs written in place flow through the captured graph
    g["x"].copy_(synth.normal(77, synth.STREAM_X, tuple(g["x"].shape), 1.0, cfg.torch_dtype))
    graph.replay()
    run_ref = out.clone()
    run()
    torch.cuda.synchronize()
    assert torch.equal(out, run_ref)
    assert B.device_status(ws) == B.OK
    del graph
