"""Parity of the rows built past the layer itself: the router's load statistics
(moe_route_stats) and the one-expert-per-token matmul (moe_expert_matmul),
each against both CPU oracles."""
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from oracle import moe_oracle_cpp as OC
from routing_grouped_expert_moe_b200 import synth
from tests.helpers import TOL, as_np, gapped_inputs, rel_err

pytestmark = pytest.mark.gpu


def B():
    from routing_grouped_expert_moe_b200 import binding
    return binding


# ---------------------------------------------------------------- router load statistics

STATS_CFGS = [
    synth.CONFIGS["tiny_f32"],
    replace(synth.CONFIGS["page1_gelu"], name="stats_e8", T=1000, H=256, seed=3001),
    replace(synth.CONFIGS["e128_skew"], name="stats_e128", T=1500, H=256, seed=3002),
    replace(synth.CONFIGS["e32_long"], name="stats_e32_bias", T=777, H=128, seed=3003),
    synth.CONFIGS["e128_skew"],
    synth.CONFIGS["e32_long"],
]


@pytest.mark.parametrize("cfg", STATS_CFGS, ids=lambda c: c.name)
def test_route_stats(cfg):
    d = gapped_inputs(cfg, with_weights=False)
    x, wg = d["x"].cuda(), d["w_gate"].cuda()
    b = None if d["gate_bias"] is None else d["gate_bias"].cuda()
    idx, gate, counts, prob, ws = B().route_stats(x, wg, b, cfg.top_k)
    assert B().device_status(ws) == B().OK
    # selection equals the oracle's (the inputs keep a 1e-3 gap between ranks)
    lg_ref = O.router_logits(as_np(d["x"]), as_np(d["w_gate"]),
                             None if d["gate_bias"] is None else as_np(d["gate_bias"]))
    np.testing.assert_array_equal(as_np(idx), O.topk_select(lg_ref, cfg.top_k))
    # statistics against each oracle, from the logits the GPU router produced
    _, _, lg = B().route(x, wg, b, top_k=cfg.top_k, logits_out=True)
    for orc in (O, OC):
        ref = orc.router_load_stats(as_np(lg), as_np(idx), cfg.E)
        np.testing.assert_array_equal(as_np(counts), ref["counts"])
        pm = as_np(prob)
        assert np.max(np.abs(pm - ref["prob_mean"])) <= 1e-5 * np.max(ref["prob_mean"])
    # fixed-order reductions: a second call gives the same bits
    _, _, counts2, prob2, _ = B().route_stats(x, wg, b, cfg.top_k, ws=ws)
    assert torch.equal(counts, counts2) and torch.equal(prob.view(torch.int32), prob2.view(torch.int32))


# ---------------------------------------------------------------- one expert per token

MATMUL_CASES = [
    # T, H, I, E, dtype, ids drawn from experts [0, E_used)
    (300, 200, 136, 8, "bf16", 6),     # H not a multiple of 64, I not of 256, 2 empty experts
    (257, 128, 256, 1, "bf16", 1),     # one expert: a dense matmul
    (1000, 512, 384, 16, "bf16", 16),
    (100, 64, 40, 4, "f32", 4),
]


def _matmul_inputs(T, H, I, E, dtype, e_used, seed):
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = synth.normal(seed, synth.STREAM_X, (T, H), 1.0, td)
    w = synth.normal(seed, synth.STREAM_W1, (E, H, I), H ** -0.5, td)
    ids = synth.random_expert_ids(seed, T, e_used, 1)[:, 0].contiguous()
    return x, w, ids


@pytest.mark.parametrize("case", MATMUL_CASES, ids=lambda c: "x".join(map(str, c[:4])) + c[4])
def test_expert_matmul_full_compare(case):
    T, H, I, E, dtype, e_used = case
    x, w, ids = _matmul_inputs(T, H, I, E, dtype, e_used, seed=4000 + T)
    out, ws = B().expert_matmul(x.cuda(), w.cuda(), ids.cuda())
    assert B().device_status(ws) == B().OK
    for orc in (O, OC):
        ref = orc.expert_matmul(as_np(x), as_np(w), ids.numpy(), dtype)
        err = rel_err(as_np(out), ref)
        assert err <= TOL[dtype], err


def test_expert_matmul_page_shape_sampled():
    # x[1024, 4096], expert_weight[8, 4096, 14336], int32 ids: the interface's own example
    T, H, I, E = 1024, 4096, 14336, 8
    x, w, ids = _matmul_inputs(T, H, I, E, "bf16", E, seed=4100)
    out, ws = B().expert_matmul(x.cuda(), w.cuda(), ids.cuda())
    assert B().device_status(ws) == B().OK
    toks = np.array([0, 1, 2, 511, 777, 1023])
    ref = O.expert_matmul(as_np(x[toks]), as_np(w), ids.numpy()[toks], "bf16")
    err = rel_err(as_np(out[torch.from_numpy(toks)]), ref)
    assert err <= TOL["bf16"], err


def test_expert_matmul_bad_id_gives_zero_row_and_status():
    T, H, I, E = 64, 128, 64, 4
    x, w, ids = _matmul_inputs(T, H, I, E, "bf16", E, seed=4200)
    ids[5] = E          # out of range: an error, never clamped
    ids[9] = -1
    out, ws = B().expert_matmul(x.cuda(), w.cuda(), ids.cuda())
    assert B().device_status(ws) == B().ERR_INDEX_OUT_OF_RANGE
    got = as_np(out)
    assert np.all(got[[5, 9]] == 0)
    keep = np.setdiff1d(np.arange(T), [5, 9])
    ref = O.expert_matmul(as_np(x[torch.from_numpy(keep)]), as_np(w), ids.numpy()[keep], "bf16")
    assert rel_err(got[keep], ref) <= TOL["bf16"]
