"""Parity of the rows built past the layer itself: the router's load statistics
(moe_route_stats), the one-expert-per-token matmul (moe_expert_matmul) and
threshold gating (moe_threshold_select, moe_forward_threshold), each against
both CPU oracles."""
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from oracle import moe_oracle_cpp as OC
from routing_grouped_expert_moe_b200 import synth
from tests.helpers import TOL, Guarded, as_np, gapped_inputs, guarded_workspace, rel_err

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
    wsg = guarded_workspace(B()._lib.moe_route_stats_workspace_bytes(cfg.T, cfg.E))
    idx, gate, counts, prob, ws = B().route_stats(x, wg, b, cfg.top_k, ws=wsg.t)
    assert B().device_status(ws) == B().OK
    wsg.check("workspace")
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
    og = Guarded((T, I), x.dtype)
    wsg = guarded_workspace(B()._lib.moe_expert_matmul_workspace_bytes(T, H, I, E,
                                                                       B()._dt(x)))
    out, ws = B().expert_matmul(x.cuda(), w.cuda(), ids.cuda(), out=og.t, ws=wsg.t)
    assert B().device_status(ws) == B().OK
    og.check("out")
    wsg.check("workspace")
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


# ---------------------------------------------------------------- threshold gating

@pytest.mark.parametrize("E,k_max", [(8, 4), (32, 8), (128, 8), (5, 5)])
def test_threshold_select_from_logits(E, k_max):
    from tests.helpers import threshold_margin_violations
    T = 3000
    delta = float(np.float32(1.0 / E))
    lg = synth.random_logits(5000 + E, T, E, scale=2.0).numpy()
    for attempt in range(20):                         # keep probabilities away from delta
        bad = threshold_margin_violations(lg, delta)
        if len(bad) == 0:
            break
        lg[bad] = synth.random_logits(5100 + attempt, len(bad), E, scale=2.0).numpy()
    assert len(threshold_margin_violations(lg, delta)) == 0
    idx, gate, n, offs = B().threshold_select(torch.from_numpy(lg).cuda(), k_max, token_offsets=True)
    for orc in (O, OC):
        ref = orc.threshold_select(lg, k_max)
        np.testing.assert_array_equal(as_np(idx), ref["topk_idx"])
        np.testing.assert_array_equal(as_np(n), ref["n_sel"])
        assert np.max(np.abs(as_np(gate) - ref["topk_gate"])) <= 1e-6
    np.testing.assert_array_equal(as_np(offs), np.concatenate([[0], np.cumsum(as_np(n))]))
    assert 1 <= as_np(n).min() and as_np(n).max() <= k_max


THR_CFGS = [
    (replace(synth.CONFIGS["mixtral_e8"], name="thr_e8", T=400, H=256, F=384, seed=6001), 4, 0.0),
    (replace(synth.CONFIGS["e32_long"], name="thr_e32", T=600, H=128, F=136, seed=6002), 8, 0.0),
    (replace(synth.CONFIGS["page1_gelu"], name="thr_gelu_cap", T=512, H=256, F=256, seed=6003), 3,
     0.9),
    (synth.CONFIGS["tiny_f32"], 3, 0.0),
]


@pytest.mark.parametrize("cfg,k_max,cf", THR_CFGS, ids=lambda c: getattr(c, "name", str(c)))
def test_forward_threshold(cfg, k_max, cf):
    from tests.helpers import threshold_inputs
    delta = float(np.float32(1.0 / cfg.E))
    d = threshold_inputs(cfg, delta, k_max)
    g = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    ig = Guarded((cfg.T, k_max), torch.int32)
    ng = Guarded((cfg.T,), torch.int32)
    og = Guarded((cfg.T, cfg.H), cfg.torch_dtype)
    wsg = guarded_workspace(B()._lib.moe_forward_threshold_workspace_bytes(
        cfg.T, cfg.H, cfg.F, cfg.E, k_max, B().ACT[cfg.act], B()._dt(d["x"])))
    idx, n = ig.t, ng.t
    out, ws = B().forward_threshold(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"],
                                    k_max, 0.0, cf, cfg.act, out=og.t, ws=wsg.t,
                                    topk_idx_out=idx, n_selected_out=n)
    assert B().device_status(ws) == B().OK
    for buf, name in ((ig, "topk_idx"), (ng, "n_selected"), (og, "out"), (wsg, "workspace")):
        buf.check(name)
    f = lambda t: None if t is None else as_np(t)  # noqa: E731
    for orc in (O, OC):
        ref = orc.moe_forward_threshold(f(d["x"]), f(d["w_gate"]), f(d["gate_bias"]), f(d["w1"]),
                                        f(d["w3"]), f(d["w2"]), k_max, None, cf, cfg.act, cfg.dtype)
        np.testing.assert_array_equal(as_np(idx), ref["topk_idx"])
        np.testing.assert_array_equal(as_np(n), ref["n_sel"])
        err = rel_err(as_np(out), ref["out"])
        assert err <= TOL[cfg.dtype], err
    nn = as_np(n)
    assert nn.min() >= 1 and (nn.max() > 1 or k_max == 1)
