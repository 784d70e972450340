"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test ties one oracle function to brute force, a closed form, a library
routine on a special case, or a hand-derived fixture under tests/golden/, so
that a dropped term, a wrong sign or index, or a transposed operand fails.
"""
import json
import math
import os
from itertools import combinations

import numpy as np
import pytest
import torch
from scipy.special import expit, softmax

from oracle import moe_oracle as PY
from oracle import moe_oracle_cpp as CPP

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


@pytest.fixture(params=["numpy", "cpp"])
def O(request):
    """Every pin runs on both oracles: the numpy one and the plain C++ one."""
    return PY if request.param == "numpy" else CPP


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- rounding

def test_bf16_rounding_golden(O):
    for c in _load("bf16_rounding_cases.json")["cases"]:
        got = float(O.round_to_bf16(np.array([c["value"]]))[0])
        assert got == c["expect"], c


def test_bf16_rounding_matches_library_on_fp32_values(O):
    # fp32 -> bf16 is a single rounding in torch (round to nearest even), so on
    # values exactly representable in fp32 the oracle's one-step rounding must agree.
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        rng.integers(-70000, 70000, 5000).astype(np.float64),
    ]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_to_bf16(v.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_rounding_subnormal_and_overflow(O):
    assert O.round_to_bf16(np.array([2.0 ** -133]))[0] == 2.0 ** -133
    assert O.round_to_bf16(np.array([2.0 ** -135]))[0] == 0.0          # below half spacing
    assert math.isinf(O.round_to_bf16(np.array([3.5e38]))[0])
    big = float(torch.tensor(3.38e38).to(torch.bfloat16).item())
    assert O.round_to_bf16(np.array([big]))[0] == big


# ---------------------------------------------------------------- logits

def test_router_logits_match_library_matmul(O):
    x = torch.randn(37, 96, dtype=torch.float64).to(torch.bfloat16).to(torch.float64)
    w = torch.randn(96, 5, dtype=torch.float64).to(torch.bfloat16).to(torch.float64)
    b = torch.randn(5, dtype=torch.float64).float().double()
    ref = (x @ w + b).float().numpy()
    got = O.router_logits(x.numpy(), w.numpy(), b.numpy())
    np.testing.assert_array_equal(got, ref)


def test_router_logits_orientation_and_bias_exact(O):
    # Integer inputs: every partial sum is exact, so the result is known exactly.
    x = np.array([[1, 2, 3]], dtype=np.float64)             # [T=1, H=3]
    w = np.array([[1, 0], [0, 1], [1, 1]], dtype=np.float64)  # [H=3, E=2]
    got = O.router_logits(x, w, np.array([0.5, -1.0]))
    np.testing.assert_array_equal(got, np.array([[4.5, 4.0]], dtype=np.float32))


# ---------------------------------------------------------------- top-k

@pytest.mark.parametrize("E", [2, 3, 4, 5, 6, 8])
def test_topk_matches_bruteforce(O, E):
    for k in range(1, min(3, E) + 1):
        lg = rng.standard_normal((200, E)).astype(np.float32)
        idx = O.topk_select(lg, k)
        for t in range(lg.shape[0]):
            assert tuple(idx[t]) == PY.topk_select_bruteforce(lg[t], k)
            # independent check: the chosen set has the largest sum over all subsets
            best = max(combinations(range(E), k), key=lambda s: sum(float(lg[t, e]) for e in s))
            assert set(idx[t]) == set(best)


def test_topk_k_equals_E_is_descending_sort(O):
    lg = rng.standard_normal((50, 7)).astype(np.float32)
    idx = O.topk_select(lg, 7)
    np.testing.assert_array_equal(idx, np.argsort(-lg, axis=1, kind="stable"))


def test_topk_k1_is_argmax_with_low_id_ties(O):
    lg = rng.integers(0, 3, (300, 6)).astype(np.float32)     # many ties
    idx = O.topk_select(lg, 1)
    np.testing.assert_array_equal(idx[:, 0], np.argmax(lg, axis=1))


def test_topk_ties_and_nan(O):
    lg = np.array([[1.0, 2.0, 2.0, 0.5],
                   [np.nan, -np.inf, 1.0, np.nan]], dtype=np.float32)
    idx = O.topk_select(lg, 4)
    assert list(idx[0]) == [1, 2, 0, 3]
    assert list(idx[1]) == [2, 1, 0, 3]


# ---------------------------------------------------------------- gates

def test_gates_sum_to_one_and_closed_forms(O):
    lg = (rng.standard_normal((500, 8)) * 3).astype(np.float32)
    for k in (1, 2, 3):
        idx = O.topk_select(lg, k)
        g = O.topk_gates(lg, idx).astype(np.float64)
        assert np.all(np.abs(g.sum(1) - 1.0) <= 1e-6)
        assert np.all(g[:, :-1] >= g[:, 1:])          # descending, like the logits
        if k == 1:
            np.testing.assert_array_equal(g[:, 0], 1.0)
        if k == 2:
            sel = np.take_along_axis(lg.astype(np.float64), idx.astype(np.int64), 1)
            np.testing.assert_allclose(g[:, 0], expit(sel[:, 0] - sel[:, 1]), rtol=1e-7)


def test_gates_equal_full_softmax_then_renormalise(O):
    lg = (rng.standard_normal((300, 16)) * 2).astype(np.float32)
    idx = O.topk_select(lg, 2)
    p = softmax(lg.astype(np.float64), axis=1)               # library softmax over all E
    sel = np.take_along_axis(p, idx.astype(np.int64), 1)
    ref = sel / sel.sum(1, keepdims=True)
    np.testing.assert_allclose(O.topk_gates(lg, idx), ref, rtol=1e-7, atol=0)
    np.testing.assert_allclose(O.topk_gates_literal(lg, idx), ref, rtol=1e-12, atol=0)


# ---------------------------------------------------------------- dispatch

def test_capacity_values(O):
    assert O.capacity(1.2, 4096, 2, 8) == 1229
    assert O.capacity(1.25, 32768, 2, 32) == 2560
    assert O.capacity(0.5, 512, 2, 8) == 64
    assert O.capacity(1.0, 8, 1, 2) == 4
    assert O.capacity(0.0, 8, 1, 2) is None
    assert O.capacity(-1.0, 8, 1, 2) is None
    # the factor is the float32 the library receives: fp32(1.1) * 10 > 11
    assert O.capacity(1.1, 10, 1, 1) == 12
    assert O.capacity(1e-9, 8, 1, 2) == 1


@pytest.mark.parametrize("case", _load("capacity_cases.json")["cases"], ids=lambda c: c["name"])
def test_permute_golden(O, case):
    idx = np.array(case["topk_idx"], dtype=np.int32)
    cap = O.capacity(case["capacity_factor"], case["T"], case["k"], case["E"])
    assert cap == case["capacity"]
    p = O.permute(idx, case["E"], cap)
    for key in ("counts", "kept", "offsets", "row_token", "row_slot", "row_map"):
        np.testing.assert_array_equal(p[key], np.array(case[key]), err_msg=key)
    assert p["dropped"] == case["dropped"]


def test_counts_match_bincount(O):
    idx = rng.integers(0, 13, (1000, 3)).astype(np.int32)
    np.testing.assert_array_equal(O.expert_counts(idx, 13), np.bincount(idx.ravel(), minlength=13))


def test_index_out_of_range_is_an_error(O):
    with pytest.raises(O.IndexOutOfRange):
        O.permute(np.array([[0, 4]], dtype=np.int32), 4, None)
    with pytest.raises(O.IndexOutOfRange):
        O.permute(np.array([[-1, 1]], dtype=np.int32), 4, None)


def _distinct_ids(T, E, k, skew=0.0):
    w = np.exp(-skew * np.arange(E)); w /= w.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=w) for _ in range(T)]).astype(np.int32)


def test_permute_no_limit_is_stable_sort_by_expert(O):
    T, E, k = 400, 9, 3
    idx = _distinct_ids(T, E, k)
    p = O.permute(idx, E, None)
    order = np.argsort(idx.ravel(), kind="stable")            # library stable sort
    np.testing.assert_array_equal(p["row_token"], order // k)
    np.testing.assert_array_equal(p["row_slot"], order % k)
    assert p["dropped"] == 0


@pytest.mark.parametrize("cf", [0.0, 0.5, 0.8, 1.0, 1.3])
def test_permute_invariants(O, cf):
    T, E, k = 600, 8, 2
    idx = _distinct_ids(T, E, k, skew=0.3)
    cap = O.capacity(cf, T, k, E)
    p = O.permute(idx, E, cap)
    counts = np.bincount(idx.ravel(), minlength=E)
    np.testing.assert_array_equal(p["counts"], counts)
    kept_expected = counts if cap is None else np.minimum(counts, cap)
    np.testing.assert_array_equal(p["kept"], kept_expected)
    assert p["R"] == T * k - p["dropped"] == kept_expected.sum()
    assert np.all(np.diff(p["offsets"]) >= 0) and p["offsets"][0] == 0
    for e in range(E):
        seg = p["row_token"][p["offsets"][e]:p["offsets"][e + 1]]
        assert np.all(np.diff(seg) > 0)                          # stable, one row per token
        assert np.all(idx[seg, p["row_slot"][p["offsets"][e]:p["offsets"][e + 1]]] == e)
    # row_map o row_token is the identity on kept rows
    r = np.arange(p["R"])
    np.testing.assert_array_equal(p["row_map"][p["row_token"], p["row_slot"]], r)
    # drops are first-come: a dropped pair's expert already had C earlier pairs kept
    if cap is not None:
        for t, s in zip(*np.nonzero(p["row_map"] < 0)):
            e = idx[t, s]
            earlier = p["row_token"][p["offsets"][e]:p["offsets"][e + 1]]
            assert len(earlier) == cap and np.all(earlier < t + (s > 0))
    # permute then unpermute gives x back on every kept slot
    x = rng.standard_normal((T, 5))
    x_perm = x[p["row_token"]]
    for t in range(T):
        for s in range(k):
            if p["row_map"][t, s] >= 0:
                np.testing.assert_array_equal(x_perm[p["row_map"][t, s]], x[t])


# ---------------------------------------------------------------- expert FFN / combine

def test_activations_match_library(O):
    z = np.linspace(-8, 8, 1001)
    zt = torch.from_numpy(z)
    np.testing.assert_allclose(O.gelu(z), torch.nn.functional.gelu(zt).numpy(), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(O.silu(z), torch.nn.functional.silu(zt).numpy(), rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_single_expert_k1_equals_dense_ffn(O, act):
    # E=1, k=1, no capacity: every gate is 1 and the layer is the dense FFN.
    T, H, F = 33, 24, 40                                       # H != F: a transpose fails
    x = rng.standard_normal((T, H)).astype(np.float32).astype(np.float64)
    wg = rng.standard_normal((H, 1))
    w1 = rng.standard_normal((1, H, F)) / math.sqrt(H)
    w3 = rng.standard_normal((1, H, F)) / math.sqrt(H) if act == "swiglu" else None
    w2 = rng.standard_normal((1, F, H)) / math.sqrt(F)
    res = O.moe_forward(x, wg, None, w1, w3, w2, 1, 0.0, act, "f32")
    xt = torch.from_numpy(x)
    z1 = xt @ torch.from_numpy(w1[0])
    if act == "gelu":
        h = torch.nn.functional.gelu(z1)
    else:
        h = torch.nn.functional.silu(z1) * (xt @ torch.from_numpy(w3[0]))
    ref = (h.float().double() @ torch.from_numpy(w2[0])).numpy()
    np.testing.assert_array_equal(res["topk_gate"], 1.0)
    np.testing.assert_allclose(res["out"], ref, rtol=2e-6, atol=2e-6 * np.abs(ref).max())


def test_identity_experts_give_x_times_kept_gate_sum(O):
    T, H, E, k = 120, 16, 6, 2
    x = O.round_to_bf16(rng.standard_normal((T, H)))
    lg = rng.standard_normal((T, E)).astype(np.float32)
    for cf in (0.0, 0.6):
        res = O.moe_forward(x, None, None, None, None, None, k, cf, "identity", "f32", logits=lg)
        g = res["topk_gate"].astype(np.float64) * (res["row_map"] >= 0)
        ref = x * g.sum(1, keepdims=True)
        np.testing.assert_allclose(res["out"], ref, rtol=1e-7, atol=1e-7)
        if cf == 0.0:
            np.testing.assert_allclose(res["out"], x, rtol=1e-6, atol=1e-6)
        else:
            assert res["dropped"] > 0
            all_dropped = np.all(res["row_map"] < 0, axis=1)
            assert np.all(res["out"][all_dropped] == 0)


def test_combine_is_linear_in_y(O):
    T, H, k = 50, 8, 2
    row_map = np.arange(T * k).reshape(T, k)
    row_map[3, 1] = -1
    g = rng.random((T, k)).astype(np.float32)
    y1, y2 = rng.standard_normal((T * k, H)), rng.standard_normal((T * k, H))
    a, b = 0.75, -2.5
    lhs = O.combine(a * y1 + b * y2, g, row_map, "f32")
    rhs = a * O.combine(y1, g, row_map, "f32") + b * O.combine(y2, g, row_map, "f32")
    np.testing.assert_allclose(lhs, rhs, rtol=1e-5, atol=1e-5)


def test_layer_matches_per_token_pseudocode(O):
    """The grouped (permute -> expert loop -> combine) oracle equals the pages'
    per-token form: softmax over all experts, top-k, renormalise, sum of
    gate-weighted expert outputs — written here with torch float64 ops."""
    T, H, F, E, k = 40, 16, 24, 5, 2
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((H, E))
    w1 = rng.standard_normal((E, H, F)) / 4
    w3 = rng.standard_normal((E, H, F)) / 4
    w2 = rng.standard_normal((E, F, H)) / 5
    res = O.moe_forward(x, wg, None, w1, w3, w2, k, 0.0, "swiglu", "f32")
    xt, wgt = torch.from_numpy(x), torch.from_numpy(wg)
    for t in range(T):
        logits = (xt[t] @ wgt).float().double()
        p = torch.softmax(logits, 0)
        top = torch.topk(p, k)
        gates = top.values / top.values.sum()
        acc = torch.zeros(H, dtype=torch.float64)
        for gi, e in zip(gates, top.indices.tolist()):
            h = torch.nn.functional.silu(xt[t] @ torch.from_numpy(w1[e])) * (xt[t] @ torch.from_numpy(w3[e]))
            acc += gi * (h.float().double() @ torch.from_numpy(w2[e])).float().double()
        assert list(res["topk_idx"][t]) == top.indices.tolist()
        np.testing.assert_allclose(res["out"][t], acc.numpy(), rtol=1e-5, atol=1e-6)


def test_sampled_rows_equal_full_layer(O):
    T, H, F, E, k = 64, 16, 32, 4, 2
    x = O.round_to_bf16(rng.standard_normal((T, H)))
    wg = O.round_to_bf16(rng.standard_normal((H, E)) / 4)
    w1 = O.round_to_bf16(rng.standard_normal((E, H, F)) / 4)
    w2 = O.round_to_bf16(rng.standard_normal((E, F, H)) / 5)
    for cf in (0.0, 0.7):
        full = O.moe_forward(x, wg, None, w1, None, w2, k, cf, "gelu", "bf16")
        toks = np.array([0, 5, 17, 63])
        samp = O.moe_forward_sampled(x, full["logits"], w1, None, w2, k, cf, "gelu", "bf16", toks)
        np.testing.assert_array_equal(samp["out_rows"], full["out"][toks])


@pytest.mark.parametrize("act,cf", [("gelu", 0.6), ("swiglu", 0.0)])
def test_numpy_and_cpp_oracles_agree(act, cf):
    """The two oracles are written independently (numpy with library matmuls,
    C++ with plain loops): on the same bf16 inputs they agree exactly on every
    index, count and gate, and on the outputs up to the rare bf16 rounding
    decision that a different float64 summation order can flip."""
    T, H, F, E, k = 96, 64, 80, 8, 2
    x = PY.round_to_bf16(rng.standard_normal((T, H)))
    wg = PY.round_to_bf16(rng.standard_normal((H, E)) / 8)
    w1 = PY.round_to_bf16(rng.standard_normal((E, H, F)) / 8)
    w3 = PY.round_to_bf16(rng.standard_normal((E, H, F)) / 8) if act == "swiglu" else None
    w2 = PY.round_to_bf16(rng.standard_normal((E, F, H)) / 9)
    la, lb = PY.router_logits(x, wg), CPP.router_logits(x, wg)
    assert np.all(np.abs(la.astype(np.float64) - lb) <= np.spacing(np.abs(la)))
    a = PY.moe_forward(x, wg, None, w1, w3, w2, k, cf, act, "bf16", logits=la)
    b = CPP.moe_forward(x, wg, None, w1, w3, w2, k, cf, act, "bf16", logits=la)
    for key in ("topk_idx", "topk_gate", "counts", "kept", "offsets", "row_token", "row_slot",
                "row_map"):
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)
    assert a["capacity"] == b["capacity"] and a["dropped"] == b["dropped"]
    np.testing.assert_allclose(b["out"], a["out"], rtol=2.0 ** -7, atol=1e-30)
    assert np.mean(a["out"] == b["out"]) > 0.98


# ---------------------------------------------------------------- router load statistics

def test_load_stats_match_library_softmax_and_closed_forms(O):
    lg = (rng.standard_normal((400, 12)) * 2).astype(np.float32)
    idx = O.topk_select(lg, 2)
    st = O.router_load_stats(lg, idx, 12)
    np.testing.assert_array_equal(st["counts"], np.bincount(idx.ravel(), minlength=12))
    ref = softmax(lg.astype(np.float64), axis=1).mean(0)            # library softmax
    np.testing.assert_allclose(st["prob_mean"], ref, rtol=1e-12, atol=0)
    assert abs(st["prob_mean"].sum() - 1.0) <= 1e-12
    # equal logits: uniform
    flat = np.full((7, 5), 0.25, dtype=np.float32)
    np.testing.assert_allclose(O.router_load_stats(flat, O.topk_select(flat, 1), 5)["prob_mean"],
                               0.2, rtol=1e-15)
    # two experts: p_0 is the logistic function of the logit difference
    two = rng.standard_normal((300, 2)).astype(np.float32)
    p0 = O.router_load_stats(two, O.topk_select(two, 1), 2)["prob_mean"][0]
    np.testing.assert_allclose(p0, expit(two[:, 0].astype(np.float64) - two[:, 1]).mean(), rtol=1e-13)


# ---------------------------------------------------------------- one expert per token

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_expert_matmul_matches_per_token_library_matmul(O, dtype):
    T, H, I, E = 50, 24, 40, 5                                      # H != I: a transpose fails
    x = PY.round_to_bf16(rng.standard_normal((T, H)))
    w = PY.round_to_bf16(rng.standard_normal((E, H, I)) / 4)
    ids = rng.integers(0, E, T).astype(np.int32)
    ids[:3] = 2                                                      # and expert 4 maybe empty
    got = O.expert_matmul(x, w, ids, dtype)
    xt, wt = torch.from_numpy(x), torch.from_numpy(w)
    ref = torch.stack([xt[t] @ wt[int(ids[t])] for t in range(T)])
    ref = ref.float() if dtype == "f32" else ref.to(torch.bfloat16)
    np.testing.assert_allclose(got, ref.double().numpy(), rtol=2.0 ** -7 if dtype == "bf16" else 1e-6,
                               atol=0)
    assert np.mean(got == ref.double().numpy()) > 0.97


def test_expert_matmul_one_expert_is_dense_and_ids_are_checked(O):
    x = rng.standard_normal((9, 16)).astype(np.float32).astype(np.float64)
    w = rng.standard_normal((1, 16, 8)).astype(np.float32).astype(np.float64)
    got = O.expert_matmul(x, w, np.zeros(9, dtype=np.int32), "f32")
    np.testing.assert_allclose(got, (torch.from_numpy(x) @ torch.from_numpy(w[0])).float().numpy(),
                               rtol=1e-6)
    with pytest.raises(O.IndexOutOfRange):
        O.expert_matmul(x, w, np.array([0] * 8 + [1], dtype=np.int32), "f32")


# ---------------------------------------------------------------- threshold gating

def _threshold_reference(lg, k_max, delta):
    """The definition written with library calls: softmax (scipy), a stable sort
    by descending logit, the prefix of experts above delta (at least one)."""
    p = softmax(lg.astype(np.float64), axis=1)
    T, E = lg.shape
    order = np.argsort(-lg, axis=1, kind="stable")
    idx = np.full((T, k_max), -1)
    for t in range(T):
        n = 1
        while n < k_max and p[t, order[t, n]] > delta:
            n += 1
        idx[t, :n] = order[t, :n]
    return idx, p


@pytest.mark.parametrize("E,k_max", [(4, 4), (8, 3), (16, 8), (32, 8)])
def test_threshold_select_matches_definition(O, E, k_max):
    lg = (rng.standard_normal((300, E)) * 1.5).astype(np.float32)
    sel = O.threshold_select(lg, k_max)                              # default delta = 1/E
    idx_ref, p = _threshold_reference(lg, k_max, 1.0 / E)
    np.testing.assert_array_equal(sel["topk_idx"], idx_ref)
    np.testing.assert_array_equal(sel["n_sel"], (idx_ref >= 0).sum(1))
    g = sel["topk_gate"].astype(np.float64)
    kept = idx_ref >= 0
    assert np.all(np.abs(g.sum(1) - 1.0) <= 1e-6) and np.all(g[~kept] == 0)
    pk = np.where(kept, np.take_along_axis(p, np.maximum(idx_ref, 0), 1), 0.0)
    np.testing.assert_allclose(g, pk / pk.sum(1, keepdims=True), rtol=1e-6, atol=1e-7)


def test_threshold_select_limits(O):
    lg = rng.standard_normal((100, 6)).astype(np.float32)
    # delta >= 1: nothing exceeds it, so only the largest is kept, with gate 1
    one = O.threshold_select(lg, 4, 1.5)
    np.testing.assert_array_equal(one["n_sel"], 1)
    np.testing.assert_array_equal(one["topk_idx"][:, 0], np.argmax(lg, axis=1))
    np.testing.assert_array_equal(one["topk_gate"][:, 0], 1.0)
    # delta tiny and k_max = E: every expert kept, gates = the full softmax
    every = O.threshold_select(lg, 6, 1e-30)
    np.testing.assert_array_equal(every["topk_idx"], np.argsort(-lg, axis=1, kind="stable"))
    np.testing.assert_allclose(np.sort(every["topk_gate"], axis=1),
                               np.sort(softmax(lg.astype(np.float64), axis=1), axis=1), rtol=1e-6)


def test_threshold_forward_reduces_to_topk_when_all_pass(O):
    # delta tiny: every one of the k_max slots is used, so the layer is top-k_max gating
    T, H, F, E, k = 48, 16, 24, 6, 2
    x = PY.round_to_bf16(rng.standard_normal((T, H)))
    wg = PY.round_to_bf16(rng.standard_normal((H, E)) / 4)
    w1 = PY.round_to_bf16(rng.standard_normal((E, H, F)) / 4)
    w3 = PY.round_to_bf16(rng.standard_normal((E, H, F)) / 4)
    w2 = PY.round_to_bf16(rng.standard_normal((E, F, H)) / 5)
    thr = O.moe_forward_threshold(x, wg, None, w1, w3, w2, k, 1e-30, 0.0, "swiglu", "bf16")
    top = O.moe_forward(x, wg, None, w1, w3, w2, k, 0.0, "swiglu", "bf16")
    np.testing.assert_array_equal(thr["topk_idx"], top["topk_idx"])
    np.testing.assert_array_equal(thr["out"], top["out"])


def test_permute_empty_slots(O):
    idx = np.array([[1, -1, -1], [0, 2, -1], [2, 1, 0]], dtype=np.int32)
    p = O.permute(idx, 3, None, empty_slots=True)
    np.testing.assert_array_equal(p["counts"], [2, 2, 2])
    np.testing.assert_array_equal(p["row_token"], [1, 2, 0, 2, 1, 2])
    np.testing.assert_array_equal(p["row_map"], [[2, -1, -1], [0, 4, -1], [5, 3, 1]])
    assert p["dropped"] == 0 and p["R"] == 6
    with pytest.raises(O.IndexOutOfRange):
        O.permute(idx, 3, None)                                     # -1 is an error otherwise
