"""The pins are strong enough: each test here plants one plausible mistake in
the numpy oracle (on the CPU, through monkeypatch, undone afterwards) and
checks that the pin guarding that step fails on it."""
import math

import numpy as np
import pytest

from oracle import moe_oracle as PY
from tests import test_oracle_pins as P

_orig = {name: getattr(PY, name) for name in dir(PY) if not name.startswith("__")}


def _round_truncating(a):
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)
    e = np.maximum(e, -125)
    return np.where(np.isfinite(a), np.ldexp(np.trunc(np.ldexp(a, 8 - e)), e - 8), a)


def _logits_without_bias(x, w_gate, gate_bias=None):
    return _orig["router_logits"](x, w_gate, None)


def _topk_ascending(logits, k):
    idx = _orig["topk_select"](logits, logits.shape[1])
    return np.ascontiguousarray(idx[:, ::-1][:, :k])


def _topk_high_id_ties(logits, k):
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    out = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        out[t] = sorted(range(E), key=lambda e: (-float(lg[t, e]), -e))[:k]
    return out


def _gates_not_renormalised(logits, idx):
    lg = np.asarray(logits, dtype=np.float64)
    p = np.exp(lg - lg.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    return np.take_along_axis(p, np.asarray(idx, dtype=np.int64), 1).astype(np.float32)


def _gates_wrong_sign(logits, idx):
    lg = np.asarray(logits, dtype=np.float64)
    sel = np.take_along_axis(lg, np.asarray(idx, dtype=np.int64), 1)
    z = np.exp(sel[:, :1] - sel)
    return (z / z.sum(1, keepdims=True)).astype(np.float32)


def _capacity_floor(cf, T, k, E):
    cf = float(np.float32(cf))
    return None if cf <= 0 else int(math.floor(cf * T * k / E))


def _permute_last_come_first_kept(idx, E, cap=None, empty_slots=False):
    idx = np.asarray(idx)
    T, k = idx.shape
    rev = _orig["permute"](idx[::-1].copy(), E, cap, empty_slots)
    # map the reversed walk back: keep what the reversed walk kept
    kept_pairs = rev["row_map"][::-1] >= 0
    ids = np.where(kept_pairs, idx, -1)
    return _orig["permute"](ids, E, None, True)


def _permute_unstable(idx, E, cap=None, empty_slots=False):
    p = _orig["permute"](idx, E, cap, empty_slots)
    rt, rs, rm = p["row_token"].copy(), p["row_slot"].copy(), p["row_map"].copy()
    for e in range(E):
        a, b = int(p["offsets"][e]), int(p["offsets"][e + 1])
        rt[a:b], rs[a:b] = rt[a:b][::-1].copy(), rs[a:b][::-1].copy()
    for r in range(len(rt)):
        rm[rt[r], rs[r]] = r
    return {**p, "row_token": rt, "row_slot": rs, "row_map": rm}


def _gelu_tanh(z):
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)))


def _ffn_w1_w3_swapped(x_rows, w1_e, w3_e, w2_e, act, dtype):
    if act == "swiglu":
        return _orig["expert_ffn"](x_rows, w3_e, w1_e, w2_e, act, dtype)
    return _orig["expert_ffn"](x_rows, w1_e, w3_e, w2_e, act, dtype)


def _combine_slots_crossed(y, gates, row_map, dtype):
    g = np.asarray(gates)
    return _orig["combine"](y, g[:, ::-1].copy(), row_map, dtype)


def _combine_renormalised_after_drop(y, gates, row_map, dtype):
    g = np.asarray(gates, dtype=np.float64) * (np.asarray(row_map) >= 0)
    s = g.sum(1, keepdims=True)
    g = np.where(s > 0, g / np.where(s > 0, s, 1), 0)
    return _orig["combine"](y, g.astype(np.float32), row_map, dtype)


def _threshold_inverted(logits, k_max, delta=None):
    sel = _orig["threshold_select"](-np.asarray(logits, dtype=np.float32), k_max, delta)
    return sel


def _stats_from_topk_gates(logits, idx, E):
    st = _orig["router_load_stats"](logits, idx, E)
    g = _orig["topk_gates"](logits, idx)
    pm = np.zeros(E)
    np.add.at(pm, np.asarray(idx).ravel(), np.asarray(g, dtype=np.float64).ravel())
    return {**st, "prob_mean": pm / len(idx)}


def _matmul_wrong_expert(x, w, ids, dtype):
    E = np.asarray(w).shape[0]
    return _orig["expert_matmul"](x, w, (np.asarray(ids) + 1) % E, dtype)


MUTATIONS = [
    ("round_to_bf16", _round_truncating, P.test_bf16_rounding_golden, {}),
    ("router_logits", _logits_without_bias, P.test_router_logits_orientation_and_bias_exact, {}),
    ("topk_select", _topk_ascending, P.test_topk_matches_bruteforce, {"E": 5}),
    ("topk_select", _topk_high_id_ties, P.test_topk_k1_is_argmax_with_low_id_ties, {}),
    ("topk_gates", _gates_not_renormalised, P.test_gates_sum_to_one_and_closed_forms, {}),
    ("topk_gates", _gates_wrong_sign, P.test_gates_equal_full_softmax_then_renormalise, {}),
    ("capacity", _capacity_floor, P.test_capacity_values, {}),
    ("permute", _permute_last_come_first_kept, P.test_permute_invariants, {"cf": 0.5}),
    ("permute", _permute_unstable, P.test_permute_no_limit_is_stable_sort_by_expert, {}),
    ("gelu", _gelu_tanh, P.test_activations_match_library, {}),
    ("expert_ffn", _ffn_w1_w3_swapped, P.test_single_expert_k1_equals_dense_ffn, {"act": "swiglu"}),
    ("combine", _combine_slots_crossed, P.test_layer_matches_per_token_pseudocode, {}),
    ("combine", _combine_renormalised_after_drop,
     P.test_identity_experts_give_x_times_kept_gate_sum, {}),
    ("threshold_select", _threshold_inverted, P.test_threshold_select_matches_definition,
     {"E": 8, "k_max": 3}),
    ("router_load_stats", _stats_from_topk_gates,
     P.test_load_stats_match_library_softmax_and_closed_forms, {}),
    ("expert_matmul", _matmul_wrong_expert, P.test_expert_matmul_matches_per_token_library_matmul,
     {"dtype": "f32"}),
]


@pytest.mark.parametrize("target,mutant,pin,kw", MUTATIONS,
                         ids=[f"{m[0]}:{m[1].__name__.lstrip('_')}" for m in MUTATIONS])
def test_pin_catches_planted_mistake(target, mutant, pin, kw, monkeypatch):
    pin(PY, **kw)                       # the pin passes on the oracle as written
    monkeypatch.setattr(PY, target, mutant)
    with pytest.raises((AssertionError, ValueError, IndexError)):
        pin(PY, **kw)
