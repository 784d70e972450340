"""The C++ CPU oracle (moe_oracle.cpp) behind the numpy oracle's function names.

TEST INFRASTRUCTURE.  Argument marshalling only: every step of the layer runs in
the C++ library (plain loops, float64 sums, OpenMP over rows).  Only the test
suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use
it; the product path never does.  It shares nothing with the CUDA path and does
not import the numpy oracle either, so the two oracles check each other.

The passages each function restates are cited in moe_oracle.cpp; the function
names, arguments and returned dicts are those of moe_oracle.py.  x and the
weights are handed over as float32 (the storage values of the layer's bf16 or
fp32 tensors are exact there); results are float64.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libmoe_oracle.so")


def _load():
    if not os.path.exists(LIB_PATH):
        from oracle import build_oracle
        build_oracle.build()
    return ctypes.CDLL(LIB_PATH)


_lib = _load()
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
for _name, _args in {
    "oracle_round_bf16": [_P, _I64, _P],
    "oracle_router_logits": [_P, _P, _P, _I, _I, _I, _P],
    "oracle_topk_select": [_P, _I, _I, _I, _P],
    "oracle_topk_gates": [_P, _P, _I, _I, _I, _P],
    "oracle_topk_gates_literal": [_P, _P, _I, _I, _I, _P],
    "oracle_capacity": [ctypes.c_float, _I, _I, _I, _P],
    "oracle_permute": [_P, _I, _I, _I, _I64, _I, _P, _P, _P, _P, _P, _P, _P],
    "oracle_threshold_select": [_P, _I, _I, _I, ctypes.c_float, _P, _P, _P],
    "oracle_grouped_ffn": [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I, _I, _P],
    "oracle_combine": [_P, _I, _P, _P, _I, _I, _I, _P],
    "oracle_activation": [_P, _I64, _I, _P],
    "oracle_router_prob_mean": [_P, _I, _I, _P],
    "oracle_expert_matmul": [_P, _P, _P, _I, _I, _I, _I, _I, _P],
    "oracle_num_threads": [],
}.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int

_DT = {"f32": 0, "bf16": 1}
_ACT = {"swiglu": 0, "gelu": 1, "identity": 2}


class IndexOutOfRange(ValueError):
    """An expert id outside [0, E): an error, never clamped."""


def _c(a, dtype):
    """A C-contiguous array of dtype (a copy only when needed) and its pointer."""
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(_P)


def _check(st, what):
    if st == 2:
        raise IndexOutOfRange("expert id outside [0, E)")
    if st != 0:
        raise ValueError(f"{what}: bad argument")


def num_threads() -> int:
    return int(_lib.oracle_num_threads())


def round_to_bf16(a) -> np.ndarray:
    a, pa = _c(a, np.float64)
    out = np.empty_like(a)
    _check(_lib.oracle_round_bf16(pa, a.size, out.ctypes.data_as(_P)), "round_to_bf16")
    return out


def round_to_f32(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to(dtype: str, a) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16(a)
    if dtype == "f32":
        return round_to_f32(a)
    raise ValueError(dtype)


def router_logits(x, w_gate, gate_bias=None) -> np.ndarray:
    x, px = _c(x, np.float32)
    w, pw = _c(w_gate, np.float32)
    T, H = x.shape
    E = w.shape[1]
    pb = None
    if gate_bias is not None:
        b, pb = _c(gate_bias, np.float32)
    out = np.empty((T, E), dtype=np.float32)
    _check(_lib.oracle_router_logits(px, pw, pb, T, H, E, out.ctypes.data_as(_P)), "router_logits")
    return out


def topk_select(logits, k: int) -> np.ndarray:
    lg, pl = _c(logits, np.float32)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("top_k must lie in [1, E]")
    idx = np.empty((T, k), dtype=np.int32)
    _check(_lib.oracle_topk_select(pl, T, E, k, idx.ctypes.data_as(_P)), "topk_select")
    return idx


def topk_gates(logits, idx) -> np.ndarray:
    lg, pl = _c(logits, np.float32)
    ix, pi = _c(idx, np.int32)
    T, E = lg.shape
    k = ix.shape[1]
    g = np.empty((T, k), dtype=np.float32)
    _check(_lib.oracle_topk_gates(pl, pi, T, E, k, g.ctypes.data_as(_P)), "topk_gates")
    return g


def topk_gates_literal(logits, idx) -> np.ndarray:
    lg, pl = _c(logits, np.float32)
    ix, pi = _c(idx, np.int32)
    T, E = lg.shape
    k = ix.shape[1]
    g = np.empty((T, k), dtype=np.float64)
    _check(_lib.oracle_topk_gates_literal(pl, pi, T, E, k, g.ctypes.data_as(_P)),
           "topk_gates_literal")
    return g


def capacity(capacity_factor: float, T: int, k: int, E: int):
    cap = np.zeros(1, dtype=np.int64)
    _check(_lib.oracle_capacity(ctypes.c_float(capacity_factor), T, k, E, cap.ctypes.data_as(_P)),
           "capacity")
    return None if cap[0] < 0 else int(cap[0])


def permute(idx, E: int, cap=None, empty_slots: bool = False) -> dict:
    ix, pi = _c(idx, np.int32)
    T, k = ix.shape
    n = T * k
    counts = np.zeros(E, dtype=np.int64)
    kept = np.zeros(E, dtype=np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    row_token = np.full(max(n, 1), -1, dtype=np.int64)
    row_slot = np.full(max(n, 1), -1, dtype=np.int64)
    row_map = np.full((T, k), -1, dtype=np.int64)
    R = np.zeros(1, dtype=np.int64)
    p = lambda a: a.ctypes.data_as(_P)  # noqa: E731
    _check(_lib.oracle_permute(pi, T, k, E, -1 if cap is None else int(cap), int(empty_slots),
                               p(counts), p(kept), p(offsets), p(row_token), p(row_slot),
                               p(row_map), p(R)), "permute")
    R = int(R[0])
    return {"counts": counts, "kept": kept, "offsets": offsets, "row_token": row_token[:R].copy(),
            "row_slot": row_slot[:R].copy(), "row_map": row_map,
            "dropped": int(counts.sum() - R), "R": R}


def expert_counts(idx, E: int, empty_slots: bool = False) -> np.ndarray:
    return permute(idx, E, None, empty_slots)["counts"]


def threshold_select(logits, k_max: int, delta=None) -> dict:
    lg, pl = _c(logits, np.float32)
    T, E = lg.shape
    if not 1 <= k_max <= E:
        raise ValueError("k_max must lie in [1, E]")
    idx = np.empty((T, k_max), dtype=np.int32)
    gate = np.empty((T, k_max), dtype=np.float32)
    n_sel = np.empty(T, dtype=np.int32)
    d = 0.0 if delta is None else float(delta)
    p = lambda a: a.ctypes.data_as(_P)  # noqa: E731
    _check(_lib.oracle_threshold_select(pl, T, E, k_max, ctypes.c_float(d), p(idx), p(gate),
                                        p(n_sel)), "threshold_select")
    return {"topk_idx": idx, "topk_gate": gate, "n_sel": n_sel}


def moe_forward_threshold(x, w_gate, gate_bias, w1, w3, w2, k_max: int, delta,
                          capacity_factor: float, act: str, dtype: str, logits=None) -> dict:
    x = np.asarray(x)
    T = x.shape[0]
    if logits is None:
        logits = router_logits(x, w_gate, gate_bias)
    E = logits.shape[1]
    sel = threshold_select(logits, k_max, delta)
    cap = capacity(capacity_factor, T, k_max, E)
    perm = permute(sel["topk_idx"], E, cap, empty_slots=True)
    y = grouped_ffn(x, perm, w1, w3, w2, act, dtype, E)
    out = combine(y, sel["topk_gate"], perm["row_map"], dtype)
    return {"logits": logits, **sel, "capacity": cap, "y": y, "out": out, **perm}


def _activation(z, which: int) -> np.ndarray:
    z, pz = _c(z, np.float64)
    out = np.empty_like(z)
    _check(_lib.oracle_activation(pz, z.size, which, out.ctypes.data_as(_P)), "activation")
    return out


def silu(z) -> np.ndarray:
    return _activation(z, 0)


def gelu(z) -> np.ndarray:
    return _activation(z, 1)


def grouped_ffn(x, perm: dict, w1, w3, w2, act: str, dtype: str, E: int) -> np.ndarray:
    x, px = _c(x, np.float32)
    T, H = x.shape
    R = int(perm["R"])
    offs, po = _c(perm["offsets"], np.int64)
    rt, pr = _c(perm["row_token"] if R else np.zeros(1), np.int64)
    F = 0
    ptrs = []
    keep = []
    for w in (w1, w3, w2):
        if w is None:
            ptrs.append(None)
        else:
            a, pa = _c(w, np.float32)
            keep.append(a)
            ptrs.append(pa)
    if w1 is not None:
        F = np.asarray(w1).shape[2]
    y = np.zeros((max(R, 1), H), dtype=np.float64)
    _check(_lib.oracle_grouped_ffn(px, T, H, F, E, po, pr, ptrs[0], ptrs[1], ptrs[2], _ACT[act],
                                   _DT[dtype], y.ctypes.data_as(_P)), "grouped_ffn")
    return y[:R]


def combine(y, gates, row_map, dtype: str) -> np.ndarray:
    y = np.asarray(y, dtype=np.float64)
    rm, pm = _c(row_map, np.int64)
    g, pg = _c(gates, np.float32)
    T, k = rm.shape
    H = y.shape[1] if y.ndim == 2 else 0
    yy, py = _c(y if y.size else np.zeros((1, max(H, 1))), np.float64)
    out = np.zeros((T, H), dtype=np.float64)
    _check(_lib.oracle_combine(py, H, pg, pm, T, k, _DT[dtype], out.ctypes.data_as(_P)), "combine")
    return out


def router_load_stats(logits, idx, E: int) -> dict:
    lg, pl = _c(logits, np.float32)
    T = lg.shape[0]
    prob = np.zeros(E, dtype=np.float64)
    _check(_lib.oracle_router_prob_mean(pl, T, E, prob.ctypes.data_as(_P)), "router_load_stats")
    return {"counts": expert_counts(idx, E), "prob_mean": prob}


def expert_matmul(x, expert_weight, token_expert_idx, dtype: str) -> np.ndarray:
    x, px = _c(x, np.float32)
    w, pw = _c(expert_weight, np.float32)
    ids, pi = _c(token_expert_idx, np.int32)
    T, H = x.shape
    E, _, I = w.shape
    out = np.zeros((T, I), dtype=np.float64)
    _check(_lib.oracle_expert_matmul(px, pw, pi, T, H, I, E, _DT[dtype], out.ctypes.data_as(_P)),
           "expert_matmul")
    return out


def moe_forward(x, w_gate, gate_bias, w1, w3, w2, top_k: int, capacity_factor: float,
                act: str, dtype: str, logits=None) -> dict:
    x = np.asarray(x)
    T = x.shape[0]
    if logits is None:
        logits = router_logits(x, w_gate, gate_bias)
    E = logits.shape[1]
    idx = topk_select(logits, top_k)
    gates = topk_gates(logits, idx)
    cap = capacity(capacity_factor, T, top_k, E)
    perm = permute(idx, E, cap)
    y = grouped_ffn(x, perm, w1, w3, w2, act, dtype, E)
    out = combine(y, gates, perm["row_map"], dtype)
    return {"logits": logits, "topk_idx": idx, "topk_gate": gates, "capacity": cap,
            "y": y, "out": out, **perm}


def moe_forward_sampled(x, logits, w1, w3, w2, top_k: int, capacity_factor: float,
                        act: str, dtype: str, tokens) -> dict:
    """Output rows for a sample of tokens: routing and the permutation for all
    tokens, the expert FFN and the combine only for the sampled tokens' rows."""
    x = np.asarray(x)
    T, E = logits.shape
    idx = topk_select(logits, top_k)
    gates = topk_gates(logits, idx)
    cap = capacity(capacity_factor, T, top_k, E)
    perm = permute(idx, E, cap)
    tokens = np.asarray(tokens, dtype=np.int64)
    # a small permutation holding only the sampled tokens' kept rows, expert-major
    rows = [(int(idx[t, s]), i, s) for i, t in enumerate(tokens) for s in range(top_k)
            if perm["row_map"][t, s] >= 0]
    rows.sort()
    sub_offsets = np.zeros(E + 1, dtype=np.int64)
    for e, _, _ in rows:
        sub_offsets[e + 1] += 1
    sub_offsets = np.cumsum(sub_offsets)
    sub = {"offsets": sub_offsets, "row_token": np.array([i for _, i, _ in rows], dtype=np.int64),
           "R": len(rows)}
    xs = np.stack([np.asarray(x[t], dtype=np.float32) for t in tokens]) if len(tokens) else \
        np.zeros((0, x.shape[1]), dtype=np.float32)
    ys = grouped_ffn(xs, sub, w1, w3, w2, act, dtype, E)
    sub_map = np.full((len(tokens), top_k), -1, dtype=np.int64)
    for r, (_, i, s) in enumerate(rows):
        sub_map[i, s] = r
    out_rows = combine(ys, gates[tokens], sub_map, dtype)
    return {"topk_idx": idx, "topk_gate": gates, "capacity": cap, "out_rows": out_rows,
            "tokens": tokens, **perm}
