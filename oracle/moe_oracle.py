"""CPU oracle for the forward pass of one Mixture-of-Experts layer.

TEST INFRASTRUCTURE.  This is a plain, slow, obviously-correct restatement of
what the layer computes, used only to check the CUDA path.  Only the test suite,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import it;
the product path never does.  It shares no code with the CUDA path and imports
nothing from it.

Sources (the pages this restates):
  [P2] "MoE模型高效推理：CANN算子库优化实践" (intelliparadigm.com) — §2.1, the MoE
       layer pseudo-code: gates = softmax(x @ W_gate), pick the top-2 experts,
       sum gate-weighted expert outputs; §3.2.1: renormalise the kept gates.
  [P3] "ops-transformer 仓库 - MoE 算子优化实战" (gitcode.csdn.net) — "核心代码解析":
       MoEOperator::Forward = routing scores -> top-k -> for each expert: mask,
       SparseGather, expert forward, SparseScatterAdd.
  [P4] lshu.cn/news/82007, calling the MoE fused operators through torch_npu —
       §3: x[tokens, hidden], expert_weight[num_experts, hidden, intermediate],
       int32 token_expert_idx; §4: preprocess (permute) / matmul / postprocess;
       §5.2: indices must be int32 in [0, num_experts); §5.3: a fixed-size buffer
       per expert that skewed routing overflows.
  [P1] hnwysp.cn/news/132341 (ops-transformer MoE operators) — §3.2: top_k=2,
       capacity_factor=1.2 as an over-allocation coefficient.
  [P5] "ops-transformer 算子精讲：昇腾 NPU 上的注意力机制与融合算子实现" (mhpn.cn) —
       ch.8: moe_router(x, router_weight, expert_weights, top_k,
       normalize_scores=True, capacity_factor=1.2).

Readings where the pages are silent:
  * capacity C = ceil(cf*T*k/E) per expert per call, cf <= 0 meaning no limit
    (the hnwysp.cn article names only an over-allocation coefficient);
  * overflow dropped first come, first kept, in token order then slot order
    (the workloads state "overflow dropped in token-index order");
  * no second renormalisation after a drop: a dropped slot contributes nothing
    and a token whose every slot dropped gives a zero row;
  * selection on the fp32 logits (softmax is increasing, so the set and order
    are those of the probabilities), ties to the lower expert id, NaN below
    -inf, slot 0 = the largest logit;
  * exact erf GELU, z * Phi(z); SwiGLU = silu(x W1) * (x W3), no expert biases;
  * h, y and out rounded to the storage dtype (round to nearest even) where
    the layer stores them;
  * threshold gating keeps at most k_max experts, the largest always, and
    decides p > delta on the float64 softmax.

Arithmetic: every sum is float64.  Inputs arrive as float arrays holding the
exact stored values (bf16 and fp32 values are exact in float64).  Rounding to
the storage dtype happens only where the layer stores a tensor.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(brute force, closed forms, library special cases, hand-built fixtures).
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
from scipy.special import erfc as _erfc

# --------------------------------------------------------------------------
# Rounding to the storage dtype.
# --------------------------------------------------------------------------


def round_to_bf16(a) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), in one step.

    bf16 keeps 8 significant bits.  For a normal value v = m * 2**e with
    0.5 <= |m| < 1, the representable neighbours are multiples of 2**(e-8), so
    v rounds to rint(m * 2**8) * 2**(e-8) (np.rint rounds half to even).  The
    smallest normal bf16 exponent is -126 (spacing 2**-133 below it).
    """
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)
    e = np.maximum(e, -125)            # subnormal range: fixed spacing 2**-133
    q = np.rint(np.ldexp(a, 8 - e))
    r = np.ldexp(q, e - 8)
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, a), r)   # overflow
    return np.where(np.isfinite(a), r, a)


def round_to_f32(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to(dtype: str, a) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16(a)
    if dtype == "f32":
        return round_to_f32(a)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# Router: logits, top-k selection, renormalised gates.   [P2] §2.1, §3.2.1
# --------------------------------------------------------------------------


def router_logits(x, w_gate, gate_bias=None) -> np.ndarray:
    """logits[t,e] = fp32( sum_h x[t,h] * W_gate[h,e] + b[e] ), the sum in float64.

    [P2] §2.1: the gate scores are x @ W_gate.  The bias term (absent on the
    pages) is added before selection when the workload has one.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_gate, dtype=np.float64)
    l = x @ w
    if gate_bias is not None:
        l = l + np.asarray(gate_bias, dtype=np.float64)[None, :]
    return l.astype(np.float32)


def _rank_key(v: float):
    """Sort key: larger logit first; NaN ranks below -inf."""
    if math.isnan(v):
        return (1, 0.0)
    return (0, -v)


def topk_select(logits, k: int) -> np.ndarray:
    """Top-k expert ids per token, slot 0 = highest logit.

    [P2] §2.1 (top_k(gates, k=2)); [P3] TopKRouting.  Ties go to the lower expert
    id.  Selecting on logits picks the same set, in the same order, as selecting
    on softmax probabilities, because softmax is strictly increasing.
    """
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("top_k must lie in [1, E]")
    idx = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        row = [float(v) for v in lg[t]]
        order = sorted(range(E), key=lambda e: (_rank_key(row[e]), e))
        idx[t] = order[:k]
    return idx


def topk_select_bruteforce(logits_row, k: int) -> tuple:
    """Brute force for one token: the k-subset with the largest logit sum.

    Among subsets with equal sum the lexicographically smallest id list wins;
    the winner is returned in descending-logit order (ties: lower id first).
    Only for small E (it enumerates every k-subset).
    """
    from itertools import combinations
    row = [float(v) for v in logits_row]
    best, best_sum = None, None
    for sub in combinations(range(len(row)), k):
        s = sum(row[e] for e in sub)
        if best is None or s > best_sum:
            best, best_sum = sub, s
    return tuple(sorted(best, key=lambda e: (-row[e], e)))


def topk_gates(logits, idx) -> np.ndarray:
    """Renormalised gates g[t,s] = exp(l_s - l_0) / sum_j exp(l_j - l_0), j over the k kept.

    [P2] §2.1 applies softmax over all experts; §3.2.1 renormalises the kept
    ones; [P5] ch.8 normalize_scores=True.  The full softmax denominator cancels,
    so only the k selected logits matter.  Computed in float64, stored fp32.
    """
    lg = np.asarray(logits, dtype=np.float64)
    sel = np.take_along_axis(lg, np.asarray(idx, dtype=np.int64), axis=1)
    z = np.exp(sel - sel[:, :1])
    g = z / z.sum(axis=1, keepdims=True)
    return g.astype(np.float32)


def topk_gates_literal(logits, idx) -> np.ndarray:
    """The literal reading: p = softmax over all E, then p_s / sum of kept p (float64)."""
    lg = np.asarray(logits, dtype=np.float64)
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, np.asarray(idx, dtype=np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------
# Dispatch: counts, capacity, stable permutation.   [P4] §4, §5.2, §5.3; [P3]
# --------------------------------------------------------------------------


class IndexOutOfRange(ValueError):
    """An expert id outside [0, E): an error, never clamped ([P4] §5.2, §7)."""


def expert_counts(idx, E: int, empty_slots: bool = False) -> np.ndarray:
    """count[e] = number of (token, slot) pairs routed to expert e.

    With empty_slots, id -1 marks an unused slot (threshold gating) and is skipped.
    """
    idx = np.asarray(idx)
    flat = idx.reshape(-1)
    if empty_slots:
        flat = flat[flat != -1]
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise IndexOutOfRange("expert id outside [0, E)")
    c = np.zeros(E, dtype=np.int64)
    for e in flat:
        c[int(e)] += 1
    return c


def capacity(capacity_factor: float, T: int, k: int, E: int):
    """Per-expert capacity C = ceil(cf * T * k / E); None (no limit) when cf <= 0.

    [P1] §3.2 names capacity_factor an over-allocation coefficient over the fair
    share T*k/E; [P4] §5.3 describes the fixed per-expert buffer.  cf is taken
    as the float32 value the library receives and the ceiling is exact.
    """
    cf = float(np.float32(capacity_factor))
    if cf <= 0:
        return None
    q = Fraction(cf) * T * k / E
    return int(math.ceil(q))


def permute(idx, E: int, cap=None, empty_slots: bool = False) -> dict:
    """Stable, capacity-limited permutation of (token, slot) pairs into expert-major rows.

    Walk tokens t = 0..T-1 and, within a token, slots s = 0..k-1.  The pair
    (t, s) routed to e is kept when fewer than C pairs of e were kept before it
    (first come, first kept; [P4] §5.3 overflow of the fixed buffer).  Kept pairs
    of expert e occupy rows offsets[e] .. offsets[e+1]-1 in arrival order, so
    row_token is increasing inside each expert segment ([P3] SparseGather keeps
    token order within an expert).

    Returns counts (pre-drop), kept, offsets[E+1], row_token[R], row_slot[R],
    row_map[T,k] (row index or -1 when dropped) and the number dropped.  With
    empty_slots, slots holding id -1 are unused: not counted, not dropped,
    row_map -1 (threshold gating leaves a token's trailing slots empty).
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    counts = expert_counts(idx, E, empty_slots)
    limit = cap if cap is not None else T * k
    kept = np.zeros(E, dtype=np.int64)
    arrival = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):
        for s in range(k):
            e = int(idx[t, s])
            if e == -1 and empty_slots:
                continue
            if kept[e] < limit:
                arrival[t, s] = kept[e]
                kept[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + kept[e]
    R = int(offsets[E])
    row_token = np.full(R, -1, dtype=np.int64)
    row_slot = np.full(R, -1, dtype=np.int64)
    row_map = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):
        for s in range(k):
            if arrival[t, s] >= 0:
                r = offsets[int(idx[t, s])] + arrival[t, s]
                row_token[r] = t
                row_slot[r] = s
                row_map[t, s] = r
    used = int(counts.sum())
    return {"counts": counts, "kept": kept, "offsets": offsets, "row_token": row_token,
            "row_slot": row_slot, "row_map": row_map, "dropped": int(used - R), "R": R}


# --------------------------------------------------------------------------
# Expert FFN.   [P4] §3 (up-projection to intermediate, activation, down-projection)
# --------------------------------------------------------------------------


def gelu(z) -> np.ndarray:
    """Exact GELU: z * Phi(z) = 0.5 z (1 + erf(z / sqrt 2)), evaluated as
    0.5 z erfc(-z / sqrt 2) (the same function; 1 + erf(x) = erfc(-x) avoids the
    cancellation that loses all relative precision for z below about -5)."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * _erfc(-z / math.sqrt(2.0))


def silu(z) -> np.ndarray:
    """SiLU: z / (1 + exp(-z))."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def expert_ffn(x_rows, w1_e, w3_e, w2_e, act: str, dtype: str) -> np.ndarray:
    """One expert on a block of rows: y = act(x W1 [, x W3]) W2.

    [P4] §3: x[tokens, hidden] times expert_weight[hidden, intermediate], then an
    activation and the down-projection.  GELU: h = gelu(x W1).  SwiGLU:
    h = silu(x W1) * (x W3).  "identity": y = x (test experts).  h and y are
    rounded to the storage dtype where the layer stores them.
    """
    x = np.asarray(x_rows, dtype=np.float64)
    if act == "identity":
        return x.copy()
    z1 = x @ np.asarray(w1_e, dtype=np.float64)
    if act == "gelu":
        h = gelu(z1)
    elif act == "swiglu":
        z3 = x @ np.asarray(w3_e, dtype=np.float64)
        h = silu(z1) * z3
    else:
        raise ValueError(act)
    h = round_to(dtype, h)
    y = h @ np.asarray(w2_e, dtype=np.float64)
    return round_to(dtype, y)


def grouped_ffn(x, perm: dict, w1, w3, w2, act: str, dtype: str, E: int) -> np.ndarray:
    """y[R,H]: every kept row through its expert, one expert at a time ([P3] expert loop)."""
    x = np.asarray(x)
    offs, row_token = perm["offsets"], perm["row_token"]
    H = x.shape[1]
    y = np.zeros((perm["R"], H), dtype=np.float64)
    for e in range(E):
        a, b = int(offs[e]), int(offs[e + 1])
        if b > a:
            y[a:b] = expert_ffn(x[row_token[a:b]], None if w1 is None else w1[e],
                                None if w3 is None else w3[e],
                                None if w2 is None else w2[e], act, dtype)
    return y


# --------------------------------------------------------------------------
# Combine.   [P2] §2.1 sum of gate-weighted expert outputs; [P3] SparseScatterAdd
# --------------------------------------------------------------------------


def combine(y, gates, row_map, dtype: str) -> np.ndarray:
    """out[t] = sum over slots s = 0..k-1 (in that order) of g[t,s] * y[row_map[t,s]].

    Dropped slots (row -1) contribute nothing and the kept gates are not
    renormalised again.  The sum is float64; out is rounded once to dtype.
    """
    y = np.asarray(y, dtype=np.float64)
    g = np.asarray(gates, dtype=np.float64)
    row_map = np.asarray(row_map)
    T, k = row_map.shape
    H = y.shape[1] if y.ndim == 2 else 0
    out = np.zeros((T, H), dtype=np.float64)
    for s in range(k):
        r = row_map[:, s]
        m = r >= 0
        out[m] += g[m, s][:, None] * y[r[m]]
    return round_to(dtype, out)


# --------------------------------------------------------------------------
# Threshold gating.   [P2] §3.2.1: compute all experts' gate scores, keep the
# experts whose score exceeds delta (default 1/E), renormalise the kept ones.
# --------------------------------------------------------------------------


def threshold_select(logits, k_max: int, delta=None) -> dict:
    """Per token: p = softmax over all E (float64); keep the experts with p > delta,
    largest first (ties to the lower id), at most k_max; when none exceeds delta
    the largest alone is kept.  Gates g_s = exp(l_s - l_0) / sum_kept exp(l_j - l_0).
    delta None or <= 0: the default 1/E (as the float32 the library uses).
    Returns idx [T,k_max] (-1 pads), gate [T,k_max] fp32 (0 pads), n_sel [T]."""
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    if not 1 <= k_max <= E:
        raise ValueError("k_max must lie in [1, E]")
    d = float(np.float32(1.0 / E)) if delta is None or delta <= 0 else float(np.float32(delta))
    idx = np.full((T, k_max), -1, dtype=np.int32)
    gate = np.zeros((T, k_max), dtype=np.float32)
    n_sel = np.zeros(T, dtype=np.int32)
    for t in range(T):
        row = [float(v) for v in lg[t]]
        order = sorted(range(E), key=lambda e: (_rank_key(row[e]), e))
        l64 = np.asarray(row, dtype=np.float64)
        z = np.exp(l64 - np.nanmax(l64))
        p = z / np.nansum(z)
        kept = [order[0]]
        for e in order[1:k_max]:
            if not p[e] > d:
                break
            kept.append(e)
        zk = np.exp(l64[kept] - l64[kept[0]])
        n_sel[t] = len(kept)
        idx[t, :len(kept)] = kept
        gate[t, :len(kept)] = (zk / zk.sum()).astype(np.float32)
    return {"topk_idx": idx, "topk_gate": gate, "n_sel": n_sel}


def moe_forward_threshold(x, w_gate, gate_bias, w1, w3, w2, k_max: int, delta,
                          capacity_factor: float, act: str, dtype: str, logits=None) -> dict:
    """The layer with threshold gating: unused slots (-1) carry no row; capacity
    C = ceil(cf * T * k_max / E)."""
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


# --------------------------------------------------------------------------
# Router load statistics.   [P3] "实战中的坑与解法" (track each expert's load) /
# [P4] §5.3 (auxiliary load-balancing loss named, formula not given: the two
# per-expert statistics it is built from)
# --------------------------------------------------------------------------


def router_load_stats(logits, idx, E: int) -> dict:
    """counts[e] = pairs routed to e (pre-drop); prob_mean[e] = mean over tokens
    of softmax(logits[t])[e], the softmax over all E experts, in float64."""
    lg = np.asarray(logits, dtype=np.float64)
    T = lg.shape[0]
    counts = expert_counts(idx, E)
    prob_sum = np.zeros(E, dtype=np.float64)
    for t in range(T):
        z = np.exp(lg[t] - lg[t].max())
        prob_sum += z / z.sum()
    return {"counts": counts, "prob_mean": prob_sum / T if T else prob_sum}


# --------------------------------------------------------------------------
# One expert per token, up-projection only.   [P4] §3 (x[tokens, hidden],
# expert_weight[num_experts, hidden, intermediate], int32 token_expert_idx), §5.2
# --------------------------------------------------------------------------


def expert_matmul(x, expert_weight, token_expert_idx, dtype: str) -> np.ndarray:
    """out[t] = x[t] @ expert_weight[token_expert_idx[t]], float64 sum, rounded once to dtype."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(expert_weight)
    ids = np.asarray(token_expert_idx)
    E = w.shape[0]
    if ids.size and (ids.min() < 0 or ids.max() >= E):
        raise IndexOutOfRange("expert id outside [0, E)")
    out = np.zeros((x.shape[0], w.shape[2]), dtype=np.float64)
    for e in range(E):
        rows = np.nonzero(ids == e)[0]
        if rows.size:
            out[rows] = x[rows] @ np.asarray(w[e], dtype=np.float64)
    return round_to(dtype, out)


# --------------------------------------------------------------------------
# The whole layer.   [P3] MoEOperator::Forward; [P5] ch.8 moe_router
# --------------------------------------------------------------------------


def moe_forward(x, w_gate, gate_bias, w1, w3, w2, top_k: int, capacity_factor: float,
                act: str, dtype: str, logits=None) -> dict:
    """Route, permute, run the experts and combine, returning every intermediate.

    When ``logits`` is given (fp32 [T,E]) the router matmul is skipped and the
    selection starts from those logits.
    """
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
    """The layer's output rows for a sample of tokens only.

    Routing and the permutation are computed for every token (the capacity
    decision for a token depends on all earlier tokens); the expert FFN and the
    combine run only for the sampled tokens' kept rows.
    """
    x = np.asarray(x)
    T, E = logits.shape
    idx = topk_select(logits, top_k)
    gates = topk_gates(logits, idx)
    cap = capacity(capacity_factor, T, top_k, E)
    perm = permute(idx, E, cap)
    tokens = np.asarray(tokens, dtype=np.int64)
    H = x.shape[1]
    # expert outputs of the sampled tokens' kept slots, one expert at a time
    yrows = {}
    for e in range(E):
        pairs = [(int(t), s) for t in tokens for s in range(top_k)
                 if perm["row_map"][t, s] >= 0 and int(idx[t, s]) == e]
        if not pairs:
            continue
        xe = np.stack([np.asarray(x[t], dtype=np.float64) for t, _ in pairs])
        ye = expert_ffn(xe, None if w1 is None else w1[e], None if w3 is None else w3[e],
                        None if w2 is None else w2[e], act, dtype)
        for (t, s), yr in zip(pairs, ye):
            yrows[(t, s)] = yr
    out_rows = np.zeros((len(tokens), H), dtype=np.float64)
    for i, t in enumerate(tokens):
        acc = np.zeros(H, dtype=np.float64)
        for s in range(top_k):
            if (int(t), s) in yrows:
                acc += float(gates[t, s]) * yrows[(int(t), s)]
        out_rows[i] = round_to(dtype, acc)
    return {"topk_idx": idx, "topk_gate": gates, "capacity": cap, "out_rows": out_rows,
            "tokens": tokens, **perm}
