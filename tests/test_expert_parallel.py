"""Expert-parallel forward (rank r of G owns experts [r*E/G, (r+1)*E/G)): its
exchange logic on CPU ranks over gloo.

The per-rank compute steps here are the oracle's (the product runs the C ABI's
kernels in their place); what is under test is what the expert-parallel path
adds: split sizes, the count exchange, the row exchanges both ways, the regroup
by local expert and its inverse, and the overlapped variant's point-to-point
rounds per expert group.  Each rank's result must equal one single-device
oracle forward of that rank's tokens over all E experts.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as O
from routing_grouped_expert_moe_b200 import expert_parallel as EP
from routing_grouped_expert_moe_b200 import synth
from tests.helpers import TOL, as_np, rel_err


# ---------------------------------------------------------------- host logic, no ranks
def test_split_rows_by_owning_rank():
    offsets = np.array([0, 3, 3, 7, 12, 12, 13, 20, 21])       # E = 8
    assert EP.split_rows(offsets, 1).tolist() == [21]
    assert EP.split_rows(offsets, 2).tolist() == [12, 9]
    assert EP.split_rows(offsets, 4).tolist() == [3, 9, 1, 8]
    assert EP.split_rows(offsets, 8).tolist() == [3, 0, 4, 5, 0, 1, 7, 1]
    with pytest.raises(ValueError):
        EP.split_rows(offsets, 3)


def test_local_expert_ids_follow_source_then_expert_order():
    recv = np.array([[2, 0, 1], [1, 3, 0]])                    # 2 sources, 3 local experts
    assert EP.local_expert_ids(recv).tolist() == [0, 0, 2, 0, 1, 1, 1]
    assert EP.local_expert_ids(np.zeros((2, 2), dtype=np.int64)).size == 0


# ---------------------------------------------------------------- oracle steps
class OracleSteps:
    """The per-rank compute steps through the oracle (CPU tensors in, CPU tensors out)."""

    def __init__(self, dtype: str):
        self.dtype = dtype
        self.host_reads = 0

    def _store(self, a, like):
        return torch.from_numpy(np.asarray(a, dtype=np.float64)).to(like.dtype)

    def route(self, x, w_gate, gate_bias, top_k):
        lg = O.router_logits(as_np(x), as_np(w_gate),
                             None if gate_bias is None else as_np(gate_bias))
        idx = O.topk_select(lg, top_k)
        return (torch.from_numpy(idx.astype(np.int32)),
                torch.from_numpy(O.topk_gates(lg, idx).astype(np.float32)))

    def permute(self, x, idx, E, capacity_factor):
        T, k = idx.shape
        p = O.permute(idx.numpy(), E, O.capacity(capacity_factor, T, k, E))
        x_perm = x[torch.from_numpy(p["row_token"])]
        return (x_perm, torch.from_numpy(p["offsets"].astype(np.int32)),
                torch.from_numpy(p["row_map"].astype(np.int32)))

    def grouped_ffn(self, x_rows, offsets, w1, w3, w2, act):
        xr = as_np(x_rows)
        off = offsets.numpy()
        y = np.zeros(xr.shape, dtype=np.float64)
        for e in range(off.size - 1):
            a, b = int(off[e]), int(off[e + 1])
            if b > a:
                y[a:b] = O.expert_ffn(xr[a:b], as_np(w1[e]), None if w3 is None else as_np(w3[e]),
                                      as_np(w2[e]), act, self.dtype)
        return self._store(y, x_rows)

    def unpermute(self, y, row_map):
        assert row_map.shape[1] == 1 and bool((row_map >= 0).all())
        return y[row_map[:, 0].long()]

    def combine(self, y, gate, row_map):
        return self._store(O.combine(as_np(y), gate.numpy(), row_map.numpy(), self.dtype), y)

    def to_host(self, t):
        self.host_reads += 1
        return t.numpy()

    def from_host(self, a, like):
        return torch.from_numpy(np.ascontiguousarray(a))


# ---------------------------------------------------------------- ranks
CASES = {
    # name: (T per rank, H, F, E, k, act, dtype, cf, bias)
    "f32_swiglu": ((64, 40), 128, 256, 4, 2, "swiglu", "f32", 0.0, None),
    "bf16_gelu_drops": ((96, 96), 64, 128, 8, 2, "gelu", "bf16", 0.5, None),
    "empty_rank": ((50, 0), 64, 64, 4, 2, "swiglu", "bf16", 1.25, None),
    "one_rank_gets_nothing": ((40, 40), 64, 64, 4, 2, "swiglu", "bf16", 0.0, "first_half"),
    "top1_many_experts": ((70, 33), 32, 64, 16, 1, "gelu", "f32", 1.0, None),
    # four ranks
    "four_ranks_drops": ((48, 0, 31, 64), 64, 128, 8, 2, "swiglu", "bf16", 0.75, None),
    "four_ranks_top3": ((20, 45, 33, 7), 32, 64, 16, 3, "gelu", "f32", 0.0, None),
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case_inputs(name, rank):
    (Ts, H, F, E, k, act, dtype, cf, bias) = CASES[name]
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    seed = 4100 + sorted(CASES).index(name)
    x = synth.normal(seed + 17 * (rank + 1), synth.STREAM_X, (Ts[rank], H), 1.0, td)
    wg = synth.normal(seed, synth.STREAM_WG, (H, E), H ** -0.5, td)
    w1 = synth.normal(seed, synth.STREAM_W1, (E, H, F), H ** -0.5, td)
    w3 = synth.normal(seed, synth.STREAM_W3, (E, H, F), H ** -0.5, td) if act == "swiglu" else None
    w2 = synth.normal(seed, synth.STREAM_W2, (E, F, H), F ** -0.5, td)
    b = None
    if bias == "first_half":   # every token picks its k experts among the first E/2 (rank 0's)
        b = torch.zeros(E, dtype=torch.float32)
        b[: E // 2] = 100.0
    return dict(x=x, w_gate=wg, gate_bias=b, w1=w1, w3=w3, w2=w2, E=E, k=k, act=act,
                dtype=dtype, cf=cf)


def _rank_main(rank: int, world: int, port: int, names, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        for name in names:
            d = _case_inputs(name, rank)
            E, el = d["E"], d["E"] // world
            sl = slice(rank * el, (rank + 1) * el)
            local = lambda w: None if w is None else w[sl].contiguous()  # noqa: E731
            outs = []
            for ov in (False, True):
                steps = OracleSteps(d["dtype"])
                outs.append(EP.ep_forward(d["x"], d["w_gate"], d["gate_bias"], local(d["w1"]),
                                          local(d["w3"]), local(d["w2"]), d["k"], d["cf"],
                                          d["act"], E, steps=steps, overlap=ov))
                # split sizes reach the host once per forward
                assert steps.host_reads == 1, (name, ov, steps.host_reads)
            for out in outs:
                assert out.shape == d["x"].shape and out.dtype == d["x"].dtype
            # the overlapped exchange moves the same rows: the same bits
            assert torch.equal(outs[0], outs[1]), name
            if d["x"].shape[0] == 0:
                q.put((name, rank, 0.0, 1.0))
                continue
            f = lambda t: None if t is None else as_np(t)  # noqa: E731
            ref = O.moe_forward(f(d["x"]), f(d["w_gate"]), f(d["gate_bias"]), f(d["w1"]),
                                f(d["w3"]), f(d["w2"]), d["k"], d["cf"], d["act"], d["dtype"])
            got = as_np(outs[1])
            same = float(np.mean(got == ref["out"]))
            q.put((name, rank, rel_err(got, ref["out"]), same))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_equals_single_device_forward(world):
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    names = sorted(n for n in CASES if len(CASES[n][0]) == world)
    mp.start_processes(_rank_main, args=(world, _free_port(), names, q), nprocs=world,
                       start_method="spawn", join=True)
    res = [q.get() for _ in range(world * len(names))]
    assert len(res) == world * len(names)
    for name, rank, err, same in res:
        assert err <= TOL[CASES[name][6]], (name, rank, err)
        assert same >= 0.999, (name, rank, same)   # the same arithmetic row for row
