"""The multi-rank host logic of bench.py, on CPU with two gloo ranks.

The layer shards by tokens with no data-path collective (replicas), so what a
multi-GPU run adds is host logic: per-rank inputs (same weights, own tokens),
the max-over-ranks time, whole-job throughput, and the reference arm that only
rank 0 runs.  Those are checked here without a GPU."""
import contextlib
import io
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from routing_grouped_expert_moe_b200 import synth  # noqa: E402

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _digest(t: torch.Tensor) -> torch.Tensor:
    t = t.float().reshape(-1)
    w = torch.arange(1, t.numel() + 1, dtype=torch.float64)
    return torch.stack([t.double().sum(), (t.double() * w).sum()])


def _rank_main(rank: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        cfg = synth.CONFIGS["tiny_f32"]
        d = bench.rank_inputs(cfg, rank)
        dig = {k: _digest(d[k]) for k in ("x", "w_gate", "w1", "w3", "w2")}
        gathered = {}
        for k, v in dig.items():
            parts = [torch.zeros_like(v) for _ in range(WORLD)]
            dist.all_gather(parts, v)
            gathered[k] = [p.tolist() for p in parts]
        # the slowest rank sets the time
        my_ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(my_ms, dist, torch.device("cpu"))
        value = bench.job_tokens_per_s(cfg.T, WORLD, 4, mx)
        # the reference arm: rank 0 prints one line, the others exit 0 without work
        args = bench.parse_args(["--impl", "reference", "--gpus", str(WORLD), "--steps", "1",
                                 "--warmup", "1", "--config", "tiny_f32"])
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            rc = bench.run_reference(args, cfg)
        q.put((rank, {"digests": gathered, "max_ms": mx, "value": value, "ref_rc": rc,
                      "ref_out": buf.getvalue()}))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def rank_results():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(WORLD):
        r, v = q.get(timeout=240)
        res[r] = v
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_weights_replicated_tokens_distinct(rank_results):
    dg = rank_results[0]["digests"]
    for k in ("w_gate", "w1", "w3", "w2"):
        assert dg[k][0] == dg[k][1], k
    assert dg["x"][0] != dg["x"][1]
    # rank 0's tokens are the workload's own seeded draw
    cfg = synth.CONFIGS["tiny_f32"]
    assert dg["x"][0] == _digest(synth.make_inputs(cfg)["x"]).tolist()


def test_time_is_max_over_ranks_and_value_is_whole_job(rank_results):
    for r in range(WORLD):
        assert rank_results[r]["max_ms"] == 15.0
        # 64 tokens x 2 ranks x 4 steps in 15 ms
        assert rank_results[r]["value"] == pytest.approx(64 * 2 * 4 / 0.015)


def test_reference_arm_runs_on_rank0_only(rank_results):
    assert rank_results[0]["ref_rc"] == 0 and rank_results[1]["ref_rc"] == 0
    assert rank_results[1]["ref_out"] == ""
    lines = [ln for ln in rank_results[0]["ref_out"].splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == WORLD
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
