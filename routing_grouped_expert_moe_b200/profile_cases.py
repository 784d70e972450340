"""Run one entry point of the library a few times on seeded inputs, for profiling.

    python -m routing_grouped_expert_moe_b200.profile_cases CASE [N]

A profiler (ncu) is pointed at this process and picks the launches it wants
with its kernel filter and launch counts.  Cases:

  fwd:<workload>  the fused forward (moe_forward) on a named workload
                  (tiny_f32, page1_gelu, mixtral_e8, e32_long, e128_skew)
  f32             the fused forward in fp32 storage (T=2048, H=1024, F=1024, E=8)
  permute         moe_permute alone: T=32768, top-2 over 32 experts, H=4096, capacity 1.25
  threshold       moe_forward_threshold: T=8192, H=2048, F=1024, 32 experts, k_max=4
  stats           moe_route_stats on the 32-expert long-sequence router
  gather          moe_grouped_ffn with row_token: 8 GELU experts, 8192 rows,
                  H=2048, F=8192, gathered from 4096 token rows
  matmul          moe_expert_matmul: x[1024,4096], expert_weight[8,4096,14336]

Exits non-zero when the device status after the last call is not MOE_OK.
"""
from __future__ import annotations

import sys
from dataclasses import replace

import torch

from routing_grouped_expert_moe_b200 import binding as B
from routing_grouped_expert_moe_b200 import synth


def _cuda(d, dev):
    return {k: (None if v is None else v.to(dev)) for k, v in d.items()}


def run(case: str, n: int) -> int:
    dev = torch.device("cuda:0")
    if case.startswith("fwd:") or case == "f32":
        if case == "f32":
            cfg = replace(synth.CONFIGS["tiny_f32"], name="f32_mid", T=2048, H=1024, F=1024, E=8,
                          seed=8001, wg_std=1024 ** -0.5, w1_std=1024 ** -0.5,
                          w2_std=1024 ** -0.5)
        else:
            cfg = synth.CONFIGS[case[4:]]
        g = _cuda(synth.make_inputs(cfg), dev)
        ws = B.alloc_workspace(B.workspace_bytes(cfg.T, cfg.H, cfg.F, cfg.E, cfg.top_k, cfg.act,
                                                 g["x"].dtype), dev)
        out = torch.empty_like(g["x"])
        for _ in range(n):
            B.forward(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"], g["w2"], cfg.top_k,
                      cfg.capacity_factor, cfg.act, out=out, ws=ws)
        return B.device_status(ws)
    if case == "permute":
        T, E, k, H = 32768, 32, 2, 4096
        ids = synth.random_expert_ids(1, T, E, k).to(dev)
        x = synth.normal(1, 0, (T, H), 1.0, torch.bfloat16).to(dev)
        for _ in range(n):
            r = B.permute(ids, E, capacity_factor=1.25, x=x)
        return B.device_status(r["ws"])
    if case == "threshold":
        cfg = replace(synth.CONFIGS["e32_long"], name="thr", T=8192, H=2048, F=1024, seed=8002)
        g = _cuda(synth.make_inputs(cfg), dev)
        for _ in range(n):
            _, ws = B.forward_threshold(g["x"], g["w_gate"], g["gate_bias"], g["w1"], g["w3"],
                                        g["w2"], 4, 0.0, 0.0, cfg.act)
        return B.device_status(ws)
    if case == "stats":
        cfg = synth.CONFIGS["e32_long"]
        g = _cuda(synth.make_inputs(cfg, with_weights=False), dev)
        for _ in range(n):
            res = B.route_stats(g["x"], g["w_gate"], g["gate_bias"], cfg.top_k)
        return B.device_status(res[4])
    if case == "gather":
        E, H, F, R = 8, 2048, 8192, 8192
        off = torch.arange(0, R + 1, R // E, dtype=torch.int32, device=dev)
        x = synth.normal(2, 0, (R // 2, H), 1.0, torch.bfloat16).to(dev)
        rt = (torch.arange(R, dtype=torch.int32, device=dev) * 7919) % (R // 2)
        w1 = synth.normal(2, 2, (E, H, F), H ** -0.5, torch.bfloat16).to(dev)
        w2 = synth.normal(2, 4, (E, F, H), F ** -0.5, torch.bfloat16).to(dev)
        ws = B.alloc_workspace(B._lib.moe_grouped_ffn_workspace_bytes(R, H, F, B.ACT["gelu"],
                                                                      B.BF16, 1), dev)
        for _ in range(n):
            B.grouped_ffn(off, w1, None, w2, "gelu", x=x, row_token=rt, ws=ws)
        return B.device_status(ws)
    if case == "matmul":
        T, H, I, E = 1024, 4096, 14336, 8
        x = synth.normal(3, 0, (T, H), 1.0, torch.bfloat16).to(dev)
        w = synth.normal(3, 2, (E, H, I), H ** -0.5, torch.bfloat16).to(dev)
        ids = synth.random_expert_ids(3, T, E, 1)[:, 0].contiguous().to(dev)
        for _ in range(n):
            _, ws = B.expert_matmul(x, w, ids)
        return B.device_status(ws)
    raise SystemExit(f"unknown case {case!r}")


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    if not argv:
        print(__doc__)
        return 2
    st = run(argv[0], int(argv[1]) if len(argv) > 1 else 3)
    print(argv[0], "status", B.status_string(st))
    return 0 if st == B.OK else 1


if __name__ == "__main__":
    sys.exit(main())
