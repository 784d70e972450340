"""moe_permute_noalloc: the permute step for callers that cannot allocate.

Hosts such as an engine plugin that runs on memory planned before the model
starts, or a serving process that reserved its device budget up front, can
neither call cudaMalloc nor hand the library a workspace.  This entry point
keeps its scratch in a library-owned device array instead.  The test calls it
through the C ABI and checks that two calls in a row give exactly the outputs
of moe_permute (which uses a caller workspace) — integer outputs, so the
tolerance is exact equality.
"""
import ctypes

import numpy as np
import pytest
import torch

from routing_grouped_expert_moe_b200 import synth

pytestmark = pytest.mark.gpu


def _lib():
    from routing_grouped_expert_moe_b200 import binding
    return binding


def _noalloc(B, ids, E, cf, x, status):
    T, k = ids.shape
    H = x.shape[1]
    out = {"counts": torch.full((E,), -7, dtype=torch.int32, device="cuda"),
           "offsets": torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
           "row_token": torch.full((T * k,), -1, dtype=torch.int32, device="cuda"),
           "row_map": torch.full((T, k), -7, dtype=torch.int32, device="cuda"),
           "x_perm": torch.zeros(T * k, H, dtype=x.dtype, device="cuda")}
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = B._lib.moe_permute_noalloc(p(x), p(ids), T, H, E, k, ctypes.c_float(cf), B.BF16,
                                    p(out["x_perm"]), p(out["counts"]), p(out["offsets"]),
                                    p(out["row_token"]), p(out["row_map"]), p(status),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == B.OK, B.status_string(st)
    return out


def test_noalloc_permute_matches_workspace_permute_twice():
    B = _lib()
    cases = [(3000, 32, 2, 1.25, 0.0, 11), (1500, 8, 2, 0.5, 0.4, 12)]
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    for T, E, k, cf, skew, seed in cases:               # two calls in a row, different shapes
        ids = synth.random_expert_ids(seed, T, E, k, skew=skew).cuda()
        x = synth.normal(seed, 0, (T, 64), 1.0, torch.bfloat16).cuda()
        ref = B.permute(ids, E, capacity_factor=cf, x=x)
        got = _noalloc(B, ids, E, cf, x, status)
        torch.cuda.synchronize()
        R = int(ref["offsets"][-1].item())
        assert torch.equal(got["counts"], ref["counts"])
        assert torch.equal(got["offsets"], ref["offsets"])
        assert torch.equal(got["row_token"][:R], ref["row_token"][:R])
        assert torch.equal(got["row_map"], ref["row_map"])
        assert torch.equal(got["x_perm"][:R], ref["x_perm"][:R])
        assert int(status.item()) == B.OK
        assert B.device_status(ref["ws"]) == B.OK


def test_noalloc_permute_reports_bad_ids_and_rejects_oversize():
    B = _lib()
    T, E, k = 700, 8, 2
    ids = synth.random_expert_ids(5, T, E, k).cuda()
    ids[3, 1] = E                                          # out of range: dropped, reported
    x = synth.normal(5, 0, (T, 32), 1.0, torch.bfloat16).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _noalloc(B, ids, E, 0.0, x, status)
    torch.cuda.synchronize()
    assert int(status.item()) == B.ERR_INDEX_OUT_OF_RANGE
    assert int(got["row_map"][3, 1].item()) == -1
    assert int(got["counts"].sum().item()) == T * k - 1
    # ceil(T/128) * E beyond the fixed scratch: rejected on the host, nothing launched
    big_T = 128 * (262080 // 256 + 1)
    p = ctypes.c_void_p(0x10000)
    st = B._lib.moe_permute_noalloc(None, p, big_T, 8, 256, 2, ctypes.c_float(0.0), B.BF16,
                                    None, p, p, p, p, None, None)
    assert st == B.ERR_UNSUPPORTED


def test_noalloc_python_wrapper_matches_permute():
    """binding.permute_noalloc (argument order, output allocation, the x = None
    form and status_out) gives exactly what binding.permute gives."""
    B = _lib()
    T, E, k, cf = 999, 16, 2, 1.0
    ids = synth.random_expert_ids(21, T, E, k, skew=0.2).cuda()
    x = synth.normal(21, 0, (T, 128), 1.0, torch.bfloat16).cuda()
    for with_x in (True, False):
        for with_status in (True, False):
            status = torch.full((1,), 99, dtype=torch.int32, device="cuda") if with_status else None
            got = B.permute_noalloc(ids, E, capacity_factor=cf, x=x if with_x else None,
                                    status_out=status)
            ref = B.permute(ids, E, capacity_factor=cf, x=x if with_x else None)
            torch.cuda.synchronize()
            R = int(ref["offsets"][-1].item())
            for name in ("counts", "offsets", "row_map"):
                assert torch.equal(got[name], ref[name]), name
            assert torch.equal(got["row_token"][:R], ref["row_token"][:R])
            assert ("x_perm" in got) == with_x
            if with_x:
                assert torch.equal(got["x_perm"][:R], ref["x_perm"][:R])
            if with_status:
                assert int(status.item()) == B.OK
