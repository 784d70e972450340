"""Per-stage parity of the CUDA path against the oracle, through the C ABI.

Integer outputs (expert ids, counts, offsets, row maps) must match bit for bit;
floating point outputs within max|gpu - oracle| / max|oracle| <= 1e-4 (fp32) or
2e-2 (bf16).  Sizes span several tiles and a ragged tail.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from routing_grouped_expert_moe_b200 import synth
from tests.helpers import Guarded, guarded_workspace, TOL, as_np, gap_violations, rel_err

pytestmark = pytest.mark.gpu


def B():
    from routing_grouped_expert_moe_b200 import binding
    return binding


# ---------------------------------------------------------------- router

@pytest.mark.parametrize("T,E,k", [(1, 4, 1), (37, 8, 2), (300, 32, 2), (1000, 128, 2),
                                   (129, 256, 8), (77, 5, 5), (64, 12, 3)])
def test_route_from_logits_bit_exact(T, E, k):
    lg = synth.random_logits(100 + T, T, E, scale=2.0)
    lg[0, :] = 0.5                         # a token of all-equal logits: lower ids win
    if T > 2:
        lg[1, 0] = float("nan")
        lg[2, E - 1] = float("-inf")
    idx, gate = B().route_from_logits(lg.cuda(), k)
    ref_idx = O.topk_select(lg.numpy(), k)
    np.testing.assert_array_equal(as_np(idx), ref_idx)
    ok = np.isfinite(lg.numpy()).all(axis=1)
    ref_g = O.topk_gates(lg.numpy(), ref_idx)
    np.testing.assert_allclose(as_np(gate)[ok], ref_g[ok], rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("dtype,T,H,E,k", [
    ("bf16", 1000, 512, 8, 2), ("bf16", 333, 1024, 32, 2), ("bf16", 517, 256, 128, 2),
    ("bf16", 64, 4096, 8, 2),                       # few tiles: H split over a cluster
    ("bf16", 96, 200, 16, 4),                       # H not a multiple of the 64-wide k-block
    ("bf16", 20000, 128, 8, 2),                     # enough tiles: no H split
    ("bf16", 300, 256, 256, 8),                     # 256 experts (MMA N = 256), top-8
    ("bf16", 19000, 192, 128, 2),                   # 128 experts, no H split, ragged tail
    ("bf16", 50, 64, 12, 3),                        # E not a multiple of 8 (CUDA-core path)
    ("bf16", 777, 2048, 16, 2),                     # few experts: H split in a cluster, ragged tile
    ("bf16", 129, 768, 8, 3),                       # few experts, one CTA per tile
    ("bf16", 4096, 256, 16, 1),                     # few experts, top-1
    ("f32", 257, 128, 4, 2), ("f32", 100, 96, 40, 3),
])
def test_route_from_x(dtype, T, H, E, k):
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = synth.normal(7, 0, (T, H), 1.0, dt)
    wg = synth.normal(7, 1, (H, E), H ** -0.5, dt)
    bias = synth.normal(7, 2, (E,), 0.1, torch.float32)
    idx, gate, lg = B().route(x.cuda(), wg.cuda(), bias.cuda(), top_k=k, logits_out=True)
    ref_lg = O.router_logits(as_np(x), as_np(wg), as_np(bias))
    # logits: fp32 accumulation in a different order than the float64 oracle
    assert rel_err(as_np(lg), ref_lg) < 1e-5
    # selection from the GPU's own logits follows the selection rule exactly
    np.testing.assert_array_equal(as_np(idx), O.topk_select(as_np(lg).astype(np.float32), k))
    # and agrees with the oracle's selection wherever the top-k gaps are clear
    clear = np.setdiff1d(np.arange(T), gap_violations(ref_lg, k))
    np.testing.assert_array_equal(as_np(idx)[clear], O.topk_select(ref_lg, k)[clear])
    np.testing.assert_allclose(as_np(gate)[clear],
                               O.topk_gates(ref_lg, O.topk_select(ref_lg, k))[clear],
                               rtol=1e-4, atol=1e-6)


# ---------------------------------------------------------------- permute

def _perm_check(ids, E, cf, x=None):
    """moe_permute against the oracle bit for bit, every output and the
    workspace sentinel-guarded; row_token entries and x_perm rows past R must
    stay unwritten."""
    T, k = ids.shape
    H = 8 if x is None else x.shape[1]
    g = {"counts": Guarded((E,), torch.int32), "offsets": Guarded((E + 1,), torch.int32),
         "row_token": Guarded((T * k,), torch.int32), "row_map": Guarded((T, k), torch.int32)}
    if x is not None:
        g["x_perm"] = Guarded((T * k, H), x.dtype)
    ws = guarded_workspace(B().workspace_bytes(T, H, 8, E, k, "identity",
                                               torch.bfloat16 if x is None else x.dtype))
    r = B().permute(ids.cuda(), E, capacity_factor=cf, x=None if x is None else x.cuda(),
                    ws=ws.t, out={n: v.t for n, v in g.items()})
    cap = O.capacity(cf, T, k, E)
    ref = O.permute(ids.numpy(), E, cap)
    np.testing.assert_array_equal(as_np(r["counts"]), ref["counts"])
    np.testing.assert_array_equal(as_np(r["offsets"]), ref["offsets"])
    R = ref["R"]
    np.testing.assert_array_equal(as_np(r["row_token"])[:R], ref["row_token"])
    np.testing.assert_array_equal(as_np(r["row_map"]), ref["row_map"])
    assert B().device_status(r["ws"]) == B().OK
    if x is not None:
        np.testing.assert_array_equal(as_np(r["x_perm"])[:R], as_np(x)[ref["row_token"]])
        g["x_perm"].untouched(R * H * x.element_size(), T * k * H * x.element_size(),
                              "x_perm rows past R")
    g["row_token"].untouched(R * 4, T * k * 4, "row_token past R")
    for n, v in g.items():
        v.check(n)
    ws.check("workspace")
    return r, ref


@pytest.mark.parametrize("T,E,k,cf,skew", [
    (1, 4, 2, 0.0, 0.0), (1000, 8, 2, 0.0, 0.0), (4097, 32, 2, 1.25, 0.0),
    (3000, 128, 2, 0.0, 0.05), (777, 8, 2, 0.5, 0.3), (2000, 16, 4, 1.0, 0.2),
    (513, 256, 8, 0.0, 0.0), (300, 3, 1, 0.8, 1.0),
])
def test_permute_bit_exact(T, E, k, cf, skew):
    ids = synth.random_expert_ids(T + E, T, E, k, skew=skew)
    x = synth.normal(3, 0, (T, 64), 1.0, torch.bfloat16)
    _perm_check(ids, E, cf, x)


def test_permute_golden_cases():
    import json, os
    here = os.path.join(os.path.dirname(__file__), "golden", "capacity_cases.json")
    for c in json.load(open(here))["cases"]:
        ids = torch.tensor(c["topk_idx"], dtype=torch.int32)
        r, _ = _perm_check(ids, c["E"], c["capacity_factor"])
        np.testing.assert_array_equal(as_np(r["row_map"]), np.array(c["row_map"]))


def test_permute_all_to_one_expert_with_capacity():
    T, E, k = 5000, 8, 2
    ids = torch.stack([torch.zeros(T, dtype=torch.int32), torch.ones(T, dtype=torch.int32)], 1)
    _perm_check(ids, E, 1.0)                         # C = 1250: 3750 pairs dropped per expert


def test_permute_out_of_range_is_reported():
    ids = synth.random_expert_ids(1, 300, 8, 2)
    ids[17, 1] = 8
    ids[200, 0] = -3
    r = B().permute(ids.cuda(), 8)
    assert B().device_status(r["ws"]) == B().ERR_INDEX_OUT_OF_RANGE
    rm = as_np(r["row_map"])
    assert rm[17, 1] == -1 and rm[200, 0] == -1
    assert as_np(r["counts"]).sum() == 300 * 2 - 2
    assert B().device_status(r["ws"]) == B().OK      # reading clears it


# ---------------------------------------------------------------- grouped FFN

def _ffn_case(dtype, act, E, rows_per_expert, H, F, seed=11):
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    T = max(1, sum(rows_per_expert))
    x = synth.normal(seed, 0, (T, H), 1.0, dt)
    w1 = synth.normal(seed, 2, (E, H, F), H ** -0.5, dt)
    w3 = synth.normal(seed, 3, (E, H, F), H ** -0.5, dt) if act == "swiglu" else None
    w2 = synth.normal(seed, 4, (E, F, H), F ** -0.5, dt)
    # a k=1 assignment with the requested rows per expert, tokens shuffled
    ids = np.concatenate([np.full(n, e, dtype=np.int32) for e, n in enumerate(rows_per_expert)])
    ids = np.random.default_rng(seed).permutation(ids)[:, None].astype(np.int32)
    perm = O.permute(ids, E, None)
    return dt, x, w1, w3, w2, perm


@pytest.mark.parametrize("dtype,act,gather", [
    ("bf16", "swiglu", False), ("bf16", "gelu", False), ("bf16", "swiglu", True),
    ("bf16", "gelu", True), ("f32", "swiglu", True), ("f32", "gelu", False),
], ids=["bf16-swiglu-dense", "bf16-gelu-dense", "bf16-swiglu-gather", "bf16-gelu-gather",
        "f32-swiglu-gather", "f32-gelu-dense"])
@pytest.mark.parametrize("shape", [
    (4, [0, 1, 130, 257], 256, 384),       # empty expert, 1-row expert, ragged m tiles
    (3, [200, 64, 129], 200, 136),         # K tail (200 % 64), N tail (136 % 128)
    (2, [300, 45], 512, 1376),             # F of the 32-expert workload (N tail 1376 % 256)
    (5, [512, 640, 383, 0, 129], 384, 512),   # even / odd m-tile counts per expert
])
@pytest.mark.parametrize("variant", ["rows128", "rows256_pair", "tokens_pair",
                                     "tokens_pair_nosplit"])
def test_grouped_ffn(dtype, act, gather, shape, variant, gemm_variant):
    """Every kernel against the oracle, with R_max - R = 37 spare rows: the spare
    rows of x_perm hold NaN (a kernel that mixes rows would spread them), the
    spare rows of y and the bytes around y and the workspace hold sentinels
    that must survive."""
    if dtype == "f32" and variant != "rows128":
        pytest.skip("the fp32 path has a single CUDA-core kernel")
    if gather and variant.startswith("tokens_pair"):
        pytest.skip("gathered rows always use the row-tiled kernels")
    gemm_variant(variant)
    E, rows, H, F = shape
    dt, x, w1, w3, w2, perm = _ffn_case(dtype, act, E, rows, H, F)
    xo = as_np(x)
    ref = O.grouped_ffn(xo, perm, as_np(w1), None if w3 is None else as_np(w3), as_np(w2), act,
                        dtype, E)
    R = perm["R"]
    R_max = R + 37
    offs = torch.from_numpy(perm["offsets"].astype(np.int32)).cuda()
    rt = torch.full((R_max,), 0, dtype=torch.int32)
    rt[:R] = torch.from_numpy(perm["row_token"].astype(np.int32))
    esz = 2 if dtype == "bf16" else 4
    y = Guarded((R_max, H), dt)
    # the smallest workspace: gathered rows are read by the GEMM itself
    ws = guarded_workspace(256 + R_max * F * esz)
    if gather:
        B().grouped_ffn(offs, w1.cuda(), None if w3 is None else w3.cuda(), w2.cuda(), act,
                        x=x.cuda(), row_token=rt.cuda(), R_max=R_max, ws=ws.t, y=y.t)
    else:
        x_perm = torch.full((R_max, H), float("nan"), dtype=dt)
        x_perm[:R] = x[torch.from_numpy(perm["row_token"])]
        B().grouped_ffn(offs, w1.cuda(), None if w3 is None else w3.cuda(), w2.cuda(), act,
                        x_perm=x_perm.cuda(), R_max=R_max, ws=ws.t, y=y.t)
    torch.cuda.synchronize()
    got = as_np(y.t)[:R]
    assert np.all(np.isfinite(got))
    assert rel_err(got, ref) <= TOL[dtype]
    y.check("y")
    y.untouched(R * H * esz, R_max * H * esz, "y rows past R")
    ws.check("workspace")


def test_grouped_ffn_ksplit_tail(gemm_variant):
    """With room in the workspace the SwiGLU GEMM-1 cuts its last partial wave of
    tiles in two along K: here 3 token groups x 2 output-column blocks = 6 tiles,
    all of them in that wave, so all are split.  Against the oracle; bit-identical
    on a second run (a sum of two fp32 parts does not depend on which part
    finished first); within tolerance of the unsplit kernel, and different from it
    in some element (the split's summation order ran); sentinels around y and the
    workspace, split sums and tickets included."""
    E, rows, H, F = 3, [256, 200, 77], 2048, 512
    dt, x, w1, w3, w2, perm = _ffn_case("bf16", "swiglu", E, rows, H, F, seed=23)
    ref = O.grouped_ffn(as_np(x), perm, as_np(w1), as_np(w3), as_np(w2), "swiglu", "bf16", E)
    R = perm["R"]
    offs = torch.from_numpy(perm["offsets"].astype(np.int32)).cuda()
    x_perm = x[torch.from_numpy(perm["row_token"])].contiguous().cuda()
    nbytes = B()._lib.moe_grouped_ffn_workspace_bytes(R, H, F, B().ACT["swiglu"], B().BF16, 0)
    outs = []
    for variant in ("tokens_pair", "tokens_pair", "tokens_pair_nosplit"):
        gemm_variant(variant)
        ws = guarded_workspace(nbytes)
        y = Guarded((R, H), dt)
        B().grouped_ffn(offs, w1.cuda(), w3.cuda(), w2.cuda(), "swiglu", x_perm=x_perm, ws=ws.t,
                        y=y.t)
        assert B().device_status(ws.t) == B().OK
        y.check("y")
        ws.check("workspace")
        outs.append(y.t.clone())
    for o in outs:
        assert rel_err(as_np(o), ref) <= TOL["bf16"]
    assert torch.equal(outs[0], outs[1])
    assert not torch.equal(outs[0], outs[2])


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_grouped_ffn_gather_with_room_equals_dense(act):
    """With room for the gathered rows in ws, the gathered form copies them into
    expert order and runs the dense kernel: bit-identical to passing x_perm."""
    E, rows, H, F = 5, [512, 640, 383, 0, 129], 384, 512
    dt, x, w1, w3, w2, perm = _ffn_case("bf16", act, E, rows, H, F)
    offs = torch.from_numpy(perm["offsets"].astype(np.int32)).cuda()
    rt = torch.from_numpy(perm["row_token"].astype(np.int32)).cuda()
    R = perm["R"]
    w3c = None if w3 is None else w3.cuda()
    ws = guarded_workspace(B()._lib.moe_grouped_ffn_workspace_bytes(R, H, F, B().ACT[act],
                                                                    B().BF16, 1))
    yg = Guarded((R, H), dt)
    B().grouped_ffn(offs, w1.cuda(), w3c, w2.cuda(), act, x=x.cuda(), row_token=rt, ws=ws.t,
                    y=yg.t)
    x_perm = x[torch.from_numpy(perm["row_token"])].contiguous().cuda()
    yd = B().grouped_ffn(offs, w1.cuda(), w3c, w2.cuda(), act, x_perm=x_perm)
    assert B().device_status(ws.t) == B().OK
    assert torch.equal(yg.t, yd)
    yg.check("y")
    ws.check("workspace")


def test_grouped_ffn_identity_and_gemm_only_rows():
    dt, x, *_ , perm = _ffn_case("bf16", "gelu", 3, [5, 0, 70], 64, 64)
    offs = torch.from_numpy(perm["offsets"].astype(np.int32)).cuda()
    rt = torch.from_numpy(perm["row_token"].astype(np.int32)).cuda()
    y = B().grouped_ffn(offs, None, None, None, "identity", x=x.cuda(), row_token=rt)
    np.testing.assert_array_equal(as_np(y), as_np(x)[perm["row_token"]])


# ---------------------------------------------------------------- combine

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,H,k", [(1, 8, 1), (1000, 2048, 2), (333, 136, 4), (64, 4096, 8)])
def test_combine(dtype, T, H, k):
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    R = T * k
    y = synth.normal(5, 0, (R, H), 1.0, dt)
    rng = np.random.default_rng(T)
    row_map = rng.permutation(R).reshape(T, k).astype(np.int32)
    row_map[rng.random((T, k)) < 0.1] = -1          # some dropped slots
    gate = torch.from_numpy(rng.random((T, k)).astype(np.float32))
    og = Guarded((T, H), dt)
    out = B().unpermute_combine(y.cuda(), gate.cuda(), torch.from_numpy(row_map).cuda(),
                                out=og.t)
    ref = O.combine(as_np(y), gate.numpy(), row_map, dtype)
    assert rel_err(as_np(out), ref) <= (1e-6 if dtype == "f32" else 8e-3)
    og.check("out")
    # deterministic: a second run is bit-identical
    out2 = B().unpermute_combine(y.cuda(), gate.cuda(), torch.from_numpy(row_map).cuda())
    assert torch.equal(out, out2)


def test_epilogue_activations_error_bounds():
    """The bf16 epilogue's GELU (erfc by the Numerical Recipes Chebyshev fit,
    fractional error < 1.2e-7, hardware exp) and SiLU (hardware exp and
    reciprocal) stay within a few 1e-6 relative of the exact values (the
    oracle's float64 functions) over the range an accumulator reaches — far
    below the 2^-8 spacing of the bf16 h they are rounded to."""
    from routing_grouped_expert_moe_b200 import binding as Bd
    z = torch.cat([torch.linspace(-12, 12, 400001), torch.tensor([0.0, -0.0, 1e-30, -1e-30, 80.0,
                                                                   -80.0, 200.0, -200.0])])
    g, s = Bd.epilogue_activations(z.cuda())
    z64 = z.double().numpy()
    g_exact, s_exact = O.gelu(z64), O.silu(z64)
    g_gpu, s_gpu = g.cpu().double().numpy(), s.cpu().double().numpy()
    assert np.all(np.isfinite(g_gpu)) and np.all(np.isfinite(s_gpu))
    # the hardware exponential's error grows with |argument| (up to ~75 here)
    m = np.abs(g_exact) > 1e-35
    rel_g = np.abs(g_gpu - g_exact)[m] / np.abs(g_exact)[m]
    assert rel_g.max() <= 3e-5, rel_g.max()
    assert np.max(np.abs(g_gpu - g_exact)) <= 1e-6
    sm = np.abs(z64) <= 20
    rel_s = np.abs(s_gpu - s_exact)[sm] / np.maximum(np.abs(s_exact[sm]), 1e-30)
    assert rel_s.max() <= 5e-6, rel_s.max()
    assert np.max(np.abs(s_gpu - s_exact)) <= 1e-5


def test_bounded_wait_times_out_and_context_survives():
    """A pipeline wait that nothing satisfies gives up after its 1 s limit and
    reports MOE_ERR_TIMEOUT through the status word; the context stays usable."""
    import time
    ws = B().alloc_workspace(256)
    torch.cuda.synchronize()
    t0 = time.time()
    B().selftest_bounded_wait(ws)
    assert B().device_status(ws) == B().ERR_TIMEOUT
    assert 0.9 <= time.time() - t0 < 30
    assert B().device_status(ws) == B().OK          # reading the status cleared it
    # the context still works: a small routing call matches the oracle
    lg = synth.random_logits(9, 64, 8, scale=2.0)
    idx, _ = B().route_from_logits(lg.cuda(), 2)
    np.testing.assert_array_equal(as_np(idx), O.topk_select(lg.numpy(), 2))
