"""The debug build and the launch-plan log, on the GPU.

libmoe_b200_debug.so is the library compiled with MOE_DEBUG: kernels check
internal indices before the accesses they guard and report MOE_ERR_BOUNDS
instead of trapping.  On valid inputs no check may fire and every result must
equal the release build's bit for bit (the checks only guard accesses).
MOE_LOG=1 prints one line per launch and per plan decision to stderr.
"""
import ctypes
import os
import subprocess
import sys

import pytest
import torch

from routing_grouped_expert_moe_b200 import binding as B
from routing_grouped_expert_moe_b200 import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def small_cfg(base_name, **kw):
    from dataclasses import replace
    return replace(synth.CONFIGS[base_name], **kw)


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _forward_with(lib, cfg, g):
    """moe_forward through one build of the library; returns out, ids, counts, status."""
    T, H, F, E, k = cfg.T, cfg.H, cfg.F, cfg.E, cfg.top_k
    dt = g["x"].dtype
    out = torch.full_like(g["x"], float("nan"))
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    nbytes = lib.moe_workspace_bytes(T, H, F, E, k, B.ACT[cfg.act], B._dt(g["x"]))
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    st = lib.moe_forward(_p(g["x"]), _p(g["w_gate"]), _p(g["gate_bias"]), _p(g["w1"]),
                         _p(g["w3"]), _p(g["w2"]), T, H, F, E, k,
                         ctypes.c_float(cfg.capacity_factor), B.ACT[cfg.act], B._dt(g["x"]),
                         _p(out), _p(idx), _p(counts), _p(ws), nbytes,
                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == B.OK, B.status_string(st)
    dev_status = lib.moe_get_device_status(_p(ws), ctypes.c_void_p(
        torch.cuda.current_stream().cuda_stream))
    assert out.dtype == dt
    return out, idx, counts, dev_status


CASES = [
    small_cfg("mixtral_e8", name="dbg_swiglu", T=600, H=256, F=384, seed=7101),
    small_cfg("page1_gelu", name="dbg_gelu_drop", T=900, H=256, F=512, capacity_factor=0.6,
              seed=7102),
    small_cfg("e128_skew", name="dbg_skew", T=1200, H=128, F=256, seed=7103),
    small_cfg("tiny_f32", name="dbg_f32", T=300, seed=7104),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_debug_build_matches_release_and_raises_nothing(cfg):
    dbg = B.load_library(B.DEBUG_LIB_PATH)
    g = {k: (None if v is None else v.cuda()) for k, v in synth.make_inputs(cfg).items()}
    rel = _forward_with(B._lib, cfg, g)
    got = _forward_with(dbg, cfg, g)
    assert rel[3] == B.OK and got[3] == B.OK, (B.status_string(rel[3]), B.status_string(got[3]))
    for a, b in zip(rel[:3], got[:3]):
        assert torch.equal(a, b)


def test_debug_build_reports_bad_ids_like_release():
    """Caller errors the release build reports keep their own code in the
    debug build (its bounds checks guard internal indices only)."""
    dbg = B.load_library(B.DEBUG_LIB_PATH)
    T, E, k, H = 500, 8, 2, 64
    ids = synth.random_expert_ids(7, T, E, k).cuda()
    ids[10, 0] = E + 3
    x = synth.normal(7, 0, (T, H), 1.0, torch.bfloat16).cuda()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for lib in (B._lib, dbg):
        counts = torch.empty(E, dtype=torch.int32, device="cuda")
        offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        rt = torch.empty(T * k, dtype=torch.int32, device="cuda")
        rm = torch.empty(T * k, dtype=torch.int32, device="cuda")
        xp = torch.empty(T * k, H, dtype=torch.bfloat16, device="cuda")
        nbytes = lib.moe_workspace_bytes(T, H, 8, E, k, B.ACT["identity"], B.BF16)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        st = lib.moe_permute(_p(x), _p(ids), T, H, E, k, ctypes.c_float(0.0), B.BF16, _p(xp),
                             _p(counts), _p(offs), _p(rt), _p(rm), _p(ws), nbytes, s)
        assert st == B.OK
        assert lib.moe_get_device_status(_p(ws), s) == B.ERR_INDEX_OUT_OF_RANGE
        assert int(rm[10 * k].item()) == -1


def test_launch_plan_log():
    """MOE_LOG=1 (read when the library loads, so in a child process): the
    router, scatter, GEMM and combine plans and every launch appear on stderr."""
    code = (
        "import torch\n"
        "from routing_grouped_expert_moe_b200 import binding as B, synth\n"
        "from dataclasses import replace\n"
        "cfg = replace(synth.CONFIGS['mixtral_e8'], name='log', T=256, H=256, F=512, seed=7105)\n"
        "g = {k: (None if v is None else v.cuda()) for k, v in synth.make_inputs(cfg).items()}\n"
        "B.forward(g['x'], g['w_gate'], g['gate_bias'], g['w1'], g['w3'], g['w2'], cfg.top_k,\n"
        "          cfg.capacity_factor, cfg.act)\n"
        "torch.cuda.synchronize()\n")
    env = dict(os.environ, MOE_LOG="1", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stderr.splitlines() if ln.startswith("[moe] ")]
    text = "\n".join(lines)
    for part in ("router T=256", "scatter T=256", "grouped GEMM mode=1 (SwiGLU)",
                 "grouped GEMM mode=2 (down)", "token-as-N GEMM", "combine T=256",
                 "launch moe::k_clear_status", "launch moe::k_scatter", "launch moe::k_combine",
                 "launch moe::k_gemm_tokn<1, 2"):
        assert part in text, (part, text)
    assert sum(ln.startswith("[moe] launch ") for ln in lines) == 6  # the fused forward's launches


def test_fuzz_through_the_debug_build():
    """The seeded random shapes of test_gpu_fuzz.py (T from 1, E up to 256, top-1
    to top-8, both activations and storage types, capacity limits, threshold
    gating, the k = 1 matmul) through the debug build, in a child process: every
    case asserts MOE_OK, so no device bounds check may fire."""
    env = dict(os.environ, MOE_LIBRARY="debug", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_fuzz.py")],
                       env=env, capture_output=True, text=True, timeout=1200, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
