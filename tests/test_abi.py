"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/moe_b200.h declares, and rejects bad arguments on the host
before any CUDA call."""
import ctypes
import os
import re

import pytest

from routing_grouped_expert_moe_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")

FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced on these paths
MISALIGNED = ctypes.c_void_p(0x10008)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_header_functions_are_exported():
    names = declared_functions()
    assert len(names) >= 12
    lib = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTED)


def test_debug_build_exports_the_same_functions():
    """libmoe_b200_debug.so (MOE_DEBUG device bounds checks) is a drop-in
    replacement: same entry points, same host-side argument checks."""
    assert os.path.exists(B.DEBUG_LIB_PATH), "build with `python -m routing_grouped_expert_moe_b200.build --debug`"
    dbg = B.load_library(B.DEBUG_LIB_PATH)
    for n in declared_functions():
        assert hasattr(dbg, n), n
    assert dbg.moe_status_string(B.ERR_BOUNDS) == b"MOE_ERR_BOUNDS"
    # host-side rejection before any CUDA call, as in the release build
    assert dbg.moe_route(None, None, None, 4, 64, 8, 9, B.BF16, None, None, None, None) == \
        B.ERR_INVALID_ARG


def test_status_strings_and_version():
    assert B.status_string(B.OK) == "MOE_OK"
    assert B.status_string(B.ERR_INDEX_OUT_OF_RANGE) == "MOE_ERR_INDEX_OUT_OF_RANGE"
    assert B.status_string(B.ERR_TIMEOUT) == "MOE_ERR_TIMEOUT"
    assert B.status_string(B.ERR_BOUNDS) == "MOE_ERR_BOUNDS"
    assert "sm_100a" in B.version()


def test_workspace_bytes_monotone_and_aligned():
    a = B._lib.moe_workspace_bytes(1024, 4096, 14336, 8, 2, 0, 1)
    b = B._lib.moe_workspace_bytes(2048, 4096, 14336, 8, 2, 0, 1)
    assert a > 0 and b > a and a % 256 == 0
    # h + y + x_perm dominate: R*(F + 2H)*2 bytes
    R = 1024 * 2
    assert a >= R * (14336 + 2 * 4096) * 2
    host = B._lib.moe_forward_host_workspace_bytes(1024, 4096, 14336, 8, 2, 0, 1)
    assert host >= a + 2 * 1024 * 4096 * 2
    assert B._lib.moe_workspace_bytes(-1, 8, 8, 1, 1, 0, 1) == 0


def _fwd(T=64, H=128, F=256, E=4, k=2, cf=0.0, act=0, dt=1, x=FAKE, w1=FAKE, w3=FAKE, w2=FAKE,
         out=FAKE, ws=FAKE, ws_bytes=1 << 40):
    return B._lib.moe_forward(x, FAKE, None, w1, w3, w2, T, H, F, E, k, ctypes.c_float(cf), act, dt,
                              out, None, None, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(k=5, E=4), B.ERR_INVALID_ARG),            # top_k > E
    (dict(k=0), B.ERR_INVALID_ARG),
    (dict(H=100), B.ERR_INVALID_ARG),               # H not a multiple of 8
    (dict(F=100), B.ERR_INVALID_ARG),
    (dict(E=300, k=2), B.ERR_UNSUPPORTED),          # E > 256
    (dict(E=16, k=9), B.ERR_UNSUPPORTED),           # top_k > 8
    (dict(dt=7), B.ERR_INVALID_ARG),
    (dict(act=9), B.ERR_INVALID_ARG),
    (dict(x=None), B.ERR_INVALID_ARG),
    (dict(w3=None), B.ERR_INVALID_ARG),             # SwiGLU needs W3
    (dict(x=MISALIGNED), B.ERR_INVALID_ARG),
    (dict(ws_bytes=1024), B.ERR_WORKSPACE),
    (dict(T=1 << 20, H=4096, F=8192), B.ERR_UNSUPPORTED),   # T*k*F >= 2^31
])
def test_forward_rejects_on_host(kw, expect):
    assert _fwd(**kw) == expect


def test_forward_gelu_needs_no_w3_and_empty_input_is_ok():
    # GELU with w3 NULL passes validation up to the workspace check
    assert _fwd(act=1, w3=None, ws_bytes=16) == B.ERR_WORKSPACE
    # T = 0: nothing to do, no launch
    assert _fwd(T=0) == B.OK


def test_other_entry_points_reject_on_host():
    L = B._lib
    assert L.moe_route(FAKE, FAKE, None, 8, 64, 4, 5, 1, FAKE, FAKE, None, None) == B.ERR_INVALID_ARG
    assert L.moe_route(None, FAKE, None, 8, 64, 4, 2, 1, FAKE, FAKE, None, None) == B.ERR_INVALID_ARG
    assert L.moe_route(FAKE, FAKE, None, 0, 64, 4, 2, 1, FAKE, FAKE, None, None) == B.OK
    assert L.moe_route_from_logits(FAKE, 8, 300, 2, FAKE, FAKE, None) == B.ERR_UNSUPPORTED
    assert L.moe_permute(None, FAKE, 8, 64, 4, 2, ctypes.c_float(0), 1, None, FAKE, FAKE, FAKE,
                         FAKE, FAKE, 16, None) == B.ERR_WORKSPACE
    assert L.moe_permute(None, None, 8, 64, 4, 2, ctypes.c_float(0), 1, None, FAKE, FAKE, FAKE,
                         FAKE, FAKE, 1 << 20, None) == B.ERR_INVALID_ARG
    assert L.moe_grouped_ffn(FAKE, None, None, FAKE, FAKE, FAKE, FAKE, 16, 0, 64, 100, 4, 0, 1, FAKE,
                             FAKE, 1 << 20, None) == B.ERR_INVALID_ARG          # F % 8
    assert L.moe_grouped_ffn(FAKE, None, None, FAKE, FAKE, FAKE, FAKE, 16, 0, 64, 128, 4, 0, 1, FAKE,
                             FAKE, 300, None) == B.ERR_WORKSPACE
    assert L.moe_unpermute_combine(FAKE, FAKE, FAKE, 8, 64, 9, 1, FAKE, None) == B.ERR_UNSUPPORTED
    assert L.moe_unpermute_combine(MISALIGNED, FAKE, FAKE, 8, 64, 2, 1, FAKE, None) == B.ERR_INVALID_ARG
    assert L.moe_get_device_status(None, None) == B.ERR_INVALID_ARG


def test_binding_rejects_int64_indices_and_cpu_tensors():
    import torch
    with pytest.raises((TypeError, ValueError)):
        B.permute(torch.zeros(4, 2, dtype=torch.int64), 4)
    with pytest.raises(ValueError):
        B.route(torch.zeros(4, 8, dtype=torch.bfloat16), torch.zeros(8, 2, dtype=torch.bfloat16))


def test_route_stats_and_expert_matmul_reject_on_host():
    L = B._lib
    need = L.moe_route_stats_workspace_bytes(64, 8)
    assert need >= 64 * 8 * 4 and need % 256 == 0
    assert L.moe_route_stats_workspace_bytes(-1, 8) == 0
    args = lambda ws_bytes, prob=FAKE: (FAKE, FAKE, None, 64, 128, 8, 2, 1, FAKE, FAKE, FAKE,  # noqa: E731
                                        prob, FAKE, ws_bytes, None)
    assert L.moe_route_stats(*args(need - 1)) == B.ERR_WORKSPACE
    assert L.moe_route_stats(*args(need, prob=None)) == B.ERR_INVALID_ARG
    assert L.moe_route_stats(FAKE, FAKE, None, 64, 128, 8, 9, 1, FAKE, FAKE, FAKE, FAKE, FAKE,
                             need, None) == B.ERR_INVALID_ARG                 # top_k > E
    mneed = L.moe_expert_matmul_workspace_bytes(64, 128, 256, 8, 1)
    assert mneed >= 64 * (128 + 256) * 2 and L.moe_expert_matmul_workspace_bytes(64, 128, 0, 8, 1) == 0
    mm = lambda I=256, ws_bytes=mneed, T=64, w=FAKE: L.moe_expert_matmul(  # noqa: E731
        FAKE, w, FAKE, T, 128, I, 8, 1, FAKE, FAKE, ws_bytes, None)
    assert mm(I=100) == B.ERR_INVALID_ARG                                    # I not a multiple of 8
    assert mm(ws_bytes=mneed - 1) == B.ERR_WORKSPACE
    assert mm(w=MISALIGNED) == B.ERR_INVALID_ARG
    assert mm(T=0) == B.OK


def test_host_batches_rejects_on_host():
    L = B._lib
    need = L.moe_forward_host_batches_workspace_bytes(64, 128, 256, 4, 2, 0, 1)
    base = L.moe_workspace_bytes(64, 128, 256, 4, 2, 0, 1)
    assert need == base + 4 * 64 * 128 * 2 and need % 256 == 0
    assert L.moe_forward_host_batches_workspace_bytes(64, 128, 0, 4, 2, 0, 1) == 0
    ptrs = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    holes = (ctypes.c_void_p * 2)(0x10000, None)

    def call(n=2, xs=ptrs, outs=ptrs, k=2, ws_bytes=need, F=256):
        return L.moe_forward_host_batches(xs, outs, n, FAKE, None, FAKE, FAKE, FAKE, 64, 128, F, 4,
                                          k, ctypes.c_float(0), 0, 1, FAKE, ws_bytes, None, None,
                                          None)
    assert call(ws_bytes=need - 1) == B.ERR_WORKSPACE
    assert call(n=-1) == B.ERR_INVALID_ARG
    assert call(n=0) == B.OK                                                 # nothing to do
    assert call(xs=holes) == B.ERR_INVALID_ARG                               # a null batch
    assert call(outs=None) == B.ERR_INVALID_ARG
    assert call(k=5) == B.ERR_INVALID_ARG                                    # top_k > E
    assert call(F=100) == B.ERR_INVALID_ARG
