"""Python binding of the C ABI in include/moe_b200.h (ctypes; argument marshalling only).

Every function here checks tensor dtypes, devices, shapes and contiguity, turns
tensors into raw pointers and calls the entry point of the same name on the
current CUDA stream.  All arithmetic happens in the CUDA library; there is no
fallback: importing this module raises if ``lib/libmoe_b200.so`` is missing.
With ``MOE_LIBRARY=debug`` in the environment the module loads the debug build
``lib/libmoe_b200_debug.so`` instead (device bounds checks that report
MOE_ERR_BOUNDS; same results otherwise).

Tensors are allocated with torch (PyTorch is used for device memory and streams
only).  Expert ids are int32, as the MoE fused operators require (an int64
index tensor is rejected, lshu.cn torch_npu article §5.2).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
RELEASE_LIB_PATH = os.path.join(_PKG, "lib", "libmoe_b200.so")
DEBUG_LIB_PATH = os.path.join(_PKG, "lib", "libmoe_b200_debug.so")
LIB_PATH = DEBUG_LIB_PATH if os.environ.get("MOE_LIBRARY") == "debug" else RELEASE_LIB_PATH

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m routing_grouped_expert_moe_b200.build`")


# status codes (moe_status)
OK, ERR_INVALID_ARG, ERR_INDEX_OUT_OF_RANGE, ERR_WORKSPACE, ERR_UNSUPPORTED, ERR_CUDA, \
    ERR_TIMEOUT, ERR_BOUNDS = range(8)
F32, BF16 = 0, 1
ACT = {"swiglu": 0, "gelu": 1, "identity": 2}

_p, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "moe_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "moe_forward_host_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "moe_grouped_ffn_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "moe_route": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _p, _p, _p, _p]),
    "moe_route_from_logits": (_i, [_p, _i, _i, _i, _p, _p, _p]),
    "moe_permute": (_i, [_p, _p, _i, _i, _i, _i, _f, _i, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "moe_permute_noalloc": (_i, [_p, _p, _i, _i, _i, _i, _f, _i, _p, _p, _p, _p, _p, _p, _p]),
    "moe_grouped_ffn": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p, _sz,
                             _p]),
    "moe_unpermute_combine": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _p]),
    "moe_forward": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _i, _p, _p, _p, _p,
                         _sz, _p]),
    "moe_forward_timed": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _i, _p, _p,
                               _sz, _p, _p, _i]),
    "moe_forward_host": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _i, _p, _p, _sz,
                              _p]),
    "moe_forward_host_batches_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "moe_forward_host_batches": (_i, [_p, _p, _i, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i,
                                      _i, _p, _sz, _p, _p, _p]),
    "moe_route_stats_workspace_bytes": (_sz, [_i, _i]),
    "moe_route_stats": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _sz, _p]),
    "moe_expert_matmul_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "moe_expert_matmul": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "moe_threshold_select": (_i, [_p, _i, _i, _i, _f, _p, _p, _p, _p, _p]),
    "moe_forward_threshold_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "moe_forward_threshold": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _f, _i, _i, _p,
                                   _p, _p, _p, _sz, _p]),
    "moe_selftest_epilogue_activations": (_i, [_p, _i, _p, _p, _p]),
    "moe_selftest_bounded_wait": (_i, [_p, _p]),
    "moe_workspace_section": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _p, _p]),
    "moe_set_gemm_variant": (_i, [_i]),
    "moe_get_device_status": (_i, [_p, _p]),
    "moe_status_string": (ctypes.c_char_p, [_i]),
    "moe_version": (ctypes.c_char_p, []),
}


def load_library(path: str) -> ctypes.CDLL:
    """Opens a build of the library and declares every entry point's signature."""
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library(LIB_PATH)

EXPORTED = tuple(_SIGS)


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def status_string(s: int) -> str:
    return _lib.moe_status_string(int(s)).decode()


def version() -> str:
    return _lib.moe_version().decode()


def _check(status: int, where: str):
    if status != OK:
        raise MoEError(status, where)


def _ptr(t):
    """The tensor's address for the C ABI.  A device tensor must live on the current
    device: the kernels run there, and another GPU's memory is not theirs to read."""
    if t is None:
        return None
    if t.is_cuda and t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported element type {t.dtype} (bf16 or fp32)")


def _need(t, name, dtype=None, dim=None, cuda=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def workspace_bytes(T, H, F, E, top_k, act="swiglu", dtype=torch.bfloat16) -> int:
    return int(_lib.moe_workspace_bytes(T, H, F, E, top_k, ACT[act],
                                        BF16 if dtype == torch.bfloat16 else F32))


def forward_host_workspace_bytes(T, H, F, E, top_k, act="swiglu", dtype=torch.bfloat16) -> int:
    return int(_lib.moe_forward_host_workspace_bytes(T, H, F, E, top_k, ACT[act],
                                                     BF16 if dtype == torch.bfloat16 else F32))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def route(x, w_gate, gate_bias=None, top_k=2, logits_out=False):
    """Router: returns (topk_idx int32 [T,k], topk_gate fp32 [T,k][, logits fp32 [T,E]])."""
    _need(x, "x", dim=2)
    _need(w_gate, "w_gate", dtype=x.dtype, dim=2)
    T, H = x.shape
    E = w_gate.shape[1]
    if gate_bias is not None:
        _need(gate_bias, "gate_bias", dtype=torch.float32, dim=1)
    idx = torch.empty(T, top_k, dtype=torch.int32, device=x.device)
    gate = torch.empty(T, top_k, dtype=torch.float32, device=x.device)
    lg = torch.empty(T, E, dtype=torch.float32, device=x.device) if logits_out else None
    _check(_lib.moe_route(_ptr(x), _ptr(w_gate), _ptr(gate_bias), T, H, E, top_k, _dt(x),
                          _ptr(idx), _ptr(gate), _ptr(lg), _stream()), "moe_route")
    return (idx, gate, lg) if logits_out else (idx, gate)


def route_from_logits(logits, top_k):
    _need(logits, "logits", dtype=torch.float32, dim=2)
    T, E = logits.shape
    idx = torch.empty(T, top_k, dtype=torch.int32, device=logits.device)
    gate = torch.empty(T, top_k, dtype=torch.float32, device=logits.device)
    _check(_lib.moe_route_from_logits(_ptr(logits), T, E, top_k, _ptr(idx), _ptr(gate),
                                      _stream()), "moe_route_from_logits")
    return idx, gate


def permute(token_expert_idx, num_experts, capacity_factor=0.0, x=None, ws=None, out=None):
    """Dispatch: returns dict(counts, offsets, row_token, row_map[, x_perm]).
    out: optional dict of preallocated output tensors under those names."""
    _need(token_expert_idx, "token_expert_idx", dtype=torch.int32, dim=2)
    T, k = token_expert_idx.shape
    dev = token_expert_idx.device
    E = int(num_experts)
    if x is not None:
        _need(x, "x", dim=2)
        H, dt = x.shape[1], _dt(x)
    else:
        H, dt = 8, BF16
    out = out or {}
    counts = out.get("counts", torch.empty(E, dtype=torch.int32, device=dev))
    offsets = out.get("offsets", torch.empty(E + 1, dtype=torch.int32, device=dev))
    row_token = out.get("row_token", torch.full((T * k,), -1, dtype=torch.int32, device=dev))
    row_map = out.get("row_map", torch.empty(T, k, dtype=torch.int32, device=dev))
    x_perm = None
    if x is not None:
        x_perm = out.get("x_perm", torch.empty(T * k, H, dtype=x.dtype, device=dev))
    for name, t, n in (("counts", counts, E), ("offsets", offsets, E + 1),
                       ("row_token", row_token, T * k), ("row_map", row_map, T * k)):
        _need(t, name, dtype=torch.int32)
        if t.numel() != n or not t.is_contiguous():
            raise ValueError(f"{name}: {n} contiguous int32 entries expected")
    if ws is None:
        ws = alloc_workspace(workspace_bytes(T, H, 8, E, k, "identity",
                                             torch.bfloat16 if dt == BF16 else torch.float32), dev)
    _check(_lib.moe_permute(_ptr(x), _ptr(token_expert_idx), T, H, E, k,
                            ctypes.c_float(capacity_factor), dt, _ptr(x_perm), _ptr(counts),
                            _ptr(offsets), _ptr(row_token), _ptr(row_map), _ptr(ws), ws.numel(),
                            _stream()), "moe_permute")
    out = {"counts": counts, "offsets": offsets, "row_token": row_token, "row_map": row_map,
           "ws": ws}
    if x_perm is not None:
        out["x_perm"] = x_perm
    return out


def permute_noalloc(token_expert_idx, num_experts, capacity_factor=0.0, x=None,
                    status_out=None):
    """moe_permute without a workspace (library-owned scratch); same outputs as permute()."""
    _need(token_expert_idx, "token_expert_idx", dtype=torch.int32, dim=2)
    T, k = token_expert_idx.shape
    dev = token_expert_idx.device
    E = int(num_experts)
    if x is not None:
        _need(x, "x", dim=2)
        H, dt = x.shape[1], _dt(x)
    else:
        H, dt = 8, BF16
    if status_out is not None:
        _need(status_out, "status_out", dtype=torch.int32)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_token = torch.full((T * k,), -1, dtype=torch.int32, device=dev)
    row_map = torch.empty(T, k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * k, H, dtype=x.dtype, device=dev) if x is not None else None
    _check(_lib.moe_permute_noalloc(_ptr(x), _ptr(token_expert_idx), T, H, E, k,
                                    ctypes.c_float(capacity_factor), dt, _ptr(x_perm),
                                    _ptr(counts), _ptr(offsets), _ptr(row_token), _ptr(row_map),
                                    _ptr(status_out), _stream()), "moe_permute_noalloc")
    out = {"counts": counts, "offsets": offsets, "row_token": row_token, "row_map": row_map}
    if x_perm is not None:
        out["x_perm"] = x_perm
    return out


def grouped_ffn(expert_offsets, w1, w3, w2, act="swiglu", x_perm=None, x=None, row_token=None,
                R_max=None, ws=None, y=None):
    """Grouped expert FFN over expert-ordered rows; returns y [R_max, H]."""
    _need(expert_offsets, "expert_offsets", dtype=torch.int32, dim=1)
    E = expert_offsets.numel() - 1
    if row_token is not None:
        _need(row_token, "row_token", dtype=torch.int32)
        src = _need(x, "x", dim=2)
        R_max = int(R_max if R_max is not None else row_token.numel())
    else:
        src = _need(x_perm, "x_perm", dim=2)
        R_max = int(R_max if R_max is not None else x_perm.shape[0])
    H = src.shape[1]
    T = x.shape[0] if x is not None else 0
    if act == "identity":
        F = 8
    else:
        _need(w1, "w1", dtype=src.dtype, dim=3)
        _need(w2, "w2", dtype=src.dtype, dim=3)
        if act == "swiglu":
            _need(w3, "w3", dtype=src.dtype, dim=3)
        F = w1.shape[2]
    if y is None:
        y = torch.empty(R_max, H, dtype=src.dtype, device=src.device)
    if ws is None:
        ws = alloc_workspace(_lib.moe_grouped_ffn_workspace_bytes(
            R_max, H, F, ACT[act], _dt(src), 1 if row_token is not None else 0), src.device)
    _check(_lib.moe_grouped_ffn(_ptr(x_perm), _ptr(row_token), _ptr(x), _ptr(w1), _ptr(w3),
                                _ptr(w2), _ptr(expert_offsets), R_max, T, H, F, E, ACT[act],
                                _dt(src), _ptr(y), _ptr(ws), ws.numel(), _stream()),
           "moe_grouped_ffn")
    return y


def unpermute_combine(y, topk_gate, row_map, out=None):
    """out[t] = sum_s topk_gate[t,s] * y[row_map[t,s]]; topk_gate None means weights of 1."""
    _need(y, "y", dim=2)
    if topk_gate is not None:
        _need(topk_gate, "topk_gate", dtype=torch.float32, dim=2)
    _need(row_map, "row_map", dtype=torch.int32, dim=2)
    T, k = row_map.shape
    H = y.shape[1]
    if out is None:
        out = torch.empty(T, H, dtype=y.dtype, device=y.device)
    _check(_lib.moe_unpermute_combine(_ptr(y), _ptr(topk_gate), _ptr(row_map), T, H, k, _dt(y),
                                      _ptr(out), _stream()), "moe_unpermute_combine")
    return out


def forward(x, w_gate, gate_bias, w1, w3, w2, top_k, capacity_factor=0.0, act="swiglu",
            out=None, ws=None, topk_idx_out=None, expert_counts_out=None):
    """The whole layer; returns out [T,H] (same dtype as x)."""
    _need(x, "x", dim=2)
    _need(w_gate, "w_gate", dtype=x.dtype, dim=2)
    T, H = x.shape
    E = w_gate.shape[1]
    if gate_bias is not None:
        _need(gate_bias, "gate_bias", dtype=torch.float32, dim=1)
    if act == "identity":
        F = 8
    else:
        _need(w1, "w1", dtype=x.dtype, dim=3)
        _need(w2, "w2", dtype=x.dtype, dim=3)
        if act == "swiglu":
            _need(w3, "w3", dtype=x.dtype, dim=3)
        F = w1.shape[2]
    if out is None:
        out = torch.empty_like(x)
    if ws is None:
        ws = alloc_workspace(workspace_bytes(T, H, F, E, top_k, act, x.dtype), x.device)
    if topk_idx_out is not None:
        _need(topk_idx_out, "topk_idx_out", dtype=torch.int32)
    if expert_counts_out is not None:
        _need(expert_counts_out, "expert_counts_out", dtype=torch.int32)
    _check(_lib.moe_forward(_ptr(x), _ptr(w_gate), _ptr(gate_bias), _ptr(w1), _ptr(w3), _ptr(w2),
                            T, H, F, E, top_k, ctypes.c_float(capacity_factor), ACT[act], _dt(x),
                            _ptr(out), _ptr(topk_idx_out), _ptr(expert_counts_out), _ptr(ws),
                            ws.numel(), _stream()), "moe_forward")
    return out


def forward_timed(x, w_gate, gate_bias, w1, w3, w2, top_k, capacity_factor, act, out, ws,
                  events):
    """moe_forward recording 7 torch.cuda.Event objects at its stage boundaries
    (None entries are not recorded)."""
    for ev in events:
        if ev is not None and ev.cuda_event == 0:   # torch creates the CUDA event on first record
            ev.record()
    handles = (ctypes.c_void_p * len(events))(*[None if ev is None else ev.cuda_event
                                                for ev in events])
    T, H = x.shape
    E = w_gate.shape[1]
    F = 8 if act == "identity" else w1.shape[2]
    _check(_lib.moe_forward_timed(_ptr(x), _ptr(w_gate), _ptr(gate_bias), _ptr(w1), _ptr(w3),
                                  _ptr(w2), T, H, F, E, top_k, ctypes.c_float(capacity_factor),
                                  ACT[act], _dt(x), _ptr(out), _ptr(ws), ws.numel(), _stream(),
                                  handles, len(events)), "moe_forward_timed")
    return out


def forward_host(x_host, w_gate, gate_bias, w1, w3, w2, top_k, capacity_factor=0.0,
                 act="swiglu", out_host=None, ws=None):
    """The whole layer with x and out in page-locked host memory (copies on the stream)."""
    _need(x_host, "x_host", dim=2, cuda=False)
    T, H = x_host.shape
    E = w_gate.shape[1]
    F = 8 if act == "identity" else w1.shape[2]
    if out_host is None:
        out_host = torch.empty_like(x_host, pin_memory=True)
    if ws is None:
        ws = alloc_workspace(forward_host_workspace_bytes(T, H, F, E, top_k, act, x_host.dtype),
                             w_gate.device)
    _check(_lib.moe_forward_host(_ptr(x_host), _ptr(w_gate), _ptr(gate_bias), _ptr(w1), _ptr(w3),
                                 _ptr(w2), T, H, F, E, top_k, ctypes.c_float(capacity_factor),
                                 ACT[act], _dt(x_host), _ptr(out_host), _ptr(ws), ws.numel(),
                                 _stream()), "moe_forward_host")
    return out_host


def forward_host_batches_workspace_bytes(T, H, F, E, top_k, act="swiglu",
                                         dtype=torch.bfloat16) -> int:
    return int(_lib.moe_forward_host_batches_workspace_bytes(
        T, H, F, E, top_k, ACT[act], BF16 if dtype == torch.bfloat16 else F32))


def forward_host_batches(x_hosts, w_gate, gate_bias, w1, w3, w2, top_k, capacity_factor=0.0,
                         act="swiglu", out_hosts=None, ws=None, copy_streams="new"):
    """Independent layer forwards over a list of page-locked host batches [T, H] (all the
    same shape), copy-in / layer / copy-out overlapped on three streams.  copy_streams:
    (copy_in, copy_out) torch streams, "new" for two fresh ones, None for no overlap.
    Returns the list of host outputs, valid once the current stream is synchronised; the
    host buffers must stay alive until then (the copies are asynchronous)."""
    xs = list(x_hosts)
    if not xs:
        return []
    for i, xh in enumerate(xs):
        _need(xh, f"x_hosts[{i}]", dtype=xs[0].dtype, dim=2, cuda=False)
        if xh.is_cuda:
            raise ValueError(f"x_hosts[{i}] must be in host memory")
        if xh.shape != xs[0].shape:
            raise ValueError(f"x_hosts[{i}] has shape {tuple(xh.shape)}, "
                             f"x_hosts[0] {tuple(xs[0].shape)}")
    T, H = xs[0].shape
    E = w_gate.shape[1]
    F = 8 if act == "identity" else w1.shape[2]
    if out_hosts is None:
        out_hosts = [torch.empty_like(xh, pin_memory=True) for xh in xs]
    outs = list(out_hosts)
    if len(outs) != len(xs):
        raise ValueError(f"{len(xs)} input batches but {len(outs)} outputs")
    for i, oh in enumerate(outs):
        _need(oh, f"out_hosts[{i}]", dtype=xs[0].dtype, dim=2, cuda=False)
        if oh.is_cuda:
            raise ValueError(f"out_hosts[{i}] must be in host memory")
        if oh.shape != xs[0].shape:
            raise ValueError(f"out_hosts[{i}] has shape {tuple(oh.shape)}")
    if ws is None:
        ws = alloc_workspace(forward_host_batches_workspace_bytes(T, H, F, E, top_k, act,
                                                                  xs[0].dtype), w_gate.device)
    if copy_streams == "new":
        copy_streams = (torch.cuda.Stream(w_gate.device), torch.cuda.Stream(w_gate.device))
    cin, cout = (None, None) if copy_streams is None else copy_streams
    for st in (cin, cout):
        if st is not None and st.device.index != torch.cuda.current_device():
            raise ValueError(f"copy stream on {st.device}, but the current device is "
                             f"cuda:{torch.cuda.current_device()}")
    xp = (ctypes.c_void_p * len(xs))(*[xh.data_ptr() for xh in xs])
    op = (ctypes.c_void_p * len(outs))(*[oh.data_ptr() for oh in outs])
    _check(_lib.moe_forward_host_batches(
        xp, op, len(xs), _ptr(w_gate), _ptr(gate_bias), _ptr(w1), _ptr(w3), _ptr(w2), T, H, F,
        E, top_k, ctypes.c_float(capacity_factor), ACT[act], _dt(xs[0]), _ptr(ws), ws.numel(),
        _stream(), None if cin is None else cin.cuda_stream,
        None if cout is None else cout.cuda_stream), "moe_forward_host_batches")
    return outs


def route_stats(x, w_gate, gate_bias=None, top_k=2, ws=None):
    """Router plus its load statistics: returns (topk_idx, topk_gate, expert_counts int32 [E],
    prob_mean fp32 [E]) and the workspace (for device_status)."""
    _need(x, "x", dim=2)
    _need(w_gate, "w_gate", dtype=x.dtype, dim=2)
    T, H = x.shape
    E = w_gate.shape[1]
    if gate_bias is not None:
        _need(gate_bias, "gate_bias", dtype=torch.float32, dim=1)
    dev = x.device
    idx = torch.empty(T, top_k, dtype=torch.int32, device=dev)
    gate = torch.empty(T, top_k, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    prob = torch.empty(E, dtype=torch.float32, device=dev)
    if ws is None:
        ws = alloc_workspace(_lib.moe_route_stats_workspace_bytes(T, E), dev)
    _check(_lib.moe_route_stats(_ptr(x), _ptr(w_gate), _ptr(gate_bias), T, H, E, top_k, _dt(x),
                                _ptr(idx), _ptr(gate), _ptr(counts), _ptr(prob), _ptr(ws),
                                ws.numel(), _stream()), "moe_route_stats")
    return idx, gate, counts, prob, ws


def expert_matmul(x, expert_weight, token_expert_idx, out=None, ws=None):
    """out[t] = x[t] @ expert_weight[token_expert_idx[t]] (one expert per token).
    Returns (out [T, I], ws)."""
    _need(x, "x", dim=2)
    _need(expert_weight, "expert_weight", dtype=x.dtype, dim=3)
    _need(token_expert_idx, "token_expert_idx", dtype=torch.int32, dim=1)
    T, H = x.shape
    E, H2, I = expert_weight.shape
    if H2 != H or token_expert_idx.shape[0] != T:
        raise ValueError("shape mismatch between x, expert_weight and token_expert_idx")
    dev = x.device
    if out is None:
        out = torch.empty(T, I, dtype=x.dtype, device=dev)
    if ws is None:
        ws = alloc_workspace(_lib.moe_expert_matmul_workspace_bytes(T, H, I, E, _dt(x)), dev)
    _check(_lib.moe_expert_matmul(_ptr(x), _ptr(expert_weight), _ptr(token_expert_idx), T, H, I, E,
                                  _dt(x), _ptr(out), _ptr(ws), ws.numel(), _stream()),
           "moe_expert_matmul")
    return out, ws


def threshold_select(logits, k_max, delta=0.0, token_offsets=False):
    """Threshold gating from fp32 logits: (idx [T,k_max] (-1 pads), gate [T,k_max],
    n_selected [T][, token_offsets [T+1]])."""
    _need(logits, "logits", dtype=torch.float32, dim=2)
    T, E = logits.shape
    dev = logits.device
    idx = torch.empty(T, k_max, dtype=torch.int32, device=dev)
    gate = torch.empty(T, k_max, dtype=torch.float32, device=dev)
    n = torch.empty(T, dtype=torch.int32, device=dev)
    offs = torch.empty(T + 1, dtype=torch.int32, device=dev) if token_offsets else None
    _check(_lib.moe_threshold_select(_ptr(logits), T, E, k_max, ctypes.c_float(delta), _ptr(idx),
                                     _ptr(gate), _ptr(n), _ptr(offs), _stream()),
           "moe_threshold_select")
    return (idx, gate, n, offs) if token_offsets else (idx, gate, n)


def forward_threshold(x, w_gate, gate_bias, w1, w3, w2, k_max, delta=0.0, capacity_factor=0.0,
                      act="swiglu", out=None, ws=None, topk_idx_out=None, n_selected_out=None):
    """The layer with threshold gating; returns (out, ws)."""
    _need(x, "x", dim=2)
    T, H = x.shape
    E = w_gate.shape[1]
    F = 8 if act == "identity" else w1.shape[2]
    if out is None:
        out = torch.empty_like(x)
    if ws is None:
        ws = alloc_workspace(_lib.moe_forward_threshold_workspace_bytes(T, H, F, E, k_max, ACT[act],
                                                                         _dt(x)), x.device)
    _check(_lib.moe_forward_threshold(_ptr(x), _ptr(w_gate), _ptr(gate_bias), _ptr(w1), _ptr(w3),
                                      _ptr(w2), T, H, F, E, k_max, ctypes.c_float(delta),
                                      ctypes.c_float(capacity_factor), ACT[act], _dt(x), _ptr(out),
                                      _ptr(topk_idx_out), _ptr(n_selected_out), _ptr(ws),
                                      ws.numel(), _stream()), "moe_forward_threshold")
    return out, ws


def epilogue_activations(z):
    """(gelu, silu) of fp32 z as the bf16 GEMM epilogue computes them (self-test hook)."""
    _need(z, "z", dtype=torch.float32)
    z = z.contiguous()
    g, s = torch.empty_like(z), torch.empty_like(z)
    _check(_lib.moe_selftest_epilogue_activations(_ptr(z), z.numel(), _ptr(g), _ptr(s), _stream()),
           "moe_selftest_epilogue_activations")
    return g, s


def selftest_bounded_wait(ws):
    """Enqueue the self-test whose bounded wait must time out (see device_status)."""
    _check(_lib.moe_selftest_bounded_wait(_ptr(ws), _stream()), "moe_selftest_bounded_wait")


def device_status(ws) -> int:
    """Synchronises the current stream and returns (and clears) the kernels' status word."""
    return int(_lib.moe_get_device_status(_ptr(ws), _stream()))


WS_SECTIONS = {"topk_idx": 0, "topk_gate": 1, "counts": 2, "offsets": 3, "row_token": 4,
               "row_map": 5, "x_perm": 6, "h": 7, "y": 8}
GEMM_VARIANTS = {"auto": 0, "rows128": 1, "rows256_pair": 2, "tokens_pair": 3,
                 "tokens_pair_nosplit": 4}


def workspace_section(ws, name, T, H, F, E, top_k, act="swiglu", dtype=torch.bfloat16):
    """The view of section `name` of a fused-forward workspace (uint8 tensor
    `ws`), per moe_workspace_section: read it once the forward has completed."""
    off, nb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(_lib.moe_workspace_section(T, H, F, E, top_k, ACT[act], BF16 if dtype == torch.bfloat16 else F32,
                                      WS_SECTIONS[name], ctypes.byref(off), ctypes.byref(nb)),
           "moe_workspace_section")
    return ws[off.value:off.value + nb.value]


def set_gemm_variant(variant) -> None:
    """Select the bf16 grouped-GEMM kernel process-wide ("auto", "rows128",
    "rows256_pair", "tokens_pair", or 0..3), per moe_set_gemm_variant."""
    v = GEMM_VARIANTS[variant] if isinstance(variant, str) else int(variant)
    _check(_lib.moe_set_gemm_variant(v), "moe_set_gemm_variant")
