"""Thin ctypes binding over libjanus.so (the C ABI declared in include/janus.h).

Argument marshalling only: every function checks tensor placement/dtype,
allocates outputs and workspaces with PyTorch (device memory is PyTorch's
job here), passes raw device pointers and the current CUDA stream, and turns a
non-zero ``janus_status`` into ``JanusError``.  Every step of the computation
runs in the library's CUDA kernels; there is no CPU or PyTorch fallback, and
importing this module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjanus.so")
# the debug build (index arrays checked on the device, see janus_debug_check)
DEBUG_LIB_PATH = os.path.join(_HERE, "libjanus_debug.so")

JANUS_OK = 0
JANUS_ERR_INVALID_ARG = 1
JANUS_ERR_MISALIGNED = 2
JANUS_ERR_CUDA = 3
JANUS_ERR_DATA = 4

JANUS_FFN_FP32_SIMT = 0
JANUS_FFN_3XTF32 = 1

# Every entry point declared in include/janus.h.
SYMBOLS = (
    "janus_status_string", "janus_version", "janus_check",
    "janus_route_workspace_size", "janus_route",
    "janus_route_layers_workspace_size", "janus_route_layers", "janus_active_experts",
    "janus_dispatch", "janus_dispatch_split_workspace_size", "janus_dispatch_split",
    "janus_quant_by_type_workspace_size", "janus_quant_by_type", "janus_quant_by_type_noalloc",
    "janus_dequant_by_type", "janus_dispatch_row_scales",
    "janus_expert_ffn_workspace_size", "janus_expert_ffn_fwd", "janus_expert_ffn_vjp",
    "janus_expert_ffn_fwd_rows", "janus_expert_ffn_vjp_rows", "janus_expert_ffn_fwd_ex",
    "janus_expert_ffn_packed_workspace_size", "janus_expert_ffn_fwd_packed", "janus_expert_ffn_f16_min_rows_per_expert",
    "janus_expert_weights_f16_size", "janus_expert_weights_f16",
    "janus_expert_ffn_split_workspace_size", "janus_expert_ffn_fwd_split", "janus_expert_ffn_vjp_split",
    "janus_expert_ffn_weight_grad_workspace_size", "janus_expert_ffn_weight_grad",
    "janus_expert_ffn_vjp_vjp_workspace_size", "janus_expert_ffn_vjp_vjp",
    "janus_combine", "janus_edge_aggregate", "janus_edge_broadcast", "janus_neighbor_aggregate",
    "janus_ep_layout", "janus_ep_dispatch_quant", "janus_ep_dispatch", "janus_ep_dequant_rows",
    "janus_ep_return", "janus_ep_return_rows",
    "janus_ipc_get_handle", "janus_ipc_open_handle", "janus_ipc_close_handle",
    "janus_debug_build", "janus_debug_check", "janus_debug_inject_launch_failures",
    "janus_trace_start", "janus_trace_stop", "janus_trace_count", "janus_trace_get", "janus_trace_release",
)


JANUS_EP_MAX_RANKS = 8


class IpcHandle(ctypes.Structure):
    """janus_ipc_handle: the allocation's CUDA IPC handle and the byte offset
    of the pointer inside it."""
    _fields_ = [("bytes", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64)]


class JanusError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_lib = None
_loaded = {}


def _load(path: str) -> ctypes.CDLL:
    if path not in _loaded:
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m element_routed_moe_b200.build`"
                " (nvcc, sm_100a; --debug for the debug build); there is no fallback implementation")
        L = ctypes.CDLL(path)
        _declare(L)
        _loaded[path] = L
    return _loaded[path]


def lib() -> ctypes.CDLL:
    """The library every wrapper here calls: libjanus.so, or the debug build
    when the environment sets JANUS_DEBUG_LIB=1 (or after use_library)."""
    global _lib
    if _lib is None:
        _lib = _load(DEBUG_LIB_PATH if os.environ.get("JANUS_DEBUG_LIB") == "1" else LIB_PATH)
    return _lib


def use_library(debug: bool) -> ctypes.CDLL:
    """Route every wrapper to the debug build (True) or the release build."""
    global _lib
    _lib = _load(DEBUG_LIB_PATH if debug else LIB_PATH)
    return _lib


def _declare(L):
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    psz = ctypes.POINTER(ctypes.c_size_t)
    st = ctypes.c_int
    sig = {
        "janus_status_string": (ctypes.c_char_p, [st]),
        "janus_version": (i32, []),
        "janus_check": (st, [vp, vp]),
        "janus_route_workspace_size": (st, [i64, i32, i32, i32, psz]),
        "janus_route": (st, [vp, i64, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "janus_route_layers_workspace_size": (st, [i64, i32, i32, i32, i32, psz]),
        "janus_route_layers": (st, [vp, i64, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz,
                                    vp]),
        "janus_active_experts": (st, [vp, i32, i32, vp, vp, vp]),
        "janus_dispatch": (st, [vp, i64, i32, i32, vp, vp, vp, vp]),
        "janus_dispatch_split_workspace_size": (st, [i64, psz]),
        "janus_dispatch_split": (st, [vp, i64, i32, i32, vp, vp, vp, vp, vp, sz, vp]),
        "janus_quant_by_type_workspace_size": (st, [i32, psz]),
        "janus_quant_by_type": (st, [vp, i64, i32, i32, vp, i32, vp, vp, vp, vp, sz, vp]),
        "janus_quant_by_type_noalloc": (st, [vp, i64, i32, i32, vp, i32, vp, vp, vp, vp]),
        "janus_dequant_by_type": (st, [vp, i64, i32, i32, vp, i32, vp, vp, vp, vp]),
        "janus_dispatch_row_scales": (st, [i64, i32, vp, i32, vp, vp, vp, vp]),
        "janus_expert_ffn_workspace_size": (st, [i64, i32, i32, i32, i32, i32, ctypes.c_int, psz]),
        "janus_expert_ffn_fwd": (st, [vp, vp, i32, i64, i32, i32, vp, vp, vp, vp, ctypes.c_int,
                                      vp, sz, vp]),
        "janus_expert_ffn_vjp": (st, [vp, vp, vp, vp, i32, i64, i32, i32, vp, vp, vp,
                                      ctypes.c_int, vp, sz, vp]),
        "janus_expert_ffn_fwd_rows": (st, [vp, vp, i32, i64, i32, i32, vp, vp, vp, vp, ctypes.c_int,
                                           vp, sz, vp]),
        "janus_expert_ffn_vjp_rows": (st, [vp, vp, vp, vp, i32, i64, i32, i32, vp, vp, vp,
                                           ctypes.c_int, vp, sz, vp]),
        "janus_expert_ffn_fwd_ex": (st, [vp, vp, i32, i64, i32, i32, vp, vp, vp, vp, vp, ctypes.c_uint32,
                                         ctypes.c_int, vp, sz, vp]),
        "janus_expert_ffn_packed_workspace_size": (st, [i64, i32, i32, i32, ctypes.c_int, psz]),
        "janus_expert_ffn_f16_min_rows_per_expert": (i32, []),
        "janus_expert_weights_f16_size": (st, [i32, i32, i32, psz]),
        "janus_expert_weights_f16": (st, [vp, vp, i32, i32, i32, ctypes.c_uint32, vp, sz, vp]),
        "janus_expert_ffn_fwd_packed": (st, [vp, vp, vp, i32, i64, i32, i32, vp, vp, vp, vp, vp, vp, sz,
                                             ctypes.c_int, vp, sz, vp]),
        "janus_expert_ffn_split_workspace_size": (st, [i64, i32, i32, i32, psz]),
        "janus_expert_ffn_fwd_split": (st, [vp, vp, vp, i32, i64, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp, sz,
                                            vp]),
        "janus_expert_ffn_vjp_split": (st, [vp, vp, vp, vp, i32, i64, i32, i32, vp, vp, vp, vp, vp, sz, vp, sz,
                                            vp]),
        "janus_expert_ffn_weight_grad_workspace_size": (st, [i64, i32, i32, psz]),
        "janus_expert_ffn_weight_grad": (st, [vp, vp, vp, vp, i32, i64, i32, i32, vp, vp, vp, vp,
                                              ctypes.c_int, vp, sz, vp]),
        "janus_expert_ffn_vjp_vjp_workspace_size": (st, [i64, i32, i32, i32, psz]),
        "janus_expert_ffn_vjp_vjp": (st, [vp, vp, vp, vp, vp, i32, i64, i32, i32, vp, vp, vp, vp, vp, vp,
                                          i32, vp, sz, vp]),
        "janus_combine": (st, [vp, vp, vp, i64, i32, i32, vp, vp]),
        "janus_edge_aggregate": (st, [vp, i64, vp, i64, i32, vp, vp]),
        "janus_edge_broadcast": (st, [vp, vp, i64, i32, vp, i64, vp]),
        "janus_neighbor_aggregate": (st, [vp, vp, vp, i64, i64, i32, vp, vp]),
        "janus_ep_layout": (st, [vp, i32, i32, i64, vp, vp, vp, vp]),
        "janus_ep_dispatch_quant": (st, [vp, i64, i32, i32, vp, i32, vp, vp, vp, vp, i32, i32, i32, i64, vp, vp,
                                         vp, vp, sz, vp]),
        "janus_ep_dispatch": (st, [vp, i64, i32, i32, vp, vp, vp, vp, vp, i32, i32, i32, i64, vp, vp, vp]),
        "janus_ep_dequant_rows": (st, [vp, vp, vp, i32, i32, i32, i64, i32, vp, vp]),
        "janus_ep_return": (st, [vp, vp, vp, vp, vp, i32, i32, i32, i64, i32, vp, vp]),
        "janus_ep_return_rows": (st, [vp, vp, vp, i32, i32, i32, i64, i32, vp, vp, vp]),
        "janus_ipc_get_handle": (st, [vp, ctypes.POINTER(IpcHandle)]),
        "janus_ipc_open_handle": (st, [ctypes.POINTER(IpcHandle), ctypes.POINTER(ctypes.c_void_p)]),
        "janus_ipc_close_handle": (st, [vp, ctypes.c_uint64]),
        "janus_debug_build": (i32, []),
        "janus_debug_check": (st, [vp]),
        "janus_debug_inject_launch_failures": (None, [i32]),
        "janus_trace_start": (st, [i32]),
        "janus_trace_stop": (st, []),
        "janus_trace_count": (st, [ctypes.POINTER(ctypes.c_int32)]),
        "janus_trace_get": (st, [i32, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float)]),
        "janus_trace_release": (st, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args


def status_string(status: int) -> str:
    return lib().janus_status_string(int(status)).decode()


def version() -> int:
    return int(lib().janus_version())


def _raise(status: int, where: str):
    if status != JANUS_OK:
        raise JanusError(status, where)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _p(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr() if t.numel() > 0 else None


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


def _workspace(nbytes, device, ws):
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError("workspace too small")
        return ws
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# --------------------------------------------------------------------------
# routing
# --------------------------------------------------------------------------
def janus_route_workspace_size(n_atoms: int, n_types: int, n_experts: int, top_k: int) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_route_workspace_size(n_atoms, n_types, n_experts, top_k, ctypes.byref(b)),
           "janus_route_workspace_size")
    return b.value


def janus_route(types, gate, top_k, *, out=None, workspace=None, stream=None):
    """Static per-element top-K routing; returns a dict of device tensors
    (topk_expert, topk_weight, counts, offsets, perm, slot_of, workspace)."""
    dev = gate.device
    N = types.shape[0]
    T, E = gate.shape
    K = int(top_k)
    R = N * K
    if out is None:
        out = dict(topk_expert=_empty((N, K), torch.int32, dev),
                   topk_weight=_empty((N, K), torch.float32, dev),
                   counts=_empty((E,), torch.int32, dev),
                   offsets=_empty((E + 1,), torch.int32, dev),
                   perm=_empty((R,), torch.int32, dev),
                   slot_of=_empty((R,), torch.int32, dev))
    nb = janus_route_workspace_size(N, T, E, K)
    ws = _workspace(nb, dev, workspace)
    _raise(lib().janus_route(_p(types, torch.int32, "types"), N, _p(gate, torch.float32, "gate"),
                             T, E, K, _p(out["topk_expert"]), _p(out["topk_weight"]),
                             _p(out["counts"]), _p(out["offsets"]), _p(out["perm"]),
                             _p(out["slot_of"]), _p(ws), nb, _stream(stream)), "janus_route")
    out["workspace"] = ws
    return out


def janus_route_layers_workspace_size(n_atoms, n_types, n_experts, top_k, n_layers) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_route_layers_workspace_size(n_atoms, n_types, n_experts, top_k, n_layers,
                                                   ctypes.byref(b)), "janus_route_layers_workspace_size")
    return b.value


def janus_route_layers(types, gates, top_k, *, workspace=None, stream=None):
    """Routes gates [L,T,E] for the same atoms; returns per-layer stacked
    device tensors (topk_expert [L,N,K], ..., offsets [L,E+1], perm [L,R])."""
    dev = gates.device
    N = types.shape[0]
    L, T, E = gates.shape
    K = int(top_k)
    R = N * K
    out = dict(topk_expert=_empty((L, N, K), torch.int32, dev),
               topk_weight=_empty((L, N, K), torch.float32, dev),
               counts=_empty((L, E), torch.int32, dev),
               offsets=_empty((L, E + 1), torch.int32, dev),
               perm=_empty((L, R), torch.int32, dev),
               slot_of=_empty((L, R), torch.int32, dev))
    nb = janus_route_layers_workspace_size(N, T, E, K, L)
    ws = _workspace(nb, dev, workspace)
    _raise(lib().janus_route_layers(_p(types, torch.int32, "types"), N, _p(gates, torch.float32, "gates"),
                                    L, T, E, K, _p(out["topk_expert"]), _p(out["topk_weight"]),
                                    _p(out["counts"]), _p(out["offsets"]), _p(out["perm"]),
                                    _p(out["slot_of"]), _p(ws), nb, _stream(stream)), "janus_route_layers")
    out["workspace"] = ws
    return out


def janus_check(workspace, stream=None):
    _raise(lib().janus_check(_p(workspace), _stream(stream)), "janus_check")


# --------------------------------------------------------------------------
# dispatch / combine
# --------------------------------------------------------------------------
def janus_active_experts(counts, *, active=None, n_active=None, stream=None):
    """Per layer, the ids of the experts with routed rows (ascending) and their
    number: (active [L,E] (first n_active[l] valid), n_active [L])."""
    c = counts.reshape(-1, counts.shape[-1])
    L, E = c.shape
    if active is None:
        active = torch.full((L, E), -1, dtype=torch.int32, device=counts.device)
    if n_active is None:
        n_active = _empty((L,), torch.int32, counts.device)
    _raise(lib().janus_active_experts(_p(c.contiguous(), torch.int32, "counts"), L, E,
                                      _p(active, torch.int32, "active"), _p(n_active, torch.int32, "n_active"),
                                      _stream(stream)), "janus_active_experts")
    return active, n_active


def janus_dispatch(x, slot_of, top_k, topk_weight=None, *, out=None, stream=None):
    N, d = x.shape
    K = int(top_k)
    if out is None:
        out = _empty((N * K, d), torch.float32, x.device)
    _raise(lib().janus_dispatch(_p(x, torch.float32, "x"), N, d, K,
                                _p(slot_of, torch.int32, "slot_of"),
                                _p(topk_weight, torch.float32, "topk_weight"),
                                _p(out, torch.float32, "xd"), _stream(stream)), "janus_dispatch")
    return out


def janus_dispatch_split_workspace_size(n_atoms) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_dispatch_split_workspace_size(int(n_atoms), ctypes.byref(b)),
           "janus_dispatch_split_workspace_size")
    return b.value


def janus_dispatch_split(x, slot_of, top_k, topk_weight=None, *, out=None, row_scale=None, workspace=None,
                         stream=None):
    """Dispatch into two FP16 terms per value with a per-row power-of-two
    scale: returns (rows16 [2R, d] float16 = [hi | mid], row_scale [R])."""
    N, d = x.shape
    K = int(top_k)
    R = N * K
    if out is None:
        out = _empty((2 * R, d), torch.float16, x.device)
    if row_scale is None:
        row_scale = _empty((R,), torch.float32, x.device)
    nb = janus_dispatch_split_workspace_size(N)
    ws = _workspace(nb, x.device, workspace)
    _raise(lib().janus_dispatch_split(_p(x, torch.float32, "x"), N, d, K, _p(slot_of, torch.int32, "slot_of"),
                                      _p(topk_weight, torch.float32, "topk_weight"), _p(out, torch.float16, "rows16"),
                                      _p(row_scale, torch.float32, "row_scale"), _p(ws), nb, _stream(stream)),
           "janus_dispatch_split")
    return out, row_scale


def janus_combine(yd, slot_of, top_k, topk_weight=None, *, out=None, stream=None):
    K = int(top_k)
    R, d = yd.shape
    N = slot_of.shape[0] // K
    if out is None:
        out = _empty((N, d), torch.float32, yd.device)
    _raise(lib().janus_combine(_p(yd, torch.float32, "yd"), _p(slot_of, torch.int32, "slot_of"),
                               _p(topk_weight, torch.float32, "topk_weight"), N, K, d,
                               _p(out, torch.float32, "y"), _stream(stream)), "janus_combine")
    return out


# --------------------------------------------------------------------------
# expert-parallel exchange (rank o owns experts [o*E/P, (o+1)*E/P))
# --------------------------------------------------------------------------
def _ptr_array(ptrs):
    """Host array of device pointers (index = rank) from tensors or ints."""
    vals = [t.data_ptr() if isinstance(t, torch.Tensor) else int(t) for t in ptrs]
    return (ctypes.c_void_p * len(vals))(*vals)


def janus_ep_layout(counts_all, n_experts, recv_cap, *, src_off=None, dst_off=None, recv_off=None, stream=None):
    """Exchange layout from the gathered counts [P, E] for receive buffers of
    recv_cap rows: (src_off [P, E+1], dst_off [P, E], recv_off [P, E/P+1]),
    device int32 (recv_off clamped to recv_cap)."""
    P = counts_all.shape[0]
    E = int(n_experts)
    dev = counts_all.device
    if src_off is None:
        src_off = _empty((P, E + 1), torch.int32, dev)
    if dst_off is None:
        dst_off = _empty((P, E), torch.int32, dev)
    if recv_off is None:
        recv_off = _empty((P, E // max(P, 1) + 1), torch.int32, dev)
    _raise(lib().janus_ep_layout(_p(counts_all, torch.int32, "counts_all"), P, E, int(recv_cap),
                                 _p(src_off, torch.int32, "src_off"), _p(dst_off, torch.int32, "dst_off"),
                                 _p(recv_off, torch.int32, "recv_off"), _stream(stream)), "janus_ep_layout")
    return src_off, dst_off, recv_off


def janus_ep_dispatch_quant(x, types, n_types, route, layout, rank, recv_cap, recv_payload, recv_scale, *,
                            scale=None, workspace=None, stream=None):
    """FP16-pack this rank's routed rows and store them in their owners'
    receive buffers of recv_cap rows (recv_payload / recv_scale: one per rank,
    index = rank).  Returns (scale [T], workspace); janus_check(workspace)
    reports rows that did not fit."""
    N, d = x.shape
    K = route["topk_expert"].shape[1]
    src_off, dst_off, _ = layout
    P, E = dst_off.shape
    if scale is None:
        scale = _empty((int(n_types),), torch.float32, x.device)
    nb = janus_quant_by_type_workspace_size(n_types)
    ws = _workspace(nb, x.device, workspace)
    _raise(lib().janus_ep_dispatch_quant(_p(x, torch.float32, "x"), N, d, K, _p(types, torch.int32, "types"),
                                         int(n_types), _p(route["slot_of"], torch.int32, "slot_of"),
                                         _p(route["topk_expert"], torch.int32, "topk_expert"),
                                         _p(src_off, torch.int32, "src_off"), _p(dst_off, torch.int32, "dst_off"),
                                         int(rank), P, E, int(recv_cap), _ptr_array(recv_payload),
                                         _ptr_array(recv_scale),
                                         _p(scale, torch.float32, "scale"), _p(ws), nb, _stream(stream)),
           "janus_ep_dispatch_quant")
    return scale, ws


def janus_ep_dispatch(x, route, layout, rank, recv_cap, recv_rows, *, weighted=False, workspace=None, stream=None):
    """FP32 send of this rank's rows (times the gate weight when weighted) to
    their owners' receive buffers of recv_cap rows; rows that do not fit are
    recorded in workspace's error word when a workspace is given."""
    N, d = x.shape
    K = route["topk_expert"].shape[1]
    src_off, dst_off, _ = layout
    P, E = dst_off.shape
    _raise(lib().janus_ep_dispatch(_p(x, torch.float32, "x"), N, d, K, _p(route["slot_of"], torch.int32, "slot_of"),
                                   _p(route["topk_expert"], torch.int32, "topk_expert"),
                                   _p(route["topk_weight"] if weighted else None, torch.float32, "topk_weight"),
                                   _p(src_off, torch.int32, "src_off"), _p(dst_off, torch.int32, "dst_off"),
                                   int(rank), P, E, int(recv_cap), _ptr_array(recv_rows), _p(workspace),
                                   _stream(stream)), "janus_ep_dispatch")


def janus_ep_dequant_rows(payload, row_scale, layout, rank, *, out=None, stream=None):
    """Owner side of the FP16 send: received rows times their scales."""
    max_rows, d = payload.shape
    _, dst_off, recv_off = layout
    P, E = dst_off.shape
    if out is None:
        out = _empty((max_rows, d), torch.float32, payload.device)
    _raise(lib().janus_ep_dequant_rows(_p(payload, torch.float16, "payload"), _p(row_scale, torch.float32, "row_scale"),
                                       _p(recv_off, torch.int32, "recv_off"), int(rank), P, E, max_rows, d,
                                       _p(out, torch.float32, "xd"), _stream(stream)), "janus_ep_dequant_rows")
    return out


def janus_ep_return(yd, counts_all, layout, rank, ret_rows, *, stream=None):
    """Owner side of the return: each received row's result to its sender."""
    max_rows, d = yd.shape
    src_off, dst_off, recv_off = layout
    P, E = dst_off.shape
    _raise(lib().janus_ep_return(_p(yd, torch.float32, "yd"), _p(counts_all, torch.int32, "counts_all"),
                                 _p(src_off, torch.int32, "src_off"), _p(dst_off, torch.int32, "dst_off"),
                                 _p(recv_off, torch.int32, "recv_off"), int(rank), P, E, max_rows, d,
                                 _ptr_array(ret_rows), _stream(stream)), "janus_ep_return")


def janus_ep_return_rows(layout, rank, ret_rows, max_rows, d, *, out=None, stream=None):
    """Row table of the fused return: int64 device tensor [max_rows] holding,
    for each received row, its address in the sender's return buffer (entries
    past the received count stay as they were; a new table starts at 0)."""
    src_off, dst_off, recv_off = layout
    P, E = dst_off.shape
    if out is None:
        out = torch.zeros((max_rows,), dtype=torch.int64, device=src_off.device)
    if out.dtype != torch.int64 or out.numel() < max_rows:
        raise ValueError("out must be an int64 tensor of at least max_rows entries")
    _raise(lib().janus_ep_return_rows(_p(src_off, torch.int32, "src_off"), _p(dst_off, torch.int32, "dst_off"),
                                      _p(recv_off, torch.int32, "recv_off"), int(rank), P, E, int(max_rows),
                                      int(d), _ptr_array(ret_rows), _p(out, torch.int64, "rows"),
                                      _stream(stream)), "janus_ep_return_rows")
    return out


def janus_ipc_get_handle(t) -> bytes:
    """Serialised janus_ipc_handle of a device tensor's storage."""
    h = IpcHandle()
    _raise(lib().janus_ipc_get_handle(ctypes.c_void_p(t.data_ptr()), ctypes.byref(h)), "janus_ipc_get_handle")
    return bytes(h)


def janus_ipc_open_handle(blob: bytes) -> tuple:
    """Map another process's buffer: returns (device pointer, offset)."""
    h = IpcHandle.from_buffer_copy(blob)
    p = ctypes.c_void_p(0)
    _raise(lib().janus_ipc_open_handle(ctypes.byref(h), ctypes.byref(p)), "janus_ipc_open_handle")
    return p.value, int(h.offset)


def janus_ipc_close_handle(ptr: int, offset: int):
    _raise(lib().janus_ipc_close_handle(ctypes.c_void_p(ptr), ctypes.c_uint64(offset)), "janus_ipc_close_handle")


# --------------------------------------------------------------------------
# per-element-type FP16 packing
# --------------------------------------------------------------------------
def janus_quant_by_type_workspace_size(n_types: int) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_quant_by_type_workspace_size(n_types, ctypes.byref(b)),
           "janus_quant_by_type_workspace_size")
    return b.value


def janus_quant_by_type(x, types, n_types, slot_of, top_k, *, payload=None, scale=None,
                        workspace=None, stream=None):
    """Returns (payload [R,d] float16 (binary16 bits), scale [T] float32, workspace)."""
    N, d = x.shape
    K = int(top_k)
    if payload is None:
        payload = _empty((N * K, d), torch.float16, x.device)
    if scale is None:
        scale = _empty((n_types,), torch.float32, x.device)
    nb = janus_quant_by_type_workspace_size(n_types)
    ws = _workspace(nb, x.device, workspace)
    _raise(lib().janus_quant_by_type(_p(x, torch.float32, "x"), N, d, K,
                                     _p(types, torch.int32, "types"), int(n_types),
                                     _p(slot_of, torch.int32, "slot_of"), _p(payload, None, "payload"),
                                     _p(scale, torch.float32, "scale"), _p(ws), nb,
                                     _stream(stream)), "janus_quant_by_type")
    return payload, scale, ws


def janus_quant_by_type_noalloc(x, types, n_types, slot_of, top_k, *, payload=None, scale=None,
                                stream=None):
    """janus_quant_by_type without a workspace, for callers that cannot
    allocate device memory where they pack.  The library keeps its own
    16,640-byte scratch per GPU; calls that overlap on the GPU race.
    payload/scale are allocated here only when not given (pass them to keep
    the call allocation-free).  Returns (payload, scale)."""
    N, d = x.shape
    K = int(top_k)
    if payload is None:
        payload = _empty((N * K, d), torch.float16, x.device)
    if scale is None:
        scale = _empty((n_types,), torch.float32, x.device)
    _raise(lib().janus_quant_by_type_noalloc(_p(x, torch.float32, "x"), N, d, K,
                                             _p(types, torch.int32, "types"), int(n_types),
                                             _p(slot_of, torch.int32, "slot_of"),
                                             _p(payload, None, "payload"),
                                             _p(scale, torch.float32, "scale"), _stream(stream)),
           "janus_quant_by_type_noalloc")
    return payload, scale


def janus_dequant_by_type(payload, types, n_types, perm, top_k, scale, *, out=None, stream=None):
    R, d = payload.shape
    K = int(top_k)
    N = types.shape[0]
    if out is None:
        out = _empty((R, d), torch.float32, payload.device)
    _raise(lib().janus_dequant_by_type(_p(payload, None, "payload"), N, d, K,
                                       _p(types, torch.int32, "types"), int(n_types),
                                       _p(perm, torch.int32, "perm"),
                                       _p(scale, torch.float32, "scale"),
                                       _p(out, torch.float32, "xd"), _stream(stream)),
           "janus_dequant_by_type")
    return out


def janus_dispatch_row_scales(types, n_types, perm, top_k, scale, *, out=None, stream=None):
    """row_scale [R] = scale[type of dispatch row p] (the per-row scales the
    packed forward takes)."""
    K = int(top_k)
    N = types.shape[0]
    if out is None:
        out = _empty((N * K,), torch.float32, types.device)
    _raise(lib().janus_dispatch_row_scales(N, K, _p(types, torch.int32, "types"), int(n_types),
                                           _p(perm, torch.int32, "perm"), _p(scale, torch.float32, "scale"),
                                           _p(out, torch.float32, "row_scale"), _stream(stream)),
           "janus_dispatch_row_scales")
    return out


# --------------------------------------------------------------------------
# grouped expert MLP
# --------------------------------------------------------------------------
def janus_expert_ffn_workspace_size(n_rows, d, h, n_experts, vjp, have_act,
                                    mode=JANUS_FFN_FP32_SIMT) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_expert_ffn_workspace_size(n_rows, d, h, n_experts, int(bool(vjp)),
                                                 int(bool(have_act)), int(mode), ctypes.byref(b)),
           "janus_expert_ffn_workspace_size")
    return b.value


def janus_expert_ffn_fwd(xd, offsets, w1, w2, *, mode=JANUS_FFN_FP32_SIMT, want_act=False,
                         out=None, act=None, workspace=None, stream=None):
    """yd = silu(xd W1[e]) W2[e] per expert segment; returns (yd, act-or-None)."""
    R, d = xd.shape
    E, _, h = w1.shape
    if out is None:
        out = _empty((R, d), torch.float32, xd.device)
    if want_act and act is None:
        act = _empty((R, h), torch.float32, xd.device)
    nb = janus_expert_ffn_workspace_size(R, d, h, E, False, act is not None, mode)
    ws = _workspace(nb, xd.device, workspace)
    _raise(lib().janus_expert_ffn_fwd(_p(xd, torch.float32, "xd"),
                                      _p(offsets, torch.int32, "offsets"), E, R, d, h,
                                      _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                      _p(out, torch.float32, "yd"), _p(act, torch.float32, "act"),
                                      int(mode), _p(ws), nb, _stream(stream)),
           "janus_expert_ffn_fwd")
    return out, act


def janus_expert_ffn_vjp(xd, gd, offsets, w1, w2, *, act=None, mode=JANUS_FFN_FP32_SIMT,
                         out=None, workspace=None, stream=None):
    R, d = xd.shape
    E, _, h = w1.shape
    if out is None:
        out = _empty((R, d), torch.float32, xd.device)
    nb = janus_expert_ffn_workspace_size(R, d, h, E, True, act is not None, mode)
    ws = _workspace(nb, xd.device, workspace)
    _raise(lib().janus_expert_ffn_vjp(_p(xd, torch.float32, "xd"), _p(gd, torch.float32, "gd"),
                                      _p(act, torch.float32, "act"),
                                      _p(offsets, torch.int32, "offsets"), E, R, d, h,
                                      _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                      _p(out, torch.float32, "dxd"), int(mode), _p(ws), nb,
                                      _stream(stream)), "janus_expert_ffn_vjp")
    return out


def _row_table(rows, R):
    if rows.dtype != torch.int64 or rows.dim() != 1 or rows.numel() < R:
        raise ValueError("the row table must be a 1-D int64 tensor of at least n_rows addresses")
    return _p(rows, torch.int64, "rows")


def janus_expert_ffn_fwd_rows(xd, offsets, w1, w2, yd_rows, *, mode=JANUS_FFN_FP32_SIMT, want_act=False,
                              act=None, workspace=None, stream=None):
    """janus_expert_ffn_fwd with output row p stored at address yd_rows[p]
    (int64 device tensor of 16-byte aligned device addresses with room for d
    floats each, e.g. from janus_ep_return_rows); returns act-or-None."""
    R, d = xd.shape
    E, _, h = w1.shape
    if want_act and act is None:
        act = _empty((R, h), torch.float32, xd.device)
    nb = janus_expert_ffn_workspace_size(R, d, h, E, False, act is not None, mode)
    ws = _workspace(nb, xd.device, workspace)
    _raise(lib().janus_expert_ffn_fwd_rows(_p(xd, torch.float32, "xd"),
                                           _p(offsets, torch.int32, "offsets"), E, R, d, h,
                                           _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                           _row_table(yd_rows, R), _p(act, torch.float32, "act"),
                                           int(mode), _p(ws), nb, _stream(stream)),
           "janus_expert_ffn_fwd_rows")
    return act


JANUS_FFN_X_DEQUANTIZED = 1


def janus_expert_ffn_fwd_ex(xd, offsets, w1, w2, *, out=None, out_rows=None, flags=0, mode=JANUS_FFN_FP32_SIMT,
                            want_act=False, act=None, workspace=None, stream=None):
    """The general forward: output rows to `out` (allocated when both out and
    out_rows are None) or to the addresses in `out_rows`; flags as in the C
    header (JANUS_FFN_X_DEQUANTIZED).  Returns (out-or-None, act-or-None)."""
    R, d = xd.shape
    E, _, h = w1.shape
    if out is not None and out_rows is not None:
        raise ValueError("give out or out_rows, not both")
    if out is None and out_rows is None:
        out = _empty((R, d), torch.float32, xd.device)
    if want_act and act is None:
        act = _empty((R, h), torch.float32, xd.device)
    nb = janus_expert_ffn_workspace_size(R, d, h, E, False, act is not None, mode)
    ws = _workspace(nb, xd.device, workspace)
    _raise(lib().janus_expert_ffn_fwd_ex(_p(xd, torch.float32, "xd"), _p(offsets, torch.int32, "offsets"), E, R, d,
                                         h, _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                         _p(out, torch.float32, "yd"),
                                         None if out_rows is None else _row_table(out_rows, R),
                                         _p(act, torch.float32, "act"), int(flags), int(mode), _p(ws), nb,
                                         _stream(stream)), "janus_expert_ffn_fwd_ex")
    return out, act


def janus_expert_ffn_packed_workspace_size(n_rows, n_experts, d, h, mode=JANUS_FFN_FP32_SIMT) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_expert_ffn_packed_workspace_size(n_rows, n_experts, d, h, int(mode), ctypes.byref(b)),
           "janus_expert_ffn_packed_workspace_size")
    return b.value


def janus_expert_ffn_f16_min_rows_per_expert() -> int:
    """Rows per expert from which the packed and split MLP calls run both GEMMs
    of a direction on the FP16 tensor path (the library's rule)."""
    return int(lib().janus_expert_ffn_f16_min_rows_per_expert())


JANUS_W16_FWD = 1
JANUS_W16_VJP = 2


def janus_expert_weights_f16_size(n_experts, d, h) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_expert_weights_f16_size(int(n_experts), int(d), int(h), ctypes.byref(b)),
           "janus_expert_weights_f16_size")
    return b.value


def janus_expert_weights_f16(w1, w2, which=JANUS_W16_FWD | JANUS_W16_VJP, *, out=None, stream=None):
    """The FP16 splits of w1 [E,d,h] and w2 [E,h,d] for the FP16 MLP calls
    (their `weights16`): the forward's parts, the input VJP's, or both from
    one read of each weight tensor.  Returns the set (uint8 device tensor)."""
    E, d, h = w1.shape
    nb = janus_expert_weights_f16_size(E, d, h)
    out = _workspace(nb, w1.device, out)
    _raise(lib().janus_expert_weights_f16(_p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"), E, d, h,
                                          int(which), _p(out), out.numel() * out.element_size(), _stream(stream)),
           "janus_expert_weights_f16")
    return out


def _w16(weights16):
    if weights16 is None:
        return None, 0
    return _p(weights16, torch.uint8, "weights16"), weights16.numel()


def janus_expert_ffn_fwd_packed(payload, row_scale, offsets, w1, w2, *, out=None, out_rows=None,
                                mode=JANUS_FFN_FP32_SIMT, want_act=False, act=None, weights16=None, workspace=None,
                                stream=None):
    """The forward on the FP16 payload [R,d] with per-row scales [R] (3xTF32
    mode: the first GEMM on the FP16 tensor path against an FP16 split of
    w1, the call's own or weights16's, a set from janus_expert_weights_f16);
    output as in janus_expert_ffn_fwd_ex.  Returns (out-or-None,
    act-or-None)."""
    R, d = payload.shape
    E, _, h = w1.shape
    if payload.dtype not in (torch.float16, torch.int16, torch.uint16):
        raise ValueError("payload must hold 16-bit FP16 words")
    if out is not None and out_rows is not None:
        raise ValueError("give out or out_rows, not both")
    if out is None and out_rows is None:
        out = _empty((R, d), torch.float32, payload.device)
    if want_act and act is None:
        act = _empty((R, h), torch.float32, payload.device)
    nb = janus_expert_ffn_packed_workspace_size(R, E, d, h, mode)
    ws = _workspace(nb, payload.device, workspace)
    _raise(lib().janus_expert_ffn_fwd_packed(_p(payload, None, "payload"), _p(row_scale, torch.float32, "row_scale"),
                                             _p(offsets, torch.int32, "offsets"), E, R, d, h,
                                             _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                             _p(out, torch.float32, "yd"),
                                             None if out_rows is None else _row_table(out_rows, R),
                                             _p(act, torch.float32, "act"), *_w16(weights16), int(mode), _p(ws), nb,
                                             _stream(stream)),
           "janus_expert_ffn_fwd_packed")
    return out, act


def janus_expert_ffn_split_workspace_size(n_rows, n_experts, d, h) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_expert_ffn_split_workspace_size(int(n_rows), int(n_experts), int(d), int(h),
                                                       ctypes.byref(b)), "janus_expert_ffn_split_workspace_size")
    return b.value


def janus_expert_ffn_fwd_split(rows16, row_scale, offsets, w1, w2, *, out=None, out_rows=None, want_act=False,
                               act=None, weights16=None, workspace=None, stream=None):
    """The forward on split rows (janus_dispatch_split): the first GEMM on the
    FP16 tensor path, the second on 3xTF32, or on the FP16 path too from
    janus_expert_ffn_f16_min_rows_per_expert() rows per expert with h % 8 == 0.
    weights16: a set from janus_expert_weights_f16 (forward parts), else the
    call splits the weights itself.  Returns (out-or-None, act-or-None)."""
    R2, d = rows16.shape
    R = R2 // 2
    E, _, h = w1.shape
    if out is not None and out_rows is not None:
        raise ValueError("give out or out_rows, not both")
    if out is None and out_rows is None:
        out = _empty((R, d), torch.float32, rows16.device)
    if want_act and act is None:
        act = _empty((R, h), torch.float32, rows16.device)
    nb = janus_expert_ffn_split_workspace_size(R, E, d, h)
    ws = _workspace(nb, rows16.device, workspace)
    _raise(lib().janus_expert_ffn_fwd_split(_p(rows16, torch.float16, "rows16"), _p(row_scale, torch.float32, "row_scale"),
                                            _p(offsets, torch.int32, "offsets"), E, R, d, h,
                                            _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                            _p(out, torch.float32, "yd"),
                                            None if out_rows is None else _row_table(out_rows, R),
                                            _p(act, torch.float32, "act"), *_w16(weights16), _p(ws), nb,
                                            _stream(stream)),
           "janus_expert_ffn_fwd_split")
    return out, act


def janus_expert_ffn_vjp_split(gd16, gd_scale, offsets, w1, w2, act, *, out=None, out_rows=None, weights16=None,
                               workspace=None, stream=None):
    """The input VJP on split upstream-gradient rows (janus_dispatch_split,
    weighted) and the forward's pre-activations: dA = (gd W2^T) silu'(a) on
    the FP16 tensor path, dxd = dA W1^T on 3xTF32, or on the FP16 path too at
    janus_expert_ffn_f16_min_rows_per_expert() rows per expert with h % 8 == 0.
    weights16: a set from janus_expert_weights_f16 (VJP parts), else the call
    splits the weights itself.  Returns out-or-None."""
    R2, d = gd16.shape
    R = R2 // 2
    E, _, h = w1.shape
    if out is not None and out_rows is not None:
        raise ValueError("give out or out_rows, not both")
    if out is None and out_rows is None:
        out = _empty((R, d), torch.float32, gd16.device)
    nb = janus_expert_ffn_split_workspace_size(R, E, d, h)
    ws = _workspace(nb, gd16.device, workspace)
    _raise(lib().janus_expert_ffn_vjp_split(_p(gd16, torch.float16, "gd16"), _p(gd_scale, torch.float32, "gd_scale"),
                                            _p(act, torch.float32, "act"), _p(offsets, torch.int32, "offsets"), E, R,
                                            d, h, _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                            _p(out, torch.float32, "dxd"),
                                            None if out_rows is None else _row_table(out_rows, R),
                                            *_w16(weights16), _p(ws), nb, _stream(stream)),
           "janus_expert_ffn_vjp_split")
    return out


def janus_expert_ffn_vjp_rows(xd, gd, offsets, w1, w2, dxd_rows, *, act=None, mode=JANUS_FFN_FP32_SIMT,
                              workspace=None, stream=None):
    """janus_expert_ffn_vjp with row p of dxd stored at address dxd_rows[p]."""
    R, d = xd.shape
    E, _, h = w1.shape
    nb = janus_expert_ffn_workspace_size(R, d, h, E, True, act is not None, mode)
    ws = _workspace(nb, xd.device, workspace)
    _raise(lib().janus_expert_ffn_vjp_rows(_p(xd, torch.float32, "xd"), _p(gd, torch.float32, "gd"),
                                           _p(act, torch.float32, "act"),
                                           _p(offsets, torch.int32, "offsets"), E, R, d, h,
                                           _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                           _row_table(dxd_rows, R), int(mode), _p(ws), nb,
                                           _stream(stream)), "janus_expert_ffn_vjp_rows")


def janus_expert_ffn_weight_grad_workspace_size(n_rows, h, have_act) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_expert_ffn_weight_grad_workspace_size(n_rows, h, int(bool(have_act)),
                                                             ctypes.byref(b)),
           "janus_expert_ffn_weight_grad_workspace_size")
    return b.value


def janus_expert_ffn_weight_grad(xd, gd, offsets, w1, w2, *, act=None, mode=JANUS_FFN_FP32_SIMT,
                                 dw1=None, dw2=None, workspace=None, stream=None):
    """Per-expert weight gradients; returns (dw1 [E,d,h], dw2 [E,h,d])."""
    R, d = xd.shape
    E, _, h = w1.shape
    if dw1 is None:
        dw1 = _empty((E, d, h), torch.float32, w1.device)
    if dw2 is None:
        dw2 = _empty((E, h, d), torch.float32, w1.device)
    nb = janus_expert_ffn_weight_grad_workspace_size(R, h, act is not None)
    ws = _workspace(nb, w1.device, workspace)
    _raise(lib().janus_expert_ffn_weight_grad(_p(xd, torch.float32, "xd"), _p(gd, torch.float32, "gd"),
                                              _p(act, torch.float32, "act"),
                                              _p(offsets, torch.int32, "offsets"), E, R, d, h,
                                              _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                              _p(dw1, torch.float32, "dw1"), _p(dw2, torch.float32, "dw2"),
                                              int(mode), _p(ws), nb, _stream(stream)),
           "janus_expert_ffn_weight_grad")
    return dw1, dw2


def janus_expert_ffn_vjp_vjp_workspace_size(n_rows, h, have_act, want_weight_grad) -> int:
    b = ctypes.c_size_t(0)
    _raise(lib().janus_expert_ffn_vjp_vjp_workspace_size(n_rows, h, int(bool(have_act)),
                                                         int(bool(want_weight_grad)), ctypes.byref(b)),
           "janus_expert_ffn_vjp_vjp_workspace_size")
    return b.value


def janus_expert_ffn_vjp_vjp(xd, gd, vd, offsets, w1, w2, *, act=None, mode=JANUS_FFN_FP32_SIMT,
                             weight_grad=False, d_xd=None, d_gd=None, dw1=None, dw2=None,
                             workspace=None, stream=None):
    """Second-order pass for the cotangent vd of the input VJP; returns
    (d_xd, d_gd) or, with weight_grad, (d_xd, d_gd, dw1, dw2)."""
    R, d = xd.shape
    E, _, h = w1.shape
    if d_xd is None:
        d_xd = _empty((R, d), torch.float32, xd.device)
    if d_gd is None:
        d_gd = _empty((R, d), torch.float32, xd.device)
    if weight_grad:
        if dw1 is None:
            dw1 = _empty((E, d, h), torch.float32, w1.device)
        if dw2 is None:
            dw2 = _empty((E, h, d), torch.float32, w1.device)
    nb = janus_expert_ffn_vjp_vjp_workspace_size(R, h, act is not None, weight_grad)
    ws = _workspace(nb, w1.device, workspace)
    _raise(lib().janus_expert_ffn_vjp_vjp(_p(xd, torch.float32, "xd"), _p(gd, torch.float32, "gd"),
                                          _p(vd, torch.float32, "vd"), _p(act, torch.float32, "act"),
                                          _p(offsets, torch.int32, "offsets"), E, R, d, h,
                                          _p(w1, torch.float32, "w1"), _p(w2, torch.float32, "w2"),
                                          _p(d_xd, torch.float32, "d_xd"), _p(d_gd, torch.float32, "d_gd"),
                                          _p(dw1 if weight_grad else None, torch.float32, "dw1"),
                                          _p(dw2 if weight_grad else None, torch.float32, "dw2"),
                                          int(mode), _p(ws), nb, _stream(stream)),
           "janus_expert_ffn_vjp_vjp")
    if weight_grad:
        return d_xd, d_gd, dw1, dw2
    return d_xd, d_gd


# --------------------------------------------------------------------------
# edge aggregation
# --------------------------------------------------------------------------
def janus_edge_aggregate(msg, row_ptr, *, out=None, stream=None):
    """out[i] = sum of receiver i's edge messages (msg [Ed,d], row_ptr [N+1])."""
    N = row_ptr.shape[0] - 1
    Ed, d = msg.shape
    if out is None:
        out = _empty((N, d), torch.float32, msg.device)
    _raise(lib().janus_edge_aggregate(_p(msg, torch.float32, "msg"), Ed,
                                      _p(row_ptr, torch.int64, "row_ptr"), N, d,
                                      _p(out, torch.float32, "out"), _stream(stream)),
           "janus_edge_aggregate")
    return out


def janus_edge_broadcast(dx, row_ptr, *, out=None, stream=None):
    """dmsg[e] = dx[receiver(e)] over a receiver-sorted CSR."""
    N, d = dx.shape
    if out is None:
        out = _empty((int(row_ptr[-1].item()) if row_ptr.numel() else 0, d), torch.float32, dx.device)
    _raise(lib().janus_edge_broadcast(_p(dx, torch.float32, "dx"), _p(row_ptr, torch.int64, "row_ptr"),
                                      N, d, _p(out, torch.float32, "dmsg"), out.shape[0], _stream(stream)),
           "janus_edge_broadcast")
    return out


def janus_neighbor_aggregate(x, row_ptr, senders, *, out=None, stream=None):
    """out[i] = sum over row i's edges of x[senders[e]]."""
    N, d = x.shape
    if out is None:
        out = _empty((N, d), torch.float32, x.device)
    _raise(lib().janus_neighbor_aggregate(_p(x, torch.float32, "x"), _p(row_ptr, torch.int64, "row_ptr"),
                                          _p(senders, torch.int32, "senders"), senders.shape[0], N, d,
                                          _p(out, torch.float32, "out"), _stream(stream)),
           "janus_neighbor_aggregate")
    return out


def janus_debug_build() -> bool:
    """True when the loaded library is the debug build."""
    return bool(lib().janus_debug_build())


def janus_debug_check(stream=None):
    """Raise JanusError(JANUS_ERR_DATA) if a call without a workspace found a
    bad index since the last check (debug build; never in the release build)."""
    _raise(lib().janus_debug_check(_stream(stream)), "janus_debug_check")


def janus_debug_inject_launch_failures(n_calls: int):
    lib().janus_debug_inject_launch_failures(int(n_calls))


def janus_trace_start(capacity: int):
    """Start recording up to `capacity` traced launches (CUDA events on each
    launch's stream; the current device)."""
    _raise(lib().janus_trace_start(int(capacity)), "janus_trace_start")


def janus_trace_stop():
    _raise(lib().janus_trace_stop(), "janus_trace_stop")


def janus_trace_records():
    """[(kernel name, ms)] of the recorded launches, in launch order (waits
    for each record's end event)."""
    n = ctypes.c_int32(0)
    _raise(lib().janus_trace_count(ctypes.byref(n)), "janus_trace_count")
    out = []
    name, ms = ctypes.c_char_p(), ctypes.c_float()
    for i in range(n.value):
        _raise(lib().janus_trace_get(i, ctypes.byref(name), ctypes.byref(ms)), "janus_trace_get")
        out.append((name.value.decode(), float(ms.value)))
    return out


def janus_trace_release():
    _raise(lib().janus_trace_release(), "janus_trace_release")
