"""CPU oracle for the element-routed MoE layer and edge aggregation.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the package's smoke() check
and by bench.py's CPU-baseline leg, never by the product path.  It shares no
code with the CUDA library.  Each wrapper takes and returns NumPy arrays and
calls the plain C++ definitions in ``janus_oracle.cpp`` (see that file's header
for the sources and the readings taken where the pages are silent).
"""
import ctypes
import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        _setup(_lib)
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _setup(L):
    vp, i64, i32, u16, dbl = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                              ctypes.c_uint16, ctypes.c_double)
    L.orc_num_threads.restype = ctypes.c_int
    L.orc_fp16_from_double.argtypes = [dbl]
    L.orc_fp16_from_double.restype = u16
    L.orc_fp16_to_double.argtypes = [u16]
    L.orc_fp16_to_double.restype = dbl
    L.orc_route.argtypes = [vp, i64, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    L.orc_route.restype = ctypes.c_int
    L.orc_dispatch.argtypes = [vp, i64, i32, i32, vp, vp, vp]
    L.orc_quant_by_type.argtypes = [vp, i64, i32, i32, vp, i32, vp, vp, vp]
    L.orc_quant_by_type.restype = ctypes.c_int
    L.orc_dequant_by_type.argtypes = [vp, i64, i32, i32, vp, vp, vp, vp]
    L.orc_expert_ffn_fwd.argtypes = [vp, vp, i32, i64, i32, i32, vp, vp, vp, i64, vp, vp]
    L.orc_expert_ffn_vjp.argtypes = [vp, vp, vp, i32, i64, i32, i32, vp, vp, vp, i64, vp]
    L.orc_expert_ffn_weight_grad.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, vp, vp]
    L.orc_expert_ffn_vjp_vjp.argtypes = [vp, vp, vp, vp, i32, i64, i32, i32, vp, vp, vp, i64, vp, vp]
    L.orc_expert_ffn_vjp_vjp_weight_grad.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, vp]
    L.orc_combine.argtypes = [vp, vp, vp, i64, i32, i32, vp]
    L.orc_ep_layout.argtypes = [vp, i32, i32, vp, vp, vp]
    L.orc_ep_layout.restype = ctypes.c_int
    L.orc_edge_aggregate.argtypes = [vp, vp, i64, i32, vp]
    L.orc_edge_broadcast.argtypes = [vp, vp, i64, i32, vp]
    L.orc_neighbor_aggregate.argtypes = [vp, vp, vp, i64, i32, vp]
    L.orc_neighbor_aggregate.restype = ctypes.c_int


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().orc_num_threads()


def fp16_from_double(x: float) -> int:
    return int(lib().orc_fp16_from_double(float(x)))


def fp16_to_double(b: int) -> float:
    return float(lib().orc_fp16_to_double(int(b)))


def route(types, gate, top_k):
    """Per-atom top-K experts/weights, per-expert counts, offsets, stable perm."""
    types = _c(types, np.int32)
    gate = _c(gate, np.float32)
    N = types.shape[0]
    T, E = gate.shape
    K = int(top_k)
    R = N * K
    te = np.empty((N, K), np.int32)
    tw = np.empty((N, K), np.float32)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(R, np.int32)
    slot_of = np.empty(R, np.int32)
    rc = lib().orc_route(_p(types), N, _p(gate), T, E, K, _p(te), _p(tw),
                         _p(counts), _p(offsets), _p(perm), _p(slot_of))
    if rc != 0:
        raise ValueError("oracle route: element type id out of range")
    return dict(topk_expert=te, topk_weight=tw, counts=counts, offsets=offsets,
                perm=perm, slot_of=slot_of)


def dispatch(x, perm, top_k, topk_weight=None):
    x = _c(x, np.float32)
    perm = _c(perm, np.int32)
    N, d = x.shape
    xd = np.empty((perm.shape[0], d), np.float32)
    w = None if topk_weight is None else _c(topk_weight, np.float32)
    lib().orc_dispatch(_p(x), N, d, int(top_k), _p(perm), _p(w), _p(xd))
    return xd


def quant_by_type(x, types, n_types, perm, top_k):
    x = _c(x, np.float32)
    types = _c(types, np.int32)
    perm = _c(perm, np.int32)
    N, d = x.shape
    payload = np.empty((perm.shape[0], d), np.uint16)
    scale = np.empty(int(n_types), np.float32)
    rc = lib().orc_quant_by_type(_p(x), N, d, int(top_k), _p(types), int(n_types),
                                 _p(perm), _p(payload), _p(scale))
    if rc != 0:
        raise ValueError(f"oracle quant_by_type: data error {rc}")
    return payload, scale


def dequant_by_type(payload, types, perm, top_k, scale):
    payload = _c(payload, np.uint16)
    types = _c(types, np.int32)
    perm = _c(perm, np.int32)
    scale = _c(scale, np.float32)
    R, d = payload.shape
    N = types.shape[0]
    xd = np.empty((R, d), np.float32)
    lib().orc_dequant_by_type(_p(payload), N, d, int(top_k), _p(types), _p(perm),
                              _p(scale), _p(xd))
    return xd


def expert_ffn_fwd(xd, offsets, w1, w2, rows=None, want_act=False):
    xd = _c(xd, np.float32)
    offsets = _c(offsets, np.int32)
    w1 = _c(w1, np.float32)
    w2 = _c(w2, np.float32)
    R, d = xd.shape
    E, _, h = w1.shape
    r = None if rows is None else _c(rows, np.int64)
    n_out = R if r is None else r.shape[0]
    yd = np.empty((n_out, d), np.float32)
    act = np.empty((n_out, h), np.float32) if want_act else None
    lib().orc_expert_ffn_fwd(_p(xd), _p(offsets), E, R, d, h, _p(w1), _p(w2),
                             _p(r), 0 if r is None else r.shape[0], _p(yd), _p(act))
    return (yd, act) if want_act else yd


def expert_ffn_vjp(xd, gd, offsets, w1, w2, rows=None):
    xd = _c(xd, np.float32)
    gd = _c(gd, np.float32)
    offsets = _c(offsets, np.int32)
    w1 = _c(w1, np.float32)
    w2 = _c(w2, np.float32)
    R, d = xd.shape
    E, _, h = w1.shape
    r = None if rows is None else _c(rows, np.int64)
    n_out = R if r is None else r.shape[0]
    dxd = np.empty((n_out, d), np.float32)
    lib().orc_expert_ffn_vjp(_p(xd), _p(gd), _p(offsets), E, R, d, h, _p(w1), _p(w2),
                             _p(r), 0 if r is None else r.shape[0], _p(dxd))
    return dxd


def expert_ffn_weight_grad(xd, gd, offsets, w1, w2):
    """Per-expert weight gradients (dW1 [E,d,h], dW2 [E,h,d]) of
    L = sum_p <yd[p], gd[p]> for the bias-free Linear-SiLU-Linear experts."""
    xd = _c(xd, np.float32)
    gd = _c(gd, np.float32)
    offsets = _c(offsets, np.int32)
    w1 = _c(w1, np.float32)
    w2 = _c(w2, np.float32)
    E, d, h = w1.shape
    dw1 = np.empty((E, d, h), np.float32)
    dw2 = np.empty((E, h, d), np.float32)
    lib().orc_expert_ffn_weight_grad(_p(xd), _p(gd), _p(offsets), E, d, h, _p(w1), _p(w2),
                                     _p(dw1), _p(dw2))
    return dw1, dw2


def expert_ffn_vjp_vjp(xd, gd, vd, offsets, w1, w2, rows=None):
    """Second-order pass: gradients w.r.t. xd and gd of L = <dxd(xd, gd), vd>,
    where dxd is the expert MLP's input VJP.  Returns (d_xd, d_gd), [n_out, d]."""
    xd, gd, vd = _c(xd, np.float32), _c(gd, np.float32), _c(vd, np.float32)
    offsets = _c(offsets, np.int32)
    w1, w2 = _c(w1, np.float32), _c(w2, np.float32)
    R, d = xd.shape
    E, _, h = w1.shape
    r = None if rows is None else _c(rows, np.int64)
    n_out = R if r is None else r.shape[0]
    d_xd = np.empty((n_out, d), np.float32)
    d_gd = np.empty((n_out, d), np.float32)
    lib().orc_expert_ffn_vjp_vjp(_p(xd), _p(gd), _p(vd), _p(offsets), E, R, d, h, _p(w1), _p(w2),
                                 _p(r), 0 if r is None else r.shape[0], _p(d_xd), _p(d_gd))
    return d_xd, d_gd


def expert_ffn_vjp_vjp_weight_grad(xd, gd, vd, offsets, w1, w2):
    """Weight part of the second-order pass: (dW1 [E,d,h], dW2 [E,h,d]) of
    L = <dxd(xd, gd; W1, W2), vd>."""
    xd, gd, vd = _c(xd, np.float32), _c(gd, np.float32), _c(vd, np.float32)
    offsets = _c(offsets, np.int32)
    w1, w2 = _c(w1, np.float32), _c(w2, np.float32)
    E, d, h = w1.shape
    dw1 = np.empty((E, d, h), np.float32)
    dw2 = np.empty((E, h, d), np.float32)
    lib().orc_expert_ffn_vjp_vjp_weight_grad(_p(xd), _p(gd), _p(vd), _p(offsets), E, d, h,
                                             _p(w1), _p(w2), _p(dw1), _p(dw2))
    return dw1, dw2


def ep_layout(counts_all):
    """Expert-parallel exchange layout from the all-gathered counts [P, E]:
    (src_off [P, E+1], dst_off [P, E], recv_off [P, E/P+1])."""
    c = _c(counts_all, np.int32)
    P, E = c.shape
    if E % P:
        raise ValueError("E must be a multiple of the number of ranks")
    src = np.empty((P, E + 1), np.int32)
    dst = np.empty((P, E), np.int32)
    recv = np.empty((P, E // P + 1), np.int32)
    if lib().orc_ep_layout(_p(c), P, E, _p(src), _p(dst), _p(recv)) != 0:
        raise ValueError("bad layout arguments")
    return src, dst, recv


def combine(yd, slot_of, top_k, topk_weight=None):
    yd = _c(yd, np.float32)
    slot_of = _c(slot_of, np.int32)
    K = int(top_k)
    N = slot_of.shape[0] // K
    d = yd.shape[1]
    y = np.empty((N, d), np.float32)
    w = None if topk_weight is None else _c(topk_weight, np.float32)
    lib().orc_combine(_p(yd), _p(slot_of), _p(w), N, K, d, _p(y))
    return y


def edge_aggregate(msg, row_ptr):
    msg = _c(msg, np.float32)
    row_ptr = _c(row_ptr, np.int64)
    N = row_ptr.shape[0] - 1
    d = msg.shape[1]
    out = np.empty((N, d), np.float32)
    lib().orc_edge_aggregate(_p(msg), _p(row_ptr), N, d, _p(out))
    return out


def edge_broadcast(dx, row_ptr):
    """dmsg[e] = dx[receiver(e)] (the gradient of the edge aggregation)."""
    dx = _c(dx, np.float32)
    row_ptr = _c(row_ptr, np.int64)
    N, d = dx.shape
    dmsg = np.empty((int(row_ptr[-1]), d), np.float32)
    lib().orc_edge_broadcast(_p(dx), _p(row_ptr), N, d, _p(dmsg))
    return dmsg


def neighbor_aggregate(x, row_ptr, senders):
    """out[i] = sum over row i's edges of x[senders[e]]."""
    x = _c(x, np.float32)
    row_ptr = _c(row_ptr, np.int64)
    senders = _c(senders, np.int32)
    N, d = x.shape
    out = np.empty((N, d), np.float32)
    if lib().orc_neighbor_aggregate(_p(x), _p(row_ptr), _p(senders), N, d, _p(out)) != 0:
        raise ValueError("oracle neighbor_aggregate: sender index out of range")
    return out
