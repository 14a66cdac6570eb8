"""GPU tests of the debug build, libjanus_debug.so (compiled with -DJANUS_DEBUG).

It stands in for the memory checker that this pool does not offer: every
kernel checks the index arrays it is given (slot_of, perm, offsets, row_ptr,
senders, the expert-parallel tables) before using them, records a data fault
and skips the access.  Two things are checked here:

  * on valid inputs it gives the same results as the release build (the
    tiny layer chain and random shapes against the oracle, bit-exact against
    the release library where the release tests are bit-exact);
  * on a corrupted index array it reports JANUS_ERR_DATA and touches nothing
    outside its buffers: every output sits inside a larger NaN-filled
    allocation whose guard rows must stay NaN.

Corrupted index arrays are only ever given to the debug build.
"""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, host, rel_fro, to_dev

pytestmark = pytest.mark.gpu

GUARD = 64


@pytest.fixture(scope="module", autouse=True)
def debug_library():
    from element_routed_moe_b200 import build as jbuild
    jbuild.build(debug=True)
    J.use_library(debug=True)
    yield
    torch.cuda.synchronize()
    J.use_library(debug=False)


def _guarded(rows, d, dtype=torch.float32):
    """A [rows, d] view at the start of a NaN-filled [rows + GUARD, d] buffer."""
    buf = torch.full((rows + GUARD, d), float("nan"), dtype=dtype, device=DEV)
    return buf, buf[:rows]


def _guard_intact(buf, rows):
    return bool(torch.isnan(buf[rows:].float()).all().item())


def test_library_is_the_debug_build():
    assert J.janus_debug_build()
    J.janus_debug_check()


@pytest.mark.parametrize("mode", [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32])
def test_tiny_layer_chain_matches_the_oracle(mode):
    cfg = synth.CONFIGS["tiny"]
    inp = synth.layer_inputs(cfg, seed=3, device="cpu")
    N, T, K = cfg.n_atoms, cfg.n_types, cfg.top_k
    types, gate = to_dev(inp["types"]), to_dev(inp["gate"])
    w1, w2 = inp["w1"].to(DEV), inp["w2"].to(DEV)
    msg, rp, g = inp["msg"].to(DEV), to_dev(inp["row_ptr"]), inp["g"].to(DEV)
    x = J.janus_edge_aggregate(msg, rp)
    r = J.janus_route(types, gate, K)
    payload, scale, qws = J.janus_quant_by_type(x, types, T, r["slot_of"], K)
    xq = J.janus_dequant_by_type(payload, types, T, r["perm"], K, scale)
    xd = J.janus_dispatch(x, r["slot_of"], K)
    yd, act = J.janus_expert_ffn_fwd(xd, r["offsets"], w1, w2, mode=mode, want_act=True)
    y = J.janus_combine(yd, r["slot_of"], K, r["topk_weight"])
    gd = J.janus_dispatch(g, r["slot_of"], K, r["topk_weight"])
    dxd = J.janus_expert_ffn_vjp(xd, gd, r["offsets"], w1, w2, act=act, mode=mode)
    dx = J.janus_combine(dxd, r["slot_of"], K)
    J.janus_check(r["workspace"])
    J.janus_check(qws)
    J.janus_debug_check()
    hx = oracle.edge_aggregate(inp["msg"].numpy(), inp["row_ptr"])
    assert rel_fro(host(x), hx) <= TOL_FP32
    o = oracle.route(inp["types"], inp["gate"], K)
    for k in ("counts", "offsets", "perm", "slot_of", "topk_expert"):
        assert np.array_equal(host(r[k]), o[k]), k
    xh = host(x)
    q, sc = oracle.quant_by_type(xh, inp["types"], T, o["perm"], K)
    assert np.array_equal(host(payload).view(np.uint16), q) and np.array_equal(host(scale), sc)
    assert np.array_equal(host(xq), oracle.dequant_by_type(q, inp["types"], o["perm"], K, sc))
    hw1, hw2 = inp["w1"].numpy(), inp["w2"].numpy()
    oxd = oracle.dispatch(xh, o["perm"], K)
    assert np.array_equal(host(xd), oxd)
    oy = oracle.combine(oracle.expert_ffn_fwd(oxd, o["offsets"], hw1, hw2), o["slot_of"], K, o["topk_weight"])
    assert rel_fro(host(y), oy) <= TOL_FP32
    ogd = oracle.dispatch(inp["g"].numpy(), o["perm"], K, o["topk_weight"])
    odx = oracle.combine(oracle.expert_ffn_vjp(oxd, ogd, o["offsets"], hw1, hw2), o["slot_of"], K)
    assert rel_fro(host(dx), odx) <= TOL_FP32


@pytest.mark.parametrize("seed", [11, 12])
def test_random_shapes_bit_exact_with_the_release_build(seed):
    rng = np.random.default_rng(seed)
    N, T, E = int(rng.integers(1, 700)), int(rng.integers(1, 40)), int(rng.integers(2, 30))
    K, d, h = int(rng.integers(1, min(E, 9) + 1)), 4 * int(rng.integers(1, 60)), 4 * int(rng.integers(1, 60))
    types = to_dev(synth.types_zipf(N, T, seed=seed))
    gate = to_dev(synth.gate_table(T, E, seed + 1))
    w1, w2 = synth.expert_weights(E, d, h, seed + 2, DEV)
    x = synth.normal((N, d), seed + 3, DEV)

    def chain():
        r = J.janus_route(types, gate, K)
        xd = J.janus_dispatch(x, r["slot_of"], K)
        yd, act = J.janus_expert_ffn_fwd(xd, r["offsets"], w1, w2, mode=J.JANUS_FFN_3XTF32, want_act=True)
        y = J.janus_combine(yd, r["slot_of"], K, r["topk_weight"])
        dxd = J.janus_expert_ffn_vjp(xd, xd, r["offsets"], w1, w2, act=act, mode=J.JANUS_FFN_3XTF32)
        return r, y, J.janus_combine(dxd, r["slot_of"], K)

    r_dbg, y_dbg, dx_dbg = chain()
    J.janus_debug_check()
    J.use_library(debug=False)
    try:
        r_rel, y_rel, dx_rel = chain()
        torch.cuda.synchronize()
    finally:
        J.use_library(debug=True)
    for k in ("perm", "slot_of", "offsets"):
        assert torch.equal(r_dbg[k], r_rel[k]), k
    assert torch.equal(y_dbg, y_rel) and torch.equal(dx_dbg, dx_rel)


def _small_route(N=300, T=9, E=12, K=3, d=20, seed=5):
    types = to_dev(synth.types_zipf(N, T, seed=seed))
    gate = to_dev(synth.gate_table(T, E, seed + 1))
    r = J.janus_route(types, gate, K)
    x = synth.normal((N, d), seed + 2, DEV)
    return types, gate, r, x, N, T, E, K, d


def test_corrupted_slot_of_in_dispatch_combine_and_pack():
    types, gate, r, x, N, T, E, K, d = _small_route()
    R = N * K
    bad = r["slot_of"].clone()
    bad[5] = R + 3
    bad[17] = -2
    buf, xd = _guarded(R, d)
    J.janus_dispatch(x, bad, K, out=xd)
    with pytest.raises(J.JanusError) as e:
        J.janus_debug_check()
    assert e.value.status == J.JANUS_ERR_DATA
    assert _guard_intact(buf, R)
    ybuf, y = _guarded(N, d)
    J.janus_combine(synth.normal((R, d), 9, DEV), bad, K, r["topk_weight"], out=y)
    with pytest.raises(J.JanusError):
        J.janus_debug_check()
    assert _guard_intact(ybuf, N)
    pbuf, payload = _guarded(R, d, torch.float16)
    _, _, qws = J.janus_quant_by_type(x, types, T, bad, K, payload=payload)
    with pytest.raises(J.JanusError) as e:
        J.janus_check(qws)
    assert e.value.status == J.JANUS_ERR_DATA
    assert _guard_intact(pbuf, R)
    # the uncorrupted call afterwards is clean again
    J.janus_dispatch(x, r["slot_of"], K, out=xd)
    J.janus_debug_check()


def test_corrupted_perm_in_dequant_and_row_scales():
    types, gate, r, x, N, T, E, K, d = _small_route()
    R = N * K
    payload, scale, _ = J.janus_quant_by_type(x, types, T, r["slot_of"], K)
    bad = r["perm"].clone()
    bad[0] = R
    bad[R - 1] = -7
    buf, xd = _guarded(R, d)
    J.janus_dequant_by_type(payload, types, T, bad, K, scale, out=xd)
    with pytest.raises(J.JanusError):
        J.janus_debug_check()
    assert _guard_intact(buf, R)
    sbuf = torch.full((R + GUARD,), float("nan"), device=DEV)
    J.janus_dispatch_row_scales(types, T, bad, K, scale, out=sbuf[:R])
    with pytest.raises(J.JanusError):
        J.janus_debug_check()
    assert torch.isnan(sbuf[R:]).all().item()


@pytest.mark.parametrize("mode", [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32])
@pytest.mark.parametrize("corrupt", ["decreasing", "past_rows", "negative"])
def test_corrupted_offsets_in_the_expert_mlp(mode, corrupt):
    E, d, h = 5, 64, 48
    counts = np.array([40, 0, 130, 7, 90])
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offs[-1])
    if corrupt == "decreasing":
        offs[2] = offs[1] - 10
    elif corrupt == "past_rows":
        offs[-1] = R + 500
    else:
        offs[0] = -64
    w1, w2 = synth.expert_weights(E, d, h, 1, DEV)
    xd = synth.normal((R, d), 2, DEV)
    ybuf, yd = _guarded(R, d)
    abuf, act = _guarded(R, h)
    nb = J.janus_expert_ffn_workspace_size(R, d, h, E, False, True, mode)
    ws = torch.zeros(nb, dtype=torch.uint8, device=DEV)
    J.janus_expert_ffn_fwd(xd, to_dev(offs), w1, w2, mode=mode, out=yd, act=act, workspace=ws)
    torch.cuda.synchronize()
    faulted = False
    for check in (lambda: J.janus_check(ws), J.janus_debug_check):
        try:
            check()
        except J.JanusError as err:
            assert err.status == J.JANUS_ERR_DATA
            faulted = True
    assert faulted
    assert _guard_intact(ybuf, R) and _guard_intact(abuf, R)


def test_corrupted_offsets_in_the_weight_gradient():
    E, d, h = 4, 32, 40
    offs = np.array([0, 50, 20, 90, 120], np.int32)          # decreasing at expert 1
    R = 120
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    xd = synth.normal((R, d), 4, DEV)
    gd = synth.normal((R, d), 5, DEV)
    J.janus_expert_ffn_weight_grad(xd, gd, to_dev(offs), w1, w2, mode=J.JANUS_FFN_FP32_SIMT)
    with pytest.raises(J.JanusError):
        J.janus_debug_check()


def test_corrupted_row_ptr_and_senders_in_the_edge_kernels():
    N, d = 200, 36
    rp, send, _ = synth.edges_random(N, 8, 7)
    Ed = int(rp[-1])
    msg = synth.normal((Ed, d), 8, DEV)
    bad = rp.copy()
    bad[50] = bad[49] - 3          # decreasing
    bad[120] = Ed + 1000           # past the edge count
    out = J.janus_edge_aggregate(msg, to_dev(bad))
    with pytest.raises(J.JanusError):
        J.janus_debug_check()
    assert torch.isfinite(out).all().item()
    dbuf, dmsg = _guarded(Ed, d)
    J.janus_edge_broadcast(synth.normal((N, d), 9, DEV), to_dev(bad), out=dmsg)
    with pytest.raises(J.JanusError):
        J.janus_debug_check()
    assert _guard_intact(dbuf, Ed)
    s_bad = send.astype(np.int32)
    s_bad[3] = N + 4
    s_bad[9] = -1
    J.janus_neighbor_aggregate(synth.normal((N, d), 10, DEV), to_dev(rp), to_dev(s_bad))
    with pytest.raises(J.JanusError):
        J.janus_debug_check()
    # the valid CSR is clean
    J.janus_edge_aggregate(msg, to_dev(rp))
    J.janus_debug_check()


def test_corrupted_topk_expert_in_the_expert_parallel_send():
    types, gate, r, x, N, T, E, K, d = _small_route(E=12)
    R = N * K
    counts_all = r["counts"].reshape(1, -1).contiguous()
    lay = J.janus_ep_layout(counts_all, E, R)
    bad = dict(r)
    te = r["topk_expert"].clone()
    te.view(-1)[4] = E + 2
    te.view(-1)[11] = -1
    bad["topk_expert"] = te
    pbuf, pay = _guarded(R, d, torch.float16)
    rs = torch.full((R + GUARD,), float("nan"), device=DEV)
    _, ws = J.janus_ep_dispatch_quant(x, types, T, bad, lay, 0, R, [pay], [rs[:R]])
    with pytest.raises(J.JanusError):
        J.janus_check(ws)
    assert _guard_intact(pbuf, R) and torch.isnan(rs[R:]).all().item()
