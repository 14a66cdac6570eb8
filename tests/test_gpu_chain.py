"""GPU parity of the interaction-block slice: edge aggregation -> routing ->
FP16-packed dispatch -> expert MLP forward -> combine, then the input VJP
(dispatch of the gate-weighted upstream gradient -> expert VJP -> combine),
all chained on one stream (block order: paper review 'Breaking the Training
Barrier of Billion-Parameter Universal Machine Learning Interatomic
Potentials', section 3.4, Figure 3 timeline).

Checks: (1) the FP16 payload is bit-exact against the oracle's packing of the
same features; (2) the layer output and input gradient are within 1e-5 of an
oracle chain that also packs to FP16; (3) within 2e-3 of an FP32-only oracle
chain (the packed path's tolerance)."""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP16_PATH, TOL_FP32, host, rel_fro, to_dev

pytestmark = pytest.mark.gpu


def _gpu_chain(msg, rp, types, gate, T, K, w1, w2, g, mode):
    s = torch.cuda.current_stream()
    x = J.janus_edge_aggregate(msg, rp)
    r = J.janus_route(types, gate, K)
    payload, scale, qws = J.janus_quant_by_type(x, types, T, r["slot_of"], K)
    xd = J.janus_dequant_by_type(payload, types, T, r["perm"], K, scale)
    yd, act = J.janus_expert_ffn_fwd(xd, r["offsets"], w1, w2, mode=mode, want_act=True)
    y = J.janus_combine(yd, r["slot_of"], K, r["topk_weight"])
    gdd = J.janus_dispatch(g, r["slot_of"], K, r["topk_weight"])
    dxd = J.janus_expert_ffn_vjp(xd, gdd, r["offsets"], w1, w2, act=act, mode=mode)
    dx = J.janus_combine(dxd, r["slot_of"], K)
    s.synchronize()
    J.janus_check(r["workspace"])
    J.janus_check(qws)
    return dict(x=x, route=r, payload=payload, scale=scale, xd=xd, y=y, dx=dx)


def _oracle_chain(x, types, gate, T, K, w1, w2, g, quant):
    r = oracle.route(types, gate, K)
    if quant:
        p, s = oracle.quant_by_type(x, types, T, r["perm"], K)
        xd = oracle.dequant_by_type(p, types, r["perm"], K, s)
    else:
        p, s = None, None
        xd = oracle.dispatch(x, r["perm"], K)
    yd = oracle.expert_ffn_fwd(xd, r["offsets"], w1, w2)
    y = oracle.combine(yd, r["slot_of"], K, r["topk_weight"])
    gd = oracle.dispatch(g, r["perm"], K, r["topk_weight"])
    dxd = oracle.expert_ffn_vjp(xd, gd, r["offsets"], w1, w2)
    dx = oracle.combine(dxd, r["slot_of"], K)
    return dict(route=r, payload=p, scale=s, y=y, dx=dx)


@pytest.mark.parametrize("mode", [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32])
def test_slice_chain_small(mode):
    N, T, E, K, d = 2048, 89, 40, 8, 256
    rp, _, _ = synth.edges_pbc(N, seed=1)
    msg = synth.normal((int(rp[-1]), d), 2, DEV)
    types = synth.types_zipf(N, T, seed=3)
    gate = synth.gate_table(T, E, 4)
    w1, w2 = synth.expert_weights(E, d, d, 5, DEV)
    g = synth.normal((N, d), 6, DEV)
    out = _gpu_chain(msg, to_dev(rp), to_dev(types), to_dev(gate), T, K, w1, w2, g, mode)
    x_ref = oracle.edge_aggregate(host(msg), rp)
    assert rel_fro(host(out["x"]), x_ref) <= TOL_FP32
    # the rest of the chain starts from the GPU's aggregated features
    x = host(out["x"])
    hw1, hw2, hg = host(w1), host(w2), host(g)
    q = _oracle_chain(x, types, gate, T, K, hw1, hw2, hg, quant=True)
    assert np.array_equal(host(out["payload"]).view(np.uint16), q["payload"])
    assert np.array_equal(host(out["scale"]), q["scale"])
    assert rel_fro(host(out["y"]), q["y"]) <= TOL_FP32
    assert rel_fro(host(out["dx"]), q["dx"]) <= TOL_FP32
    f = _oracle_chain(x_ref, types, gate, T, K, hw1, hw2, hg, quant=False)
    assert rel_fro(host(out["y"]), f["y"]) <= TOL_FP16_PATH
    assert rel_fro(host(out["dx"]), f["dx"]) <= TOL_FP16_PATH


@pytest.mark.parametrize("mode", [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32])
def test_slice_chain_full_size_sampled(mode):
    cfg = synth.CONFIGS["slice"]
    N, T, E, K, d = cfg.n_atoms, cfg.n_types, cfg.n_experts, cfg.top_k, cfg.d
    rp, _, _ = synth.edges_pbc(N, seed=1)
    msg = synth.normal((int(rp[-1]), d), 2, DEV)
    types = synth.types_zipf(N, T, seed=3)
    gate = synth.gate_table(T, E, 4)
    w1, w2 = synth.expert_weights(E, d, cfg.h, 5, DEV)
    g = synth.normal((N, d), 6, DEV)
    out = _gpu_chain(msg, to_dev(rp), to_dev(types), to_dev(gate), T, K, w1, w2, g, mode)
    del msg
    r = oracle.route(types, gate, K)
    for k in ("counts", "offsets", "perm", "slot_of", "topk_expert"):
        assert np.array_equal(host(out["route"][k]), r[k]), k
    x = host(out["x"])
    p_ref, s_ref = oracle.quant_by_type(x, types, T, r["perm"], K)
    assert np.array_equal(host(out["scale"]), s_ref)
    assert np.array_equal(host(out["payload"]).view(np.uint16), p_ref)
    # sampled atoms: the oracle computes their K expert rows one by one
    atoms = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(9).integers(0, N, 48)]))
    slots = (atoms[:, None] * K + np.arange(K)[None, :]).ravel()
    rows = r["slot_of"][slots].astype(np.int64)
    xd = oracle.dequant_by_type(p_ref, types, r["perm"], K, s_ref)
    hw1, hw2 = host(w1), host(w2)
    yd_rows = oracle.expert_ffn_fwd(xd, r["offsets"], hw1, hw2, rows=rows)
    gd = oracle.dispatch(host(g), r["perm"], K, r["topk_weight"])
    dxd_rows = oracle.expert_ffn_vjp(xd, gd, r["offsets"], hw1, hw2, rows=rows)
    # rows are listed atom by atom, k ascending: combine them with a compact slot map
    compact = np.arange(len(atoms) * K, dtype=np.int32)
    y_ref = oracle.combine(yd_rows, compact, K, r["topk_weight"][atoms])
    dx_ref = oracle.combine(dxd_rows, compact, K)
    assert rel_fro(host(out["y"])[atoms], y_ref) <= TOL_FP32
    assert rel_fro(host(out["dx"])[atoms], dx_ref) <= TOL_FP32
