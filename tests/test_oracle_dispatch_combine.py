"""Pins for the oracle's dispatch, combine and edge aggregation (CPU only).

Dispatch/combine: paper review 'Breaking the Training Barrier of
Billion-Parameter Universal Machine Learning Interatomic Potentials', section
3.5 (CNIS high-performance kernels, MoE dispatch/combine); gate-weighted sum:
'MatRIS-MoE与Janus框架' section 3.2.  Edge aggregation: same review, section
3.5 (neighbour / edge aggregation).  Checked against NumPy gathers,
np.add.at brute force, and the identities the pages' method implies.
"""
import numpy as np

import oracle
from element_routed_moe_b200 import synth


def _layer(N=300, T=11, E=12, K=3, d=20, seed=0):
    gate = synth.gate_table(T, E, seed + 1)
    types = synth.types_zipf(N, T, seed=seed + 2)
    x = synth.normal((N, d), seed + 3).numpy()
    r = oracle.route(types, gate, K)
    return x, types, r, K


def test_dispatch_is_numpy_gather():
    x, types, r, K = _layer()
    xd = oracle.dispatch(x, r["perm"], K)
    assert np.array_equal(xd, x[r["perm"] // K])
    w = r["topk_weight"].ravel()
    xdw = oracle.dispatch(x, r["perm"], K, r["topk_weight"])
    ref = x[r["perm"] // K] * w[r["perm"]][:, None]      # float32 products (RN)
    assert np.array_equal(xdw, ref)


def test_combine_of_dispatch_identity_experts_returns_input():
    x, types, r, K = _layer(seed=5)
    xd = oracle.dispatch(x, r["perm"], K)
    y = oracle.combine(xd, r["slot_of"], K, r["topk_weight"])
    np.testing.assert_allclose(y, x, rtol=1e-6, atol=1e-6)
    # unweighted combine of an unweighted dispatch: K * x exactly (K = 2^m)
    x2, _, r2, K2 = _layer(K=4, seed=6)
    y2 = oracle.combine(oracle.dispatch(x2, r2["perm"], K2), r2["slot_of"], K2)
    assert np.array_equal(y2, 4.0 * x2)


def test_combine_dispatch_adjoint():
    x, types, r, K = _layer(seed=9)
    R, d = r["perm"].shape[0], x.shape[1]
    yd = synth.normal((R, d), 31).numpy()
    g = synth.normal((x.shape[0], d), 32).numpy()
    w = r["topk_weight"]
    lhs = np.sum(oracle.combine(yd, r["slot_of"], K, w).astype(np.float64) * g)
    rhs = np.sum(yd.astype(np.float64) * oracle.dispatch(g, r["perm"], K, w))
    assert abs(lhs - rhs) <= 1e-5 * np.sqrt(np.sum(yd.astype(np.float64) ** 2) * np.sum(g.astype(np.float64) ** 2))


def test_combine_k_order_single_expert_rows():
    # K = 1: combine is the inverse gather with weight 1 -> bit-exact
    x, types, r, K = _layer(K=1, seed=12)
    xd = oracle.dispatch(x, r["perm"], K)
    assert np.array_equal(oracle.combine(xd, r["slot_of"], K, r["topk_weight"]), x)


def test_edge_aggregate_brute_force_coo():
    N, d = 257, 12
    rp, send, recv = synth.edges_random(N, 16, seed=4)
    msg = synth.normal((int(rp[-1]), d), 5).numpy()
    out = oracle.edge_aggregate(msg, rp)
    ref = np.zeros((N, d), np.float64)
    np.add.at(ref, recv, msg.astype(np.float64))
    assert np.array_equal(out, ref.astype(np.float32))
    # column sums are conserved
    np.testing.assert_allclose(out.astype(np.float64).sum(0), msg.astype(np.float64).sum(0),
                               rtol=1e-6, atol=1e-4)
    deg = np.diff(rp)
    for i in np.nonzero(deg == 1)[0]:
        assert np.array_equal(out[i], msg[rp[i]])
    assert np.all(out[deg == 0] == 0)


def test_edge_aggregate_pbc_degrees():
    # periodic cell at 0.08 atoms/A^3, cutoff 6 A: mean degree ~ 0.08*4/3*pi*216
    rp, send, recv = synth.edges_pbc(2000, seed=1)
    deg = np.diff(rp)
    expect = 0.08 * 4.0 / 3.0 * np.pi * 6.0 ** 3
    assert abs(deg.mean() - expect * (1999 / 2000)) < 0.05 * expect
    assert np.all(recv[:-1] <= recv[1:])
    assert not np.any(send == recv)


def test_edge_broadcast_is_adjoint_of_edge_aggregate():
    N, d = 300, 10
    rp, send, recv = synth.edges_random(N, 12, seed=7)
    msg = synth.normal((int(rp[-1]), d), 8).numpy()
    dx = synth.normal((N, d), 9).numpy()
    dmsg = oracle.edge_broadcast(dx, rp)
    assert np.array_equal(dmsg, dx[recv])                 # NumPy gather, bit-exact
    lhs = np.sum(oracle.edge_aggregate(msg, rp).astype(np.float64) * dx)
    rhs = np.sum(msg.astype(np.float64) * dmsg)
    assert abs(lhs - rhs) <= 1e-6 * (abs(lhs) + 1.0)


def test_neighbor_aggregate_brute_force():
    N, d = 257, 12
    rp, send, recv = synth.edges_random(N, 16, seed=10)
    x = synth.normal((N, d), 11).numpy()
    out = oracle.neighbor_aggregate(x, rp, send.astype(np.int32))
    ref = np.zeros((N, d), np.float64)
    np.add.at(ref, recv, x[send].astype(np.float64))
    assert np.array_equal(out, ref.astype(np.float32))
    # the same as aggregating the gathered messages
    assert np.array_equal(out, oracle.edge_aggregate(x[send], rp))
    import pytest
    bad = send.astype(np.int32).copy()
    bad[3] = N
    with pytest.raises(ValueError):
        oracle.neighbor_aggregate(x, rp, bad)
