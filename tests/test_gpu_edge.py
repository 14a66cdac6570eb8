"""GPU parity: edge -> atom aggregation vs the oracle (paper review 'Breaking
the Training Barrier of Billion-Parameter Universal Machine Learning
Interatomic Potentials', section 3.5: neighbour / edge aggregation)."""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, host, poison_like, rel_fro, to_dev

pytestmark = pytest.mark.gpu


def _run(msg, rp):
    N = rp.shape[0] - 1
    out = poison_like((N, msg.shape[1]), torch.float32)
    J.janus_edge_aggregate(msg, to_dev(rp), out=out)
    return out


def test_edge_tiny_random():
    rp, _, _ = synth.edges_random(512, 16, seed=6)
    msg = synth.normal((int(rp[-1]), 64), 8, DEV)
    got = host(_run(msg, rp))
    ref = oracle.edge_aggregate(host(msg), rp)
    assert rel_fro(got, ref) <= TOL_FP32
    deg = np.diff(rp)
    assert np.all(got[deg == 0] == 0)
    for i in np.nonzero(deg == 1)[0]:
        assert np.array_equal(got[i], host(msg)[rp[i]])


def test_edge_degenerate_degrees():
    # zero-degree atoms, one receiver with 4096 edges, odd degrees, ragged d
    deg = np.array([0, 1, 4096, 0, 3, 5, 7, 0, 2, 9, 0], np.int64)
    rp = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    for d in (4, 4 * 37, 4 * 300):
        msg = synth.normal((int(rp[-1]), d), 3, DEV)
        got = host(_run(msg, rp))
        ref = oracle.edge_aggregate(host(msg), rp)
        assert rel_fro(got, ref) <= TOL_FP32
        assert np.all(got[deg == 0] == 0)
        assert np.array_equal(got[1], host(msg)[0])


def test_edge_no_edges():
    rp = np.zeros(6, np.int64)
    msg = torch.empty((0, 8), dtype=torch.float32, device=DEV)
    out = poison_like((5, 8), torch.float32)
    J.janus_edge_aggregate(msg, to_dev(rp), out=out)
    assert torch.all(out == 0).item()


@pytest.mark.parametrize("name", ["L", "slice"])
def test_edge_full_size_sampled_atoms(name):
    cfg = synth.CONFIGS[name]
    rp, _, _ = synth.edges_pbc(cfg.n_atoms, seed=6)
    Ed = int(rp[-1])
    msg = synth.normal((Ed, cfg.d), 8, DEV)
    out = _run(msg, rp)
    assert torch.isfinite(out).all().item()
    atoms = np.unique(np.concatenate([[0, cfg.n_atoms - 1],
                                      np.random.default_rng(3).integers(0, cfg.n_atoms, 512)]))
    # compact CSR of the sampled atoms' contiguous message blocks
    deg = rp[atoms + 1] - rp[atoms]
    sub_rp = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    idx = np.concatenate([np.arange(rp[a], rp[a + 1]) for a in atoms])
    sub_msg = host(msg[torch.as_tensor(idx, device=DEV)])
    ref = oracle.edge_aggregate(sub_msg, sub_rp)
    assert rel_fro(host(out)[atoms], ref) <= TOL_FP32
    # column sums are conserved over the whole layer (property at any size)
    colsum_out = _colsum64(out)
    colsum_msg = _colsum64(msg)
    assert rel_fro(host(colsum_out), host(colsum_msg)) <= 1e-6


def _colsum64(t, chunk=1 << 18):
    acc = torch.zeros(t.shape[1], dtype=torch.float64, device=t.device)
    for i in range(0, t.shape[0], chunk):
        acc += t[i:i + chunk].to(torch.float64).sum(0)
    return acc


# ---- gradient of the edge aggregation, and neighbour aggregation by sender ----

def test_edge_broadcast_bit_exact():
    deg = np.array([0, 1, 4096, 0, 3, 5, 7, 0, 2, 9, 0], np.int64)
    rp = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    for d in (4, 4 * 37, 4 * 300):
        dx = synth.normal((len(deg), d), 5, DEV)
        out = poison_like((int(rp[-1]), d), torch.float32)
        J.janus_edge_broadcast(dx, to_dev(rp), out=out)
        assert np.array_equal(host(out), oracle.edge_broadcast(host(dx), rp))


def test_edge_broadcast_adjoint_on_gpu():
    rp, _, _ = synth.edges_random(512, 16, seed=6)
    msg = synth.normal((int(rp[-1]), 64), 8, DEV)
    dx = synth.normal((512, 64), 9, DEV)
    x = J.janus_edge_aggregate(msg, to_dev(rp))
    dmsg = J.janus_edge_broadcast(dx, to_dev(rp))
    lhs = float((x.double() * dx.double()).sum())
    rhs = float((msg.double() * dmsg.double()).sum())
    assert abs(lhs - rhs) <= 1e-5 * (abs(lhs) + 1.0)


@pytest.mark.parametrize("d", [4, 64, 4 * 37, 4 * 300])
def test_neighbor_aggregate_small(d):
    rp, send, _ = synth.edges_random(700, 16, seed=12)
    x = synth.normal((700, d), 13, DEV)
    out = poison_like((700, d), torch.float32)
    J.janus_neighbor_aggregate(x, to_dev(rp), to_dev(send.astype(np.int32)), out=out)
    ref = oracle.neighbor_aggregate(host(x), rp, send.astype(np.int32))
    assert rel_fro(host(out), ref) <= TOL_FP32
    deg = np.diff(rp)
    assert np.all(host(out)[deg == 0] == 0)


def test_neighbor_aggregate_degenerate_and_bad_senders():
    deg = np.array([0, 1, 4096, 0, 33, 31, 32, 64, 0], np.int64)
    rp = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    N = len(deg)
    send = np.random.default_rng(3).integers(0, N, int(rp[-1])).astype(np.int32)
    x = synth.normal((N, 4 * 40), 14, DEV)
    out = J.janus_neighbor_aggregate(x, to_dev(rp), to_dev(send))
    assert rel_fro(host(out), oracle.neighbor_aggregate(host(x), rp, send)) <= TOL_FP32
    # out-of-range senders add nothing
    bad = send.copy()
    bad[5] = N + 7
    bad[100] = -2
    out2 = J.janus_neighbor_aggregate(x, to_dev(rp), to_dev(bad))
    mask = (bad < 0) | (bad >= N)
    xs = np.vstack([host(x), np.zeros((1, x.shape[1]), np.float32)])   # row N is zero
    ref2 = oracle.edge_aggregate(xs[np.where(mask, N, bad)], rp)
    assert rel_fro(host(out2), ref2) <= TOL_FP32


def test_neighbor_aggregate_full_size_L():
    cfg = synth.CONFIGS["L"]
    rp, send, _ = synth.edges_pbc(cfg.n_atoms, seed=6)
    x = synth.normal((cfg.n_atoms, cfg.d), 8, DEV)
    out = J.janus_neighbor_aggregate(x, to_dev(rp), to_dev(send.astype(np.int32)))
    ref = oracle.neighbor_aggregate(host(x), rp, send.astype(np.int32))
    assert rel_fro(host(out), ref) <= TOL_FP32
