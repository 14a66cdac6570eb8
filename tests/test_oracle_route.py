"""Pins for the oracle's routing (CPU only).

Element-type routing: each element type has a fixed top-K expert set (paper
review 'Breaking the Training Barrier of Billion-Parameter Universal Machine
Learning Interatomic Potentials', section 3.2, sparse MoE design).  The oracle
is checked against brute force over all K-subsets, NumPy's stable argsort,
SciPy's softmax and closed forms, never against its own formulas.
"""
import itertools

import numpy as np
import pytest
import scipy.special

import oracle
from element_routed_moe_b200 import synth


def _dominant_subset(g, K):
    """Brute force: the unique K-subset S with every selected logit beating
    every unselected one (ties: the lower expert id wins)."""
    E = len(g)
    found = []
    for S in itertools.combinations(range(E), K):
        rest = [b for b in range(E) if b not in S]
        ok = all(g[a] > g[b] or (g[a] == g[b] and a < b) for a in S for b in rest)
        if ok:
            found.append(set(S))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("E,K", [(8, 2), (8, 1), (8, 8), (6, 3), (5, 4)])
def test_route_topk_matches_brute_force(E, K):
    T = 7
    gate = synth.gate_table(T, E, seed=11)
    gate[3, 1] = gate[3, 4]            # plant a tie
    gate[5, :] = 0.25                  # an all-tied row
    types = synth.types_uniform(200, T, seed=12)
    r = oracle.route(types, gate, K)
    te = r["topk_expert"]
    for i, t in enumerate(types):
        assert set(te[i].tolist()) == _dominant_subset(gate[t].tolist(), K)
        # order within K: descending logit, then ascending id
        lg = gate[t, te[i]]
        for k in range(K - 1):
            assert lg[k] > lg[k + 1] or (lg[k] == lg[k + 1] and te[i, k] < te[i, k + 1])


def test_route_weights_library_softmax_and_invariants():
    T, E, K = 9, 16, 5
    gate = synth.gate_table(T, E, seed=3)
    types = synth.types_uniform(300, T, seed=4)
    r = oracle.route(types, gate, K)
    te, tw = r["topk_expert"], r["topk_weight"]
    for i, t in enumerate(types):
        ref = scipy.special.softmax(gate[t, te[i]].astype(np.float64))
        np.testing.assert_allclose(tw[i], ref, rtol=1e-6, atol=0)
        assert abs(float(tw[i].astype(np.float64).sum()) - 1.0) < 1e-6
        assert np.all(np.diff(tw[i]) <= 0)


def test_route_weight_closed_forms():
    gate = np.array([[0.5, -1.0, 2.0, 0.0]], np.float32)
    types = np.zeros(3, np.int32)
    r1 = oracle.route(types, gate, 1)
    assert np.all(r1["topk_weight"] == 1.0)           # K = 1: exactly one
    assert np.all(r1["topk_expert"] == 2)
    r2 = oracle.route(types, gate, 2)
    # K = 2: the weights are the logistic function of the logit gap
    l0, l1 = 2.0, 0.5
    assert np.all(r2["topk_expert"][0] == [2, 0])
    np.testing.assert_allclose(r2["topk_weight"][0, 0], 1.0 / (1.0 + np.exp(l1 - l0)), rtol=1e-7)
    z = np.zeros((1, 8), np.float32)                    # all tied: 1/K, lowest ids
    r4 = oracle.route(types, z, 4)
    assert np.all(r4["topk_weight"] == 0.25)
    assert np.all(r4["topk_expert"] == [0, 1, 2, 3])


def test_route_counts_offsets_perm():
    T, E, K, N = 89, 40, 8, 4000
    gate = synth.gate_table(T, E, seed=21)
    types = synth.types_zipf(N, T, seed=22)
    r = oracle.route(types, gate, K)
    te = r["topk_expert"]
    # closed form: counts[e] = sum_t hist[t] * [e in S_t]
    hist = np.bincount(types, minlength=T)
    cf = np.zeros(E, np.int64)
    for t in range(T):
        if hist[t]:
            for e in _top_set(gate[t], K):
                cf[e] += hist[t]
    assert np.array_equal(r["counts"], cf)
    assert r["counts"].sum() == N * K
    assert np.array_equal(r["offsets"], np.concatenate([[0], np.cumsum(cf)]))
    # stable permutation = NumPy's stable argsort of the flat expert keys
    assert np.array_equal(r["perm"], np.argsort(te.ravel(), kind="stable"))
    R = N * K
    assert np.array_equal(np.sort(r["perm"]), np.arange(R))
    assert np.array_equal(r["slot_of"][r["perm"]], np.arange(R))
    # atom index strictly increases inside each expert segment
    off = r["offsets"]
    for e in range(E):
        atoms = r["perm"][off[e]:off[e + 1]] // K
        assert np.all(np.diff(atoms) > 0)
        assert np.all(te.ravel()[r["perm"][off[e]:off[e + 1]]] == e)


def _top_set(row, K):
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return order[:K]


def test_route_K_equals_E_and_single_type():
    E = 6
    gate = synth.gate_table(1, E, seed=5)
    types = np.zeros(50, np.int32)
    r = oracle.route(types, gate, E)
    assert np.all(r["counts"] == 50)
    assert sorted(r["topk_expert"][0].tolist()) == list(range(E))
    # every expert not chosen by any type gets an empty segment
    gate2 = np.array([[5, 4, -9, -9], [5, 4, -9, -9]], np.float32)
    r2 = oracle.route(np.array([0, 1, 1], np.int32), gate2, 2)
    assert list(r2["counts"]) == [3, 3, 0, 0]
    assert list(r2["offsets"]) == [0, 3, 6, 6, 6]


def test_route_rejects_bad_type():
    gate = synth.gate_table(4, 4, seed=0)
    with pytest.raises(ValueError):
        oracle.route(np.array([0, 4], np.int32), gate, 2)
    with pytest.raises(ValueError):
        oracle.route(np.array([-1], np.int32), gate, 2)
