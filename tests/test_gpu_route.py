"""GPU parity: janus_route vs the oracle, bit-exact for indices/counts/offsets
and the stable permutation (routing by element type: paper review 'Breaking
the Training Barrier of Billion-Parameter Universal Machine Learning
Interatomic Potentials', section 3.2)."""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_WEIGHT, host, poison_like, to_dev

pytestmark = pytest.mark.gpu

CASES = {
    # name: (N, T, E, K, dist)
    "tiny": (512, 8, 8, 2, "uniform"),
    "S": (8192, 89, 72, 4, "zipf"),
    "M": (32768, 89, 40, 8, "zipf"),
    "L": (16384, 89, 72, 16, "zipf"),
    "slice": (65536, 89, 40, 8, "zipf"),
    "K1": (3000, 89, 40, 1, "zipf"),
    "K_eq_E": (2000, 13, 24, 24, "zipf"),
    "single_type": (1500, 1, 16, 4, "zipf"),
    "E256_K200": (700, 30, 256, 200, "uniform"),
    "ragged_chunks": (64 * 7 + 13, 5, 9, 3, "uniform"),
    "one_atom": (1, 3, 5, 2, "uniform"),
    "large_N_multichunk": (300_000, 89, 40, 1, "zipf"),
}


def _inputs(N, T, E, K, dist, seed):
    types = synth.types_uniform(N, T, seed) if dist == "uniform" else synth.types_zipf(N, T, seed=seed)
    gate = synth.gate_table(T, E, seed + 1)
    return types, gate


def _gpu_route(types, gate, K):
    N = types.shape[0]
    T, E = gate.shape
    R = N * K
    out = dict(topk_expert=poison_like((N, K), torch.int32),
               topk_weight=poison_like((N, K), torch.float32),
               counts=poison_like((E,), torch.int32),
               offsets=poison_like((E + 1,), torch.int32),
               perm=poison_like((R,), torch.int32),
               slot_of=poison_like((R,), torch.int32))
    r = J.janus_route(to_dev(types), to_dev(gate), K, out=out)
    J.janus_check(r["workspace"])
    return {k: host(v) for k, v in r.items() if k != "workspace"}


def _compare(g, o):
    for k in ("topk_expert", "counts", "offsets", "perm", "slot_of"):
        assert np.array_equal(g[k], o[k]), k
    w_g, w_o = g["topk_weight"].astype(np.float64), o["topk_weight"].astype(np.float64)
    assert np.all(np.abs(w_g - w_o) <= TOL_WEIGHT * np.abs(w_o))


@pytest.mark.parametrize("name", list(CASES))
def test_route_parity(name):
    N, T, E, K, dist = CASES[name]
    types, gate = _inputs(N, T, E, K, dist, seed=10)
    _compare(_gpu_route(types, gate, K), oracle.route(types, gate, K))


@pytest.mark.parametrize("seed", [1, 2])
def test_route_parity_more_seeds(seed):
    N, T, E, K, dist = CASES["M"]
    types, gate = _inputs(N, T, E, K, dist, seed=100 + seed)
    _compare(_gpu_route(types, gate, K), oracle.route(types, gate, K))


def test_route_ties_and_empty_experts():
    gate = np.zeros((4, 12), np.float32)
    gate[1, [3, 7, 9]] = 1.5               # ties at the top
    gate[2, :] = -np.arange(12, dtype=np.float32)
    gate[3, 5] = gate[3, 6] = 2.0
    types = synth.types_uniform(5000, 4, 3)
    for K in (1, 3, 5, 12):
        _compare(_gpu_route(types, gate, K), oracle.route(types, gate, K))


def test_route_zero_atoms():
    gate = synth.gate_table(4, 6, 0)
    r = J.janus_route(torch.empty(0, dtype=torch.int32, device=DEV), to_dev(gate), 2)
    J.janus_check(r["workspace"])
    assert np.all(host(r["counts"]) == 0) and np.all(host(r["offsets"]) == 0)


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), -float("inf")])
def test_route_non_finite_gate_logit_sets_data_error(bad):
    # a gate row with a non-finite logit has no defined top-K: reported as a
    # data fault, while the selection stays K distinct valid experts
    gate = synth.gate_table(3, 6, 1)
    gate[1, 4] = bad
    types = np.array([1, 0, 2, 1], np.int32)
    r = J.janus_route(to_dev(types), to_dev(gate), 3)
    with pytest.raises(J.JanusError) as e:
        J.janus_check(r["workspace"])
    assert e.value.status == J.JANUS_ERR_DATA
    te = host(r["topk_expert"])
    assert ((te >= 0) & (te < 6)).all()
    assert all(len(set(row)) == 3 for row in te)
    assert np.array_equal(np.sort(host(r["perm"])), np.arange(12))
    # the finite rows are routed as usual
    o = oracle.route(np.array([0, 2], np.int32), np.where(np.isfinite(gate), gate, 0).astype(np.float32), 3)
    assert np.array_equal(te[[1, 2]], o["topk_expert"])


def test_route_bad_type_sets_data_error():
    gate = synth.gate_table(4, 6, 0)
    types = np.array([0, 1, 7, 2, -3], np.int32)
    r = J.janus_route(to_dev(types), to_dev(gate), 2)
    with pytest.raises(J.JanusError) as e:
        J.janus_check(r["workspace"])
    assert e.value.status == J.JANUS_ERR_DATA
    # outputs stay well-formed: bad ids are routed as type 0
    fixed = np.where((types < 0) | (types >= 4), 0, types).astype(np.int32)
    _compare({k: host(v) for k, v in r.items() if k != "workspace"}, oracle.route(fixed, gate, 2))
    # the next good call clears the error word
    r2 = J.janus_route(to_dev(fixed), to_dev(gate), 2, workspace=r["workspace"])
    J.janus_check(r2["workspace"])


def test_route_repeat_calls_reuse_workspace():
    N, T, E, K, dist = CASES["S"]
    types, gate = _inputs(N, T, E, K, dist, seed=5)
    ref = oracle.route(types, gate, K)
    ws = None
    for _ in range(3):
        r = J.janus_route(to_dev(types), to_dev(gate), K, workspace=ws)
        ws = r["workspace"]
        J.janus_check(ws)
        _compare({k: host(v) for k, v in r.items() if k != "workspace"}, ref)


def test_injected_failure_with_real_buffers():
    types, gate = _inputs(100, 4, 6, 2, "uniform", 0)
    J.janus_debug_inject_launch_failures(1)
    with pytest.raises(J.JanusError) as e:
        J.janus_route(to_dev(types), to_dev(gate), 2)
    assert e.value.status == J.JANUS_ERR_CUDA
    r = J.janus_route(to_dev(types), to_dev(gate), 2)
    J.janus_check(r["workspace"])


# ---- several MoE layers routed at once (JIT planning) ----

@pytest.mark.parametrize("shape", [(8192, 89, 72, 4, 12), (3001, 13, 24, 7, 3), (700, 30, 256, 200, 2)])
def test_route_layers_match_per_layer_oracle(shape):
    N, T, E, K, L = shape
    types = synth.types_zipf(N, T, seed=3)
    gates = np.stack([synth.gate_table(T, E, 100 + l) for l in range(L)])
    r = J.janus_route_layers(to_dev(types), to_dev(gates), K)
    J.janus_check(r["workspace"])
    for l in range(L):
        ref = oracle.route(types, gates[l], K)
        got = {k: host(v[l]) for k, v in r.items() if k != "workspace"}
        got["topk_expert"] = got["topk_expert"].reshape(N, K)
        got["topk_weight"] = got["topk_weight"].reshape(N, K)
        _compare(got, ref)


def test_route_layers_zero_atoms_and_bad_type():
    gates = np.stack([synth.gate_table(4, 6, l) for l in range(3)])
    r = J.janus_route_layers(torch.empty(0, dtype=torch.int32, device=DEV), to_dev(gates), 2)
    J.janus_check(r["workspace"])
    assert np.all(host(r["counts"]) == 0) and np.all(host(r["offsets"]) == 0)
    r = J.janus_route_layers(to_dev(np.array([0, 9, 1], np.int32)), to_dev(gates), 2)
    with pytest.raises(J.JanusError) as e:
        J.janus_check(r["workspace"])
    assert e.value.status == J.JANUS_ERR_DATA


# ---- active-expert lists (JIT planning: the experts a batch activates) ----

@pytest.mark.parametrize("E", [1, 7, 32, 72, 256])
def test_active_experts_match_numpy_nonzero(E):
    g = np.random.default_rng(E)
    L = 13
    counts = g.integers(0, 4, size=(L, E)).astype(np.int32)
    counts[g.random((L, E)) < 0.5] = 0
    counts[0] = 0                     # a layer with no active expert
    counts[1] = 1                     # a layer with every expert active
    active, n_active = J.janus_active_experts(to_dev(counts))
    a, n = host(active), host(n_active)
    for l in range(L):
        ref = np.nonzero(counts[l])[0]
        assert n[l] == ref.size
        assert np.array_equal(a[l, :n[l]], ref)
        assert np.all(a[l, n[l]:] == -1)     # entries past the count untouched


def test_active_experts_of_routed_layers():
    N, T, E, K, L = 3000, 13, 24, 3, 4
    types = synth.types_zipf(N, T, seed=9)
    gates = np.stack([synth.gate_table(T, E, 300 + l) for l in range(L)])
    r = J.janus_route_layers(to_dev(types), to_dev(gates), K)
    active, n_active = J.janus_active_experts(r["counts"])
    for l in range(L):
        ref = np.nonzero(oracle.route(types, gates[l], K)["counts"])[0]
        assert np.array_equal(host(active)[l, :host(n_active)[l]], ref)
