"""Pins for the oracle's expert-parallel exchange layout (CPU only).

Experts are sharded over ranks ([Review] 'Breaking the Training Barrier of
Billion-Parameter Universal Machine Learning Interatomic Potentials', section
3.4, FSEP) and the packed dispatch rows travel to the expert's owner in an
all-to-all (section 3.5).  The layout is pinned by a brute-force simulation
that places every (sender, expert, row) token one by one, and the whole
exchange (send, expert MLP on the owner, return, combine) is checked on the
CPU against each rank's local chain: the expert MLP works row by row, so
moving rows between ranks must not change any atom's output.
"""
import numpy as np
import pytest

import oracle
from element_routed_moe_b200 import synth


def _brute(counts):
    """Owner row of every token (s, e, i): owners list received tokens by
    (local expert, sender, i); senders list theirs by (e, i)."""
    P, E = counts.shape
    El = E // P
    dst, src = {}, {}
    for o in range(P):
        toks = [(e - o * El, s, i) for e in range(o * El, (o + 1) * El) for s in range(P)
                for i in range(counts[s, e])]
        for pos, (j, s, i) in enumerate(sorted(toks)):
            dst[(s, o * El + j, i)] = pos
    for s in range(P):
        toks = [(e, i) for e in range(E) for i in range(counts[s, e])]
        for pos, (e, i) in enumerate(toks):
            src[(s, e, i)] = pos
    return src, dst


@pytest.mark.parametrize("P,E", [(1, 8), (2, 8), (4, 16), (8, 72), (3, 9)])
def test_layout_matches_token_by_token_placement(P, E):
    rng = np.random.default_rng(P * 100 + E)
    counts = rng.integers(0, 7, size=(P, E)).astype(np.int32)
    counts[rng.random((P, E)) < 0.2] = 0                      # empty (sender, expert) blocks
    src_off, dst_off, recv_off = oracle.ep_layout(counts)
    src, dst = _brute(counts)
    for (s, e, i), pos in dst.items():
        assert dst_off[s, e] + i == pos
        assert src_off[s, e] + i == src[(s, e, i)]
    El = E // P
    for o in range(P):
        per_expert = counts[:, o * El:(o + 1) * El].sum(0)
        assert np.array_equal(recv_off[o], np.concatenate([[0], np.cumsum(per_expert)]))
    assert np.array_equal(src_off[:, -1], counts.sum(1))
    assert recv_off[:, -1].sum() == counts.sum()


def test_layout_single_rank_is_the_local_dispatch_order():
    counts = np.array([[3, 0, 5, 1]], np.int32)
    src_off, dst_off, recv_off = oracle.ep_layout(counts)
    assert np.array_equal(dst_off[0], src_off[0, :-1])
    assert np.array_equal(recv_off[0], src_off[0])


def test_layout_rejects_uneven_expert_split():
    with pytest.raises(ValueError):
        oracle.ep_layout(np.ones((3, 8), np.int32))


def _ep_forward_cpu(shards, gate, K, w1, w2, d, P):
    """The EP exchange with oracle kernels: local route + quant + dequant per
    rank, rows moved to the owners by the layout, the owner's experts on the
    received rows, rows moved back, local combine."""
    E = gate.shape[1]
    El = E // P
    local = []
    for x, types in shards:
        r = oracle.route(types, gate, K)
        q, scale = oracle.quant_by_type(x, types, gate.shape[0], r["perm"], K)
        xd = oracle.dequant_by_type(q, types, r["perm"], K, scale)
        local.append((r, xd))
    counts = np.stack([r["counts"] for r, _ in local])
    src_off, dst_off, recv_off = oracle.ep_layout(counts)
    recv = [np.zeros((recv_off[o, -1], d), np.float32) for o in range(P)]
    for s, (r, xd) in enumerate(local):
        for e in range(E):
            o, n = e // El, counts[s, e]
            recv[o][dst_off[s, e]:dst_off[s, e] + n] = xd[src_off[s, e]:src_off[s, e] + n]
    outs = [oracle.expert_ffn_fwd(recv[o], recv_off[o], w1[o * El:(o + 1) * El], w2[o * El:(o + 1) * El])
            for o in range(P)]
    ys = []
    for s, (r, xd) in enumerate(local):
        back = np.zeros_like(xd)
        for e in range(E):
            o, n = e // El, counts[s, e]
            back[src_off[s, e]:src_off[s, e] + n] = outs[o][dst_off[s, e]:dst_off[s, e] + n]
        ys.append(oracle.combine(back, r["slot_of"], K, r["topk_weight"]))
    return ys


def test_ep_forward_equals_each_ranks_local_chain():
    P, N, T, E, K, d, h = 4, 96, 11, 8, 2, 8, 12
    gate = synth.gate_table(T, E, 1)
    w1, w2 = (t.numpy() for t in synth.expert_weights(E, d, h, 2))
    shards = [(synth.normal((N, d), 10 + s).numpy(), synth.types_zipf(N, T, seed=20 + s)) for s in range(P)]
    ys = _ep_forward_cpu(shards, gate, K, w1, w2, d, P)
    for s, (x, types) in enumerate(shards):
        r = oracle.route(types, gate, K)
        q, scale = oracle.quant_by_type(x, types, T, r["perm"], K)
        xd = oracle.dequant_by_type(q, types, r["perm"], K, scale)
        yd = oracle.expert_ffn_fwd(xd, r["offsets"], w1, w2)
        ref = oracle.combine(yd, r["slot_of"], K, r["topk_weight"])
        assert np.array_equal(ys[s], ref)
