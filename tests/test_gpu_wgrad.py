"""GPU parity: per-expert weight gradients dW1 = Xd^T dA, dW2 = silu(a)^T Gd
(force training differentiates the energy w.r.t. the expert weights too:
paper review 'Breaking the Training Barrier of Billion-Parameter Universal
Machine Learning Interatomic Potentials', section 3.3).  Tolerance: relative
Frobenius error <= 1e-5 per expert."""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, host, poison_like, rel_fro, to_dev

pytestmark = pytest.mark.gpu

MODES = [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32]


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


SMALL = {
    "ragged": ([37, 0, 300, 1, 129, 200], 4 * 49, 4 * 65),
    "multi_tile": ([700, 900, 17], 512, 384),
    "tiny_rows": ([0, 1, 0, 2], 16, 8),
    "k_tail_16": ([15, 16, 17, 33], 64, 96),
}


def _check(xd, gd, counts, d, h, mode, with_act):
    E = len(counts)
    offs = _offsets(counts)
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    act = None
    if with_act:
        _, act = J.janus_expert_ffn_fwd(xd, to_dev(offs), w1, w2, mode=mode, want_act=True)
    dw1 = poison_like((E, d, h), torch.float32)
    dw2 = poison_like((E, h, d), torch.float32)
    J.janus_expert_ffn_weight_grad(xd, gd, to_dev(offs), w1, w2, act=act, mode=mode, dw1=dw1, dw2=dw2)
    torch.cuda.synchronize()
    r1, r2 = oracle.expert_ffn_weight_grad(host(xd), host(gd), offs, host(w1), host(w2))
    g1, g2 = host(dw1), host(dw2)
    for e in range(E):
        if counts[e] == 0:
            assert np.all(g1[e] == 0) and np.all(g2[e] == 0)
        else:
            assert rel_fro(g1[e], r1[e]) <= TOL_FP32, (e, rel_fro(g1[e], r1[e]))
            assert rel_fro(g2[e], r2[e]) <= TOL_FP32, (e, rel_fro(g2[e], r2[e]))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("with_act", [True, False])
def test_weight_grad_small(name, mode, with_act):
    counts, d, h = SMALL[name]
    R = int(sum(counts))
    xd = synth.normal((R, d), 4, DEV)
    gd = synth.normal((R, d), 5, DEV)
    _check(xd, gd, counts, d, h, mode, with_act)


@pytest.mark.parametrize("mode", MODES)
def test_weight_grad_no_rows(mode):
    E, d, h = 3, 8, 12
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    empty = torch.empty((0, d), dtype=torch.float32, device=DEV)
    dw1, dw2 = J.janus_expert_ffn_weight_grad(empty, empty, to_dev(np.zeros(E + 1, np.int32)), w1, w2,
                                              mode=mode)
    assert torch.all(dw1 == 0).item() and torch.all(dw2 == 0).item()


@pytest.mark.parametrize("mode", MODES)
def test_weight_grad_full_size_sampled_experts(mode):
    # the S-shaped layer; the oracle checks the smallest, a median and the largest expert
    cfg = synth.CONFIGS["S"]
    types = synth.types_zipf(cfg.n_atoms, cfg.n_types, seed=1)
    gate = synth.gate_table(cfg.n_types, cfg.n_experts, 2)
    r = oracle.route(types, gate, cfg.top_k)
    offs = r["offsets"]
    cnt = np.diff(offs)
    R, d, h, E = cfg.n_rows, cfg.d, cfg.h, cfg.n_experts
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    xd = synth.normal((R, d), 4, DEV)
    gd = synth.normal((R, d), 5, DEV)
    _, act = J.janus_expert_ffn_fwd(xd, to_dev(offs), w1, w2, mode=mode, want_act=True)
    dw1, dw2 = J.janus_expert_ffn_weight_grad(xd, gd, to_dev(offs), w1, w2, act=act, mode=mode)
    torch.cuda.synchronize()
    order = np.argsort(cnt)
    picks = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])})
    hw1, hw2 = host(w1), host(w2)
    for e in picks:
        a, b = offs[e], offs[e + 1]
        sub = np.array([0, b - a], np.int32)
        r1, r2 = oracle.expert_ffn_weight_grad(host(xd[a:b]), host(gd[a:b]), sub, hw1[e:e + 1], hw2[e:e + 1])
        assert rel_fro(host(dw1[e]), r1[0]) <= TOL_FP32
        assert rel_fro(host(dw2[e]), r2[0]) <= TOL_FP32
