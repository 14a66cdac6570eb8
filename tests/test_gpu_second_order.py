"""GPU parity: the second-order pass of the expert MLP (the VJP of the input
VJP: force training fits forces, which are input gradients, so the loss
gradient flows back through the input VJP; paper review 'Breaking the
Training Barrier of Billion-Parameter Universal Machine Learning Interatomic
Potentials', section 3.3).  Outputs d_xd, d_gd [R,d] and the per-expert
dW1, dW2; tolerance: relative Frobenius error <= 1e-5 (per expert for the
weights), both FFN modes."""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, host, poison_like, rel_fro, sample_rows, to_dev

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


def _inputs(R, d, seed):
    return (synth.normal((R, d), seed, DEV), synth.normal((R, d), seed + 1, DEV),
            synth.normal((R, d), seed + 2, DEV))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("with_act", [True, False])
def test_second_order_small(name, mode, with_act):
    counts, d, h = SMALL[name]
    E, R = len(counts), int(sum(counts))
    offs = _offsets(counts)
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    xd, gd, vd = _inputs(R, d, 20)
    act = None
    if with_act:
        _, act = J.janus_expert_ffn_fwd(xd, to_dev(offs), w1, w2, mode=mode, want_act=True)
    out = dict(d_xd=poison_like((R, d), torch.float32), d_gd=poison_like((R, d), torch.float32),
               dw1=poison_like((E, d, h), torch.float32), dw2=poison_like((E, h, d), torch.float32))
    J.janus_expert_ffn_vjp_vjp(xd, gd, vd, to_dev(offs), w1, w2, act=act, mode=mode, weight_grad=True, **out)
    torch.cuda.synchronize()
    hx, hg, hv, h1, h2 = host(xd), host(gd), host(vd), host(w1), host(w2)
    rx, rg = oracle.expert_ffn_vjp_vjp(hx, hg, hv, offs, h1, h2)
    assert rel_fro(host(out["d_xd"]), rx) <= TOL_FP32
    assert rel_fro(host(out["d_gd"]), rg) <= TOL_FP32
    r1, r2 = oracle.expert_ffn_vjp_vjp_weight_grad(hx, hg, hv, offs, h1, h2)
    g1, g2 = host(out["dw1"]), host(out["dw2"])
    for e in range(E):
        if counts[e] == 0:
            assert np.all(g1[e] == 0) and np.all(g2[e] == 0)
        else:
            assert rel_fro(g1[e], r1[e]) <= TOL_FP32, (e, rel_fro(g1[e], r1[e]))
            assert rel_fro(g2[e], r2[e]) <= TOL_FP32, (e, rel_fro(g2[e], r2[e]))


@pytest.mark.parametrize("mode", MODES)
def test_second_order_without_weight_part_matches(mode):
    counts, d, h = SMALL["ragged"]
    E, R = len(counts), int(sum(counts))
    offs = to_dev(_offsets(counts))
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    xd, gd, vd = _inputs(R, d, 30)
    a_x, a_g = J.janus_expert_ffn_vjp_vjp(xd, gd, vd, offs, w1, w2, mode=mode)
    b_x, b_g, _, _ = J.janus_expert_ffn_vjp_vjp(xd, gd, vd, offs, w1, w2, mode=mode, weight_grad=True)
    # the same kernels compute the row outputs with and without the weight part
    assert torch.equal(a_x, b_x) and torch.equal(a_g, b_g)


@pytest.mark.parametrize("mode", MODES)
def test_second_order_zero_upstream_gradient(mode):
    # g = 0: d_xd, dW1, dW2 vanish exactly (dh = 0), d_gd does not
    counts, d, h = SMALL["k_tail_16"]
    E, R = len(counts), int(sum(counts))
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    xd, _, vd = _inputs(R, d, 40)
    gd = torch.zeros_like(xd)
    d_x, d_g, dw1, dw2 = J.janus_expert_ffn_vjp_vjp(xd, gd, vd, to_dev(_offsets(counts)), w1, w2, mode=mode,
                                                    weight_grad=True)
    assert torch.all(d_x == 0).item() and torch.all(dw1 == 0).item() and torch.all(dw2 == 0).item()
    assert torch.any(d_g != 0).item()


@pytest.mark.parametrize("mode", MODES)
def test_second_order_no_rows(mode):
    E, d, h = 3, 8, 12
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    empty = torch.empty((0, d), dtype=torch.float32, device=DEV)
    _, _, dw1, dw2 = J.janus_expert_ffn_vjp_vjp(empty, empty, empty, to_dev(np.zeros(E + 1, np.int32)), w1, w2,
                                                mode=mode, weight_grad=True)
    assert torch.all(dw1 == 0).item() and torch.all(dw2 == 0).item()


def test_second_order_rejects_one_weight_output():
    E, d, h, R = 2, 8, 8, 4
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    xd, gd, vd = _inputs(R, d, 50)
    offs = to_dev(_offsets([2, 2]))
    # the binding passes both weight outputs or neither; call the ABI directly
    with pytest.raises(J.JanusError) as e:
        nb = J.janus_expert_ffn_vjp_vjp_workspace_size(R, h, False, True)
        ws = torch.empty(nb, dtype=torch.uint8, device=DEV)
        out = torch.empty((R, d), device=DEV)
        dw1 = torch.empty((E, d, h), device=DEV)
        J._raise(J.lib().janus_expert_ffn_vjp_vjp(
            xd.data_ptr(), gd.data_ptr(), vd.data_ptr(), None, offs.data_ptr(), E, R, d, h, w1.data_ptr(),
            w2.data_ptr(), out.data_ptr(), out.data_ptr(), dw1.data_ptr(), None, int(J.JANUS_FFN_3XTF32),
            ws.data_ptr(), nb, None), "janus_expert_ffn_vjp_vjp")
    assert e.value.status == J.JANUS_ERR_INVALID_ARG


@pytest.mark.parametrize("mode", MODES)
def test_second_order_full_size(mode):
    # the S-shaped layer: sampled rows for d_xd and d_gd; the smallest, a
    # median and the largest expert for the weight part
    cfg = synth.CONFIGS["S"]
    types = synth.types_zipf(cfg.n_atoms, cfg.n_types, seed=1)
    gate = synth.gate_table(cfg.n_types, cfg.n_experts, 2)
    offs = oracle.route(types, gate, cfg.top_k)["offsets"]
    cnt = np.diff(offs)
    R, d, h, E = cfg.n_rows, cfg.d, cfg.h, cfg.n_experts
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    xd, gd, vd = _inputs(R, d, 60)
    _, act = J.janus_expert_ffn_fwd(xd, to_dev(offs), w1, w2, mode=mode, want_act=True)
    d_x, d_g, dw1, dw2 = J.janus_expert_ffn_vjp_vjp(xd, gd, vd, to_dev(offs), w1, w2, act=act, mode=mode,
                                                    weight_grad=True)
    torch.cuda.synchronize()
    hx, hg, hv, h1, h2 = host(xd), host(gd), host(vd), host(w1), host(w2)
    rows = sample_rows(offs, 64, seed=7, R=R)
    rx, rg = oracle.expert_ffn_vjp_vjp(hx, hg, hv, offs, h1, h2, rows=rows)
    assert rel_fro(host(d_x)[rows], rx) <= TOL_FP32
    assert rel_fro(host(d_g)[rows], rg) <= TOL_FP32
    order = np.argsort(cnt)
    for e in sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])}):
        a, b = offs[e], offs[e + 1]
        sub = np.array([0, b - a], np.int32)
        r1, r2 = oracle.expert_ffn_vjp_vjp_weight_grad(hx[a:b], hg[a:b], hv[a:b], sub, h1[e:e + 1], h2[e:e + 1])
        assert rel_fro(host(dw1[e]), r1[0]) <= TOL_FP32
        assert rel_fro(host(dw2[e]), r2[0]) <= TOL_FP32
