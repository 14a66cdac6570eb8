"""GPU parity: the grouped expert MLP forward and input VJP vs the FP64 oracle
(paper review 'Breaking the Training Barrier of Billion-Parameter Universal
Machine Learning Interatomic Potentials', section 3.1 Table II and section
3.3).  Tolerance: relative Frobenius error <= 1e-5 (FP32-accurate paths)."""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, TOL_ROW, host, max_row_rel, poison_like, rel_fro, sample_rows, to_dev

pytestmark = pytest.mark.gpu

MODES = [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32]


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


SMALL = {
    # name: (counts per expert, d, h)
    "tiny_like": ([128, 131, 0, 127, 129, 1, 256, 252], 64, 64),
    "ragged_tails": ([37, 0, 300, 1, 129, 200], 4 * 49, 4 * 65),
    "multi_tile": ([700, 900, 400], 512, 384),
    "single_row": ([0, 1, 0], 16, 8),
    "d4": ([5, 3], 4, 4),
}


def _run(xd, gd, offs, w1, w2, mode):
    R, d = xd.shape
    h = w1.shape[2]
    yd = poison_like((R, d), torch.float32)
    act = poison_like((R, h), torch.float32)
    J.janus_expert_ffn_fwd(xd, offs, w1, w2, mode=mode, out=yd, act=act)
    dxd = poison_like((R, d), torch.float32)
    J.janus_expert_ffn_vjp(xd, gd, offs, w1, w2, act=act, mode=mode, out=dxd)
    dxd2 = poison_like((R, d), torch.float32)
    J.janus_expert_ffn_vjp(xd, gd, offs, w1, w2, act=None, mode=mode, out=dxd2)
    return yd, act, dxd, dxd2


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", list(SMALL))
def test_ffn_small_full_parity(name, mode):
    counts, d, h = SMALL[name]
    E = len(counts)
    offs = _offsets(counts)
    R = int(offs[-1])
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    xd = synth.normal((R, d), 4, DEV)
    gd = synth.normal((R, d), 5, DEV)
    yd, act, dxd, dxd2 = _run(xd, gd, to_dev(offs), w1, w2, mode)
    ref_y, ref_a = oracle.expert_ffn_fwd(host(xd), offs, host(w1), host(w2), want_act=True)
    ref_dx = oracle.expert_ffn_vjp(host(xd), host(gd), offs, host(w1), host(w2))
    assert rel_fro(host(yd), ref_y) <= TOL_FP32
    assert rel_fro(host(act), ref_a) <= TOL_FP32
    assert rel_fro(host(dxd), ref_dx) <= TOL_FP32
    assert rel_fro(host(dxd2), ref_dx) <= TOL_FP32
    # every row is written (no NaN poison left) and per-expert errors are small too
    for e in range(E):
        a, b = offs[e], offs[e + 1]
        if b > a:
            assert rel_fro(host(yd)[a:b], ref_y[a:b]) <= 4 * TOL_FP32


def test_ffn_identity_experts_give_silu():
    d = 64
    offs = _offsets([100, 60])
    eye = torch.eye(d, dtype=torch.float32, device=DEV).expand(2, d, d).contiguous()
    xd = synth.normal((160, d), 8, DEV)
    yd, _ = J.janus_expert_ffn_fwd(xd, to_dev(offs), eye, eye)
    ref = host(xd) / (1.0 + np.exp(-host(xd).astype(np.float64)))
    assert rel_fro(host(yd), ref) <= 1e-6


FULL = ["S", "M", "L"]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", FULL)
def test_ffn_full_size_sampled_rows(name, mode):
    cfg = synth.CONFIGS[name]
    types = synth.types_zipf(cfg.n_atoms, cfg.n_types, seed=1)
    gate = synth.gate_table(cfg.n_types, cfg.n_experts, 2)
    r = oracle.route(types, gate, cfg.top_k)
    offs = r["offsets"]
    R = cfg.n_rows
    w1, w2 = synth.expert_weights(cfg.n_experts, cfg.d, cfg.h, 3, DEV)
    xd = synth.normal((R, cfg.d), 4, DEV)
    gd = synth.normal((R, cfg.d), 5, DEV)
    yd, act, dxd, _ = _run(xd, gd, to_dev(offs), w1, w2, mode)
    rows = sample_rows(offs, 192, seed=7, R=R)
    hw1, hw2 = host(w1), host(w2)
    ref_y = oracle.expert_ffn_fwd(host(xd), offs, hw1, hw2, rows=rows)
    ref_dx = oracle.expert_ffn_vjp(host(xd), host(gd), offs, hw1, hw2, rows=rows)
    assert rel_fro(host(yd)[rows], ref_y) <= TOL_FP32
    assert rel_fro(host(dxd)[rows], ref_dx) <= TOL_FP32
    assert max_row_rel(host(yd)[rows], ref_y) <= TOL_ROW
    assert max_row_rel(host(dxd)[rows], ref_dx) <= TOL_ROW
    # every row was written
    assert torch.isfinite(yd).all().item() and torch.isfinite(dxd).all().item()
