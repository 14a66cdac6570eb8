"""GPU tests of the weight-split set (janus_expert_weights_f16): the FP16
splits of W1 and W2 for the forward's and the input VJP's kind::f16 GEMMs,
written once ahead of the MLP calls that read them (their `weights16`).

The FP16 tensor path is the FP32-accurate form of the expert MLP and its input
gradient (paper review 'Breaking the Training Barrier of Billion-Parameter
Universal Machine Learning Interatomic Potentials', section 3.1 Table II and
section 3.3); the split is this library's arithmetic, so the checks here are
equalities with the calls that split the weights themselves (whose results are
held to the oracle by the split-path tests):

* the set written by the one-read kernel (both flags) is byte for byte the set
  written by the per-orientation kernels (one flag at a time), on shapes with
  K tails in both orientations, rows and columns spread over 2^+-40, and
  all-zero 256 x 256 blocks;
* fwd_split, fwd_packed and vjp_split return bit-identical results with the
  set and without it, with the second GEMM on both of its paths;
* the set's call launches one kernel per weight tensor (two with one flag),
  and the MLP calls given a set launch no split of the weights.
"""
import numpy as np
import pytest
import torch

from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, to_dev

pytestmark = pytest.mark.gpu


def _wide(w, seed):
    """w with each row and each column scaled by its own power of two
    (2^-20 .. 2^20) and one 256 x 256 block of the first expert zeroed."""
    g = np.random.default_rng(seed)
    E, A, B = w.shape
    ra = np.ldexp(1.0, g.integers(-20, 21, size=(E, A, 1))).astype(np.float32)
    cb = np.ldexp(1.0, g.integers(-20, 21, size=(E, 1, B))).astype(np.float32)
    out = w * to_dev(ra) * to_dev(cb)
    out[0, :min(A, 256), :min(B, 256)] = 0
    return out.contiguous()


def _set(w1, w2, which):
    E, d, h = w1.shape
    out = torch.zeros(J.janus_expert_weights_f16_size(E, d, h), dtype=torch.uint8, device=DEV)
    return J.janus_expert_weights_f16(w1, w2, which, out=out)


SHAPES = [(2, 264, 328), (3, 512, 256), (1, 96, 776)]


@pytest.mark.parametrize("E,d,h", SHAPES)
@pytest.mark.parametrize("wide", [False, True])
def test_one_read_set_equals_the_per_orientation_splits(E, d, h, wide):
    w1, w2 = synth.expert_weights(E, d, h, 11 + d, DEV)
    if wide:
        w1, w2 = _wide(w1, 5), _wide(w2, 6)
    both = _set(w1, w2, J.JANUS_W16_FWD | J.JANUS_W16_VJP)
    sep = _set(w1, w2, J.JANUS_W16_FWD)
    J.janus_expert_weights_f16(w1, w2, J.JANUS_W16_VJP, out=sep)
    torch.cuda.synchronize()
    assert torch.equal(both, sep)
    # a one-flag set leaves the other parts as they were (zeros here)
    fwd_only = _set(w1, w2, J.JANUS_W16_FWD)
    assert torch.count_nonzero(fwd_only).item() < torch.count_nonzero(both).item()


def _ragged_offsets(E, R, seed):
    g = np.random.default_rng(seed)
    cuts = np.sort(g.integers(0, R + 1, size=E - 1))
    return to_dev(np.concatenate([[0], cuts, [R]]).astype(np.int32))


@pytest.mark.parametrize("E,d,h,R", [(2, 264, 328, 1000), (3, 512, 256, 700)])
def test_mlp_calls_with_the_set_are_bit_identical(E, d, h, R):
    # R = 1000 over 2 experts puts the second GEMM on the FP16 path (>= the
    # library's rows-per-expert threshold), 700 over 3 keeps it on 3xTF32
    w1, w2 = synth.expert_weights(E, d, h, 21, DEV)
    offs = _ragged_offsets(E, R, 22)
    x = synth.normal((R, d), 23, DEV)
    g = synth.normal((R, d), 24, DEV)
    ident = torch.arange(R, dtype=torch.int32, device=DEV)
    x16, xs = J.janus_dispatch_split(x, ident, 1)
    g16, gs = J.janus_dispatch_split(g, ident, 1)
    ws = _set(w1, w2, J.JANUS_W16_FWD | J.JANUS_W16_VJP)
    y0, a0 = J.janus_expert_ffn_fwd_split(x16, xs, offs, w1, w2, want_act=True)
    y1, a1 = J.janus_expert_ffn_fwd_split(x16, xs, offs, w1, w2, want_act=True, weights16=ws)
    dx0 = J.janus_expert_ffn_vjp_split(g16, gs, offs, w1, w2, a0)
    dx1 = J.janus_expert_ffn_vjp_split(g16, gs, offs, w1, w2, a0, weights16=ws)
    # the packed forward: FP16 payload rows with a per-row scale
    p16 = x16[:R].contiguous()
    yp0, _ = J.janus_expert_ffn_fwd_packed(p16, xs, offs, w1, w2, mode=J.JANUS_FFN_3XTF32)
    yp1, _ = J.janus_expert_ffn_fwd_packed(p16, xs, offs, w1, w2, mode=J.JANUS_FFN_3XTF32, weights16=ws)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1) and torch.equal(a0, a1)
    assert torch.equal(dx0, dx1)
    assert torch.equal(yp0, yp1)
    assert torch.isfinite(y1).all().item() and torch.isfinite(dx1).all().item()


def test_set_launches_and_no_split_in_the_calls():
    E, d, h, R = 2, 264, 328, 1000
    w1, w2 = synth.expert_weights(E, d, h, 31, DEV)
    offs = _ragged_offsets(E, R, 32)
    x = synth.normal((R, d), 33, DEV)
    ident = torch.arange(R, dtype=torch.int32, device=DEV)
    x16, xs = J.janus_dispatch_split(x, ident, 1)
    ws = torch.zeros(J.janus_expert_weights_f16_size(E, d, h), dtype=torch.uint8, device=DEV)
    torch.cuda.synchronize()
    J.janus_trace_start(16)
    try:
        J.janus_expert_weights_f16(w1, w2, J.JANUS_W16_FWD | J.JANUS_W16_VJP, out=ws)
        J.janus_expert_weights_f16(w1, w2, J.JANUS_W16_VJP, out=ws)
        y, a = J.janus_expert_ffn_fwd_split(x16, xs, offs, w1, w2, want_act=True, weights16=ws)
        J.janus_expert_ffn_vjp_split(x16, xs, offs, w1, w2, a, weights16=ws)
        recs = J.janus_trace_records()
    finally:
        J.janus_trace_release()
    names = [n for n, _ in recs]
    assert names[:4] == ["w16_split both", "w16_split both", "w16_split rows", "w16_split rows"]
    assert not any(n.startswith("w16_split") for n in names[4:])
    assert names[4:] == ["tc_gemm x.W store f16x3", "act_split silu", "tc_gemm x.W store f16x3",
                         "tc_gemm x.W store f16x3", "act_split dsilu", "tc_gemm x.W store f16x3"]
