"""GPU tests of the expert MLP's FP16 tensor path on split rows.

janus_dispatch_split writes each dispatch row as two binary16 terms with a
per-row power-of-two scale; janus_expert_ffn_fwd_split / _vjp_split run the
first GEMM of each direction on the tcgen05 kind::f16 path (three products
against a two-term FP16 split of the weights) and the second on 3xTF32, or,
in the forward above the library's rows-per-expert threshold, on the same FP16 path
(paper review 'Breaking the Training Barrier of Billion-Parameter Universal
Machine Learning Interatomic Potentials', section 3.1 Table II and section 3.3:
the expert MLP and its input gradient, FP32-accurate).

* the split dispatch is checked bit for bit against its definition computed
  with NumPy's float32 arithmetic and float16 casts (round to nearest even),
  and the two terms rebuild the FP32 rows within 2^-21 of each row's maximum;
* the forward and the input VJP match the oracle within 1e-5 (relative
  Frobenius) with no row off by more than 1e-4, and the 3xTF32 forms of the
  same calls within the same bounds, on ragged, multi-tile, K-tail and
  narrow shapes, and on rows and weights with wide dynamic ranges.
"""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, TOL_ROW, host, max_row_rel, rel_fro, sample_rows, to_dev

pytestmark = pytest.mark.gpu


def _expected_split(x, perm, K, w=None):
    """hi, mid planes and row scales by the definition (NumPy float32/float16)."""
    x = np.asarray(x, np.float32)
    rowmax = np.abs(x).max(axis=1)
    atoms = perm // K
    v = x[atoms]
    bound = rowmax[atoms]
    if w is not None:
        wk = np.asarray(w, np.float32).reshape(-1)[perm]
        v = v * wk[:, None]
        bound = (np.abs(wk) * bound).astype(np.float32)
    b = (bound.view(np.uint32) >> 23).astype(np.int64)
    e = np.where(bound == 0, 0, np.clip(141 - np.maximum(b, 1), -126, 126))
    S = np.ldexp(np.float32(1.0), e).astype(np.float32)
    t = (v * S[:, None]).astype(np.float32)
    hi = t.astype(np.float16)
    mid = (t - hi.astype(np.float32)).astype(np.float16)
    return hi, mid, (np.float32(1.0) / S).astype(np.float32)


@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("shape", [(300, 9, 12, 3, 20), (129, 5, 40, 33, 136), (64, 3, 4, 4, 1544)])
def test_dispatch_split_is_its_definition(shape, weighted):
    N, T, E, K, d = shape
    types = to_dev(synth.types_zipf(N, T, seed=1))
    gate = to_dev(synth.gate_table(T, E, 2))
    r = J.janus_route(types, gate, K)
    x = synth.normal((N, d), 3, DEV)
    x[5] *= 1.0e-20                 # rows of very different magnitudes
    x[7] *= 1.0e20
    x[11] = 0.0
    w = r["topk_weight"] if weighted else None
    rows16, scale = J.janus_dispatch_split(x, r["slot_of"], K, w)
    torch.cuda.synchronize()
    R = N * K
    hi, mid, sc = _expected_split(host(x), host(r["perm"]), K, None if w is None else host(w))
    got = host(rows16)
    assert np.array_equal(got[:R].view(np.uint16), hi.view(np.uint16))
    assert np.array_equal(got[R:].view(np.uint16), mid.view(np.uint16))
    assert np.array_equal(host(scale), sc)
    # the two terms rebuild the FP32 rows within 2^-21 of each row's largest value
    ref = oracle.dispatch(host(x), host(r["perm"]), K, None if w is None else host(w)).astype(np.float64)
    rebuilt = (got[:R].astype(np.float64) + got[R:].astype(np.float64)) * host(scale).astype(np.float64)[:, None]
    bound = np.abs(ref).max(axis=1, keepdims=True) * 2.0 ** -21
    assert np.all(np.abs(rebuilt - ref) <= bound)


SHAPES = {
    # name: (counts per expert, d, h)
    "ragged": ([37, 0, 300, 1, 129, 200], 136, 68),
    "multi_tile": ([700, 900, 400], 512, 384),
    "k_tail": ([300, 257], 1544, 200),
    "narrow": ([5, 3, 260], 8, 4),
    # above the rows-per-expert threshold, h % 8 == 0: the forward's second GEMM on the
    # FP16 path too (K = h = 200: three 64-wide blocks and an 8-wide tail)
    "second_f16": ([3000, 0, 3300], 136, 200),
    # rows of more than 4096 values: the activation and weight-row splits
    # take their two-sweep kernel
    "long_rows": ([2100], 16, 4104),
}


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _split_rows(xd):
    """Split FP32 dispatch rows (in place of a dispatch: K = 1, identity order)."""
    R = xd.shape[0]
    ident = torch.arange(R, dtype=torch.int32, device=DEV)
    return J.janus_dispatch_split(xd, ident, 1)


@pytest.mark.parametrize("name", list(SHAPES))
def test_split_forward_and_vjp_match_the_oracle(name):
    counts, d, h = SHAPES[name]
    E = len(counts)
    offs = _offsets(counts)
    R = int(offs[-1])
    w1, w2 = synth.expert_weights(E, d, h, 5, DEV)
    xd = synth.normal((R, d), 6, DEV)
    gd = synth.normal((R, d), 7, DEV)
    xd[3] *= 1.0e-12                 # rows far apart in magnitude
    gd[4] *= 1.0e9
    o = to_dev(offs)
    x16, xs = _split_rows(xd)
    g16, gs = _split_rows(gd)
    yd, act = J.janus_expert_ffn_fwd_split(x16, xs, o, w1, w2, want_act=True)
    nb = J.janus_expert_ffn_split_workspace_size(R, E, d, h)
    ws = torch.zeros(nb, dtype=torch.uint8, device=DEV)
    dxd = J.janus_expert_ffn_vjp_split(g16, gs, o, w1, w2, act, workspace=ws)
    J.janus_check(ws)
    ref_y, ref_a = oracle.expert_ffn_fwd(host(xd), offs, host(w1), host(w2), want_act=True)
    ref_dx = oracle.expert_ffn_vjp(host(xd), host(gd), offs, host(w1), host(w2))
    for got, ref in ((act, ref_a), (yd, ref_y), (dxd, ref_dx)):
        g = host(got)
        assert rel_fro(g, ref) <= TOL_FP32
        assert max_row_rel(g, ref) <= TOL_ROW
    # the 3xTF32 forms of the same calls agree within the same bounds
    y3, a3 = J.janus_expert_ffn_fwd(xd, o, w1, w2, mode=J.JANUS_FFN_3XTF32, want_act=True)
    dx3 = J.janus_expert_ffn_vjp(xd, gd, o, w1, w2, act=a3, mode=J.JANUS_FFN_3XTF32)
    assert rel_fro(host(yd), host(y3)) <= TOL_FP32 and rel_fro(host(dxd), host(dx3)) <= TOL_FP32


def test_split_forward_full_size_sampled_rows():
    # the MatRIS-MoE(S)-shaped layer's expert MLP at full size (R = 32,768,
    # d = h = 2560, 72 Zipf-loaded experts), sampled rows against the oracle
    cfg = synth.CONFIGS["S"]
    types = synth.types_zipf(cfg.n_atoms, cfg.n_types, seed=1)
    gate = synth.gate_table(cfg.n_types, cfg.n_experts, 2)
    r = oracle.route(types, gate, cfg.top_k)
    offs = r["offsets"]
    R = cfg.n_rows
    w1, w2 = synth.expert_weights(cfg.n_experts, cfg.d, cfg.h, 3, DEV)
    xd = synth.normal((R, cfg.d), 4, DEV)
    gd = synth.normal((R, cfg.d), 5, DEV)
    o = to_dev(offs)
    x16, xs = _split_rows(xd)
    g16, gs = _split_rows(gd)
    yd, act = J.janus_expert_ffn_fwd_split(x16, xs, o, w1, w2, want_act=True)
    dxd = J.janus_expert_ffn_vjp_split(g16, gs, o, w1, w2, act)
    torch.cuda.synchronize()
    rows = sample_rows(offs, 160, seed=7, R=R)
    hw1, hw2 = host(w1), host(w2)
    ref_y = oracle.expert_ffn_fwd(host(xd), offs, hw1, hw2, rows=rows)
    ref_dx = oracle.expert_ffn_vjp(host(xd), host(gd), offs, hw1, hw2, rows=rows)
    assert rel_fro(host(yd)[rows], ref_y) <= TOL_FP32 and max_row_rel(host(yd)[rows], ref_y) <= TOL_ROW
    assert rel_fro(host(dxd)[rows], ref_dx) <= TOL_FP32 and max_row_rel(host(dxd)[rows], ref_dx) <= TOL_ROW
    assert torch.isfinite(yd).all().item() and torch.isfinite(dxd).all().item()


def test_fp16_second_gemms_handle_wide_ranges():
    # above the rows-per-expert threshold both second GEMMs run on FP16: H W2 with W2
    # split per output feature d, dA W1^T with W1 split per output feature d
    # (a row of W1[e]).  Output features whose weights are 10^6 or 10^-30
    # times the rest, or all zero, stay within the FP32 tolerance column by
    # column; so do rows of the upstream gradient 10^9 times the rest
    counts, d, h = [2100, 0, 2200, 2000], 128, 96
    E = len(counts)
    offs = _offsets(counts)
    R = int(offs[-1])
    w1, w2 = synth.expert_weights(E, d, h, 15, DEV)
    w2[:, :, 3] *= 1.0e6
    w2[:, :, 5] = 0.0
    w2[:, :, 9] *= 1.0e-30
    w1[:, 7, :] *= 1.0e6
    w1[:, 11, :] = 0.0
    w1[:, 13, :] *= 1.0e-30
    xd = synth.normal((R, d), 16, DEV)
    gd = synth.normal((R, d), 17, DEV)
    gd[40] *= 1.0e9
    o = to_dev(offs)
    x16, xs = _split_rows(xd)
    g16, gs = _split_rows(gd)
    nb = J.janus_expert_ffn_split_workspace_size(R, E, d, h)
    ws = torch.zeros(nb, dtype=torch.uint8, device=DEV)
    yd, act = J.janus_expert_ffn_fwd_split(x16, xs, o, w1, w2, want_act=True, workspace=ws)
    J.janus_check(ws)
    dxd = J.janus_expert_ffn_vjp_split(g16, gs, o, w1, w2, act, workspace=ws)
    J.janus_check(ws)
    hw1, hw2 = host(w1), host(w2)
    ref_y = oracle.expert_ffn_fwd(host(xd), offs, hw1, hw2)
    ref_dx = oracle.expert_ffn_vjp(host(xd), host(gd), offs, hw1, hw2)
    hy, hdx = host(yd).astype(np.float64), host(dxd).astype(np.float64)
    for got, ref, cols, zero in ((hy, ref_y, (0, 3, 9, 40), 5), (hdx, ref_dx, (0, 7, 13, 40), 11)):
        for f in cols:
            col, rc = got[:, f], ref[:, f].astype(np.float64)
            assert np.linalg.norm(col - rc) <= TOL_FP32 * np.linalg.norm(rc), f
        assert np.all(got[:, zero] == 0.0)
    assert max_row_rel(host(dxd), ref_dx) <= TOL_ROW and max_row_rel(host(yd), ref_y) <= TOL_ROW


@pytest.mark.parametrize("name", ["ragged", "second_f16"])
def test_split_calls_store_through_a_row_table(name):
    # the same results, row p stored at the address table[p] (the expert-
    # parallel return); second_f16 stores from the FP16 second GEMMs
    counts, d, h = SHAPES[name]
    E = len(counts)
    offs = _offsets(counts)
    R = int(offs[-1])
    w1, w2 = synth.expert_weights(E, d, h, 25, DEV)
    xd = synth.normal((R, d), 26, DEV)
    gd = synth.normal((R, d), 27, DEV)
    o = to_dev(offs)
    x16, xs = _split_rows(xd)
    g16, gs = _split_rows(gd)
    y_ref, act = J.janus_expert_ffn_fwd_split(x16, xs, o, w1, w2, want_act=True)
    dx_ref = J.janus_expert_ffn_vjp_split(g16, gs, o, w1, w2, act)
    slot = torch.as_tensor(np.random.default_rng(28).permutation(R + 3)[:R], device=DEV)
    dest_y = torch.full((R + 3, d), float("nan"), device=DEV)
    dest_dx = torch.full((R + 3, d), float("nan"), device=DEV)
    out, _ = J.janus_expert_ffn_fwd_split(x16, xs, o, w1, w2,
                                          out_rows=dest_y.data_ptr() + 4 * d * slot.to(torch.int64))
    out2 = J.janus_expert_ffn_vjp_split(g16, gs, o, w1, w2, act,
                                        out_rows=dest_dx.data_ptr() + 4 * d * slot.to(torch.int64))
    torch.cuda.synchronize()
    assert out is None and out2 is None
    assert torch.equal(dest_y[slot], y_ref) and torch.equal(dest_dx[slot], dx_ref)


def test_split_calls_check_their_arguments():
    E, d, h = 3, 12, 8                              # d % 8 != 0
    offs = to_dev(_offsets([10, 0, 6]))
    w1, w2 = synth.expert_weights(E, d, h, 9, DEV)
    x16 = torch.zeros((32, d), dtype=torch.float16, device=DEV)
    xs = torch.ones((16,), device=DEV)
    with pytest.raises(J.JanusError) as e:
        J.janus_expert_ffn_fwd_split(x16, xs, offs, w1, w2)
    assert e.value.status == J.JANUS_ERR_MISALIGNED
