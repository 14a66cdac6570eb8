"""Pins for the oracle's expert MLP forward and input VJP (CPU only).

Expert MLP: paper review 'Breaking the Training Barrier of Billion-Parameter
Universal Machine Learning Interatomic Potentials', section 3.1 Table II (MLP
hidden size); read as bias-free Linear -> SiLU -> Linear.  Input VJP: same
page, section 3.3 (forces/stress by autodiff, conservative training).
The forward is pinned to NumPy/SciPy matmul + expit; the VJP to complex-step
and central finite differences of that pinned forward.
"""
import numpy as np
import scipy.special

import oracle
from element_routed_moe_b200 import synth


def _experts(E=5, d=16, h=24, seed=0):
    w1, w2 = synth.expert_weights(E, d, h, seed)
    return w1.numpy(), w2.numpy()


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _np_forward(xd, offsets, w1, w2, dtype=np.float64):
    y = np.zeros((xd.shape[0], w2.shape[2]), dtype)
    for e in range(w1.shape[0]):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            w1e = w1[e] if np.iscomplexobj(w1) else w1[e].astype(np.float64)
            w2e = w2[e] if np.iscomplexobj(w2) else w2[e].astype(np.float64)
            pre = xd[a:b].astype(dtype) @ w1e
            if np.iscomplexobj(pre):
                hh = pre / (1.0 + np.exp(-pre))
            else:
                hh = pre * scipy.special.expit(pre)
            y[a:b] = hh @ w2e
    return y


def test_ffn_forward_matches_numpy():
    counts = [7, 0, 33, 1, 19]                      # includes an empty expert
    offs = _offsets(counts)
    w1, w2 = _experts()
    xd = synth.normal((offs[-1], 16), 3).numpy()
    yd, act = oracle.expert_ffn_fwd(xd, offs, w1, w2, want_act=True)
    ref = _np_forward(xd, offs, w1, w2)
    np.testing.assert_allclose(yd, ref, rtol=2e-6, atol=1e-7)
    for e in range(5):
        a, b = offs[e], offs[e + 1]
        np.testing.assert_allclose(act[a:b], xd[a:b].astype(np.float64) @ w1[e], rtol=2e-6, atol=1e-7)


def test_ffn_identity_and_zero_experts():
    d = 12
    offs = _offsets([10, 6])
    eye = np.stack([np.eye(d, dtype=np.float32)] * 2)
    xd = synth.normal((16, d), 8).numpy()
    yd = oracle.expert_ffn_fwd(xd, offs, eye, eye)
    np.testing.assert_allclose(yd, xd * scipy.special.expit(xd.astype(np.float64)), rtol=1e-6)
    yz = oracle.expert_ffn_fwd(xd, offs, eye, np.zeros_like(eye))
    assert np.all(yz == 0.0)


def test_ffn_row_subset_equals_full():
    offs = _offsets([9, 4, 0, 12, 3])
    w1, w2 = _experts(seed=4)
    xd = synth.normal((offs[-1], 16), 9).numpy()
    gd = synth.normal((offs[-1], 16), 10).numpy()
    full = oracle.expert_ffn_fwd(xd, offs, w1, w2)
    rows = np.array([0, 8, 9, 13, 27, 25], np.int64)
    assert np.array_equal(oracle.expert_ffn_fwd(xd, offs, w1, w2, rows=rows), full[rows])
    vfull = oracle.expert_ffn_vjp(xd, gd, offs, w1, w2)
    assert np.array_equal(oracle.expert_ffn_vjp(xd, gd, offs, w1, w2, rows=rows), vfull[rows])


def test_ffn_vjp_complex_step_and_finite_differences():
    offs = _offsets([5, 3, 0, 6])
    E, d, h = 4, 10, 14
    w1, w2 = _experts(E, d, h, seed=6)
    R = offs[-1]
    xd = synth.normal((R, d), 1).numpy().astype(np.float64)
    gd = synth.normal((R, d), 2).numpy()
    dxd = oracle.expert_ffn_vjp(xd.astype(np.float32), gd, offs, w1, w2)
    g = np.random.default_rng(0)
    for _ in range(4):
        v = g.standard_normal((R, d))
        # complex step: d/dt <Y(x + t v), G> = Im(<Y(x + i h v), G>) / h, exact to rounding
        hcs = 1e-30
        ycs = _np_forward(xd + 1j * hcs * v, offs, w1, w2, np.complex128)
        dd_cs = np.sum(ycs.imag * gd) / hcs
        got = np.sum(dxd.astype(np.float64) * v)
        assert abs(got - dd_cs) <= 1e-6 * (abs(dd_cs) + 1e-3)
        # central difference in FP64, O(eps^2) truncation
        eps = 1e-6
        lp = np.sum(_np_forward(xd + eps * v, offs, w1, w2) * gd)
        lm = np.sum(_np_forward(xd - eps * v, offs, w1, w2) * gd)
        assert abs((lp - lm) / (2 * eps) - dd_cs) <= 1e-7 * (abs(dd_cs) + 1.0)


def test_layer_vjp_finite_differences():
    # whole layer: dX = combine(vjp(dispatch_w(G))) is the gradient of <Y(X), G>
    N, T, E, K, d, h = 40, 5, 6, 2, 8, 8
    gate = synth.gate_table(T, E, 1)
    types = synth.types_uniform(N, T, 2)
    w1, w2 = _experts(E, d, h, seed=3)
    x = synth.normal((N, d), 4).numpy()
    gy = synth.normal((N, d), 5).numpy()
    r = oracle.route(types, gate, K)
    gd = oracle.dispatch(gy, r["perm"], K, r["topk_weight"])
    xd = oracle.dispatch(x, r["perm"], K)
    dxd = oracle.expert_ffn_vjp(xd, gd, r["offsets"], w1, w2)
    dx = oracle.combine(dxd, r["slot_of"], K)

    def layer(xx):
        xdd = xx[r["perm"] // K]
        ydd = _np_forward(xdd, r["offsets"], w1, w2, np.complex128)
        w = r["topk_weight"].ravel()
        y = np.zeros((N, d), np.complex128)
        for s in range(N * K):
            y[s // K] += w[s] * ydd[r["slot_of"][s]]
        return np.sum(y * gy)

    v = np.random.default_rng(1).standard_normal((N, d))
    dd = layer(x.astype(np.float64) + 1j * 1e-30 * v).imag / 1e-30
    got = np.sum(dx.astype(np.float64) * v)
    assert abs(got - dd) <= 1e-6 * abs(dd)


def test_weight_grad_complex_step():
    # d/dt <Y(W + t V), G> = <dW, V>: complex step through the pinned forward
    counts = [6, 0, 9, 4]
    offs = _offsets(counts)
    E, d, h = 4, 8, 12
    w1, w2 = _experts(E, d, h, seed=12)
    R = offs[-1]
    xd = synth.normal((R, d), 13).numpy()
    gd = synth.normal((R, d), 14).numpy()
    dw1, dw2 = oracle.expert_ffn_weight_grad(xd, gd, offs, w1, w2)
    assert np.all(dw1[1] == 0) and np.all(dw2[1] == 0)        # expert without rows
    g = np.random.default_rng(5)
    for _ in range(3):
        v1 = g.standard_normal(w1.shape)
        v2 = g.standard_normal(w2.shape)
        hcs = 1e-30
        y1 = _np_forward(xd.astype(np.complex128), offs, w1 + 1j * hcs * v1, w2, np.complex128)
        y2 = _np_forward(xd.astype(np.complex128), offs, w1, w2 + 1j * hcs * v2, np.complex128)
        d1 = np.sum(y1.imag * gd) / hcs
        d2 = np.sum(y2.imag * gd) / hcs
        assert abs(np.sum(dw1.astype(np.float64) * v1) - d1) <= 1e-6 * abs(d1)
        assert abs(np.sum(dw2.astype(np.float64) * v2) - d2) <= 1e-6 * abs(d2)


def test_weight_grad_dw2_is_numpy_outer_sum():
    counts = [5, 7]
    offs = _offsets(counts)
    w1, w2 = _experts(2, 6, 10, seed=21)
    xd = synth.normal((12, 6), 22).numpy()
    gd = synth.normal((12, 6), 23).numpy()
    _, dw2 = oracle.expert_ffn_weight_grad(xd, gd, offs, w1, w2)
    for e in range(2):
        a, b = offs[e], offs[e + 1]
        pre = xd[a:b].astype(np.float64) @ w1[e]
        hh = pre * scipy.special.expit(pre)
        np.testing.assert_allclose(dw2[e], hh.T @ gd[a:b].astype(np.float64), rtol=1e-6, atol=1e-7)
