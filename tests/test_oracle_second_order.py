"""Pins for the oracle's second-order pass (CPU only): the VJP of the expert
MLP's input VJP, which force training differentiates (paper review 'Breaking
the Training Barrier of Billion-Parameter Universal Machine Learning
Interatomic Potentials', section 3.3: forces are energy gradients fitted by a
loss, so the loss gradient flows back through the input VJP).

Every expected value comes from NumPy evaluations of the forward pass
(pinned to matmul + expit in test_oracle_ffn.py):
  * a complex-step derivative of a NumPy input VJP, which is itself checked
    here against the complex step of the forward;
  * an independent mixed second derivative of the forward (complex step in one
    direction, a 4-point central difference in the other);
  * the symmetry of the Hessian, and exact zeros when the upstream gradient is 0.
"""
import numpy as np
import pytest

import oracle
from element_routed_moe_b200 import synth


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _setup(counts=(5, 0, 7, 3), d=8, h=12, seed=0):
    offs = _offsets(counts)
    E, R = len(counts), int(offs[-1])
    w1, w2 = synth.expert_weights(E, d, h, seed)
    x = synth.normal((R, d), seed + 1).numpy()
    g = synth.normal((R, d), seed + 2).numpy()
    v = synth.normal((R, d), seed + 3).numpy()
    return offs, w1.numpy(), w2.numpy(), x, g, v


def _sig(z):
    return 1.0 / (1.0 + np.exp(-z))


def _np_forward(x, offs, w1, w2):
    """y = silu(x W1[e]) W2[e] per expert segment, complex-safe."""
    dt = np.result_type(x, w1, w2, np.float64)
    x, w1, w2 = x.astype(dt), w1.astype(dt), w2.astype(dt)
    y = np.zeros((x.shape[0], w2.shape[2]), dt)
    for e in range(w1.shape[0]):
        a, b = offs[e], offs[e + 1]
        if b > a:
            pre = x[a:b] @ w1[e]
            y[a:b] = (pre * _sig(pre)) @ w2[e]
    return y


def _np_vjp(x, g, offs, w1, w2):
    """Input VJP written from the chain rule: dx = ((g W2^T) * silu'(a)) W1^T."""
    dt = np.result_type(x, g, w1, w2, np.float64)
    x, g, w1, w2 = x.astype(dt), g.astype(dt), w1.astype(dt), w2.astype(dt)
    dx = np.zeros(x.shape, dt)
    for e in range(w1.shape[0]):
        a, b = offs[e], offs[e + 1]
        if b > a:
            pre = x[a:b] @ w1[e]
            s = _sig(pre)
            dx[a:b] = ((g[a:b] @ w2[e].T) * s * (1.0 + pre * (1.0 - s))) @ w1[e].T
    return dx


H_CS = 1e-30


def _cs(fn, base, direction):
    """d/dt fn(base + t direction) at 0 by complex step (exact to rounding)."""
    return np.imag(fn(base.astype(np.complex128) + 1j * H_CS * direction)) / H_CS


def test_numpy_vjp_matches_forward_complex_step():
    offs, w1, w2, x, g, _ = _setup(seed=30)
    x64 = x.astype(np.float64)
    dx = _np_vjp(x64, g, offs, w1, w2)
    rng = np.random.default_rng(0)
    for _ in range(3):
        dirn = rng.standard_normal(x.shape)
        ref = _cs(lambda z: np.sum(_np_forward(z, offs, w1, w2) * g), x64, dirn)
        assert abs(np.sum(dx * dirn) - ref) <= 1e-12 * (abs(ref) + 1.0)


def test_second_order_input_and_upstream_gradients_complex_step():
    offs, w1, w2, x, g, v = _setup(seed=40)
    d_x, d_g = oracle.expert_ffn_vjp_vjp(x, g, v, offs, w1, w2)
    x64, g64 = x.astype(np.float64), g.astype(np.float64)
    rng = np.random.default_rng(1)
    for _ in range(4):
        dirn = rng.standard_normal(x.shape)
        ref_x = _cs(lambda z: np.sum(_np_vjp(z, g64, offs, w1, w2) * v), x64, dirn)
        ref_g = _cs(lambda z: np.sum(_np_vjp(x64, z, offs, w1, w2) * v), g64, dirn)
        assert abs(np.sum(d_x.astype(np.float64) * dirn) - ref_x) <= 1e-6 * (abs(ref_x) + 1e-3)
        assert abs(np.sum(d_g.astype(np.float64) * dirn) - ref_g) <= 1e-6 * (abs(ref_g) + 1e-3)


def test_second_order_weight_gradients_complex_step():
    offs, w1, w2, x, g, v = _setup(seed=50)
    dw1, dw2 = oracle.expert_ffn_vjp_vjp_weight_grad(x, g, v, offs, w1, w2)
    assert np.all(dw1[1] == 0) and np.all(dw2[1] == 0)          # expert without rows
    x64, g64 = x.astype(np.float64), g.astype(np.float64)
    rng = np.random.default_rng(2)
    for _ in range(3):
        v1 = rng.standard_normal(w1.shape)
        v2 = rng.standard_normal(w2.shape)
        r1 = _cs(lambda z: np.sum(_np_vjp(x64, g64, offs, z, w2) * v), w1.astype(np.float64), v1)
        r2 = _cs(lambda z: np.sum(_np_vjp(x64, g64, offs, w1, z) * v), w2.astype(np.float64), v2)
        assert abs(np.sum(dw1.astype(np.float64) * v1) - r1) <= 1e-6 * (abs(r1) + 1e-3)
        assert abs(np.sum(dw2.astype(np.float64) * v2) - r2) <= 1e-6 * (abs(r2) + 1e-3)


def test_second_order_is_a_mixed_second_derivative_of_the_forward():
    # <d_x, w> = d/dt d/ds <Y(x + s v + t w), g>: complex step in s, 4-point
    # central difference in t (truncation O(eps^4)); no VJP formula involved
    offs, w1, w2, x, g, v = _setup(seed=60)
    d_x, _ = oracle.expert_ffn_vjp_vjp(x, g, v, offs, w1, w2)
    x64 = x.astype(np.float64)
    w = np.random.default_rng(3).standard_normal(x.shape)

    def first(t):
        return _cs(lambda z: np.sum(_np_forward(z, offs, w1, w2) * g), x64 + t * w, v.astype(np.float64))

    eps = 1e-3
    ref = (-first(2 * eps) + 8 * first(eps) - 8 * first(-eps) + first(-2 * eps)) / (12 * eps)
    assert abs(np.sum(d_x.astype(np.float64) * w) - ref) <= 1e-6 * (abs(ref) + 1e-3)


def test_hessian_symmetry():
    # d_x(v) = H v with H the Hessian of <Y(x), g>: <H v, w> = <H w, v>
    offs, w1, w2, x, g, v = _setup(seed=70)
    w = synth.normal(x.shape, 71).numpy()
    hv, _ = oracle.expert_ffn_vjp_vjp(x, g, v, offs, w1, w2)
    hw, _ = oracle.expert_ffn_vjp_vjp(x, g, w, offs, w1, w2)
    lhs = np.sum(hv.astype(np.float64) * w)
    rhs = np.sum(hw.astype(np.float64) * v)
    assert abs(lhs - rhs) <= 1e-6 * (abs(lhs) + 1e-3)


def test_zero_upstream_gradient_zeroes_the_x_and_weight_terms():
    # g = 0 -> dh = 0 -> u = t2 = 0: d_x, dW1 and dW2 vanish; d_g does not
    offs, w1, w2, x, _, v = _setup(seed=80)
    g = np.zeros_like(x)
    d_x, d_g = oracle.expert_ffn_vjp_vjp(x, g, v, offs, w1, w2)
    dw1, dw2 = oracle.expert_ffn_vjp_vjp_weight_grad(x, g, v, offs, w1, w2)
    assert np.all(d_x == 0) and np.all(dw1 == 0) and np.all(dw2 == 0)
    assert np.any(d_g != 0)
    # and the cotangent v = 0 zeroes everything
    d_x0, d_g0 = oracle.expert_ffn_vjp_vjp(x, synth.normal(x.shape, 81).numpy(), np.zeros_like(x), offs, w1, w2)
    assert np.all(d_x0 == 0) and np.all(d_g0 == 0)


def test_row_subset_equals_full():
    offs, w1, w2, x, g, v = _setup(counts=(9, 4, 0, 12, 3), seed=90)
    fx, fg = oracle.expert_ffn_vjp_vjp(x, g, v, offs, w1, w2)
    rows = np.array([0, 8, 9, 13, 27, 25], np.int64)
    sx, sg = oracle.expert_ffn_vjp_vjp(x, g, v, offs, w1, w2, rows=rows)
    assert np.array_equal(sx, fx[rows]) and np.array_equal(sg, fg[rows])


@pytest.mark.parametrize("d,h", [(1, 1), (3, 17)])
def test_odd_sizes(d, h):
    offs, w1, w2, x, g, v = _setup(counts=(2, 1), d=d, h=h, seed=100)
    d_x, d_g = oracle.expert_ffn_vjp_vjp(x, g, v, offs, w1, w2)
    x64 = x.astype(np.float64)
    dirn = np.ones(x.shape)
    ref = _cs(lambda z: np.sum(_np_vjp(z, g.astype(np.float64), offs, w1, w2) * v), x64, dirn)
    assert abs(np.sum(d_x.astype(np.float64)) - ref) <= 1e-6 * (abs(ref) + 1e-3)
