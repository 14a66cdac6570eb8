"""Pins for the oracle's per-element-type FP16 packing (CPU only).

Atom-type-aware FP16 compression: paper review 'Breaking the Training Barrier
of Billion-Parameter Universal Machine Learning Interatomic Potentials',
section 3.5 (CNIS): dispatch-buffer tokens grouped by atom type, one scale per
type, FP16 on the wire, dequantised afterwards, half the FP32 volume.
The binary16 conversion is pinned to NumPy's float64 -> float16 cast.
"""
import json
import os

import numpy as np
import pytest

import oracle
from element_routed_moe_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "table2_shapes.json")


def _special_values():
    v = [0.0, -0.0, 1.0, -1.0, 65504.0, -65504.0, 65519.99, 2.0 ** -14, 2.0 ** -24,
         2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -24 * 1.5, 2.0 ** -24 * 2.5, 1.0 + 2.0 ** -11,
         1.0 + 3 * 2.0 ** -11, 2048.0 + 1.0, 2048.0 + 3.0, 0.1, 1e-8, 6.1e-5, 6.09e-5,
         32768.0 + 16.0, 32768.0 + 48.0, 1024.5, 1025.5]
    return np.array(v, np.float64)


def test_fp16_conversion_matches_numpy():
    g = np.random.default_rng(0)
    xs = np.concatenate([
        _special_values(),
        g.standard_normal(20000) * 1000.0,
        g.standard_normal(20000) * 1e-5,          # subnormal region
        (g.integers(-60000, 60000, 5000) + 0.5),  # ties at integer halves
        np.ldexp(g.integers(1024, 2048, 5000) + 0.5, g.integers(-24, 5, 5000)),  # exact ties
    ])
    xs = xs[np.abs(xs) <= 65504.0]
    ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle.fp16_from_double(x) for x in xs], np.uint16)
    assert np.array_equal(got, ref)
    back = np.array([oracle.fp16_to_double(b) for b in ref])
    assert np.array_equal(back, ref.view(np.float16).astype(np.float64))


def _quant_case(N=400, T=13, E=10, K=3, d=24, seed=0, scale_by_type=True):
    types = synth.types_zipf(N, T, seed=seed + 1)
    gate = synth.gate_table(T, E, seed + 2)
    x = synth.normal((N, d), seed + 3).numpy()
    if scale_by_type:   # very different magnitudes per type
        x = x * (10.0 ** (types[:, None] % 7 - 3)).astype(np.float32)
    r = oracle.route(types, gate, K)
    return x, types, T, r, K


def test_quant_matches_numpy_cast_and_bounds():
    x, types, T, r, K = _quant_case()
    payload, scale = oracle.quant_by_type(x, types, T, r["perm"], K)
    rows = r["perm"] // K
    rt = types[rows]
    # payload bits == NumPy float16 cast of x / scale (exact power-of-two division)
    ref = (x[rows].astype(np.float64) / scale[rt][:, None].astype(np.float64)).astype(np.float16)
    assert np.array_equal(payload, ref.view(np.uint16))
    # scales are powers of two; amax lands in the upper binade(s) of FP16
    m, _ = np.frexp(scale)
    assert np.all(m == 0.5)
    for t in range(T):
        sel = types == t
        if not sel.any():
            assert scale[t] == 1.0
            continue
        amax = np.abs(x[sel]).max()
        q = amax / scale[t]
        assert 32752.0 < q <= 65504.0, (t, q)
        assert amax / (scale[t] / 2) > 65504.0      # smallest such power of two
    # no overflow, and the half-ulp error bound
    q16 = payload.view(np.float16)
    assert np.all(np.isfinite(q16)) and np.all(np.abs(q16.astype(np.float64)) <= 65504.0)
    deq = q16.astype(np.float64) * scale[rt][:, None]
    ulp = np.spacing(np.abs(q16)).astype(np.float64)
    err = np.abs(x[rows].astype(np.float64) - deq)
    assert np.all(err <= 0.5 * ulp * scale[rt][:, None])


def test_dequant_is_exact_numpy():
    x, types, T, r, K = _quant_case(seed=7)
    payload, scale = oracle.quant_by_type(x, types, T, r["perm"], K)
    xd = oracle.dequant_by_type(payload, types, r["perm"], K, scale)
    rt = types[r["perm"] // K]
    ref = (payload.view(np.float16).astype(np.float32) * scale[rt][:, None])
    assert np.array_equal(xd, ref)


def test_quant_relative_error_and_payload_size():
    x, types, T, r, K = _quant_case(scale_by_type=False, seed=3)
    payload, scale = oracle.quant_by_type(x, types, T, r["perm"], K)
    xd = oracle.dequant_by_type(payload, types, r["perm"], K, scale)
    ref = x[r["perm"] // K].astype(np.float64)
    rel = np.linalg.norm(xd - ref) / np.linalg.norm(ref)
    assert rel < 2e-3
    with open(GOLD) as f:
        frac = json.load(f)["fp16_payload_fraction"]["value"]
    assert payload.nbytes == frac * ref.astype(np.float32).nbytes


def test_quant_degenerate_scales():
    T, K, d = 3, 1, 8
    types = np.array([0, 0, 2, 2], np.int32)
    x = np.zeros((4, d), np.float32)
    x[2:] = np.float32(1e-40)             # FP32 subnormal amax
    perm = np.arange(4, dtype=np.int32)
    payload, scale = oracle.quant_by_type(x, types, T, perm, K)
    assert scale[0] == 1.0 and scale[1] == 1.0        # zero / absent type
    assert scale[2] == np.float32(2.0 ** -126)        # exponent clamped to normal range
    assert np.all(payload[:2] == 0)
    big = np.full((4, d), 3.0e38, np.float32)
    payload, scale = oracle.quant_by_type(big, types, T, perm, K)
    assert np.isfinite(scale[0]) and np.all(np.isfinite(payload.view(np.float16)))
    bad = np.zeros((4, d), np.float32)
    bad[1, 3] = np.inf
    with pytest.raises(ValueError):
        oracle.quant_by_type(bad, types, T, perm, K)
