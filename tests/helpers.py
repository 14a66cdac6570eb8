"""Shared helpers for the GPU parity tests (test infrastructure)."""
import numpy as np
import torch

import oracle
from element_routed_moe_b200 import synth

DEV = "cuda:0"

# Tolerances (relative Frobenius error) stated by the layer's contract:
# FP32 paths <= 1e-5, FP16-packed dispatch path <= 2e-3.
TOL_FP32 = 1e-5
TOL_FP16_PATH = 2e-3
# Gate weights: CUDA exp vs the host's exp may differ by an ulp before rounding.
TOL_WEIGHT = 1e-6


def rel_fro(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    return float(num / den) if den > 0 else float(num)


def max_row_rel(got, ref) -> float:
    """Largest per-row relative error ||got_i - ref_i|| / ||ref_i|| (a local
    error that a norm over many rows would hide)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.linalg.norm(got - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    return float(np.max(np.where(den > 0, num / np.where(den > 0, den, 1.0), num)))


# Per-row bound for the full-size sampled comparisons: the relative Frobenius
# bar over the sample stays TOL_FP32, and no single row may be off by more
# than ten times that.
TOL_ROW = 1e-4


def to_dev(a, dtype=None):
    t = torch.as_tensor(a)
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().to(DEV)


def host(t):
    return t.detach().cpu().numpy()


def poison_like(shape, dtype):
    """Output buffer pre-filled with NaN (float) / 0x7fffffff (int) so that a
    row the kernel forgets to write is caught."""
    if dtype == torch.float32:
        return torch.full(shape, float("nan"), dtype=dtype, device=DEV)
    if dtype == torch.float16:
        return torch.full(shape, float("nan"), dtype=dtype, device=DEV)
    return torch.full(shape, 0x7fffffff, dtype=dtype, device=DEV)


def small_layer(N, T, E, K, d, h, seed=0, zipf=True):
    """A layer small enough for the full oracle, as host arrays."""
    types = synth.types_zipf(N, T, seed=seed + 1) if zipf else synth.types_uniform(N, T, seed + 1)
    gate = synth.gate_table(T, E, seed + 2)
    w1, w2 = synth.expert_weights(E, d, h, seed + 3)
    x = synth.normal((N, d), seed + 4).numpy()
    g = synth.normal((N, d), seed + 5).numpy()
    return dict(types=types, gate=gate, w1=w1.numpy(), w2=w2.numpy(), x=x, g=g)


def sample_rows(offsets, n_random, seed, R):
    """Seeded row sample for full-size FFN parity: first and last rows of the
    smallest and the largest non-empty expert, plus n_random uniform rows."""
    offsets = np.asarray(offsets)
    cnt = np.diff(offsets)
    nz = np.nonzero(cnt)[0]
    picks = []
    for e in (nz[np.argmin(cnt[nz])], nz[np.argmax(cnt[nz])]):
        a, b = offsets[e], offsets[e + 1]
        picks += [a, min(a + 1, b - 1), b - 1]
    rnd = np.random.default_rng(seed).integers(0, R, n_random)
    return np.unique(np.concatenate([np.array(picks, np.int64), rnd.astype(np.int64)]))


def oracle_route(types, gate, K):
    return oracle.route(types, gate, K)
