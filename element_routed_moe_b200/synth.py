"""Seeded synthetic inputs for the element-routed MoE layer and edge aggregation.

This module only draws inputs; it holds none of the layer's arithmetic.  Both
the CUDA path and the CPU oracle are fed from the same arrays it returns.

Recipe (shapes from the model table, Table II, of the paper review
"Breaking the Training Barrier of Billion-Parameter Universal Machine Learning
Interatomic Potentials"):

* element types: uniform over T (tiny layer) or Zipf(s=1.1) over T=89, type
  id = rank - 1, drawn by inverse CDF (type 0 is the most frequent, ~24 %);
* gate table [T,E] ~ N(0,1); expert weights W1 [E,d,h], W2 [E,h,d] ~ N(0,1/d);
* node features, upstream gradients, edge messages ~ N(0,1), FP32;
* edges: tiny layer, ``per_atom * N`` receivers uniform on [0,N); periodic
  layers, atoms iid uniform in a cubic cell of side (N/rho)^(1/3) at
  rho = 0.08 atoms/A^3, every ordered pair i != j within a 6 A minimum-image
  cutoff (~72 neighbours per atom), sorted by (receiver, sender) into a CSR
  with an int64 row pointer.

Small arrays are drawn with NumPy's PCG64 (``np.random.default_rng(seed)``);
the large dense tensors (weights, features, messages) with a seeded
``torch.Generator`` on the device that will hold them, so a multi-GB layer is
generated where it lives.  Tests copy whatever they hand the oracle back to
the host, so the two sides always see identical bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


# --------------------------------------------------------------------------
# layer configurations (the five layers of the benchmark table)
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class LayerConfig:
    name: str
    n_atoms: int
    n_types: int
    n_experts: int
    top_k: int
    d: int
    h: int
    type_dist: str          # "uniform" | "zipf"
    edges: str              # "none" | "random" | "pbc"
    edges_per_atom: int = 16
    vjp: bool = True
    quant: bool = False

    @property
    def n_rows(self) -> int:
        return self.n_atoms * self.top_k


CONFIGS = {
    "tiny": LayerConfig("tiny", 512, 8, 8, 2, 64, 64, "uniform", "random", vjp=False),
    "S": LayerConfig("S", 8192, 89, 72, 4, 2560, 2560, "zipf", "none"),
    "M": LayerConfig("M", 32768, 89, 40, 8, 1536, 1536, "zipf", "none", quant=True),
    "L": LayerConfig("L", 16384, 89, 72, 16, 1920, 1920, "zipf", "pbc"),
    "slice": LayerConfig("slice", 65536, 89, 40, 8, 1536, 1536, "zipf", "pbc", quant=True),
}

PBC_DENSITY = 0.08   # atoms / A^3
PBC_CUTOFF = 6.0     # A
ZIPF_S = 1.1


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def torch_gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


# --------------------------------------------------------------------------
# element types and gate table
# --------------------------------------------------------------------------
def types_uniform(n: int, n_types: int, seed: int) -> np.ndarray:
    return rng(seed).integers(0, n_types, size=n, dtype=np.int64).astype(np.int32)


def types_zipf(n: int, n_types: int = 89, s: float = ZIPF_S, seed: int = 0) -> np.ndarray:
    ranks = np.arange(1, n_types + 1, dtype=np.float64)
    p = ranks ** (-s)
    cdf = np.cumsum(p / p.sum())
    cdf[-1] = 1.0
    u = rng(seed).random(n)
    return np.searchsorted(cdf, u, side="right").clip(0, n_types - 1).astype(np.int32)


def gate_table(n_types: int, n_experts: int, seed: int) -> np.ndarray:
    return rng(seed).standard_normal((n_types, n_experts)).astype(np.float32)


# --------------------------------------------------------------------------
# dense tensors
# --------------------------------------------------------------------------
def normal(shape, seed: int, device="cpu", std: float = 1.0) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=torch_gen(seed, device))
    return t


def expert_weights(n_experts: int, d: int, h: int, seed: int, device="cpu"):
    std = 1.0 / math.sqrt(d)
    w1 = normal((n_experts, d, h), seed, device, std)
    w2 = normal((n_experts, h, d), seed + 7919, device, std)
    return w1, w2


# --------------------------------------------------------------------------
# edges (receiver-sorted CSR)
# --------------------------------------------------------------------------
def edges_random(n: int, per_atom: int, seed: int):
    """``per_atom*n`` edges with uniform receivers (Poisson degrees)."""
    g = rng(seed)
    m = per_atom * n
    recv = g.integers(0, n, size=m, dtype=np.int64)
    send = g.integers(0, n, size=m, dtype=np.int64)
    order = np.lexsort((send, recv))
    recv, send = recv[order], send[order]
    row_ptr = np.zeros(n + 1, np.int64)
    np.cumsum(np.bincount(recv, minlength=n), out=row_ptr[1:])
    return row_ptr, send, recv


def edges_pbc(n: int, seed: int, density: float = PBC_DENSITY, cutoff: float = PBC_CUTOFF):
    """All ordered pairs within ``cutoff`` (minimum image) of ``n`` atoms placed
    iid uniform in a periodic cube at ``density``; receiver-sorted CSR."""
    from scipy.spatial import cKDTree

    side = (n / density) ** (1.0 / 3.0)
    pos = rng(seed).random((n, 3)) * side
    tree = cKDTree(pos, boxsize=side)
    pairs = tree.query_pairs(cutoff, output_type="ndarray").astype(np.int64)
    recv = np.concatenate([pairs[:, 0], pairs[:, 1]])
    send = np.concatenate([pairs[:, 1], pairs[:, 0]])
    order = np.lexsort((send, recv))
    recv, send = recv[order], send[order]
    row_ptr = np.zeros(n + 1, np.int64)
    np.cumsum(np.bincount(recv, minlength=n), out=row_ptr[1:])
    return row_ptr, send, recv


# --------------------------------------------------------------------------
# a whole layer's inputs
# --------------------------------------------------------------------------
def layer_inputs(cfg: LayerConfig, seed: int = 0, device="cpu", with_edges=True,
                 with_features=True):
    """Every input of one layer pass.  Small index/table arrays are NumPy;
    dense FP32 tensors are torch tensors on ``device``."""
    out = {}
    if cfg.type_dist == "uniform":
        out["types"] = types_uniform(cfg.n_atoms, cfg.n_types, seed + 1)
    else:
        out["types"] = types_zipf(cfg.n_atoms, cfg.n_types, ZIPF_S, seed + 1)
    out["gate"] = gate_table(cfg.n_types, cfg.n_experts, seed + 2)
    out["w1"], out["w2"] = expert_weights(cfg.n_experts, cfg.d, cfg.h, seed + 3, device)
    if with_features:
        out["x"] = normal((cfg.n_atoms, cfg.d), seed + 4, device)
        out["g"] = normal((cfg.n_atoms, cfg.d), seed + 5, device)
    if with_edges and cfg.edges != "none":
        if cfg.edges == "random":
            rp, send, _ = edges_random(cfg.n_atoms, cfg.edges_per_atom, seed + 6)
        else:
            rp, send, _ = edges_pbc(cfg.n_atoms, seed + 6)
        out["row_ptr"] = rp
        out["senders"] = send
        out["msg"] = normal((int(rp[-1]), cfg.d), seed + 8, device)
    return out
