"""GPU parity, at full size, of the layer pass the benchmark times on the
FP16-packed configurations: MoELayer(packed=True) with the per-type FP16
rows fed to the first expert GEMM as they are (janus_expert_ffn_fwd_packed),
forward and input VJP, on

  * the MatRIS-MoE(M)-shaped layer (N = 32,768, E = 40, K = 8, d = h = 1536);
  * the interaction-block slice (N = 65,536, 4.74 M edges, the same MoE shape,
    edge aggregation in front).

Sources: paper review 'Breaking the Training Barrier of Billion-Parameter
Universal Machine Learning Interatomic Potentials', section 3.1 Table II (the
M shape), section 3.4 Figure 3 (block order: aggregation before the MoE
layer), section 3.5 (atom-type-aware FP16 compression of the dispatch).

Checks, as for the unfused chain (tests/test_gpu_chain.py):
  (1) routing and the FP16 payload with its scales are bit-exact;
  (2) on sampled atoms, y and dX are within 1e-5 (relative Frobenius over
      the sample) of an oracle chain that packs the same way, and no sampled
      row is off by more than 1e-4 relative;
  (3) within 2e-3 of the FP32-only oracle chain (the packed path's bar);
  (4) slice: the aggregated features of sampled atoms match the oracle.

and of the L-shaped layer's unpacked pass on the FP16 tensor path (split
dispatches and every expert GEMM on kind::f16), against the FP32 oracle chain.
"""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from element_routed_moe_b200.layer import MoELayer
from helpers import DEV, TOL_FP16_PATH, TOL_FP32, TOL_ROW, host, max_row_rel, rel_fro, to_dev

pytestmark = pytest.mark.gpu


def _sample_atoms(N, seed):
    return np.unique(np.concatenate([[0, 1, N - 1], np.random.default_rng(seed).integers(0, N, 61)]))


@pytest.mark.parametrize("mode", [J.JANUS_FFN_3XTF32, J.JANUS_FFN_FP32_SIMT])
@pytest.mark.parametrize("name", ["M", "slice"])
def test_packed_layer_full_size_sampled(name, mode):
    cfg = synth.CONFIGS[name]
    assert cfg.quant
    N, T, E, K, d = cfg.n_atoms, cfg.n_types, cfg.n_experts, cfg.top_k, cfg.d
    edges = cfg.edges != "none"
    inp = synth.layer_inputs(cfg, seed=21, device=DEV, with_edges=edges)
    types_np, gate_np = inp["types"], inp["gate"]
    rp = inp["row_ptr"] if edges else None
    layer = MoELayer(N, K, to_dev(gate_np), inp["w1"], inp["w2"], mode=mode, packed=True,
                     row_ptr=to_dev(rp) if edges else None)
    assert layer.fused_unpack
    x_in = inp["msg"] if edges else inp["x"]
    y, dx = layer.forward_vjp(x_in, inp["g"], to_dev(types_np))
    torch.cuda.synchronize()
    J.janus_check(layer.route_ws)
    J.janus_check(layer.quant_ws)
    J.janus_check(layer.ffn_ws)
    atoms = _sample_atoms(N, 5)
    # (4) the aggregated features of the sampled atoms, from their own messages
    if edges:
        blocks = [host(inp["msg"][int(rp[i]):int(rp[i + 1])]) for i in atoms]
        mini_rp = np.concatenate([[0], np.cumsum([b.shape[0] for b in blocks])]).astype(np.int64)
        x_ref = oracle.edge_aggregate(np.concatenate(blocks), mini_rp)
        assert rel_fro(host(layer.xagg)[atoms], x_ref) <= TOL_FP32
        x = host(layer.xagg)          # the rest of the chain starts from the GPU's features
        del inp["msg"], x_in
    else:
        x = host(inp["x"])
    # (1) routing, payload and scales
    r = oracle.route(types_np, gate_np, K)
    ro = layer.route_out
    for k in ("counts", "offsets", "perm", "slot_of", "topk_expert"):
        assert np.array_equal(host(ro[k]), r[k]), k
    p_ref, s_ref = oracle.quant_by_type(x, types_np, T, r["perm"], K)
    assert np.array_equal(host(layer.scale), s_ref)
    assert np.array_equal(host(layer.payload).view(np.uint16), p_ref)
    # (2) the sampled atoms' K expert rows, one by one, through a packing oracle chain
    slots = (atoms[:, None] * K + np.arange(K)[None, :]).ravel()
    rows = r["slot_of"][slots].astype(np.int64)
    hw1, hw2, hg = host(inp["w1"]), host(inp["w2"]), host(inp["g"])
    xd = oracle.dequant_by_type(p_ref, types_np, r["perm"], K, s_ref)
    gd = oracle.dispatch(hg, r["perm"], K, r["topk_weight"])
    compact = np.arange(len(atoms) * K, dtype=np.int32)
    w_s = r["topk_weight"][atoms]
    y_q = oracle.combine(oracle.expert_ffn_fwd(xd, r["offsets"], hw1, hw2, rows=rows), compact, K, w_s)
    dx_q = oracle.combine(oracle.expert_ffn_vjp(xd, gd, r["offsets"], hw1, hw2, rows=rows), compact, K)
    y_s, dx_s = host(y)[atoms], host(dx)[atoms]
    assert rel_fro(y_s, y_q) <= TOL_FP32 and rel_fro(dx_s, dx_q) <= TOL_FP32
    assert max_row_rel(y_s, y_q) <= TOL_ROW and max_row_rel(dx_s, dx_q) <= TOL_ROW
    # (3) against the FP32-only chain (no packing) from the same features
    del xd
    xd32 = oracle.dispatch(x, r["perm"], K)
    y_f = oracle.combine(oracle.expert_ffn_fwd(xd32, r["offsets"], hw1, hw2, rows=rows), compact, K, w_s)
    dx_f = oracle.combine(oracle.expert_ffn_vjp(xd32, gd, r["offsets"], hw1, hw2, rows=rows), compact, K)
    assert rel_fro(y_s, y_f) <= TOL_FP16_PATH and rel_fro(dx_s, dx_f) <= TOL_FP16_PATH
    # every atom's output was written
    assert torch.isfinite(y).all().item() and torch.isfinite(dx).all().item()


def test_split_layer_full_size_sampled_L():
    # the L-shaped layer as the benchmark runs it: edge aggregation (1.19 M
    # edges of d = 1920 messages), unpacked rows, and every expert GEMM on
    # the FP16 tensor path (3,641 rows per expert on average: the split
    # dispatches, the activation and weight splits, the kind::f16 GEMMs)
    cfg = synth.CONFIGS["L"]
    assert not cfg.quant and cfg.edges != "none"
    N, T, E, K, d = cfg.n_atoms, cfg.n_types, cfg.n_experts, cfg.top_k, cfg.d
    inp = synth.layer_inputs(cfg, seed=23, device=DEV, with_edges=True)
    types_np, gate_np, rp = inp["types"], inp["gate"], inp["row_ptr"]
    layer = MoELayer(N, K, to_dev(gate_np), inp["w1"], inp["w2"], mode=J.JANUS_FFN_3XTF32, row_ptr=to_dev(rp))
    assert layer.split and layer.split_vjp and layer.f16_second
    y, dx = layer.forward_vjp(inp["msg"], inp["g"], to_dev(types_np))
    torch.cuda.synchronize()
    J.janus_check(layer.route_ws)
    J.janus_check(layer.ffn_ws)
    atoms = _sample_atoms(N, 6)
    blocks = [host(inp["msg"][int(rp[i]):int(rp[i + 1])]) for i in atoms]
    mini_rp = np.concatenate([[0], np.cumsum([b.shape[0] for b in blocks])]).astype(np.int64)
    assert rel_fro(host(layer.xagg)[atoms], oracle.edge_aggregate(np.concatenate(blocks), mini_rp)) <= TOL_FP32
    x = host(layer.xagg)
    del inp["msg"]
    r = oracle.route(types_np, gate_np, K)
    ro = layer.route_out
    for k in ("counts", "offsets", "perm", "slot_of", "topk_expert"):
        assert np.array_equal(host(ro[k]), r[k]), k
    slots = (atoms[:, None] * K + np.arange(K)[None, :]).ravel()
    rows = r["slot_of"][slots].astype(np.int64)
    hw1, hw2, hg = host(inp["w1"]), host(inp["w2"]), host(inp["g"])
    xd = oracle.dispatch(x, r["perm"], K)
    gd = oracle.dispatch(hg, r["perm"], K, r["topk_weight"])
    compact = np.arange(len(atoms) * K, dtype=np.int32)
    y_r = oracle.combine(oracle.expert_ffn_fwd(xd, r["offsets"], hw1, hw2, rows=rows), compact, K,
                         r["topk_weight"][atoms])
    dx_r = oracle.combine(oracle.expert_ffn_vjp(xd, gd, r["offsets"], hw1, hw2, rows=rows), compact, K)
    y_s, dx_s = host(y)[atoms], host(dx)[atoms]
    assert rel_fro(y_s, y_r) <= TOL_FP32 and rel_fro(dx_s, dx_r) <= TOL_FP32
    assert max_row_rel(y_s, y_r) <= TOL_ROW and max_row_rel(dx_s, dx_r) <= TOL_ROW
    assert torch.isfinite(y).all().item() and torch.isfinite(dx).all().item()
