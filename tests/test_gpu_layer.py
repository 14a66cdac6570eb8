"""MoELayer: the layer pass behind the public Python API (paper review
'Breaking the Training Barrier of Billion-Parameter Universal Machine Learning
Interatomic Potentials', sections 3.1-3.5).

* run_host (pinned host in and out, copies on their own streams, device
  buffers double-buffered) equals the device-resident pass bit for bit, over
  several back-to-back calls with different batches and host buffers;
* the device pass equals the oracle chain (tiny layer, full comparison).
"""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from element_routed_moe_b200.layer import MoELayer
from helpers import DEV, TOL_FP32, host, rel_fro, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32])
def test_run_host_equals_device_pass_over_several_batches(mode):
    N, T, E, K, d, h = 3000, 89, 16, 4, 256, 320
    gate = to_dev(synth.gate_table(T, E, 1))
    w1, w2 = synth.expert_weights(E, d, h, 2, DEV)
    layer = MoELayer(N, K, gate, w1, w2, mode=mode)
    batches = []
    for b in range(5):
        x = synth.normal((N, d), 10 + b).pin_memory()
        g = synth.normal((N, d), 20 + b).pin_memory()
        t = torch.as_tensor(synth.types_zipf(N, T, seed=30 + b)).pin_memory()
        y = torch.full((N, d), float("nan")).pin_memory()
        dx = torch.full((N, d), float("nan")).pin_memory()
        batches.append((x, g, t, y, dx))
    for x, g, t, y, dx in batches:                    # back to back, no sync in between
        layer.run_host(x, g, t, y, dx)
    layer.host_sync()
    torch.cuda.synchronize()
    ref = MoELayer(N, K, gate, w1, w2, mode=mode)
    for x, g, t, y, dx in batches:
        y_ref, dx_ref = ref.forward_vjp(x.to(DEV), g.to(DEV), t.to(DEV))
        assert torch.equal(y, y_ref.cpu()) and torch.equal(dx, dx_ref.cpu())


@pytest.mark.parametrize("packed", [False, True])
def test_device_pass_matches_oracle(packed):
    N, T, E, K, d, h = 512, 8, 8, 2, 64, 64
    gate_np = synth.gate_table(T, E, 3)
    w1, w2 = synth.expert_weights(E, d, h, 4, DEV)
    types_np = synth.types_uniform(N, T, 5)
    x, g = synth.normal((N, d), 6, DEV), synth.normal((N, d), 7, DEV)
    layer = MoELayer(N, K, to_dev(gate_np), w1, w2, mode=J.JANUS_FFN_3XTF32, packed=packed)
    y, dx = layer.forward_vjp(x, g, to_dev(types_np))
    torch.cuda.synchronize()
    r = oracle.route(types_np, gate_np, K)
    hx = host(x)
    if packed:
        q, sc = oracle.quant_by_type(hx, types_np, T, r["perm"], K)
        xd = oracle.dequant_by_type(q, types_np, r["perm"], K, sc)
    else:
        xd = oracle.dispatch(hx, r["perm"], K)
    yd = oracle.expert_ffn_fwd(xd, r["offsets"], host(w1), host(w2))
    assert rel_fro(host(y), oracle.combine(yd, r["slot_of"], K, r["topk_weight"])) <= TOL_FP32
    gd = oracle.dispatch(host(g), r["perm"], K, r["topk_weight"])
    dxd = oracle.expert_ffn_vjp(xd, gd, r["offsets"], host(w1), host(w2))
    assert rel_fro(host(dx), oracle.combine(dxd, r["slot_of"], K)) <= TOL_FP32


def test_edge_fed_packed_layer_matches_oracle():
    # the interaction-block slice form: edge messages aggregated per receiver,
    # FP16 per-type packing of the dispatch, then the layer
    from element_routed_moe_b200.synth import edges_random
    N, T, E, K, d, h = 700, 11, 12, 3, 96, 64
    rp, send, recv = edges_random(N, 9, seed=11)
    msg = synth.normal((int(rp[-1]), d), 12, DEV)
    gate_np = synth.gate_table(T, E, 13)
    w1, w2 = synth.expert_weights(E, d, h, 14, DEV)
    types_np = synth.types_zipf(N, T, seed=15)
    g = synth.normal((N, d), 16, DEV)
    layer = MoELayer(N, K, to_dev(gate_np), w1, w2, mode=J.JANUS_FFN_3XTF32, packed=True,
                     row_ptr=torch.as_tensor(rp, device=DEV))
    assert layer.ops[0] == "edge_aggregate" and "quant" in layer.ops
    y, dx = layer.forward_vjp(msg, g, to_dev(types_np))
    torch.cuda.synchronize()
    x = oracle.edge_aggregate(host(msg), rp)
    r = oracle.route(types_np, gate_np, K)
    q, sc = oracle.quant_by_type(x, types_np, T, r["perm"], K)
    xd = oracle.dequant_by_type(q, types_np, r["perm"], K, sc)
    yd = oracle.expert_ffn_fwd(xd, r["offsets"], host(w1), host(w2))
    assert rel_fro(host(y), oracle.combine(yd, r["slot_of"], K, r["topk_weight"])) <= TOL_FP32
    gd = oracle.dispatch(host(g), r["perm"], K, r["topk_weight"])
    dxd = oracle.expert_ffn_vjp(xd, gd, r["offsets"], host(w1), host(w2))
    assert rel_fro(host(dx), oracle.combine(dxd, r["slot_of"], K)) <= TOL_FP32


@pytest.mark.parametrize("packed", [False, True])
def test_run_host_streams_edge_messages_bit_exact(packed):
    # edge-message input from pinned host memory: the messages are uploaded
    # chunk by chunk into a small ring of device buffers (forced here to many
    # chunks, a ring that wraps several times per call, and a receiver with
    # more edges than a slot holds), aggregated per chunk, and the pass must
    # equal the device-resident pass bit for bit over back-to-back calls
    from element_routed_moe_b200.synth import edges_random
    N, T, E, K, d, h = 900, 11, 12, 3, 40, 56
    gate = to_dev(synth.gate_table(T, E, 21))
    w1, w2 = synth.expert_weights(E, d, h, 22, DEV)
    rp, _, _ = edges_random(N, 7, seed=23)
    deg = np.diff(rp)
    deg[17] += 300                                  # one receiver larger than a ring slot
    rp = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    Ed = int(rp[-1])
    layer = MoELayer(N, K, gate, w1, w2, mode=J.JANUS_FFN_3XTF32, packed=packed, row_ptr=to_dev(rp))
    layer.RING_SLOT_BYTES = 4 * d * 64             # 64 edge rows per slot
    layer.RING_SLOTS = 3
    batches = []
    for b in range(4):
        m = synth.normal((Ed, d), 40 + b).pin_memory()
        g = synth.normal((N, d), 50 + b).pin_memory()
        t = torch.as_tensor(synth.types_zipf(N, T, seed=60 + b)).pin_memory()
        y = torch.full((N, d), float("nan")).pin_memory()
        dx = torch.full((N, d), float("nan")).pin_memory()
        batches.append((m, g, t, y, dx))
    for m, g, t, y, dx in batches:
        layer.run_host(m, g, t, y, dx)
    layer.host_sync()
    torch.cuda.synchronize()
    assert len(layer._host["chunks"]) > 3 * len(layer._host["ring"])
    ref = MoELayer(N, K, gate, w1, w2, mode=J.JANUS_FFN_3XTF32, packed=packed, row_ptr=to_dev(rp))
    for m, g, t, y, dx in batches:
        y_ref, dx_ref = ref.forward_vjp(m.to(DEV), g.to(DEV), t.to(DEV))
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref.cpu()) and torch.equal(dx, dx_ref.cpu())


def test_split_forward_layer_matches_oracle_and_run_host():
    # enough routed rows per expert (4,096) for the layer to take the FP16
    # tensor path in its forward: split dispatch + janus_expert_ffn_fwd_split
    N, T, E, K, d, h = 4096, 13, 4, 4, 136, 96
    gate_np = synth.gate_table(T, E, 23)
    w1, w2 = synth.expert_weights(E, d, h, 24, DEV)
    types_np = synth.types_zipf(N, T, seed=25)
    x, g = synth.normal((N, d), 26, DEV), synth.normal((N, d), 27, DEV)
    layer = MoELayer(N, K, to_dev(gate_np), w1, w2, mode=J.JANUS_FFN_3XTF32)
    assert layer.split
    y, dx = layer.forward_vjp(x, g, to_dev(types_np))
    torch.cuda.synchronize()
    J.janus_check(layer.ffn_ws)
    r = oracle.route(types_np, gate_np, K)
    xd = oracle.dispatch(host(x), r["perm"], K)
    yd = oracle.expert_ffn_fwd(xd, r["offsets"], host(w1), host(w2))
    assert rel_fro(host(y), oracle.combine(yd, r["slot_of"], K, r["topk_weight"])) <= TOL_FP32
    gd = oracle.dispatch(host(g), r["perm"], K, r["topk_weight"])
    dxd = oracle.expert_ffn_vjp(xd, gd, r["offsets"], host(w1), host(w2))
    assert rel_fro(host(dx), oracle.combine(dxd, r["slot_of"], K)) <= TOL_FP32
    # the pinned-host pipeline gives the same bits as the device pass
    y_ref, dx_ref = host(y).copy(), host(dx).copy()
    yh = torch.full((N, d), float("nan")).pin_memory()
    dxh = torch.full((N, d), float("nan")).pin_memory()
    layer.run_host(x.cpu().pin_memory(), g.cpu().pin_memory(), torch.as_tensor(types_np).pin_memory(), yh, dxh)
    layer.host_sync()
    torch.cuda.synchronize()
    assert np.array_equal(yh.numpy(), y_ref) and np.array_equal(dxh.numpy(), dx_ref)
