"""GPU parity on seeded random shapes (paper review 'Breaking the Training
Barrier of Billion-Parameter Universal Machine Learning Interatomic
Potentials', sections 3.1-3.5): each case draws N, T, E, K, d, h and the
edge count, including empty layers, one type, K up to 32, E up to 256, and
d, h at odd multiples of 4, then checks the path step by step against the
oracle: routing and packing bit-exact, features within 1e-5; the forward on
the FP16 rows (unpack fused into the GEMM) and with the exact-row flag must
equal the plain forward on the unpacked rows bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, host, rel_fro, to_dev

pytestmark = pytest.mark.gpu


def _shape(seed):
    g = np.random.default_rng(seed)
    E = int(g.choice([1, 2, 3, 7, 16, 40, 72, 255, 256]))
    K = int(g.integers(1, min(E, 32) + 1))
    T = int(g.choice([1, 2, 5, 13, 89, 100]))
    N = int(g.choice([0, 1, 7, 64, 333, 1000, 2900]))
    d = int(4 * g.integers(1, 97))
    h = int(4 * g.integers(1, 65))
    return N, T, E, K, d, h


@pytest.mark.parametrize("seed", range(30))
def test_random_shape_chain(seed):
    N, T, E, K, d, h = _shape(seed)
    types = synth.types_zipf(N, T, seed=seed) if N else np.zeros(0, np.int32)
    gate = synth.gate_table(T, E, seed + 1)
    x = synth.normal((N, d), seed + 2, DEV)
    g = synth.normal((N, d), seed + 3, DEV)
    r = J.janus_route(to_dev(types), to_dev(gate), K)
    J.janus_check(r["workspace"])
    o = oracle.route(types, gate, K)
    for k in ("topk_expert", "counts", "offsets", "perm", "slot_of"):
        assert np.array_equal(host(r[k]).reshape(o[k].shape), o[k]), (k, seed)
    if N == 0:
        return
    hx = host(x)
    # dispatch / combine
    xd = J.janus_dispatch(x, r["slot_of"], K)
    oxd = oracle.dispatch(hx, o["perm"], K)
    assert np.array_equal(host(xd), oxd)
    # FP16 packing
    payload, scale, qws = J.janus_quant_by_type(x, to_dev(types), T, r["slot_of"], K)
    J.janus_check(qws)
    op, osc = oracle.quant_by_type(hx, types, T, o["perm"], K)
    assert np.array_equal(host(payload).view(np.uint16), op) and np.array_equal(host(scale), osc)
    xq = J.janus_dequant_by_type(payload, to_dev(types), T, r["perm"], K, scale)
    assert np.array_equal(host(xq), oracle.dequant_by_type(op, types, o["perm"], K, osc))
    # expert MLP, both modes, and the layer's combines
    w1, w2 = synth.expert_weights(E, d, h, seed + 4, DEV)
    hw1, hw2 = host(w1), host(w2)
    gd = J.janus_dispatch(g, r["slot_of"], K, r["topk_weight"])
    ogd = oracle.dispatch(host(g), o["perm"], K, o["topk_weight"])
    assert np.array_equal(host(gd), ogd)
    oyd = oracle.expert_ffn_fwd(oxd, o["offsets"], hw1, hw2)
    odxd = oracle.expert_ffn_vjp(oxd, ogd, o["offsets"], hw1, hw2)
    for mode in (J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32):
        yd, act = J.janus_expert_ffn_fwd(xd, r["offsets"], w1, w2, mode=mode, want_act=True)
        dxd = J.janus_expert_ffn_vjp(xd, gd, r["offsets"], w1, w2, act=act, mode=mode)
        assert rel_fro(host(yd), oyd) <= TOL_FP32, (mode, seed)
        assert rel_fro(host(dxd), odxd) <= TOL_FP32, (mode, seed)
    # the forward on the unpacked rows with the exact-TF32 flag: bit-identical
    # to the plain forward on them; on the FP16 rows themselves: SIMT unpacks
    # first (bit-identical), 3xTF32 runs the FP16 tensor path against a split
    # of W1 (within the FP32 tolerance of the plain forward and the oracle);
    # and the split-row forward and VJP (FP16 tensor path, d % 8 == 0)
    row_scale = J.janus_dispatch_row_scales(to_dev(types), T, r["perm"], K, scale)
    oyq = oracle.expert_ffn_fwd(host(xq), o["offsets"], hw1, hw2)
    for mode in (J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32):
        yq, _ = J.janus_expert_ffn_fwd(xq, r["offsets"], w1, w2, mode=mode)
        yf, _ = J.janus_expert_ffn_fwd_ex(xq, r["offsets"], w1, w2, flags=J.JANUS_FFN_X_DEQUANTIZED, mode=mode)
        assert torch.equal(yf, yq), (mode, seed)
        if mode == J.JANUS_FFN_FP32_SIMT or d % 8 == 0:
            yp, _ = J.janus_expert_ffn_fwd_packed(payload, row_scale, r["offsets"], w1, w2, mode=mode)
            if mode == J.JANUS_FFN_FP32_SIMT:
                assert torch.equal(yp, yq), (mode, seed)
            else:
                assert rel_fro(host(yp), host(yq)) <= TOL_FP32 and rel_fro(host(yp), oyq) <= TOL_FP32, (mode, seed)
    if d % 8 == 0:
        x16, xs = J.janus_dispatch_split(x, r["slot_of"], K)
        g16, gs = J.janus_dispatch_split(g, r["slot_of"], K, r["topk_weight"])
        ys, a_s = J.janus_expert_ffn_fwd_split(x16, xs, r["offsets"], w1, w2, want_act=True)
        dxs = J.janus_expert_ffn_vjp_split(g16, gs, r["offsets"], w1, w2, a_s)
        assert rel_fro(host(ys), oyd) <= TOL_FP32 and rel_fro(host(dxs), odxd) <= TOL_FP32, seed
    y = J.janus_combine(yd, r["slot_of"], K, r["topk_weight"])
    assert rel_fro(host(y), oracle.combine(host(yd), o["slot_of"], K, o["topk_weight"])) <= TOL_FP32
    dx = J.janus_combine(dxd, r["slot_of"], K)
    assert rel_fro(host(dx), oracle.combine(host(dxd), o["slot_of"], K)) <= TOL_FP32


@pytest.mark.parametrize("seed", range(12))
def test_random_shape_edges(seed):
    g = np.random.default_rng(1000 + seed)
    N = int(g.choice([1, 5, 100, 1000, 4000]))
    d = int(4 * g.integers(1, 129))
    per = int(g.choice([0, 1, 3, 20, 70]))
    rp, send, _ = synth.edges_random(N, per, seed=seed)
    Ed = int(rp[-1])
    msg = synth.normal((Ed, d), seed + 1, DEV)
    x = J.janus_edge_aggregate(msg, torch.as_tensor(rp, device=DEV))
    assert rel_fro(host(x), oracle.edge_aggregate(host(msg), rp)) <= TOL_FP32
    if Ed:
        dx = synth.normal((N, d), seed + 2, DEV)
        dmsg = J.janus_edge_broadcast(dx, torch.as_tensor(rp, device=DEV))
        assert np.array_equal(host(dmsg), oracle.edge_broadcast(host(dx), rp))


@pytest.mark.parametrize("seed", range(8))
def test_random_shape_fp16_second_gemms(seed):
    # >= 2048 rows per expert (above the library's threshold) with d, h % 8 == 0: both GEMMs of each direction
    # on the FP16 tensor path (split rows, the FP16 payload for the packed
    # forward), on ragged segments and random widths with K tails
    g = np.random.default_rng(2000 + seed)
    E = int(g.choice([1, 2, 3, 5]))
    counts = g.integers(0, 2 * 2048, size=E)
    counts[int(g.integers(0, E))] += 2048 * E            # at least 2048 rows per expert overall
    R = int(counts.sum())
    d = int(8 * g.integers(1, 70))
    h = int(8 * g.integers(1, 70))
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    o = to_dev(offs)
    w1, w2 = synth.expert_weights(E, d, h, 3000 + seed, DEV)
    xd = synth.normal((R, d), 3100 + seed, DEV)
    gd = synth.normal((R, d), 3200 + seed, DEV)
    ident = torch.arange(R, dtype=torch.int32, device=DEV)
    x16, xs = J.janus_dispatch_split(xd, ident, 1)
    g16, gs = J.janus_dispatch_split(gd, ident, 1)
    ys, a_s = J.janus_expert_ffn_fwd_split(x16, xs, o, w1, w2, want_act=True)
    dxs = J.janus_expert_ffn_vjp_split(g16, gs, o, w1, w2, a_s)
    hw1, hw2 = host(w1), host(w2)
    oyd, oact = oracle.expert_ffn_fwd(host(xd), offs, hw1, hw2, want_act=True)
    odxd = oracle.expert_ffn_vjp(host(xd), host(gd), offs, hw1, hw2)
    assert rel_fro(host(a_s), oact) <= TOL_FP32, seed
    assert rel_fro(host(ys), oyd) <= TOL_FP32 and rel_fro(host(dxs), odxd) <= TOL_FP32, seed
    # the packed forward: FP16 rows times a power-of-two scale per row
    payload = synth.normal((R, d), 3300 + seed, DEV).half()
    rsc = torch.as_tensor(np.ldexp(1.0, g.integers(-20, 20, size=R)).astype(np.float32), device=DEV)
    yp, _ = J.janus_expert_ffn_fwd_packed(payload, rsc, o, w1, w2, mode=J.JANUS_FFN_3XTF32)
    xq = host(payload).astype(np.float32) * host(rsc)[:, None]
    assert rel_fro(host(yp), oracle.expert_ffn_fwd(xq, offs, hw1, hw2)) <= TOL_FP32, seed
