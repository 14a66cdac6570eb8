"""GPU parity of the expert-parallel exchange ([Review] 'Breaking the Training
Barrier of Billion-Parameter Universal Machine Learning Interatomic
Potentials', sections 3.4-3.5: experts sharded over ranks, FP16-packed rows in
the all-to-all).

The P ranks are emulated in one process on one GPU: each rank's send kernel
runs in turn and stores into the other ranks' buffers (plain device pointers
here; peer-mapped ones on a node), then each owner runs its experts and the
return kernel.  No kernel waits on another.  The expert MLP works row by row,
so every rank's output must equal its own single-GPU chain (route -> pack ->
unpack -> experts -> combine) and the oracle's chain on the same shard.
"""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, host, rel_fro, to_dev

pytestmark = pytest.mark.gpu

MODES = [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32]


def _shards(P, N, T, d, seed):
    out = []
    for s in range(P):
        n = N + 7 * s                                       # ragged shards
        out.append((synth.normal((n, d), seed + 10 * s, DEV), to_dev(synth.types_zipf(n, T, seed=seed + 10 * s + 1))))
    return out


def _ep_pass(shards, gate, K, w1, w2, mode, grads=None, fused=False):
    """Forward (and with grads, the input VJP) of the emulated EP layer.  With
    fused, each owner's expert MLP stores its output rows straight into the
    senders' return buffers through the janus_ep_return_rows table.  The
    receive buffers hold the worst case (every rank's rows on one owner)."""
    P = len(shards)
    T, E = gate.shape
    El = E // P
    d = shards[0][0].shape[1]
    routes = [J.janus_route(t, gate, K) for _, t in shards]
    counts_all = torch.stack([r["counts"] for r in routes]).contiguous()
    cap = sum(x.shape[0] for x, _ in shards) * K
    layout = J.janus_ep_layout(counts_all, E, cap)
    payload = [torch.full((cap, d), float("nan"), dtype=torch.float16, device=DEV) for _ in range(P)]
    rscale = [torch.full((cap,), float("nan"), device=DEV) for _ in range(P)]
    for s, (x, t) in enumerate(shards):
        _, ws = J.janus_ep_dispatch_quant(x, t, T, routes[s], layout, s, cap, payload, rscale)
        J.janus_check(ws)
    recv_off = layout[2]
    # a rank without atoms still passes a (never written) buffer
    ret = [torch.full((max(x.shape[0] * K, 1), d), float("nan"), device=DEV) for x, _ in shards]
    dret = [torch.full((max(x.shape[0] * K, 1), d), float("nan"), device=DEV) for x, _ in shards]
    xd_recv, act_recv, yd_recv = [], [], []
    for o in range(P):
        xr = J.janus_ep_dequant_rows(payload[o], rscale[o], layout, o)
        w1o, w2o = w1[o * El:(o + 1) * El].contiguous(), w2[o * El:(o + 1) * El].contiguous()
        if fused:
            ar = J.janus_expert_ffn_fwd_rows(xr, recv_off[o], w1o, w2o,
                                             J.janus_ep_return_rows(layout, o, ret, cap, d),
                                             mode=mode, want_act=True)
        else:
            yr, ar = J.janus_expert_ffn_fwd(xr, recv_off[o], w1o, w2o, mode=mode, want_act=True)
            yd_recv.append(yr)
        xd_recv.append(xr)
        act_recv.append(ar)
    if not fused:
        for o in range(P):
            J.janus_ep_return(yd_recv[o], counts_all, layout, o, ret)
    ys = [J.janus_combine(ret[s][:shards[s][0].shape[0] * K], routes[s]["slot_of"], K, routes[s]["topk_weight"])
          for s in range(P)]
    if grads is None:
        return ys, routes, layout
    g_recv = [torch.full((cap, d), float("nan"), device=DEV) for _ in range(P)]
    for s in range(P):
        J.janus_ep_dispatch(grads[s], routes[s], layout, s, cap, g_recv, weighted=True)
    for o in range(P):
        w1o, w2o = w1[o * El:(o + 1) * El].contiguous(), w2[o * El:(o + 1) * El].contiguous()
        if fused:
            J.janus_expert_ffn_vjp_rows(xd_recv[o], g_recv[o], recv_off[o], w1o, w2o,
                                        J.janus_ep_return_rows(layout, o, dret, cap, d),
                                        act=act_recv[o], mode=mode)
        else:
            dxr = J.janus_expert_ffn_vjp(xd_recv[o], g_recv[o], recv_off[o], w1o, w2o, act=act_recv[o], mode=mode)
            J.janus_ep_return(dxr, counts_all, layout, o, dret)
    dxs = [J.janus_combine(dret[s][:shards[s][0].shape[0] * K], routes[s]["slot_of"], K) for s in range(P)]
    return ys, dxs, routes, layout


def _local_chain(x, t, gate, K, w1, w2, mode, g=None):
    T = gate.shape[0]
    r = J.janus_route(t, gate, K)
    payload, scale, _ = J.janus_quant_by_type(x, t, T, r["slot_of"], K)
    xd = J.janus_dequant_by_type(payload, t, T, r["perm"], K, scale)
    yd, act = J.janus_expert_ffn_fwd(xd, r["offsets"], w1, w2, mode=mode, want_act=True)
    y = J.janus_combine(yd, r["slot_of"], K, r["topk_weight"])
    if g is None:
        return y
    gd = J.janus_dispatch(g, r["slot_of"], K, r["topk_weight"])
    dxd = J.janus_expert_ffn_vjp(xd, gd, r["offsets"], w1, w2, act=act, mode=mode)
    return y, J.janus_combine(dxd, r["slot_of"], K)


CASES = {
    # name: (P, N per rank, T, E, K, d, h)
    "p2_small": (2, 150, 11, 8, 2, 64, 96),
    "p4_ragged": (4, 300, 89, 16, 3, 132, 68),
    "p8_s_shape": (8, 1024, 89, 72, 4, 256, 256),
    "p1": (1, 200, 13, 6, 2, 32, 32),
}


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", list(CASES))
def test_ep_forward_and_vjp_equal_local_chains(name, mode):
    P, N, T, E, K, d, h = CASES[name]
    gate = to_dev(synth.gate_table(T, E, 1))
    w1, w2 = synth.expert_weights(E, d, h, 2, DEV)
    shards = _shards(P, N, T, d, 100)
    grads = [synth.normal((x.shape[0], d), 500 + s, DEV) for s, (x, _) in enumerate(shards)]
    ys, dxs, routes, layout = _ep_pass(shards, gate, K, w1, w2, mode, grads)
    torch.cuda.synchronize()
    # the layout kernel against the oracle's layout
    counts_all = np.stack([host(r["counts"]) for r in routes])
    for got, ref in zip(layout, oracle.ep_layout(counts_all)):
        assert np.array_equal(host(got), ref)
    hw1, hw2 = host(w1), host(w2)
    for s, (x, t) in enumerate(shards):
        y_loc, dx_loc = _local_chain(x, t, gate, K, w1, w2, mode, grads[s])
        # the same rows through the same kernels, only grouped differently
        assert rel_fro(host(ys[s]), host(y_loc)) <= 1e-6, s
        assert rel_fro(host(dxs[s]), host(dx_loc)) <= 1e-6, s
        # and the oracle's chain on this shard (FP16 packing identical on both sides)
        hx, ht = host(x), host(t)
        r = oracle.route(ht, host(gate), K)
        q, sc = oracle.quant_by_type(hx, ht, T, r["perm"], K)
        xd = oracle.dequant_by_type(q, ht, r["perm"], K, sc)
        yd = oracle.expert_ffn_fwd(xd, r["offsets"], hw1, hw2)
        assert rel_fro(host(ys[s]), oracle.combine(yd, r["slot_of"], K, r["topk_weight"])) <= TOL_FP32
        gd = oracle.dispatch(host(grads[s]), r["perm"], K, r["topk_weight"])
        dxd = oracle.expert_ffn_vjp(xd, gd, r["offsets"], hw1, hw2)
        assert rel_fro(host(dxs[s]), oracle.combine(dxd, r["slot_of"], K)) <= TOL_FP32


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", ["p2_small", "p4_ragged", "p8_s_shape", "p1"])
def test_fused_return_equals_copy_return(name, mode):
    # the GEMM epilogue storing through the row table writes the same values
    # to the same sender rows as the separate return copy: bit-exact
    P, N, T, E, K, d, h = CASES[name]
    gate = to_dev(synth.gate_table(T, E, 4))
    w1, w2 = synth.expert_weights(E, d, h, 5, DEV)
    shards = _shards(P, N, T, d, 300)
    grads = [synth.normal((x.shape[0], d), 700 + s, DEV) for s, (x, _) in enumerate(shards)]
    ys, dxs, _, _ = _ep_pass(shards, gate, K, w1, w2, mode, grads)
    ys_f, dxs_f, _, _ = _ep_pass(shards, gate, K, w1, w2, mode, grads, fused=True)
    torch.cuda.synchronize()
    for s in range(P):
        assert torch.equal(ys[s], ys_f[s]) and torch.equal(dxs[s], dxs_f[s]), s


def test_return_row_table_follows_the_layout():
    # every received row's address is its sender's row in the sender's local
    # order (owner row dst_off[s][e] + i <-> sender row src_off[s][e] + i)
    P, N, T, E, K, d = 4, 120, 9, 12, 3, 36
    gate = to_dev(synth.gate_table(T, E, 6))
    shards = _shards(P, N, T, d, 400)
    routes = [J.janus_route(t, gate, K) for _, t in shards]
    counts_all = torch.stack([r["counts"] for r in routes]).contiguous()
    cap = sum(x.shape[0] for x, _ in shards) * K
    layout = J.janus_ep_layout(counts_all, E, cap)
    ret = [torch.empty((x.shape[0] * K, d), device=DEV) for x, _ in shards]
    src_off, dst_off, recv_off = oracle.ep_layout(np.stack([host(r["counts"]) for r in routes]))
    El = E // P
    for o in range(P):
        table = host(J.janus_ep_return_rows(layout, o, ret, cap, d))
        expect = np.zeros(cap, np.int64)
        for e in range(o * El, (o + 1) * El):
            for s in range(P):
                for i in range(int(src_off[s][e + 1] - src_off[s][e])):
                    expect[dst_off[s][e] + i] = ret[s].data_ptr() + 4 * d * (int(src_off[s][e]) + i)
        assert np.array_equal(table, expect), o
        assert not table[recv_off[o][El]:].any()        # past the received rows: untouched


@pytest.mark.parametrize("mode", MODES)
def test_ffn_rows_store_equals_permuted_plain_store(mode):
    # an arbitrary row table (a permutation into a larger buffer): row p of the
    # plain output lands at its table address, nothing else is written
    E, d, h = 7, 132, 68
    counts = np.array([0, 5, 300, 1, 0, 129, 64])
    offsets = to_dev(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32))
    R = int(counts.sum())
    xd = synth.normal((R, d), 31, DEV)
    gd = synth.normal((R, d), 32, DEV)
    w1, w2 = synth.expert_weights(E, d, h, 33, DEV)
    dest = torch.full((R + 50, d), float("nan"), device=DEV)
    slot = torch.as_tensor(np.random.default_rng(34).permutation(R + 50)[:R], device=DEV)
    table = dest.data_ptr() + 4 * d * slot.to(torch.int64)
    yd, act = J.janus_expert_ffn_fwd(xd, offsets, w1, w2, mode=mode, want_act=True)
    J.janus_expert_ffn_fwd_rows(xd, offsets, w1, w2, table, mode=mode)
    torch.cuda.synchronize()
    assert torch.equal(dest[slot], yd)
    untouched = torch.ones(R + 50, dtype=torch.bool, device=DEV)
    untouched[slot] = False
    assert torch.isnan(dest[untouched]).all()
    dest.fill_(float("nan"))
    dxd = J.janus_expert_ffn_vjp(xd, gd, offsets, w1, w2, act=act, mode=mode)
    J.janus_expert_ffn_vjp_rows(xd, gd, offsets, w1, w2, table, act=act, mode=mode)
    torch.cuda.synchronize()
    assert torch.equal(dest[slot], dxd)
    assert torch.isnan(dest[untouched]).all()


def test_ep_send_places_rows_by_the_layout():
    # unweighted FP32 send: every owner row is the sender's atom row, bit-exact
    P, N, T, E, K, d = 4, 90, 7, 12, 3, 20
    gate = to_dev(synth.gate_table(T, E, 3))
    shards = _shards(P, N, T, d, 200)
    routes = [J.janus_route(t, gate, K) for _, t in shards]
    counts_all = torch.stack([r["counts"] for r in routes]).contiguous()
    cap = sum(x.shape[0] for x, _ in shards) * K
    layout = J.janus_ep_layout(counts_all, E, cap)
    recv = [torch.full((cap, d), float("nan"), device=DEV) for _ in range(P)]
    for s, (x, _) in enumerate(shards):
        J.janus_ep_dispatch(x, routes[s], layout, s, cap, recv, weighted=False)
    torch.cuda.synchronize()
    src_off, dst_off, recv_off = (host(a) for a in layout)
    El = E // P
    for s, (x, _) in enumerate(shards):
        hx, perm = host(x), host(routes[s]["perm"])
        for e in range(E):
            o, n = e // El, counts_all[s, e].item()
            got = host(recv[o][dst_off[s, e]:dst_off[s, e] + n])
            assert np.array_equal(got, hx[perm[src_off[s, e]:src_off[s, e] + n] // K])
    for o in range(P):      # rows past the received count stay untouched
        assert torch.isnan(recv[o][int(recv_off[o, -1]):]).all().item()


def test_ep_experts_without_rows_and_a_rank_without_atoms():
    # rank 1 has no atoms; gate makes half the experts unreachable
    P, T, E, K, d, h = 2, 5, 8, 2, 16, 16
    g = np.full((T, E), -10.0, np.float32)
    g[:, :3] = synth.gate_table(T, 3, 4)
    gate = to_dev(g)
    w1, w2 = synth.expert_weights(E, d, h, 5, DEV)
    shards = [(synth.normal((64, d), 1, DEV), to_dev(synth.types_uniform(64, T, 2))),
              (torch.empty((0, d), device=DEV), torch.empty((0,), dtype=torch.int32, device=DEV))]
    ys, _, _ = _ep_pass(shards, gate, K, w1, w2, J.JANUS_FFN_3XTF32)
    y0 = _local_chain(shards[0][0], shards[0][1], gate, K, w1, w2, J.JANUS_FFN_3XTF32)
    assert rel_fro(host(ys[0]), host(y0)) <= 1e-6
    assert ys[1].shape[0] == 0


def test_ep_argument_checks():
    E = 9
    counts = torch.zeros((2, E), dtype=torch.int32, device=DEV)
    with pytest.raises(J.JanusError) as e:
        J.janus_ep_layout(counts, E, 100)                   # 9 experts over 2 ranks
    assert e.value.status == J.JANUS_ERR_INVALID_ARG
    with pytest.raises(J.JanusError):
        J.janus_ep_layout(torch.zeros((9, 72), dtype=torch.int32, device=DEV), 72, 100)   # > 8 ranks
    with pytest.raises(J.JanusError):
        J.janus_ep_layout(torch.zeros((2, 8), dtype=torch.int32, device=DEV), 8, -1)     # negative capacity


def test_ep_capacity_overflow_is_reported_and_stays_in_bounds():
    # P = 8 emulated ranks with receive buffers smaller than the busiest
    # owner's rows: the sends skip what does not fit and record a data fault;
    # guard rows past the capacity stay untouched, recv_off is clamped, and
    # every owner row below the capacity holds what the unbounded layout puts there
    P, N, T, E, K, d = 8, 200, 89, 16, 4, 24
    gate = to_dev(synth.gate_table(T, E, 8))
    shards = _shards(P, N, T, d, 600)
    routes = [J.janus_route(t, gate, K) for _, t in shards]
    counts_all = torch.stack([r["counts"] for r in routes]).contiguous()
    full = sum(x.shape[0] for x, _ in shards) * K
    _, _, recv_ref = oracle.ep_layout(host(counts_all))
    busiest = int(recv_ref[:, -1].max())
    cap = busiest - 37                                    # the busiest owner overflows
    guard = 64
    lay_full = J.janus_ep_layout(counts_all, E, full)
    lay = J.janus_ep_layout(counts_all, E, cap)
    torch.cuda.synchronize()
    assert np.array_equal(host(lay[2]), np.minimum(recv_ref, cap))
    assert np.array_equal(host(lay[0]), host(lay_full[0])) and np.array_equal(host(lay[1]), host(lay_full[1]))
    pay = [torch.full((cap + guard, d), float("nan"), dtype=torch.float16, device=DEV) for _ in range(P)]
    rsc = [torch.full((cap + guard,), float("nan"), device=DEV) for _ in range(P)]
    rows = [torch.full((cap + guard, d), float("nan"), device=DEV) for _ in range(P)]
    pay_f = [torch.full((full, d), float("nan"), dtype=torch.float16, device=DEV) for _ in range(P)]
    rsc_f = [torch.full((full,), float("nan"), device=DEV) for _ in range(P)]
    faults = 0
    for s, (x, t) in enumerate(shards):
        _, ws = J.janus_ep_dispatch_quant(x, t, T, routes[s], lay, s, cap, pay, rsc)
        J.janus_ep_dispatch(x, routes[s], lay, s, cap, rows, weighted=True, workspace=ws)
        try:
            J.janus_check(ws)
        except J.JanusError as err:
            assert err.status == J.JANUS_ERR_DATA
            faults += 1
        J.janus_ep_dispatch_quant(x, t, T, routes[s], lay_full, s, full, pay_f, rsc_f)
    torch.cuda.synchronize()
    assert faults >= 1
    for o in range(P):
        assert torch.isnan(pay[o][cap:].float()).all() and torch.isnan(rsc[o][cap:]).all(), o
        assert torch.isnan(rows[o][cap:]).all(), o
        n = min(int(recv_ref[o, -1]), cap)
        assert torch.equal(pay[o][:n].view(torch.int16), pay_f[o][:n].view(torch.int16)), o
        assert torch.equal(rsc[o][:n], rsc_f[o][:n]), o


@pytest.mark.parametrize("fused", [True, False])
def test_ep_layer_fp16_path_one_rank(fused):
    # one rank owning every expert, sized so that the owner's expert MLP runs
    # on the FP16 tensor path in both directions (receive rows per local
    # expert above the library's threshold): the layer's y and dX against its
    # own local chain
    from element_routed_moe_b200.ep import ExpertParallelLayer
    N, T, E, K, d, h = 2100, 13, 2, 2, 64, 64
    gate = to_dev(synth.gate_table(T, E, 41))
    w1, w2 = synth.expert_weights(E, d, h, 42, DEV)
    x = synth.normal((N, d), 43, DEV)
    types = to_dev(synth.types_zipf(N, T, seed=44))
    g = synth.normal((N, d), 45, DEV)
    layer = ExpertParallelLayer(N, d, h, T, E, K, w1, w2, mode=J.JANUS_FFN_3XTF32, device=DEV,
                                fused_return=fused, capacity_factor=1.0)
    assert layer.f16_second and layer.split_vjp
    y = layer.forward(x, types, gate)
    dx = layer.vjp(g)
    torch.cuda.synchronize()
    y_ref, dx_ref = _local_chain(x, types, gate, K, w1, w2, J.JANUS_FFN_3XTF32, g)
    assert rel_fro(host(y), host(y_ref)) <= TOL_FP32 and rel_fro(host(dx), host(dx_ref)) <= TOL_FP32
    layer.close()
