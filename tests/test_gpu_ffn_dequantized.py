"""The expert MLP forward on dequantized FP16-packed rows (paper review
'Breaking the Training Barrier of Billion-Parameter Universal Machine Learning
Interatomic Potentials', section 3.5: atom-type-aware FP16 packing of the
dispatch).

A dequantized row is an FP16 value times a power-of-two scale, so it is exact
in TF32 and its 3xTF32 residual is zero.  JANUS_FFN_X_DEQUANTIZED lets the
first GEMM skip the product with that residual.  Skipping a product that only
adds zeros leaves every accumulator bit unchanged, so the flagged forward must
equal the unflagged one bit for bit, and both the oracle within 1e-5.  Rows
that are not exact in TF32 are reported as a data fault.
"""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, TOL_ROW, host, max_row_rel, rel_fro, sample_rows, to_dev

pytestmark = pytest.mark.gpu

SHAPES = {
    # name: (N, T, E, K, d, h)
    "ragged": (700, 11, 12, 3, 132, 68),
    "M_like": (4096, 89, 40, 8, 512, 384),
}


def _packed_rows(N, T, E, K, d, seed):
    types = synth.types_zipf(N, T, seed=seed)
    gate = synth.gate_table(T, E, seed + 1)
    x = synth.normal((N, d), seed + 2, DEV)
    r = J.janus_route(to_dev(types), to_dev(gate), K)
    payload, scale, _ = J.janus_quant_by_type(x, to_dev(types), T, r["slot_of"], K)
    xd = J.janus_dequant_by_type(payload, to_dev(types), T, r["perm"], K, scale)
    return xd, r


@pytest.mark.parametrize("mode", [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32])
@pytest.mark.parametrize("name", list(SHAPES))
def test_dequantized_flag_is_bit_identical_and_matches_oracle(name, mode):
    N, T, E, K, d, h = SHAPES[name]
    xd, r = _packed_rows(N, T, E, K, d, 40)
    w1, w2 = synth.expert_weights(E, d, h, 41, DEV)
    y_plain, a_plain = J.janus_expert_ffn_fwd(xd, r["offsets"], w1, w2, mode=mode, want_act=True)
    nb = J.janus_expert_ffn_workspace_size(xd.shape[0], d, h, E, False, True, mode)
    ws = torch.zeros(nb, dtype=torch.uint8, device=DEV)
    y_flag, a_flag = J.janus_expert_ffn_fwd_ex(xd, r["offsets"], w1, w2, flags=J.JANUS_FFN_X_DEQUANTIZED,
                                               mode=mode, want_act=True, workspace=ws)
    J.janus_check(ws)                                   # the rows kept the promise
    assert torch.equal(y_flag, y_plain) and torch.equal(a_flag, a_plain)
    offs = host(r["offsets"])
    rows = sample_rows(offs, 96, seed=3, R=xd.shape[0])
    ref = oracle.expert_ffn_fwd(host(xd), offs, host(w1), host(w2), rows=rows)
    assert rel_fro(host(y_flag)[rows], ref) <= TOL_FP32


def test_dequantized_flag_into_a_row_table():
    # the flag combines with the row-table store of the expert-parallel return
    N, T, E, K, d, h = SHAPES["ragged"]
    xd, r = _packed_rows(N, T, E, K, d, 50)
    w1, w2 = synth.expert_weights(E, d, h, 51, DEV)
    R = xd.shape[0]
    y_plain, _ = J.janus_expert_ffn_fwd(xd, r["offsets"], w1, w2, mode=J.JANUS_FFN_3XTF32)
    dest = torch.full((R + 9, d), float("nan"), device=DEV)
    slot = torch.as_tensor(np.random.default_rng(52).permutation(R + 9)[:R], device=DEV)
    table = dest.data_ptr() + 4 * d * slot.to(torch.int64)
    out, _ = J.janus_expert_ffn_fwd_ex(xd, r["offsets"], w1, w2, out_rows=table,
                                       flags=J.JANUS_FFN_X_DEQUANTIZED, mode=J.JANUS_FFN_3XTF32)
    torch.cuda.synchronize()
    assert out is None and torch.equal(dest[slot], y_plain)


def test_rows_that_break_the_promise_are_reported():
    # plain FP32 rows carry bits below TF32 precision: the call still runs, and
    # janus_check reports the broken promise as a data fault
    E, d, h = 4, 64, 64
    offs = to_dev(np.array([0, 100, 100, 250, 300], np.int32))
    xd = synth.normal((300, d), 60, DEV)
    w1, w2 = synth.expert_weights(E, d, h, 61, DEV)
    nb = J.janus_expert_ffn_workspace_size(300, d, h, E, False, False, J.JANUS_FFN_3XTF32)
    ws = torch.zeros(nb, dtype=torch.uint8, device=DEV)
    J.janus_expert_ffn_fwd_ex(xd, offs, w1, w2, flags=J.JANUS_FFN_X_DEQUANTIZED, mode=J.JANUS_FFN_3XTF32,
                              workspace=ws)
    with pytest.raises(J.JanusError) as e:
        J.janus_check(ws)
    assert e.value.status == J.JANUS_ERR_DATA


# ---------------------------------------------------------------------------
# the forward on the FP16 payload itself.  SIMT: the rows are unpacked first,
# bit-identical to unpack + forward.  3xTF32: the first GEMM multiplies the
# FP16 rows on the kind::f16 tensor path against a two-term FP16 split of
# W1 (per-feature power-of-two scale), so it is compared with the oracle and
# with the unpacked 3xTF32 forward by tolerance, per row as well as overall.
# ---------------------------------------------------------------------------
PACKED = {
    # name: (N, T, E, K, d, h)
    "ragged8": (700, 11, 12, 3, 136, 68),
    "M_like": (4096, 89, 40, 8, 512, 384),
    "tails": (257, 5, 9, 2, 8, 4),
    "wide_k": (300, 7, 3, 2, 1544, 200),       # 24 full 64-wide k-blocks + an 8-wide tail
    # above the library's rows-per-expert threshold, h % 8 == 0: the second GEMM (H W2) runs on
    # the FP16 path too, over a 200-wide K (three 64-wide blocks + an 8 tail)
    "second_f16": (3200, 9, 3, 2, 136, 200),
}


def _packed_inputs(N, T, E, K, d, seed):
    types = to_dev(synth.types_zipf(N, T, seed=seed))
    gate = to_dev(synth.gate_table(T, E, seed + 1))
    x = synth.normal((N, d), seed + 2, DEV)
    r = J.janus_route(types, gate, K)
    payload, scale, _ = J.janus_quant_by_type(x, types, T, r["slot_of"], K)
    return types, r, payload, scale


@pytest.mark.parametrize("mode", [J.JANUS_FFN_FP32_SIMT, J.JANUS_FFN_3XTF32])
@pytest.mark.parametrize("name", list(PACKED))
def test_packed_forward_matches_unpack_then_forward(name, mode):
    N, T, E, K, d, h = PACKED[name]
    types, r, payload, scale = _packed_inputs(N, T, E, K, d, 70)
    w1, w2 = synth.expert_weights(E, d, h, 71, DEV)
    row_scale = J.janus_dispatch_row_scales(types, T, r["perm"], K, scale)
    # the per-row scales are the per-type scales of each row's atom
    ht, hp = host(types), host(r["perm"])
    assert np.array_equal(host(row_scale), host(scale)[ht[hp // K]])
    xd = J.janus_dequant_by_type(payload, types, T, r["perm"], K, scale)
    y_ref, a_ref = J.janus_expert_ffn_fwd_ex(xd, r["offsets"], w1, w2, flags=J.JANUS_FFN_X_DEQUANTIZED, mode=mode,
                                             want_act=True)
    nb = J.janus_expert_ffn_packed_workspace_size(xd.shape[0], E, d, h, mode)
    ws = torch.zeros(nb, dtype=torch.uint8, device=DEV)
    y, a = J.janus_expert_ffn_fwd_packed(payload, row_scale, r["offsets"], w1, w2, mode=mode, want_act=True,
                                         workspace=ws)
    J.janus_check(ws)
    if mode == J.JANUS_FFN_FP32_SIMT:
        assert torch.equal(y, y_ref) and torch.equal(a, a_ref)
    else:
        assert rel_fro(host(a), host(a_ref)) <= TOL_FP32 and rel_fro(host(y), host(y_ref)) <= TOL_FP32
        assert max_row_rel(host(y), host(y_ref)) <= TOL_ROW
        assert torch.isfinite(y).all().item()
    offs = host(r["offsets"])
    rows = sample_rows(offs, 64, seed=5, R=xd.shape[0])
    ref, ref_a = oracle.expert_ffn_fwd(host(xd), offs, host(w1), host(w2), rows=rows, want_act=True)
    assert rel_fro(host(y)[rows], ref) <= TOL_FP32 and rel_fro(host(a)[rows], ref_a) <= TOL_FP32
    assert max_row_rel(host(y)[rows], ref) <= TOL_ROW


def test_packed_forward_weight_split_handles_wide_column_ranges():
    # the FP16 split scales each weight column on its own: a column a million
    # times larger than the rest, an all-zero column, a column of values near
    # 1e-32 and a column whose one entry is 40,000 times its others all stay
    # within the FP32 tolerance of the oracle, column by column
    N, T, E, K, d, h = 600, 7, 4, 2, 128, 72
    types, r, payload, scale = _packed_inputs(N, T, E, K, d, 73)
    w1, w2 = synth.expert_weights(E, d, h, 74, DEV)
    w1[:, :, 3] *= 1.0e6
    w1[:, :, 5] = 0.0
    w1[:, :, 9] *= 1.0e-30
    w1[1, 17, 11] = 1.0e3
    row_scale = J.janus_dispatch_row_scales(types, T, r["perm"], K, scale)
    y, a = J.janus_expert_ffn_fwd_packed(payload, row_scale, r["offsets"], w1, w2, mode=J.JANUS_FFN_3XTF32,
                                         want_act=True)
    torch.cuda.synchronize()
    xd = J.janus_dequant_by_type(payload, types, T, r["perm"], K, scale)
    offs = host(r["offsets"])
    ref_y, ref_a = oracle.expert_ffn_fwd(host(xd), offs, host(w1), host(w2), want_act=True)
    # per feature column of the pre-activation: each is scaled on its own
    ha = host(a).astype(np.float64)
    for f in (0, 3, 9, 11, 40):
        col, rc = ha[:, f], ref_a[:, f].astype(np.float64)
        assert np.linalg.norm(col - rc) <= TOL_FP32 * np.linalg.norm(rc), f
    assert np.all(ha[:, 5] == 0.0)
    assert rel_fro(host(y), ref_y) <= TOL_FP32


def test_fp16_second_gemm_handles_wide_column_ranges_of_w2():
    # the second GEMM's W2 split scales each output feature on its own, and
    # H's split each row: W2 columns far apart in magnitude, an all-zero
    # column and one large entry stay within the FP32 tolerance column by
    # column (6,400 rows over 3 experts put it on the FP16 path)
    N, T, E, K, d, h = 3200, 7, 3, 2, 128, 72
    types, r, payload, scale = _packed_inputs(N, T, E, K, d, 75)
    w1, w2 = synth.expert_weights(E, d, h, 76, DEV)
    w2[:, :, 3] *= 1.0e6
    w2[:, :, 5] = 0.0
    w2[:, :, 9] *= 1.0e-30
    w2[1, 17, 11] = 1.0e3
    row_scale = J.janus_dispatch_row_scales(types, T, r["perm"], K, scale)
    nb = J.janus_expert_ffn_packed_workspace_size(N * K, E, d, h, J.JANUS_FFN_3XTF32)
    ws = torch.zeros(nb, dtype=torch.uint8, device=DEV)
    y, _ = J.janus_expert_ffn_fwd_packed(payload, row_scale, r["offsets"], w1, w2, mode=J.JANUS_FFN_3XTF32,
                                         workspace=ws)
    J.janus_check(ws)
    xd = J.janus_dequant_by_type(payload, types, T, r["perm"], K, scale)
    offs = host(r["offsets"])
    ref_y = oracle.expert_ffn_fwd(host(xd), offs, host(w1), host(w2))
    hy = host(y).astype(np.float64)
    for f in (0, 3, 9, 11, 40):
        col, rc = hy[:, f], ref_y[:, f].astype(np.float64)
        assert np.linalg.norm(col - rc) <= TOL_FP32 * np.linalg.norm(rc), f
    assert np.all(hy[:, 5] == 0.0)
    assert rel_fro(hy, ref_y) <= TOL_FP32


@pytest.mark.parametrize("name", ["ragged8", "second_f16"])
def test_packed_forward_into_a_row_table(name):
    # second_f16: the FP16 second GEMM stores through the row table
    N, T, E, K, d, h = PACKED[name]
    types, r, payload, scale = _packed_inputs(N, T, E, K, d, 80)
    w1, w2 = synth.expert_weights(E, d, h, 81, DEV)
    row_scale = J.janus_dispatch_row_scales(types, T, r["perm"], K, scale)
    R = payload.shape[0]
    y_ref, _ = J.janus_expert_ffn_fwd_packed(payload, row_scale, r["offsets"], w1, w2, mode=J.JANUS_FFN_3XTF32)
    dest = torch.full((R + 5, d), float("nan"), device=DEV)
    slot = torch.as_tensor(np.random.default_rng(82).permutation(R + 5)[:R], device=DEV)
    table = dest.data_ptr() + 4 * d * slot.to(torch.int64)
    out, _ = J.janus_expert_ffn_fwd_packed(payload, row_scale, r["offsets"], w1, w2, out_rows=table,
                                           mode=J.JANUS_FFN_3XTF32)
    torch.cuda.synchronize()
    assert out is None and torch.equal(dest[slot], y_ref)


def test_packed_forward_needs_d_multiple_of_8_on_the_tensor_cores():
    N, T, E, K, d, h = 64, 3, 4, 2, 12, 8
    types, r, payload, scale = _packed_inputs(N, T, E, K, d, 90)
    w1, w2 = synth.expert_weights(E, d, h, 91, DEV)
    row_scale = J.janus_dispatch_row_scales(types, T, r["perm"], K, scale)
    with pytest.raises(J.JanusError) as e:
        J.janus_expert_ffn_fwd_packed(payload, row_scale, r["offsets"], w1, w2, mode=J.JANUS_FFN_3XTF32)
    assert e.value.status == J.JANUS_ERR_MISALIGNED
    # the SIMT path takes any d % 4 == 0
    y, _ = J.janus_expert_ffn_fwd_packed(payload, row_scale, r["offsets"], w1, w2, mode=J.JANUS_FFN_FP32_SIMT)
    xd = J.janus_dequant_by_type(payload, types, T, r["perm"], K, scale)
    y_ref, _ = J.janus_expert_ffn_fwd(xd, r["offsets"], w1, w2, mode=J.JANUS_FFN_FP32_SIMT)
    assert torch.equal(y, y_ref)


def test_row_scales_treat_bad_type_ids_as_type_0_like_the_unpack():
    # the per-row scales and janus_dequant_by_type agree on every row,
    # including atoms whose type id is outside [0, T)
    N, T, E, K, d = 300, 6, 5, 2, 16
    types_np = synth.types_uniform(N, T, 7).astype(np.int32)
    types_np[[3, 50, 299]] = [-1, T, 1000]
    types = to_dev(types_np)
    gate = to_dev(synth.gate_table(T, E, 8))
    r = J.janus_route(to_dev(np.clip(types_np, 0, T - 1)), gate, K)
    scale = to_dev(np.exp2(np.arange(T, dtype=np.float32) - 3.0).astype(np.float32))
    row_scale = J.janus_dispatch_row_scales(types, T, r["perm"], K, scale)
    t_row = types_np[host(r["perm"]) // K]
    t_row = np.where((t_row < 0) | (t_row >= T), 0, t_row)
    assert np.array_equal(host(row_scale), host(scale)[t_row])
    payload = torch.ones((N * K, d), dtype=torch.float16, device=DEV)
    xd = J.janus_dequant_by_type(payload, types, T, r["perm"], K, scale)
    assert np.array_equal(host(xd)[:, 0], host(row_scale))
