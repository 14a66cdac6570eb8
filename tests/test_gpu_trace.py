"""GPU tests of the launch trace (janus_trace_*): the expert MLP's GEMMs and
splits are recorded in launch order with positive durations, nothing is
recorded after janus_trace_stop or past the capacity, and tracing does not
change results."""
import numpy as np
import pytest
import torch

from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, to_dev

pytestmark = pytest.mark.gpu


def _case():
    counts = [300, 0, 500, 129]
    offs = to_dev(np.array([0, 300, 300, 800, 929], dtype=np.int32))
    E, d, h = len(counts), 136, 96
    w1, w2 = synth.expert_weights(E, d, h, 3, DEV)
    xd = synth.normal((929, d), 4, DEV)
    gd = synth.normal((929, d), 5, DEV)
    return offs, w1, w2, xd, gd


def test_trace_records_the_gemms_in_order():
    offs, w1, w2, xd, gd = _case()
    y0, a0 = J.janus_expert_ffn_fwd(xd, offs, w1, w2, mode=J.JANUS_FFN_3XTF32, want_act=True)
    dx0 = J.janus_expert_ffn_vjp(xd, gd, offs, w1, w2, act=a0, mode=J.JANUS_FFN_3XTF32)
    J.janus_trace_start(16)
    try:
        y, a = J.janus_expert_ffn_fwd(xd, offs, w1, w2, mode=J.JANUS_FFN_3XTF32, want_act=True)
        dx = J.janus_expert_ffn_vjp(xd, gd, offs, w1, w2, act=a, mode=J.JANUS_FFN_3XTF32)
        J.janus_trace_stop()
        J.janus_expert_ffn_fwd(xd, offs, w1, w2, mode=J.JANUS_FFN_3XTF32)     # not recorded
        recs = J.janus_trace_records()
    finally:
        J.janus_trace_release()
    names = [n for n, _ in recs]
    assert names == ["tc_gemm x.W silu tf32x3", "tc_gemm x.W store tf32x3",
                     "tc_gemm x.Wt dsilu tf32x3", "tc_gemm x.Wt store tf32x3"]
    assert all(ms > 0 for _, ms in recs)
    assert torch.equal(y, y0) and torch.equal(a, a0) and torch.equal(dx, dx0)


def test_trace_stops_at_its_capacity_and_names_the_splits():
    offs, w1, w2, xd, gd = _case()
    R = xd.shape[0]
    ident = torch.arange(R, dtype=torch.int32, device=DEV)
    x16, xs = J.janus_dispatch_split(xd, ident, 1)
    J.janus_trace_start(2)
    try:
        J.janus_expert_ffn_fwd_split(x16, xs, offs, w1, w2)
        recs = J.janus_trace_records()
    finally:
        J.janus_trace_release()
    # the weight split, then the first GEMM; the second GEMM is past the capacity
    assert [n for n, _ in recs] == ["w16_split transposed", "tc_gemm x.W silu f16x3"]
    assert J.janus_trace_records() == []          # released
