"""GPU test of janus_quant_by_type_noalloc, the packing entry point for callers
that cannot allocate device memory where they pack.

It is called through the C ABI twice in a row, on different inputs, and each
result must equal (bit for bit, like every packing test here) what the
workspace-taking janus_quant_by_type returns for the same inputs.  The second
call uses much smaller magnitudes, so absmax words left over from the first
call in the library's shared scratch would show up as wrong scales.  This file
sorts last so that a run stopping at the first failure has run everything
else first; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _inputs(seed, magnitude):
    N, T, E, K, d = 3001, 89, 40, 8, 4 * 97
    types = synth.types_zipf(N, T, seed=seed + 1)
    gate = synth.gate_table(T, E, seed + 2)
    r = oracle.route(types, gate, K)
    x = synth.normal((N, d), seed + 3, DEV)
    per_type = torch.as_tensor(magnitude * 10.0 ** (types % 5 - 2), dtype=torch.float32, device=DEV)
    x = (x * per_type[:, None]).contiguous()
    return x, torch.as_tensor(types, device=DEV), T, torch.as_tensor(r["slot_of"], device=DEV), K


def _raw_noalloc(x, types, T, slot_of, K, payload, scale):
    """The entry point called directly through ctypes (no binding logic)."""
    N, d = x.shape
    L = J.lib()
    return L.janus_quant_by_type_noalloc(x.data_ptr(), N, d, K, types.data_ptr(), T,
                                         slot_of.data_ptr(), payload.data_ptr(), scale.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    for call, (seed, mag) in enumerate([(0, 1.0e3), (10, 1.0e-3)]):
        x, types, T, slot_of, K = _inputs(seed, mag)
        ref_p, ref_s, ws = J.janus_quant_by_type(x, types, T, slot_of, K)
        J.janus_check(ws)
        payload = torch.full_like(ref_p, float("nan"))
        scale = torch.full_like(ref_s, float("nan"))
        st = _raw_noalloc(x, types, T, slot_of, K, payload, scale)
        assert st == J.JANUS_OK, J.status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(scale, ref_s), f"call {call}: scales differ"
        assert torch.equal(payload.view(torch.int16), ref_p.view(torch.int16)), f"call {call}: payload differs"


def test_noalloc_binding_and_limits():
    x, types, T, slot_of, K = _inputs(20, 1.0)
    p, s = J.janus_quant_by_type_noalloc(x, types, T, slot_of, K)
    ref_p, ref_s, _ = J.janus_quant_by_type(x, types, T, slot_of, K)
    torch.cuda.synchronize()
    assert torch.equal(s, ref_s) and torch.equal(p.view(torch.int16), ref_p.view(torch.int16))
    # the largest type count the scratch holds is accepted and packs bit for bit
    T_max = 4096
    types_w = torch.as_tensor(synth.types_uniform(x.shape[0], T_max, 21), device=DEV)
    p4, s4 = J.janus_quant_by_type_noalloc(x, types_w, T_max, slot_of, K)
    ref_p4, ref_s4, ws4 = J.janus_quant_by_type(x, types_w, T_max, slot_of, K)
    J.janus_check(ws4)
    torch.cuda.synchronize()
    assert torch.equal(s4, ref_s4) and torch.equal(p4.view(torch.int16), ref_p4.view(torch.int16))
    # more element types than the library-owned scratch holds: rejected before any launch
    big_scale = torch.empty(4097, dtype=torch.float32, device=DEV)
    st = J.lib().janus_quant_by_type_noalloc(x.data_ptr(), x.shape[0], x.shape[1], K, types.data_ptr(),
                                             4097, slot_of.data_ptr(), p.data_ptr(), big_scale.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream)
    assert st == J.JANUS_ERR_INVALID_ARG
