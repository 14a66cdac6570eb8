"""GPU parity: dispatch, combine and the per-element-type FP16 packing vs the
oracle (paper review 'Breaking the Training Barrier of Billion-Parameter
Universal Machine Learning Interatomic Potentials', section 3.5: MoE
dispatch/combine kernels and atom-type-aware FP16 compression)."""
import numpy as np
import pytest
import torch

import oracle
from element_routed_moe_b200 import janus as J
from element_routed_moe_b200 import synth
from helpers import DEV, TOL_FP32, host, poison_like, rel_fro, to_dev

pytestmark = pytest.mark.gpu

SHAPES = {
    # name: (N, T, E, K, d)
    "tiny": (512, 8, 8, 2, 64),
    "ragged": (1000, 11, 12, 3, 4 * 37),       # d4 = 37: ragged lane chunk
    "wide": (300, 7, 9, 5, 4 * 300),           # several 128-float4 chunks + tail
    "K40": (200, 5, 48, 40, 64),               # K > 32: slots read from memory
    "S": (8192, 89, 72, 4, 2560),
    "M": (32768, 89, 40, 8, 1536),
}


def _setup(name, seed=0):
    N, T, E, K, d = SHAPES[name]
    types = synth.types_zipf(N, T, seed=seed + 1)
    gate = synth.gate_table(T, E, seed + 2)
    r = oracle.route(types, gate, K)
    x = synth.normal((N, d), seed + 3, DEV)
    return N, T, E, K, d, types, r, x


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("weighted", [False, True])
def test_dispatch_bit_exact(name, weighted):
    N, T, E, K, d, types, r, x = _setup(name)
    w = r["topk_weight"] if weighted else None
    out = poison_like((N * K, d), torch.float32)
    J.janus_dispatch(x, to_dev(r["slot_of"]), K, None if w is None else to_dev(w), out=out)
    ref = oracle.dispatch(host(x), r["perm"], K, w)
    assert np.array_equal(host(out), ref)


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("weighted", [False, True])
def test_combine_parity(name, weighted):
    N, T, E, K, d, types, r, x = _setup(name, seed=4)
    yd = synth.normal((N * K, d), 77, DEV)
    w = r["topk_weight"] if weighted else None
    out = poison_like((N, d), torch.float32)
    J.janus_combine(yd, to_dev(r["slot_of"]), K, None if w is None else to_dev(w), out=out)
    ref = oracle.combine(host(yd), r["slot_of"], K, w)
    got = host(out)
    assert np.all(np.isfinite(got))
    assert rel_fro(got, ref) <= TOL_FP32
    if K == 1 and not weighted:
        assert np.array_equal(got, ref)


def _quant_input(name, seed):
    N, T, E, K, d, types, r, x = _setup(name, seed)
    # per-type magnitudes spanning 7 decades, as different elements would
    mag = torch.as_tensor(10.0 ** (types % 7 - 3), dtype=torch.float32, device=DEV)
    return N, T, E, K, d, types, r, (x * mag[:, None]).contiguous()


@pytest.mark.parametrize("name", list(SHAPES))
def test_quant_dequant_bit_exact(name):
    N, T, E, K, d, types, r, x = _quant_input(name, seed=2)
    payload = poison_like((N * K, d), torch.float16)
    scale = poison_like((T,), torch.float32)
    tdev = to_dev(types)
    p, s, ws = J.janus_quant_by_type(x, tdev, T, to_dev(r["slot_of"]), K, payload=payload, scale=scale)
    J.janus_check(ws)
    ref_p, ref_s = oracle.quant_by_type(host(x), types, T, r["perm"], K)
    assert np.array_equal(host(s), ref_s)
    assert np.array_equal(host(p).view(np.uint16), ref_p)
    assert p.numel() * p.element_size() == (N * K * d * 4) // 2      # half the FP32 bytes
    xd = poison_like((N * K, d), torch.float32)
    J.janus_dequant_by_type(p, tdev, T, to_dev(r["perm"]), K, s, out=xd)
    ref_x = oracle.dequant_by_type(ref_p, types, r["perm"], K, ref_s)
    assert np.array_equal(host(xd), ref_x)


def test_quant_degenerate_and_faults():
    T, K, d = 6, 2, 16
    types = np.array([0, 0, 2, 2, 3], np.int32)      # types 1, 4, 5 absent
    gate = synth.gate_table(T, 4, 0)
    r = oracle.route(types, gate, K)
    x = np.zeros((5, d), np.float32)
    x[2:4] = np.float32(1e-40)                       # subnormal amax
    x[4] = np.float32(3e38)
    p, s, ws = J.janus_quant_by_type(to_dev(x), to_dev(types), T, to_dev(r["slot_of"]), K)
    J.janus_check(ws)
    ref_p, ref_s = oracle.quant_by_type(x, types, T, r["perm"], K)
    assert np.array_equal(host(s), ref_s) and np.array_equal(host(p).view(np.uint16), ref_p)
    # non-finite feature -> data error
    x[1, 3] = np.inf
    _, _, ws = J.janus_quant_by_type(to_dev(x), to_dev(types), T, to_dev(r["slot_of"]), K)
    with pytest.raises(J.JanusError) as e:
        J.janus_check(ws)
    assert e.value.status == J.JANUS_ERR_DATA
    # bad type id -> data error, outputs still written
    bad = types.copy()
    bad[0] = 9
    x[1, 3] = 0.0
    _, _, ws = J.janus_quant_by_type(to_dev(x), to_dev(bad), T, to_dev(r["slot_of"]), K)
    with pytest.raises(J.JanusError):
        J.janus_check(ws)


def test_combine_dispatch_roundtrip_identity():
    N, T, E, K, d, types, r, x = _setup("ragged", seed=9)
    xd = J.janus_dispatch(x, to_dev(r["slot_of"]), K)
    y = J.janus_combine(xd, to_dev(r["slot_of"]), K, to_dev(r["topk_weight"]))
    assert rel_fro(host(y), host(x)) <= 1e-6
