"""Host-side tests of the C ABI (no GPU needed, no kernel launched).

The library must load, export every entry point include/janus.h declares,
and reject bad arguments before launching anything.  Calls here use fake
device addresses that every checked case rejects first; they are skipped on
a machine with a CUDA device so that a validation bug can never turn into a
launch on a fake address (the GPU suite covers the same checks with real
buffers).
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from element_routed_moe_b200 import build as jbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "janus.h")

no_device = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="fake-pointer validation tests run only without a GPU")


@pytest.fixture(scope="module")
def J():
    jbuild.build()
    from element_routed_moe_b200 import janus
    janus.lib()
    return janus


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(janus_[a-z0-9_]+)\s*\(", src)))


def test_header_symbols_exported(J):
    names = _declared()
    assert "janus_route" in names and "janus_edge_aggregate" in names
    out = subprocess.run(["nm", "-D", "--defined-only", J.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(janus_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert sorted(J.SYMBOLS) == names


def test_status_strings_and_version(J):
    for s in range(5):
        assert J.status_string(s).startswith("JANUS_")
    assert J.status_string(99) == "JANUS_ERR_UNKNOWN"
    assert J.version() == 10000


def test_workspace_queries(J):
    assert J.janus_route_workspace_size(512, 8, 8, 2) >= 256
    with pytest.raises(J.JanusError) as e:
        J.janus_route_workspace_size(10, 8, 8, 9)          # K > E
    assert e.value.status == J.JANUS_ERR_INVALID_ARG
    with pytest.raises(J.JanusError):
        J.janus_route_workspace_size(10, 8, 257, 2)        # E > 256
    with pytest.raises(J.JanusError):
        J.janus_route_workspace_size(2 ** 28, 8, 16, 16)   # N*K >= 2^31
    assert J.janus_quant_by_type_workspace_size(89) == 256 + 512
    nb = J.janus_expert_ffn_workspace_size(1000, 64, 96, 4, False, False)
    assert nb >= 1000 * 96 * 4
    nb2 = J.janus_expert_ffn_workspace_size(1000, 64, 96, 4, True, False)
    assert nb2 >= 2 * 1000 * 96 * 4


FAKE = 0x7f0000000000   # 256-byte aligned fake address, never dereferenced


@no_device
def test_argument_validation_before_launch(J):
    L = J.lib()
    null = None
    # dispatch: d % 4 != 0 -> misaligned; misaligned x; null slot_of
    assert L.janus_dispatch(FAKE, 10, 6, 2, FAKE, null, FAKE, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_dispatch(FAKE + 4, 10, 8, 2, FAKE, null, FAKE, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_dispatch(FAKE, 10, 8, 2, null, null, FAKE, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_dispatch(FAKE, -1, 8, 2, FAKE, null, FAKE, null) == J.JANUS_ERR_INVALID_ARG
    # combine
    assert L.janus_combine(FAKE, FAKE, null, 10, 0, 8, FAKE, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_combine(FAKE, FAKE, null, 10, 2, 8, FAKE + 8, null) == J.JANUS_ERR_MISALIGNED
    # route: workspace too small, K > E, T out of range
    assert L.janus_route(FAKE, 10, FAKE, 4, 4, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16,
                         null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_route(FAKE, 10, FAKE, 4, 4, 5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                         1 << 20, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_route(FAKE, 10, FAKE, 0, 4, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                         1 << 20, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_route(FAKE, 10, FAKE, 4, 4, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 16,
                         1 << 20, null) == J.JANUS_ERR_MISALIGNED
    # quant: workspace too small; payload misaligned
    assert L.janus_quant_by_type(FAKE, 10, 8, 2, FAKE, 4, FAKE, FAKE, FAKE, FAKE, 8,
                                 null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_quant_by_type(FAKE, 10, 8, 2, FAKE, 4, FAKE, FAKE + 2, FAKE, FAKE, 4096,
                                 null) == J.JANUS_ERR_MISALIGNED
    # ffn: bad mode, h % 4, workspace too small
    assert L.janus_expert_ffn_fwd(FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, null, 7, FAKE,
                                  1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_ffn_fwd(FAKE, FAKE, 4, 100, 64, 66, FAKE, FAKE, FAKE, null, 0, FAKE,
                                  1 << 30, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_expert_ffn_fwd(FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, null, 0, FAKE,
                                  1024, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_ffn_vjp(FAKE, null, null, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, 0,
                                  FAKE, 1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    # ffn with a row table: table missing, table misaligned
    assert L.janus_expert_ffn_fwd_rows(FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, null, null, 0, FAKE,
                                       1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_ffn_fwd_rows(FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE + 8, null, 0, FAKE,
                                       1 << 30, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_expert_ffn_vjp_rows(FAKE, FAKE, null, FAKE, 4, 100, 64, 64, FAKE, FAKE, null, 0,
                                       FAKE, 1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    # general forward: both outputs given, unknown flag bits
    assert L.janus_expert_ffn_fwd_ex(FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, FAKE, null, 0, 0, FAKE,
                                     1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_ffn_fwd_ex(FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, null, null, 6, 1, FAKE,
                                     1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    # packed forward: d % 8 on the tensor cores, workspace too small, no row scales
    assert L.janus_expert_ffn_fwd_packed(FAKE, FAKE, FAKE, 4, 100, 12, 64, FAKE, FAKE, FAKE, null, null, null, 0,
                                         1, FAKE, 1 << 30, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_expert_ffn_fwd_packed(FAKE, FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, null, null, null, 0,
                                         0, FAKE, 1024, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_ffn_fwd_packed(FAKE, null, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, null, null, null, 0,
                                         1, FAKE, 1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    # a weight-split set: only on the tensor-core path, large enough, 256-byte aligned
    assert L.janus_expert_ffn_fwd_packed(FAKE, FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, null, null, FAKE,
                                         1 << 30, 0, FAKE, 1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_ffn_fwd_packed(FAKE, FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, null, null, FAKE,
                                         1024, 1, FAKE, 1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_ffn_fwd_split(FAKE, FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, null, null, FAKE + 16,
                                        1 << 30, FAKE, 1 << 30, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_expert_ffn_vjp_split(FAKE, FAKE, FAKE, FAKE, 4, 100, 64, 64, FAKE, FAKE, FAKE, null, FAKE,
                                        1024, FAKE, 1 << 30, null) == J.JANUS_ERR_INVALID_ARG
    # the set's own call: flags, d % 8, size, alignment
    nb = ctypes.c_size_t(0)
    assert L.janus_expert_weights_f16_size(4, 64, 96, ctypes.byref(nb)) == J.JANUS_OK
    # four parts as documented: two f16 planes [E][N][K] and 1/S [E][ceil(K/256)][N] each, 256-byte aligned
    for E, d, h in ((4, 64, 96), (72, 2560, 2560), (3, 264, 776)):
        up = lambda b: -(-b // 256) * 256
        want = sum(up(2 * 2 * E * d * h) + up(4 * E * (-(-kd // 256)) * n) for kd, n in ((d, h), (h, d), (d, h), (h, d)))
        assert J.janus_expert_weights_f16_size(E, d, h) == want
    assert L.janus_expert_weights_f16(FAKE, FAKE, 4, 64, 96, 0, FAKE, nb.value, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_weights_f16(FAKE, FAKE, 4, 64, 96, 4, FAKE, nb.value, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_weights_f16(FAKE, FAKE, 4, 60, 96, 3, FAKE, 1 << 30, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_expert_weights_f16(FAKE, FAKE, 4, 64, 96, 3, FAKE, nb.value - 1, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_expert_weights_f16(FAKE, FAKE, 4, 64, 96, 3, FAKE + 64, nb.value, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_expert_weights_f16(null, FAKE, 4, 64, 96, 3, FAKE, nb.value, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_dispatch_row_scales(10, 2, FAKE, 0, FAKE, FAKE, FAKE, null) == J.JANUS_ERR_INVALID_ARG
    # EP return table: E not a multiple of P, missing peer buffer, d % 4, misaligned table
    two = (ctypes.c_void_p * 2)(FAKE, FAKE)
    assert L.janus_ep_return_rows(FAKE, FAKE, FAKE, 0, 2, 5, 10, 8, two, FAKE, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_ep_return_rows(FAKE, FAKE, FAKE, 0, 2, 4, 10, 8, (ctypes.c_void_p * 2)(FAKE, 0), FAKE,
                                  null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_ep_return_rows(FAKE, FAKE, FAKE, 0, 2, 4, 10, 6, two, FAKE, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_ep_return_rows(FAKE, FAKE, FAKE, 0, 2, 4, 10, 8, two, FAKE + 4, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_ep_return_rows(FAKE, FAKE, FAKE, 0, 2, 4, 0, 8, two, null, null) == J.JANUS_OK
    # edge aggregate: null row_ptr, d % 4, and a null message / gradient /
    # sender array while the CSR has edges (only an edge-free CSR may pass NULL)
    assert L.janus_edge_aggregate(FAKE, 100, null, 10, 8, FAKE, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_edge_aggregate(FAKE, 100, FAKE, 10, 10, FAKE, null) == J.JANUS_ERR_MISALIGNED
    assert L.janus_edge_aggregate(null, 100, FAKE, 10, 8, FAKE, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_edge_aggregate(FAKE, -1, FAKE, 10, 8, FAKE, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_edge_broadcast(FAKE, FAKE, 10, 8, null, 100, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_edge_broadcast(FAKE, null, 10, 8, FAKE, 100, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_neighbor_aggregate(FAKE, FAKE, null, 100, 10, 8, FAKE, null) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_neighbor_aggregate(FAKE, FAKE, FAKE, 100, 10, 6, FAKE, null) == J.JANUS_ERR_MISALIGNED
    # janus_check needs a workspace
    assert L.janus_check(null, null) == J.JANUS_ERR_INVALID_ARG


@no_device
def test_injected_launch_failure_launches_nothing(J):
    L = J.lib()
    J.janus_debug_inject_launch_failures(2)
    assert L.janus_dispatch(FAKE, 10, 8, 2, FAKE, None, FAKE, None) == J.JANUS_ERR_CUDA
    assert L.janus_combine(FAKE, FAKE, None, 10, 2, 8, FAKE, None) == J.JANUS_ERR_CUDA
    J.janus_debug_inject_launch_failures(0)


def test_empty_inputs_are_no_ops(J):
    L = J.lib()
    # n_atoms == 0: nothing to launch, nothing dereferenced
    assert L.janus_dispatch(None, 0, 8, 2, None, None, None, None) == J.JANUS_OK
    assert L.janus_combine(None, None, None, 0, 2, 8, None, None) == J.JANUS_OK
    assert L.janus_edge_aggregate(None, 0, None, 0, 8, None, None) == J.JANUS_OK
    assert L.janus_edge_broadcast(None, None, 0, 8, None, 0, None) == J.JANUS_OK
    assert L.janus_neighbor_aggregate(None, None, None, 0, 0, 8, None, None) == J.JANUS_OK
    assert L.janus_dequant_by_type(None, 0, 8, 2, None, 4, None, None, None, None) == J.JANUS_OK


def test_trace_checks_its_arguments(J):
    # the checks come before any CUDA call: no GPU needed
    L = J.lib()
    assert L.janus_trace_start(0) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_trace_start((1 << 20) + 1) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_trace_count(None) == J.JANUS_ERR_INVALID_ARG
    assert J.janus_trace_records() == []          # nothing recorded
    name, ms = ctypes.c_char_p(), ctypes.c_float()
    assert L.janus_trace_get(0, ctypes.byref(name), ctypes.byref(ms)) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_trace_get(0, None, None) == J.JANUS_ERR_INVALID_ARG
    assert L.janus_trace_stop() == J.JANUS_OK and L.janus_trace_release() == J.JANUS_OK


def test_release_build_reports_no_debug_faults(J):
    assert J.janus_debug_build() is False


def test_product_path_has_no_oracle_dependency():
    pkg = os.path.join(ROOT, "element_routed_moe_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f), errors="ignore").read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "liboracle" not in txt, f
