"""Host-side logic of bench.py (no GPU): the GEMM roofline arithmetic over
mixed operand kinds, the launch-trace kind names, the split kernels'
algorithmic bytes, and the traffic record's source check."""
import importlib.util
import os
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class _J:
    JANUS_FFN_FP32_SIMT = 0
    JANUS_FFN_3XTF32 = 1


def test_trace_kind_reads_the_operand_kind(bench):
    assert bench.trace_kind("tc_gemm x.W store f16x2") == ("f16", 2)
    assert bench.trace_kind("tc_gemm x.W store f16x3") == ("f16", 3)
    assert bench.trace_kind("tc_gemm x.Wt dsilu tf32x3") == ("tf32", 3)
    assert bench.trace_kind("tc_gemm x.W silu tf32x2") == ("tf32", 2)


def test_gemm_roofline_is_the_flop_weighted_harmonic_mean(bench):
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1200.0, "sm_max_mhz": 1965.0}
    kinds = [("f16", 2), ("f16", 3), ("tf32", 3), ("tf32", 3)]
    flops = 1e12
    # per-launch peaks: FP16 = the bf16 figure, TF32 = half of it, each / products
    per = [800.0, 1600.0 / 3, 800.0 / 3, 800.0 / 3]
    ideal_s = sum(flops / (p * 1e12) for p in per)
    ms = 2.5 * ideal_s * 1e3                       # a run at 40 % of the ideal
    roof = bench.gemm_roofline(_J, _J.JANUS_FFN_3XTF32, None, kinds, peaks, "measured", flops, ms, 4)
    assert roof["peak_per_gemm"] == pytest.approx(per)
    assert roof["peak"] == pytest.approx(4 * flops / ideal_s / 1e12)
    assert roof["frac"] == pytest.approx(0.4)
    assert roof["achieved"] == pytest.approx(4 * flops / (ms * 1e-3) / 1e12)
    assert roof["frac_of_sustained_peak"] == pytest.approx(0.4 * 1600.0 / 1200.0)
    assert roof["gemm_kinds"] == ["f16x2", "f16x3", "tf32x3", "tf32x3"] and roof["bound"] == "tensor"


def test_gemm_roofline_simt_uses_the_fp32_lanes(bench):
    peaks = {"bf16_tflops": 1600.0, "sm_max_mhz": 2000.0}
    roof = bench.gemm_roofline(_J, _J.JANUS_FFN_FP32_SIMT, None, [("tf32", 3)] * 4, peaks, "measured", 1e12,
                               100.0, 4)
    assert roof["bound"] == "alu"
    assert roof["peak"] == pytest.approx(148 * 128 * 2 * 2000e6 / 1e12)


def test_split_bytes_count_one_read_and_one_write(bench):
    cfg = types.SimpleNamespace(n_rows=1000, d=64, h=32, n_experts=3)
    b = bench.split_bytes(cfg, None)
    assert b["act_split silu"] == 1000 * 32 * 4 * 2 + 1000 * 4
    assert b["act_split dsilu"] == 1000 * 32 * 4 * 3 + 1000 * 4
    assert b["w16_split rows"] == b["w16_split transposed"] == 3 * 64 * 32 * 4 * 2 + 3 * 64 * 4
    # both orientations from one read: W once, four FP16 planes, two scale tables
    assert b["w16_split both"] == 3 * 64 * 32 * 4 + 2 * (3 * 64 * 32 * 4) + 2 * 3 * 64 * 4


def test_code_hash_ignores_comments_and_blank_lines(bench):
    a = "int x = 1;  // one\n\n// a comment line\nint y = 2;\n"
    b = "int x = 1;\nint y = 2;   // two\n"
    assert bench.code_hash(a) == bench.code_hash(b)
    assert bench.code_hash(a) != bench.code_hash("int x = 1;\nint y = 3;\n")


def test_traffic_record_follows_the_gemm_source(bench, monkeypatch):
    rec = bench.GEMM_TRAFFIC[("slice", "3xtf32")]
    with open(os.path.join(ROOT, rec["src"])) as f:
        src = f.read()
    end = src.find(rec["upto"])
    assert end > 0
    # the record matches the GEMM code in the tree, and reads null otherwise
    assert bench.measured_traffic("slice", "3xtf32") == rec["bytes_per_launch"]
    bad = dict(bench.GEMM_TRAFFIC)
    bad[("slice", "3xtf32")] = dict(rec, sha256_prefix="0" * 16)
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", bad)
    assert bench.measured_traffic("slice", "3xtf32") is None
    assert bench.measured_traffic("S", "3xtf32") is None
