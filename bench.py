"""Benchmark of the element-routed MoE layer (forward + input VJP) on B200.

One step = one pass of the MoE layer over one synthetic batch:
    route -> dispatch -> expert MLP fwd -> combine            (forward)
    weighted dispatch of dY -> expert MLP VJP -> combine      (input VJP)
with the edge aggregation in front where the workload has edges (tiny, L, the
interaction-block slice) and the per-element-type FP16 packing in place of the
dispatch where it packs (M, the slice; the payload feeds the first GEMM as it
is).  --mode 3xtf32 (the default) is the FP32-accurate tensor-core mode: the
expert GEMMs run on 3xTF32, or, from 384 rows per expert, on the two-term
FP16 path; --mode simt runs them as FP32 FFMA.

Metric: routed atom-expert tokens/s (tokens = N*K routed rows) per layer pass.
Default workload: the interaction-block slice at the MatRIS-MoE(M) shape
(N=65,536 atoms in a periodic cell at 0.08 atoms/A^3, 6 A cutoff, ~4.74 M
edges with d=1536 messages -> edge aggregation -> route -> FP16-packed
dispatch -> expert MLP fwd + input VJP -> combine; T=89 Zipf(1.1), E=40, K=8,
d=h=1536), the largest configuration that fits one GPU and the only one that
chains every step.  Shapes: model table of the paper review 'Breaking the
Training Barrier of Billion-Parameter Universal Machine Learning Interatomic
Potentials', section 3.1 Table II; block order: section 3.4 Figure 3.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload slice|S|M|L|tiny]
                  [--mode simt|3xtf32] [--impl janus|reference] [--no-cpu-baseline]
Multi-GPU (weak scaling, one independent layer per rank, no collective on the
data path): python -m torch.distributed.run --nproc-per-node N bench.py --gpus N
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from element_routed_moe_b200 import synth  # noqa: E402

METRIC = "routed atom-expert tokens/sec per MoE layer (fwd+VJP)"
UNIT = "tokens/s"
L2_BYTES = 126 * 2 ** 20
SM_COUNT = 148
FP32_LANES_PER_SM = 128


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="slice", choices=list(synth.CONFIGS))
    ap.add_argument("--mode", default="3xtf32", choices=["simt", "3xtf32"])
    ap.add_argument("--impl", default="janus", choices=["janus", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cold", action="store_true", help="skip the cold-L2 timing of the memory-bound kernels")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--atoms", type=int, default=None, help="override N (profiling small cases)")
    ap.add_argument("--experts", type=int, default=None, help="override E (profiling small cases)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism over the ranks (experts split, FP16 all-to-all by peer "
                         "stores) instead of independent replicas")
    ap.add_argument("--ep-return", choices=("fused", "copy"), default="fused",
                    help="--ep: the experts' last GEMM stores into the senders' return buffers (fused) or "
                         "a separate kernel copies the rows back (copy)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip timing the weight-gradient, multi-layer routing and edge-side calls")
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="reference arm: target seconds of oracle work per step")
    return ap.parse_args()


def workload(args):
    import dataclasses
    cfg = synth.CONFIGS[args.workload]
    if args.atoms:
        cfg = dataclasses.replace(cfg, n_atoms=args.atoms)
    if args.experts:
        cfg = dataclasses.replace(cfg, n_experts=args.experts, top_k=min(cfg.top_k, args.experts))
    return cfg


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def describe(cfg) -> dict:
    w = {"tiny": "tiny layer", "S": "MatRIS-MoE(S)-shaped layer", "M": "MatRIS-MoE(M)-shaped layer",
         "L": "MatRIS-MoE(L)-shaped layer", "slice": "interaction-block slice at M shape"}[cfg.name]
    return {
        "workload": f"{w}{'' if cfg == synth.CONFIGS[cfg.name] else ' (resized)'}: "
                    f"N={cfg.n_atoms} atoms, T={cfg.n_types} element types "
                    f"({'Zipf(1.1)' if cfg.type_dist == 'zipf' else 'uniform'}), E={cfg.n_experts}, "
                    f"K={cfg.top_k}, d=h={cfg.d}, FP32, fwd+input-VJP"
                    + (", edge aggregation in front" if cfg.edges != "none" else "")
                    + (", FP16 per-type packed dispatch" if cfg.quant else ""),
        "n_atoms": cfg.n_atoms, "n_types": cfg.n_types, "n_experts": cfg.n_experts,
        "top_k": cfg.top_k, "d": cfg.d, "h": cfg.h, "routed_tokens": cfg.n_rows,
    }


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled every
    `period` seconds by a host thread through NVML (nvidia-smi's own query as
    a fallback) while the timed region runs.  Only samples taken inside the
    timed window are summarised: reading the settings, never changing them."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, uuid: str | None, index: int, period: float = 0.02):
        self.uuid, self.index, self.period = uuid, index, period
        self.samples = []
        self._stop = None
        self._thread = None
        self.source = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.uuid:
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            except pynvml.NVMLError:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def start(self):
        import threading
        try:
            nv, h = self._handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:   # no NVML here: no clock record
            self._thread = None
            return
        self.source = "nvml"
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                t = time.time()
                try:
                    mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                    self.samples.append((t, mhz, pw, rs))
                except Exception:
                    pass
                self._stop.wait(self.period)

        self._nv, self._h = nv, h
        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def sample_now(self):
        """One sample taken at once (the timed region of a small workload can
        be shorter than the sampling period)."""
        if self._thread is None:
            return
        nv, h = self._nv, self._h
        try:
            self.samples.append((time.time(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                 nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                 int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
        except Exception:
            pass

    def stop(self, wall0: float, wall1: float) -> dict | None:
        """Summary of the samples taken between wall0 and wall1 (time.time())."""
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=5)
        inside = [x for x in self.samples if wall0 <= x[0] <= wall1]
        if not inside:
            return {"samples_in_timed_region": 0, "source": self.source, "period_s": self.period,
                    "note": "no sample fell inside the timed region"}
        reasons = sorted({name for _, _, _, rs in inside for name, bit in self.REASONS if rs & bit})
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(x[1] for x in inside), "samples_in_timed_region": len(inside),
                "power_w_max": max(x[2] for x in inside), "reasons": reasons,
                "source": self.source, "period_s": self.period}


# DRAM bytes per launch of the expert-MLP GEMM (mean over a step's four
# launches), from ncu captures of a smaller case of the same workload scaled
# to full size by its routed rows; valid only for the kernel source it was
# taken on (else reported as null).
GEMM_SRC_END = "// ---- the FP16 split of the weights for the kind::f16 GEMMs"
GEMM_TRAFFIC = {
    # the M-shaped MoE layer (the slice's) captured at 12,288 and 16,384 atoms
    # on the FP16 path, each launch kind fitted as a + b * rows and taken to
    # the workload's R; mean of the step's four launches.  The hash covers the
    # GEMM kernel and its launch code (ffn_tc.cu up to the weight-split
    # section) without its comments.
    ("slice", "3xtf32"): {"src": "element_routed_moe_b200/csrc/ffn_tc.cu", "upto": GEMM_SRC_END,
                          "sha256_prefix": "9a893657e4daa214", "bytes_per_launch": 6.678e+09},
    ("M", "3xtf32"): {"src": "element_routed_moe_b200/csrc/ffn_tc.cu", "upto": GEMM_SRC_END,
                      "sha256_prefix": "9a893657e4daa214", "bytes_per_launch": 3.492e+09},
}


def code_hash(text: str) -> str:
    """sha256 prefix of source text with its // comments and blank lines removed."""
    import hashlib
    import re
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()[:16]


def measured_traffic(workload: str, mode: str):
    """The recorded DRAM bytes per GEMM launch, or None once the GEMM's code
    (the file up to the marker) differs from the code the counters came from."""
    rec = GEMM_TRAFFIC.get((workload, mode))
    if rec is None:
        return None
    with open(os.path.join(ROOT, rec["src"])) as f:
        src = f.read()
    end = src.find(rec["upto"])
    if end < 0 or code_hash(src[:end]) != rec["sha256_prefix"]:
        return None
    return rec["bytes_per_launch"]


def measured_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0}, "fallback"


# --------------------------------------------------------------------------
# the layer pass through the C ABI (device-resident inputs)
# --------------------------------------------------------------------------
class Layer:
    """Synthetic inputs of one workload and the library's MoELayer over them."""

    def __init__(self, cfg, mode: int, seed: int, dev):
        from element_routed_moe_b200 import janus as J
        from element_routed_moe_b200.layer import MoELayer
        self.J = J
        self.cfg = cfg
        self.mode = mode
        self.edges = cfg.edges != "none"  # the tiny, L and slice configs aggregate edge messages first
        self.packed = cfg.quant           # the M and slice configs name the FP16-packed dispatch
        inp = synth.layer_inputs(cfg, seed=seed, device=dev, with_edges=self.edges)
        self.inp = inp
        self.types = torch.as_tensor(inp["types"], device=dev)
        self.gate = torch.as_tensor(inp["gate"], device=dev)
        self.w1, self.w2 = inp["w1"], inp["w2"]
        self.x, self.g = inp["x"], inp["g"]
        if self.edges:
            self.msg = inp["msg"]
            self.row_ptr = torch.as_tensor(inp["row_ptr"], device=dev)
        self.core = MoELayer(cfg.n_atoms, cfg.top_k, self.gate, self.w1, self.w2, mode=mode, packed=self.packed,
                             row_ptr=self.row_ptr if self.edges else None)
        c = self.core
        self.route_out, self.route_ws = c.route_out, c.route_ws
        self.xd, self.gd, self.act, self.y, self.dx = c.xd, c.gd, c.act, c.y, c.dx
        if self.edges:
            self.xagg = c.xagg
        self.ops = c.ops
        self.launches_per_step = c.launches_per_call

    def step(self, x=None, g=None, types=None, events=None):
        """One layer pass.  events: dict op -> (start, end) CUDA events, or None."""
        x = (self.msg if self.edges else self.x) if x is None else x
        g = self.g if g is None else g
        types = self.types if types is None else types
        return self.core.forward_vjp(x, g, types, events=events)

    # algorithmic bytes (memory-bound ops) and FLOPs (expert MLP) per call
    def work(self):
        c = self.cfg
        N, R, d, h = c.n_atoms, c.n_rows, c.d, c.h
        split, split_vjp = self.core.split, self.core.split_vjp
        w = {
            # split dispatch: a first pass reads X for the row maxima; the two
            # FP16 planes are as many bytes as the FP32 rows, plus a scale per row
            "dispatch": ("bytes", 4 * d * (N + R) + 4 * R + ((4 * N * d + 4 * R) if split else 0)),
            "dispatch_w": ("bytes", 4 * d * (N + R) + 8 * R + ((4 * N * d + 4 * R) if split_vjp else 0)),
            "combine": ("bytes", 4 * d * (R + N) + 8 * R),
            "combine_vjp": ("bytes", 4 * d * (R + N) + 4 * R),
            "ffn_fwd": ("flops", 4 * R * d * h),
            "ffn_vjp": ("flops", 4 * R * d * h),
            "route": ("bytes", 4 * N + 8 * R * 2 + 8 * R),
        }
        if self.edges:
            Ed = int(self.inp["row_ptr"][-1])
            w["edge_aggregate"] = ("bytes", 4 * Ed * d + 4 * N * d + 8 * (N + 1))
        if self.packed:
            w["quant"] = ("bytes", 4 * N * d * 2 + 2 * R * d + 4 * R)
            w["dequant"] = ("bytes", 2 * R * d + 4 * R * d + 8 * R)
            w["row_scales"] = ("bytes", 12 * R)      # perm + the row's type + the scale written
        return w


# --------------------------------------------------------------------------
# CPU oracle timing (the reported CPU baseline; never the product path)
# --------------------------------------------------------------------------
def oracle_pass(cfg, host_inp, n: int) -> float:
    """Wall time of the oracle's layer pass on the first n atoms of the
    workload, with the full expert weights: the same chain as the GPU step
    (edge aggregation first where there are edges, FP16 pack and unpack in place of
    the dispatch where the config packs; route, FFN fwd, combine, weighted
    dispatch, FFN VJP, combine)."""
    import oracle
    types = host_inp["types"][:n]
    x, g = host_inp["x"][:n], host_inp["g"][:n]
    w1, w2 = host_inp["w1"], host_inp["w2"]
    K = cfg.top_k
    msg = rp = None
    if "row_ptr" in host_inp:            # the first n receivers' edge messages (copied before timing)
        rp = host_inp["row_ptr"][:n + 1]
        msg = host_inp["msg"][:int(rp[-1])].cpu().numpy()
    t0 = time.perf_counter()
    if msg is not None:
        x = oracle.edge_aggregate(msg, rp)
    r = oracle.route(types, host_inp["gate"], K)
    if cfg.quant:
        q, sc = oracle.quant_by_type(x, types, cfg.n_types, r["perm"], K)
        xd = oracle.dequant_by_type(q, types, r["perm"], K, sc)
    else:
        xd = oracle.dispatch(x, r["perm"], K)
    yd = oracle.expert_ffn_fwd(xd, r["offsets"], w1, w2)
    oracle.combine(yd, r["slot_of"], K, r["topk_weight"])
    gd = oracle.dispatch(g, r["perm"], K, r["topk_weight"])
    dxd = oracle.expert_ffn_vjp(xd, gd, r["offsets"], w1, w2)
    oracle.combine(dxd, r["slot_of"], K)
    return time.perf_counter() - t0


def oracle_calibrate(cfg, host_inp, target_s: float) -> int:
    """Number of atoms whose oracle pass takes about target_s seconds (at
    most host_inp["max_atoms"] when given)."""
    n_max = int(host_inp.get("max_atoms", cfg.n_atoms))
    n = min(4, n_max)
    dt = oracle_pass(cfg, host_inp, n)
    while dt < 0.1 * target_s and n < n_max:
        n = min(n_max, n * 4)
        dt = oracle_pass(cfg, host_inp, n)
    return int(min(n_max, max(1, n * target_s / max(dt, 1e-6))))


def host_inputs(cfg, layer):
    h = dict(types=np.asarray(layer.inp["types"]), gate=np.asarray(layer.inp["gate"]),
             x=layer.x.cpu().numpy(), g=layer.g.cpu().numpy(),
             w1=layer.w1.cpu().numpy(), w2=layer.w2.cpu().numpy())
    if layer.edges:   # the messages stay on the device; a sample's rows are copied when timed
        h.update(row_ptr=np.asarray(layer.inp["row_ptr"]), msg=layer.msg)
    return h


def cpu_descr():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# --------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# --------------------------------------------------------------------------
def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle
    cfg = workload(args)
    inp = synth.layer_inputs(cfg, seed=args.seed, device="cpu", with_edges=False)
    host = dict(types=inp["types"], gate=inp["gate"], x=inp["x"].numpy(), g=inp["g"].numpy(),
                w1=inp["w1"].numpy(), w2=inp["w2"].numpy())
    if cfg.edges != "none":
        # the same receiver-sorted CSR as the GPU arm; messages only for the
        # first atoms the sample can reach (the full tensor is 9-29 GB)
        if cfg.edges == "random":
            rp, _, _ = synth.edges_random(cfg.n_atoms, cfg.edges_per_atom, args.seed + 6)
        else:
            rp, _, _ = synth.edges_pbc(cfg.n_atoms, args.seed + 6)
        cap = min(cfg.n_atoms, 2048)
        host.update(row_ptr=rp, msg=synth.normal((int(rp[cap]), cfg.d), args.seed + 8), max_atoms=cap)
    per_step = args.ref_seconds or max(2.0, min(15.0, 150.0 / max(1, args.steps + args.warmup)))
    n_s = oracle_calibrate(cfg, host, per_step)
    times = []
    for i in range(args.warmup + args.steps):
        dt = oracle_pass(cfg, host, n_s)
        if i >= args.warmup:
            times.append(dt)
    t = float(np.mean(times))
    value = n_s * cfg.top_k / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": describe(cfg),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"first {n_s} of {cfg.n_atoms} atoms ({n_s * cfg.top_k} routed tokens) "
                                   f"per step, full expert weights; host {cpu_descr()}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# janus arm
# --------------------------------------------------------------------------
TRACE_PER_STEP = 32     # traced launches per layer pass: 4 GEMMs + up to 6 splits, with room


def trace_kind(name):
    """(operand kind, products) from a GEMM's trace name, e.g. 'tc_gemm x.W
    store f16x3' -> ('f16', 3)."""
    ops = name.split()[-1]
    return ("f16" if ops.startswith("f16") else "tf32"), int(ops[-1])


def split_bytes(cfg, layer):
    """Algorithmic bytes of one launch of each traced split kind: the
    activation split reads a (and dH for dSiLU) once and writes the two FP16
    planes and a scale per row; the weight split reads one expert matrix and
    writes its two FP16 planes and a scale per output feature; the split of
    both orientations reads it once and writes four planes and both scale
    tables."""
    R, d, h, E = cfg.n_rows, cfg.d, cfg.h, cfg.n_experts
    return {
        "act_split silu": 4 * R * h + 4 * R * h + 4 * R,
        "act_split dsilu": 8 * R * h + 4 * R * h + 4 * R,
        "w16_split transposed": 4 * E * d * h + 4 * E * d * h + 4 * E * max(d, h),
        "w16_split rows": 4 * E * d * h + 4 * E * d * h + 4 * E * max(d, h),
        "w16_split both": 4 * E * d * h + 8 * E * d * h + 8 * E * max(d, h),
    }


def gemm_roofline(J, mode, cfg, kinds, peaks, peak_src, flops_per_gemm, ms_total, launches):
    """Roofline of the grouped expert-MLP GEMM over a step's launches.

    Each launch's FP32-accurate peak is the tensor peak of the operand kind it
    runs on divided by the products it issues per k-step:
      3xTF32 (every GEMM on FP32 rows): TF32 peak / 3, with TF32 peak =
        measured burst BF16 x the nominal TF32/BF16 ratio (1.125 / 2.25);
      FP16 rows x two-term FP16 split of the weights (the packed forward's
        first GEMM): FP16 peak / 2, FP16 peak = the measured burst BF16 figure
        (the same nominal rate);
      two-term FP16 rows x two-term FP16 weights (the first GEMM of each
        direction on split rows): FP16 peak / 3;
      unpacked FP16 rows on TF32 (packed layers with d % 8 != 0): TF32 / 2.
    `kinds` lists each launch's (kind, products) in step order.
    The combined peak is the FLOP-weighted harmonic mean, so frac = (sum of
    each launch's ideal time) / (measured time).  SIMT: 148 SMs x 128 FP32
    lanes x 2 FLOP x the maximum SM clock, the same for every launch."""
    bf16 = peaks["bf16_tflops"]
    tf32 = bf16 * (1.125 / 2.25)
    if mode == J.JANUS_FFN_FP32_SIMT:
        per = [SM_COUNT * FP32_LANES_PER_SM * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12] * launches
        roof = {"bound": "alu", "peak_source": "148 SMs x 128 FP32 lanes x 2 FLOP x max SM clock"}
    else:
        per = [(bf16 if k == "f16" else tf32) / p for k, p in kinds]
        roof = {"bound": "tensor",
                "peak_source": f"{peak_src} burst bf16 (FP16 kind; x 1.125/2.25 for TF32) / products per GEMM "
                               f"{[f'{k}x{p}' for k, p in kinds]}",
                "gemm_kinds": [f"{k}x{p}" for k, p in kinds]}
    flops = flops_per_gemm * launches
    ideal_s = sum(flops_per_gemm / (pk * 1e12) for pk in per)
    peak = flops / ideal_s / 1e12
    achieved = flops / (ms_total * 1e-3) / 1e12
    roof.update({"kernel": "grouped expert-MLP GEMM", "achieved": achieved, "peak": peak,
                 "peak_per_gemm": per, "unit": "TFLOP/s", "frac": achieved / peak,
                 "frac_of_sustained_peak": achieved / (peak * peaks.get("bf16_tflops_sustained", bf16) / bf16),
                 "algorithmic_flops_per_launch": flops_per_gemm, "launches_per_step": launches})
    return roof


def run_janus(args, world, rank, local):
    from element_routed_moe_b200 import janus as J
    J.lib()   # fails loudly if the CUDA library is missing
    dev = torch.device("cuda", local)
    cfg = workload(args)
    mode = J.JANUS_FFN_3XTF32 if args.mode == "3xtf32" else J.JANUS_FFN_FP32_SIMT
    layer = Layer(cfg, mode, seed=args.seed + 1000 * rank, dev=dev)
    work = layer.work()
    peaks, peak_src = measured_peaks()

    for _ in range(args.warmup):
        layer.step()
    torch.cuda.synchronize()
    J.janus_check(layer.route_ws)

    ev = [{op: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for op in layer.ops} for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else None, local)
    sampler.start()
    time.sleep(0.1)
    barrier(world)
    torch.cuda.synchronize()
    # the library's launch trace brackets each expert-MLP GEMM (and the
    # weight / activation splits around them) with CUDA events on the
    # launching stream, so the GEMM roofline uses the kernels' own durations
    J.janus_trace_start(args.steps * TRACE_PER_STEP)
    wall0 = time.time()
    t_start.record()
    for k in range(args.steps):
        layer.step(events=ev[k])
    t_end.record()
    sampler.sample_now()        # while the enqueued steps run
    torch.cuda.synchronize()
    wall1 = time.time()
    J.janus_trace_stop()
    trace = J.janus_trace_records()
    J.janus_trace_release()
    clocks = sampler.stop(wall0, wall1)
    barrier(world)
    elapsed = t_start.elapsed_time(t_end) / 1e3
    t_max = max_over_ranks(elapsed, world)
    tokens = cfg.n_rows * args.steps * world
    value = tokens / t_max

    op_ms = {op: float(np.mean([e[op][0].elapsed_time(e[op][1]) for e in ev])) for op in layer.ops}
    kernels = {}
    for op, (kind, amount) in work.items():
        if op not in op_ms or kind != "bytes" or op == "route":
            continue
        gbs = amount / (op_ms[op] * 1e-3) / 1e9
        kernels[op] = {"ms": op_ms[op], "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                       "algorithmic_bytes": amount}
    kernels["route"] = {"ms": op_ms["route"]}

    # roofline of the dominant kernel: the grouped expert-MLP GEMM (4 launches
    # per step: two forward, two VJP, each 2*R*d*h FLOPs), each launch timed
    # by the library's trace events on the launching stream inside the timed
    # steps (the SIMT path is not traced: there the FFN calls' events)
    ffn_ms = op_ms["ffn_fwd"] + op_ms["ffn_vjp"]
    flops_per_gemm = work["ffn_fwd"][1] / 2
    gemms = [(n, ms) for n, ms in trace if n.startswith("tc_gemm")]
    if mode == J.JANUS_FFN_3XTF32 and len(gemms) == 4 * args.steps:
        kinds = [trace_kind(n) for n, _ in gemms[:4]]
        gemm_ms = sum(ms for _, ms in gemms) / args.steps
        roof = gemm_roofline(J, mode, cfg, kinds, peaks, peak_src, flops_per_gemm, gemm_ms, 4)
        per_launch = []
        for j in range(4):
            ms_j = float(np.mean([gemms[4 * k + j][1] for k in range(args.steps)]))
            tf = flops_per_gemm / (ms_j * 1e-3) / 1e12
            per_launch.append({"kernel": gemms[j][0], "ms": ms_j, "TFLOP/s": tf,
                               "frac": tf / roof["peak_per_gemm"][j]})
        roof["per_launch"] = per_launch
        roof["timing"] = "library trace events around each GEMM launch, mean over the timed steps"
        roof["ffn_calls_ms"] = ffn_ms      # the MLP calls with their weight and activation splits
    else:
        kinds = [("tf32", 3)] * 4
        roof = gemm_roofline(J, mode, cfg, kinds, peaks, peak_src, flops_per_gemm, ffn_ms, 4)
        roof["timing"] = "CUDA events around the expert-MLP calls"
    # the splits around the FP16 GEMMs: memory-bound, from the same trace
    for name, nbytes in split_bytes(cfg, layer).items():
        rec = [ms for n, ms in trace if n == name]
        if rec:
            ms = float(np.sum(rec)) / args.steps
            per = len(rec) // args.steps
            gbs = nbytes * per / (ms * 1e-3) / 1e9
            kernels[name] = {"ms": ms, "launches_per_step": per, "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                             "algorithmic_bytes": nbytes * per}
    roof["traffic"] = measured_traffic(cfg.name, args.mode) if cfg == synth.CONFIGS[cfg.name] else None
    roof["traffic_unit"] = "DRAM bytes per launch (mean of the step's 4 launches)"
    ws_gb = ((layer.w1.numel() + layer.w2.numel()) * 4 + cfg.n_rows * cfg.d * 4 * 4) / 1e9
    if layer.edges:
        ws_gb += layer.msg.numel() * 4 / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {**describe(cfg), "ffn_mode": args.mode, "parallelism": f"replicas x{world}",
                   "l2": f"no flush between steps: each step streams {ws_gb:.1f} GB (weights, activations"
                         f"{', edge messages' if layer.edges else ''}) >> the 126 MB L2; cold-L2 figures of the "
                         f"memory-bound kernels under kernels_cold_l2"},
        "roofline": roof,
        "kernels": kernels,
        "breakdown_ms": op_ms,
        "gpu_launches": layer.launches_per_step * args.steps,
        "clocks": clocks,
    }
    if not args.no_cold:
        line["kernels_cold_l2"] = run_cold_l2(layer, peaks)
    if not args.no_e2e:
        line["e2e"] = run_e2e(layer, args)
    if not args.no_extras:
        line["extras"] = run_extras(layer, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = host_inputs(cfg, layer)
        n_s = oracle_calibrate(cfg, host, 15.0)
        dt = oracle_pass(cfg, host, n_s)
        import oracle
        line["cpu_baseline"] = {
            "value": n_s * cfg.top_k / dt, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"first {n_s} of {cfg.n_atoms} atoms ({n_s * cfg.top_k} routed tokens), "
                      f"full expert weights, {dt:.1f} s; host {cpu_descr()}"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_cold_l2(layer, peaks, reps=5):
    """The memory-bound kernels of the step timed one call at a time with the
    L2 flushed before each call (a 2x-L2 buffer written in between, outside
    the timed events): median of `reps` calls, next to the in-step figures."""
    J = layer.J
    cfg = layer.cfg
    K, T = cfg.top_k, cfg.n_types
    r = layer.route_out
    core = layer.core
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=layer.x.device)
    x = core.xagg if layer.edges else layer.x
    calls = {
        "dispatch": lambda: J.janus_dispatch(x, r["slot_of"], K, out=layer.xd),
        "dispatch_w": lambda: J.janus_dispatch(layer.g, r["slot_of"], K, r["topk_weight"], out=layer.gd),
    }
    # the calls the step makes: the split dispatch on the FP16 tensor path
    if core.split:
        calls["dispatch"] = lambda: J.janus_dispatch_split(x, r["slot_of"], K, out=core.xd16, row_scale=core.xd_scale,
                                                           workspace=core.split_ws)
    if core.split_vjp:
        calls["dispatch_w"] = lambda: J.janus_dispatch_split(layer.g, r["slot_of"], K, r["topk_weight"],
                                                             out=core.gd16, row_scale=core.gd_scale,
                                                             workspace=core.split_ws)
    calls.update({
        "combine": lambda: J.janus_combine(core.yd, r["slot_of"], K, r["topk_weight"], out=layer.y),
        "combine_vjp": lambda: J.janus_combine(core.dxd, r["slot_of"], K, out=layer.dx),
    })
    if layer.edges:
        calls["edge_aggregate"] = lambda: J.janus_edge_aggregate(layer.msg, layer.row_ptr, out=core.xagg)
    if layer.packed:
        calls["quant"] = lambda: J.janus_quant_by_type(x, layer.types, T, r["slot_of"], K, payload=core.payload,
                                                       scale=core.scale, workspace=core.quant_ws)
        calls["dequant"] = lambda: J.janus_dequant_by_type(core.payload, layer.types, T, r["perm"], K, core.scale,
                                                           out=layer.xd)
    work = layer.work()
    out = {}
    for op, fn in calls.items():
        fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ms = statistics.median(ts)
        amount = work[op][1]
        out[op] = {"ms": ms, "GB/s": amount / (ms * 1e-3) / 1e9,
                   "frac_hbm": amount / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "algorithmic_bytes": amount}
    del flush
    return out


def run_ep(args, world, rank, local):
    """The layer pass with experts split over the ranks (each rank: its own
    N atoms, E/P experts); same metric, whole-job tokens per second."""
    from element_routed_moe_b200 import janus as J
    from element_routed_moe_b200.ep import ExpertParallelLayer
    J.lib()
    dev = torch.device("cuda", local)
    cfg = workload(args)
    N, T, E, K, d, h = cfg.n_atoms, cfg.n_types, cfg.n_experts, cfg.top_k, cfg.d, cfg.h
    if E % world:
        raise SystemExit(f"--ep needs E ({E}) divisible by the number of ranks ({world})")
    mode = J.JANUS_FFN_3XTF32 if args.mode == "3xtf32" else J.JANUS_FFN_FP32_SIMT
    inp = synth.layer_inputs(cfg, seed=args.seed + 1000 * rank, device=dev, with_edges=False)
    gate = torch.as_tensor(synth.gate_table(T, E, args.seed + 2), device=dev)     # the same on every rank
    w1, w2 = synth.expert_weights(E, d, h, args.seed + 3, dev)
    El = E // world
    w1l, w2l = w1[rank * El:(rank + 1) * El].contiguous(), w2[rank * El:(rank + 1) * El].contiguous()
    del w1, w2, inp["w1"], inp["w2"]
    types = torch.as_tensor(inp["types"], device=dev)
    x, g = inp["x"], inp["g"]
    layer = ExpertParallelLayer(N, d, h, T, E, K, w1l, w2l, mode=mode, device=dev,
                                fused_return=args.ep_return == "fused")
    peaks, peak_src = measured_peaks()
    for _ in range(args.warmup):
        layer.forward(x, types, gate)
        layer.vjp(g)
    torch.cuda.synchronize()
    phases = ExpertParallelLayer.PHASES_FWD + ExpertParallelLayer.PHASES_VJP
    ev = [{ph: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for ph in phases}
          for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else None, local)
    sampler.start()
    time.sleep(0.1)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.time()
    t_start.record()
    for k in range(args.steps):
        layer.forward(x, types, gate, events=ev[k])
        layer.vjp(g, events=ev[k])
    t_end.record()
    sampler.sample_now()
    torch.cuda.synchronize()
    wall1 = time.time()
    clocks = sampler.stop(wall0, wall1)
    barrier(world)
    elapsed = t_start.elapsed_time(t_end) / 1e3
    t_max = max_over_ranks(elapsed, world)
    value = N * K * world * args.steps / t_max
    ph_ms = {ph: float(np.mean([e[ph][0].elapsed_time(e[ph][1]) for e in ev])) for ph in phases}
    # this rank's expert GEMMs: 4 of 2 * R_recv * d * h FLOPs each (fwd + VJP)
    r_recv = int(layer.layout[2][rank][-1].item())
    ffn_ms = ph_ms["ffn_fwd"] + ph_ms["ffn_vjp"]
    # the owner's first forward GEMM runs on the received FP16 rows: 2 products
    kinds = [("f16", 2) if layer.fused_unpack else ("tf32", 2), ("f16", 3) if layer.f16_second else ("tf32", 3)]
    kinds += [("f16", 3)] * 2 if layer.split_vjp else [("tf32", 3)] * 2
    roof = gemm_roofline(J, mode, cfg, kinds, peaks, peak_src, 2.0 * r_recv * d * h, max(ffn_ms, 1e-9), 4)
    roof.update({"kernel": "grouped expert-MLP GEMM (rank 0's experts; ffn phases include the FP16 unpack)",
                 "traffic": None})
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {**describe(cfg), "ffn_mode": args.mode, "parallelism": f"ep{world}",
                   "experts_per_rank": El, "received_rows_rank0": r_recv, "ep_return": args.ep_return,
                   "l2": "no flush: per-step working set far above the 126 MB L2"},
        "roofline": roof,
        "breakdown_ms": ph_ms,
        "gpu_launches": layer.launches_per_step * args.steps,
        "clocks": clocks,
    }
    layer.close()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _time_ms(fn, reps=5):
    fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def run_extras(layer, peaks):
    """Calls outside the layer pass, timed separately (not part of `value`):
    expert weight gradients, routing of 12 MoE layers at once vs one by one,
    and (workloads with edges) the edge-side gradient and sender-indexed gather."""
    J = layer.J
    cfg = layer.cfg
    N, R, d, h, E, K, T = cfg.n_atoms, cfg.n_rows, cfg.d, cfg.h, cfg.n_experts, cfg.top_k, cfg.n_types
    r = layer.route_out
    out = {}
    # the weight-gradient extras take the FP32 dispatch rows, which the step
    # does not write on its FP16 tensor path (FP16 payload or split rows):
    # written here, untimed
    x_in = layer.core.xagg if layer.edges else layer.x
    if layer.core.packed:
        J.janus_dequant_by_type(layer.core.payload, layer.types, T, r["perm"], K, layer.core.scale, out=layer.xd)
    else:
        J.janus_dispatch(x_in, r["slot_of"], K, out=layer.xd)
    J.janus_dispatch(layer.g, r["slot_of"], K, r["topk_weight"], out=layer.gd)
    dw1 = torch.empty_like(layer.w1)
    dw2 = torch.empty_like(layer.w2)
    ws = torch.empty(J.janus_expert_ffn_weight_grad_workspace_size(R, h, True), dtype=torch.uint8,
                     device=layer.x.device)
    ms = _time_ms(lambda: J.janus_expert_ffn_weight_grad(layer.xd, layer.gd, r["offsets"], layer.w1, layer.w2,
                                                          act=layer.act, mode=layer.mode, dw1=dw1, dw2=dw2,
                                                          workspace=ws))
    out["expert_weight_grad"] = {"ms": ms, "gemms": 3, "TFLOP/s": 6 * R * d * h / (ms * 1e-3) / 1e12}
    # second-order pass (VJP of the input VJP) with its weight part: 7 GEMMs
    # of 2*R*d*h each (dh, v W1, t1 W2, t2 W1^T, T1^T Gd, Vd^T U, Xd^T T2)
    vd = synth.normal((R, d), 77, layer.x.device)    # cotangent of the input VJP
    d_x = torch.empty_like(layer.xd)
    d_g = torch.empty_like(layer.xd)
    ws2 = torch.empty(J.janus_expert_ffn_vjp_vjp_workspace_size(R, h, True, True), dtype=torch.uint8,
                      device=layer.x.device)
    ms2 = _time_ms(lambda: J.janus_expert_ffn_vjp_vjp(layer.xd, layer.gd, vd, r["offsets"], layer.w1,
                                                      layer.w2, act=layer.act, mode=layer.mode, weight_grad=True,
                                                      d_xd=d_x, d_gd=d_g, dw1=dw1, dw2=dw2, workspace=ws2))
    out["expert_second_order"] = {"ms": ms2, "gemms": 7, "TFLOP/s": 14 * R * d * h / (ms2 * 1e-3) / 1e12}
    del dw1, dw2, ws, d_x, d_g, ws2, vd
    L = 12   # 6 interaction blocks x 2 MoE layers
    gates = torch.as_tensor(np.stack([synth.gate_table(T, E, 500 + l) for l in range(L)]), device=layer.x.device)
    ws_l = torch.empty(J.janus_route_layers_workspace_size(N, T, E, K, L), dtype=torch.uint8,
                       device=layer.x.device)
    ms_layers = _time_ms(lambda: J.janus_route_layers(layer.types, gates, K, workspace=ws_l))
    ms_single = _time_ms(lambda: [J.janus_route(layer.types, gates[l], K, out=r, workspace=layer.route_ws)
                                  for l in range(L)])
    out["route_12_layers"] = {"ms_one_call": ms_layers, "ms_12_calls": ms_single}
    if layer.edges:
        Ed = int(layer.inp["row_ptr"][-1])
        dmsg = torch.empty_like(layer.msg)
        ms_b = _time_ms(lambda: J.janus_edge_broadcast(layer.dx, layer.row_ptr, out=dmsg), reps=3)
        bb = 4 * N * d + 4 * Ed * d + 8 * (N + 1)
        out["edge_broadcast"] = {"ms": ms_b, "GB/s": bb / (ms_b * 1e-3) / 1e9,
                                 "frac_hbm": bb / (ms_b * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        senders = torch.as_tensor(layer.inp["senders"].astype(np.int32), device=layer.x.device)
        y = torch.empty_like(layer.xagg)
        ms_n = _time_ms(lambda: J.janus_neighbor_aggregate(layer.xagg, layer.row_ptr, senders, out=y), reps=3)
        gathered = 4 * Ed * d + 4 * Ed + 8 * (N + 1) + 4 * N * d
        out["neighbor_aggregate"] = {"ms": ms_n, "gathered_GB/s": gathered / (ms_n * 1e-3) / 1e9,
                                     "note": "gathered bytes (rows re-read through L2) per second"}
        del dmsg, y
    return out


def _pinned_copy(t):
    """Host copy of device tensor t in page-locked memory, registered in place
    (cudaHostRegister: no rounding of the size, unlike the caching pinned
    allocator); release with _unpin."""
    h = torch.empty(t.shape, dtype=t.dtype)
    err = torch.cuda.cudart().cudaHostRegister(h.data_ptr(), h.numel() * h.element_size(), 0)
    if int(err) != 0:
        raise RuntimeError(f"cudaHostRegister failed ({err})")
    h.copy_(t)
    return h


def _unpin(*ts):
    torch.cuda.synchronize()
    for t in ts:
        torch.cuda.cudart().cudaHostUnregister(t.data_ptr())


def run_e2e(layer, args):
    """Same metric through the library's MoELayer.run_host with the step's
    inputs in pinned host memory: every step uploads its inputs (the node
    features x, or the edge messages where the workload aggregates them; dY;
    types) and downloads its results (y, dX) inside the timed region.  The
    copies run on their own streams: dY's upload overlaps the forward, y's
    download the VJP, the next step's upload this step's compute; edge
    messages stream through a ring of device buffers, each chunk aggregated as
    it lands.  The receiver graph (row_ptr, 8 (N+1) bytes) is the layer's own,
    uploaded once when the layer is built."""
    core = layer.core
    x_h = _pinned_copy(layer.msg if layer.edges else layer.x)
    g_h = _pinned_copy(layer.g)
    t_h = _pinned_copy(layer.types)
    y_h = _pinned_copy(layer.y)
    dx_h = _pinned_copy(layer.dx)
    try:
        for _ in range(args.warmup):
            core.run_host(x_h, g_h, t_h, y_h, dx_h)
        core.host_sync()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            core.run_host(x_h, g_h, t_h, y_h, dx_h)
        core.host_sync()
        b.record()
        torch.cuda.synchronize()
        t = a.elapsed_time(b) / 1e3
        h2d = x_h.numel() * 4 + g_h.numel() * 4 + t_h.numel() * 4
        d2h = y_h.numel() * 4 + dx_h.numel() * 4
        out = {"value": layer.cfg.n_rows * args.steps / t, "unit": UNIT, "ms_per_step": t / args.steps * 1e3,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "h2d_GB/s": h2d / (t / args.steps) / 1e9,
               "overlap": "uploads and downloads on their own streams, double-buffered on the device"
                          + ("; edge messages streamed through a device ring, aggregated chunk by chunk"
                             if layer.edges else "")}
        if layer.edges:
            out["chunks_per_step"] = len(core._host["chunks"])
    finally:
        core._host = None      # the host pipeline's device buffers and ring
        _unpin(x_h, g_h, t_h, y_h, dx_h)
    return out


def main():
    args = parse()
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.ep:
            run_ep(args, world, rank, local)
        else:
            run_janus(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
