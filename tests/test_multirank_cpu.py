"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The layer path shards by atoms with no collective on the data path, so the
only cross-rank steps are the barrier around the timed region and the
max-over-ranks of the elapsed time; the reference arm runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup()
    bench.barrier(w)
    v = bench.max_over_ranks(1.5 + r, w)      # rank 1 is the slowest
    q.put((r, w, dist.get_backend(), v))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == 2 and g[2] == "gloo" and g[3] == 2.5 for g in got)


def test_reference_arm_two_ranks_prints_one_line():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "2",
           "--warmup", "1", "--ref-seconds", "0.05"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def _ep_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from element_routed_moe_b200.ep import ExpertParallelLayer
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    out = []
    w1, w2 = torch.zeros((4, 8, 12)), torch.zeros((4, 12, 8))
    for E, a, b in ((9, w1, w2), (8, w1[:3], w2[:3]), (8, w2, w1)):
        try:
            ExpertParallelLayer(16, 8, 12, 5, E, 2, a, b)
            out.append("accepted")
        except ValueError as e:
            out.append(str(e))
    q.put((rank, out))
    dist.destroy_process_group()


def test_ep_layer_validates_the_expert_split_on_every_rank():
    # two gloo ranks: 9 experts cannot be split, each rank must pass its E/P = 4
    # experts in the [E/P, d, h] / [E/P, h, d] layout; nothing reaches CUDA
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, msgs in got:
        assert "multiple of the number of ranks" in msgs[0]
        assert "E/P experts" in msgs[1] and "E/P experts" in msgs[2]
