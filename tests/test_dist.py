"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

On N GPUs the benchmark runs N independent problems (rows are independent, so
there is no data-path collective); what is shared is the plumbing: rank
discovery from the torchrun environment, barriers, and the maximum over ranks
of the timed duration.  These run here on CPU ranks over gloo; the reference
arm is launched through torchrun exactly as the driver launches it.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    r, w, local, pg = bench.dist_init(world)
    assert (r, w, local) == (rank, world, rank) and pg is not None
    bench.barrier(pg)
    # rank r "measured" 10 + r ms: everyone must see the maximum
    m = bench.max_over_ranks(10.0 + r, pg, torch.device("cpu"))
    q.put((rank, m))
    pg.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert got == [(0, 11.0), (1, 11.0)]


def test_rank_seeds_differ_but_sources_agree():
    """Each rank draws its own query points; the sources are the workload's."""
    sys.path.insert(0, ROOT)
    import synth
    w = synth.BY_NAME["d3_10k"]
    a = synth.make_inputs(w, seed=None)
    b = synth.make_inputs(w, seed=1000 + w.wid + 7919 * 1)
    assert not torch.equal(a["x"], b["x"])
    assert a["x"].shape == b["x"].shape


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "1",
           "--workload", "d3_10k", "--cpu-seconds", "0.4"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["metric"].startswith("Gaussian kernel-sum pairs/sec")
