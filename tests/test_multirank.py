"""Multi-process paths on CPU (gloo, world size 2).

The bench runs one independent tensor per rank (weak scaling) and exchanges only timing: a
barrier and a max over ranks of the step time. A tensor split by rows across ranks would
need one exchange on the data path, the all-reduce (max) of the per-group amax, after which
every rank quantizes its rows with the global tensor scale; the test checks that this
reproduces the whole-tensor result bit for bit.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)


def _max_over_ranks_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench

    _init(rank, world, port)
    try:
        bench.barrier(world)
        q.put((rank, bench.max_over_ranks(1.5 + rank, world)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_max_over_ranks_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 2.5), (1, 2.5)]


def _sharded_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import oracle as O
    from nvfp4_block_scaled_13_b200 import synth

    _init(rank, world, port)
    try:
        x, (g, r, c) = synth.make("c3", rows=96, cols=512)
        rows = r // world
        mine = np.ascontiguousarray(x[rank * rows * c:(rank + 1) * rows * c])
        local = torch.from_numpy(O.amax(mine, 1, rows, c))
        dist.all_reduce(local, op=dist.ReduceOp.MAX)       # the one exchange of a row-sharded tensor
        out = O.quantize(mine, 1, rows, c, local.numpy(), 1, 2)
        q.put((rank, float(local[0]), out["codes"].tobytes(), out["scales"].tobytes()))
    finally:
        dist.destroy_process_group()


def test_row_sharded_amax_exchange_reproduces_whole_tensor():
    sys.path.insert(0, ROOT)
    import oracle as O
    from nvfp4_block_scaled_13_b200 import synth

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    parts = sorted(q.get(timeout=10) for _ in range(2))
    x, (g, r, c) = synth.make("c3", rows=96, cols=512)
    whole_amax = O.amax(x, g, r, c)
    whole = O.quantize(x, g, r, c, whole_amax, 1, 2)
    assert all(p[1] == float(whole_amax[0]) for p in parts)
    assert b"".join(p[2] for p in parts) == whole["codes"].tobytes()
    assert b"".join(p[3] for p in parts) == whole["scales"].tobytes()


def test_bench_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "1",
           "--rows", "256"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
