"""The N > 1 path of bench.py on CPU: ranks shard the sequences (disjoint
blocks, no data-path collective), the timing is the maximum over ranks (one
all-reduce, here over gloo with world size 2), and under torchrun only rank 0
prints a line (the reference arm, which needs no GPU, run end to end)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_rank_sequence_blocks_are_disjoint(world):
    B = 32
    seqs = [set(range(bench.rank_first_sequence(r, k, B), bench.rank_first_sequence(r, k, B) + B))
            for r in range(world) for k in (0, 1)]
    union = set().union(*seqs)
    assert len(union) == sum(len(s) for s in seqs) == 2 * world * B


def _max_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks([rank + 1.0, 10.0 - rank, 3.5], world, torch.device("cpu"))
        q.put((rank, t.tolist()))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_max_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert got[r] == [2.0, 10.0, 3.5]


def test_reference_arm_under_torchrun():
    """Two ranks launched as the driver launches them: rank 0 alone runs and
    prints the reference line, the other rank exits 0 without work."""
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
