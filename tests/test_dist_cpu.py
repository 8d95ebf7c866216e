"""The multi-process plumbing of bench.py on CPU (gloo, world size 2).

The path shards by replica (no data exchange), so the only collectives are the
benchmark's barrier and its max / sum over ranks; the reference arm runs on rank 0
alone while the other ranks leave without work.
"""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ranks(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(world)
    d.barrier()
    out[rank] = (d.max(rank + 1.5), d.sum(rank + 1.0), d.world, d.rank)
    d.barrier()
    d.close()


def test_dist_max_and_sum_over_two_gloo_ranks():
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_ranks, args=(2, free_port(), out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0] == (2.5, 3.0, 2, 0)
    assert res[1] == (2.5, 3.0, 2, 1)


def test_reference_arm_under_torchrun_prints_one_line_from_rank0():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny_relu_f32", "--ref-seconds", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "tokens/s" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
