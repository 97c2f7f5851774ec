"""World-size-2 gloo tests of the replica (data-parallel) host logic: the
max-over-ranks timing, the job throughput, and the reference arm printing one
line from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

from lossless_diffusion_speculative_b200.replicas import max_over_ranks, replica_throughput

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local = [10.0 + 5.0 * rank, 3.0 - rank]            # rank 1 is the slower one in [0]
    m = max_over_ranks(local)
    out[rank] = (m, replica_throughput(29, 100, world, m[0]))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_throughput_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        m, v = out[r]
        assert m == [15.0, 3.0]
        assert abs(v - 2 * 29 * 100 / 0.015) < 1e-6


def test_single_process_is_identity():
    assert max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert replica_throughput(10, 4, 1, 2000.0) == 20.0


def test_reference_arm_prints_one_line_from_rank0():
    port = _free_port()
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--workload", "qwen3_1p7b_layer", "--steps", "2",
           "--warmup", "1", "--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
