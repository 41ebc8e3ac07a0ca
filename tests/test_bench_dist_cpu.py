"""bench.py's multi-rank logic on CPU: world size 2 over gloo.

The bench runs independent replicas per GPU; its only cross-rank steps are a
barrier and two scalar reductions (max of elapsed time, sum of tokens). This
checks them with two gloo processes, and that the reference arm prints
nothing on a rank other than 0.
"""

import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    bench.barrier()
    mx = bench.reduce_max(10.0 + rank)
    sm = bench.reduce_sum(32.0)
    q.put((rank, mx, sm, bench.dist_env()))
    dist.destroy_process_group()


def test_reductions_over_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm, env in res:
        assert mx == 11.0 and sm == 64.0
        assert env == (2, rank, 0)


def test_reference_arm_is_silent_on_nonzero_rank():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, cwd=ROOT,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank0():
    import json
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "query-tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_causal_prefill_flops_counts_every_visible_key():
    """The FLOP count behind the prefill TFLOP/s figures: against a count of
    (query row, visible key) pairs enumerated one by one."""
    import random
    import bench
    rng = random.Random(5)
    for _ in range(20):
        ql = rng.randint(1, 300)
        L = ql + rng.randint(0, 2000)
        d, h = rng.choice([64, 128]), rng.choice([1, 8, 32])
        pairs = 0
        for j in range(ql):
            pos = L - ql + j
            pairs += sum(1 for key in range(L) if key <= pos)
        assert bench.causal_prefill_flops(L, ql, d, h) == 4 * d * h * pairs
