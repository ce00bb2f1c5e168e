"""The multi-rank plumbing of bench.py on CPU ranks (gloo, world size 2).

Token rows are independent, so the path shards by batch with no data-path
collective: every rank runs its own full batch and the only collectives are
the timing barrier and a MAX reduction of the elapsed time.  These tests run
that host logic on two CPU processes.
"""
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


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank timed its own batch; the job is as slow as its slowest rank
        mine = [0.80, 0.95][rank]
        slowest = bench.max_over_ranks(mine, world, device="cpu")
        tops = bench.job_tops(2.0e12, 10, world, slowest)
        dist.barrier()
        out.put((rank, slowest, tops))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_throughput_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, tops in res:
        assert slowest == 0.95
        assert tops == pytest.approx(2 * 2.0e12 * 10 / 0.95 / 1e12)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.job_tops(1e12, 4, 1, 2.0) == pytest.approx(2.0)


def test_reference_arm_under_torchrun_prints_once_from_rank_zero():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--reference-seconds", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"


# ------------------------------------------------------------ token-sharded linear with an all-gather


def _cp_worker(rank: int, world: int, port: int, out, cases):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    from w8a8_int8_quantized_block_b200 import context_parallel as CP

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = []
        for M, K, N in cases:
            g = torch.Generator().manual_seed(M * 100 + N)
            x = torch.randn(M, K, generator=g).to(torch.bfloat16)
            w = torch.randn(N, K, generator=g)

            def linear(xs, y):  # a CPU stand-in for the GPU linear: same rows in, same rows out
                y.copy_((xs.float() @ w.T).to(torch.bfloat16))

            s, e = CP.token_shard(M, world, rank)
            y = CP.linear_context_parallel(x[s:e].clone(), M, N, linear)
            ref = (x.float() @ w.T).to(torch.bfloat16)
            res.append(bool(torch.equal(y.view(torch.int16), ref.view(torch.int16))) and tuple(y.shape) == (M, N))
        dist.barrier()
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_token_shard_covers_every_row_once():
    sys.path.insert(0, ROOT)
    from w8a8_int8_quantized_block_b200 import context_parallel as CP

    for M in (0, 1, 7, 8, 38656, 38657):
        for world in (1, 2, 3, 8):
            rows = []
            for r in range(world):
                s, e = CP.token_shard(M, world, r)
                assert 0 <= s <= e <= M and e - s <= -(-M // world)
                rows.extend(range(s, e))
            assert rows == list(range(M))


def test_context_parallel_gather_on_two_gloo_ranks():
    # even and uneven token counts, and a rank whose shard is empty (M = 1)
    cases = [(10, 16, 6), (11, 16, 6), (1, 8, 4), (300, 64, 24)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, 2, port, q, cases)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok in res:
        assert all(ok), (rank, ok)
