"""The N>1 path of bench.py on CPU ranks (gloo, world size 2).

The decode path shards by independent sequences: no data crosses ranks.  The
only multi-rank steps are the timing reduction (max over ranks) and the
whole-job aggregate, plus rank 0 alone printing, which these tests cover.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, n, local = bench.world()
        elapsed = 0.5 + rank                      # rank 1 is the slowest
        mx = bench.reduce_max(elapsed)
        agg = bench.aggregate(tokens_per_rank=1000, elapsed_s=elapsed, steps=4, n_ranks=n)
        from bit_kv_cache_dqk_b200 import inputs as I
        w = bench.rank_workload(I.CONFIGS["tiny"], r)
        q.put((rank, r, n, local, mx, agg, w.seed))
    finally:
        dist.destroy_process_group()


def test_gloo_world2_reduce_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in procs)
    seeds = set()
    for rank, r, n, local, mx, agg, seed in res:
        assert (r, n, local) == (rank, 2, rank)
        assert mx == 1.5                          # max over ranks, seen by both
        assert agg["elapsed_s"] == 1.5
        assert agg["value"] == pytest.approx(1000 * 4 * 2 / 1.5)
        assert agg["ms_per_step"] == pytest.approx(1e3 * 1.5 / 4)
        seeds.add(seed)
    assert len(seeds) == 2                        # each rank decodes its own sequences


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(2.5) == 2.5
    agg = bench.aggregate(100, 2.0, 10, 1)
    assert agg["value"] == pytest.approx(500.0)


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "llama", "--ref-ctx", "1024"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_gpus_flag_launches_ranks_and_reports_max_over_ranks():
    """`bench.py --gpus 2` with no outer launcher runs two ranks itself (under
    torch.distributed.run); the CPU self-test step sleeps (rank + 1) ms, so the
    slowest rank sets the time and rank 0 alone prints one JSON line."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                           "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--cpu-selftest",
                        "--steps", "20", "--warmup", "3"], capture_output=True, text=True, timeout=300, env=env,
                       cwd=ROOT)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2
    assert line["ms_per_step"] >= 2.0          # rank 1's 2 ms steps, not rank 0's 1 ms
    assert line["value"] == pytest.approx(2 * 1000 / (line["ms_per_step"] / 1e3), rel=1e-6)
