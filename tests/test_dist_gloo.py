"""Host logic of the multi-GPU bench on CPU with gloo ranks: each rank runs an
independent layer (distinct seeds, no data-path collective); timings are
reduced to their max over ranks; the reference arm prints from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = [1.0 + rank, 10.0 - rank, 3.0 * rank]
        got = bench.reduce_max(mine, world)
        bench.barrier(world)
        q.put((rank, got, bench.rank_seed(0, rank)))
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_seeds_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, seed in res:
        assert got == [2.0, 10.0, 3.0]
    assert res[0][2] != res[1][2]  # independent layers per rank


def _run_bench(env_extra, args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env,
                          capture_output=True, text=True, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_line_on_rank0_only():
    args = ["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3"]
    r0 = _run_bench({"RANK": "0", "WORLD_SIZE": "2"}, args)
    assert r0.returncode == 0, r0.stderr
    lines = [line for line in r0.stdout.splitlines() if line.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "routed tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0
    r1 = _run_bench({"RANK": "1", "WORLD_SIZE": "2"}, args)
    assert r1.returncode == 0 and not r1.stdout.strip()


def test_bench_rejects_short_warmup():
    r = _run_bench({}, ["--warmup", "2"])
    assert r.returncode != 0 and "warmup" in r.stderr
