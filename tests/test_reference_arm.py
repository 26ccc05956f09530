"""CPU checks of bench.py's oracle sample (the reference arm and the cpu_baseline leg): every
timed round measures both unit costs, so a short run cannot extrapolate a step from one kind
of work alone, and the reference arm prints the contract's JSON line."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import datagen  # noqa: E402


@pytest.mark.parametrize("steps,warmup", [(1, 0), (1, 3), (2, 1)])
def test_short_samples_time_both_kinds(steps, warmup):
    w = datagen.workload("tiny")
    r = bench.oracle_sample(w, steps=steps, warmup=warmup)
    seqs = len({0, w.B - 1})
    assert r["rounds"] == steps
    assert r["n_score"] == steps * seqs and r["n_attn"] == steps * seqs
    assert r["t_step"] > 0


def test_time_bounded_sample():
    w = datagen.workload("tiny")
    r = bench.oracle_sample(w, seconds=0.2, warmup=1)
    assert r["rounds"] >= 1 and r["n_score"] >= 1 and r["n_attn"] >= 1


def test_cap_ends_a_long_request():
    w = datagen.workload("tiny")
    r = bench.oracle_sample(w, steps=10 ** 9, warmup=0, cap=0.3)
    assert 1 <= r["rounds"] < 10 ** 9 and r["elapsed"] < 30


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "steps/s" and line["value"] > 0
    assert line["steps"] == 2 and line["warmup"] == 1
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and "2 timed rounds" in line["cpu_baseline"]["sample"]


def test_dense_context_costs_more_than_the_sparse_step():
    # 128K keeps 12.5% of the tokens: the dense oracle step must be several times slower
    w = datagen.workload("128k")
    dense = bench.oracle_dense_context(w)
    sparse = bench.oracle_sample(w, seconds=1.0, warmup=1)
    assert dense["unit"] == "steps/s" and dense["cores"] == 1
    assert dense["value"] * 3 < 1.0 / sparse["t_step"]


def _ranks_worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench._barrier(world)
        q.put((rank, bench._max_over_ranks(1.5 + rank * 2.0, world)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    # the bench's timing is the maximum over ranks: every rank must report the slowest rank's time
    import multiprocessing as mp
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ranks_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 3.5, 1: 3.5}
