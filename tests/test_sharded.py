"""The chunk-sharded step's exchange logic with real collectives: world_size 2 and 3 gloo
process groups on the CPU, every rank running the phases of
learned_sparse_kv_decode_b200.sharded with an exact host backend; the result must equal the
unsharded float64 decode step (same kept ids, same output)."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import datagen
import oracle
from learned_sparse_kv_decode_b200 import sharded


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(seed):
    w = datagen.small_workload(B=2, N=(37, 64), k=(9, 20), E=32, H=2, C=8, seed=seed)
    x = datagen.make_inputs(w)
    off = w.chunk_offsets
    emb = [datagen.as_f32(x["chunk_emb"][off[b]:off[b + 1]], "f32").astype(np.float64) for b in range(w.B)]
    q_emb = [datagen.as_f32(x["q_emb"][b], "f32").astype(np.float64) for b in range(w.B)]
    q = datagen.as_f32(x["q"], "f32").astype(np.float64)
    K = [datagen.kv_rows(w, "K", off[b] * w.C + np.arange(w.L[b])).astype(np.float64) for b in range(w.B)]
    V = [datagen.kv_rows(w, "V", off[b] * w.C + np.arange(w.L[b])).astype(np.float64) for b in range(w.B)]
    return w, q_emb, emb, q, K, V


def _rank(rank, world, port, seed, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from tests._shard_oracle import OracleShardBackend
        w, q_emb, emb, q, K, V = _problem(seed)
        ln, go = sharded.split_chunks(w.N, world)[rank]
        plan = sharded.ShardPlan(w.B, 1, w.E, w.H, w.C, world, rank, w.k, ln, go, "f32", "f32")
        lemb = [emb[b][go[b]:go[b] + ln[b]] for b in range(w.B)]
        lK = [K[b][go[b] * w.C:(go[b] + ln[b]) * w.C] for b in range(w.B)]
        lV = [V[b][go[b] * w.C:(go[b] + ln[b]) * w.C] for b in range(w.B)]
        bk = OracleShardBackend(plan, lemb, lK, lV)
        out, lse = sharded.run_distributed(bk, q_emb, None, q, None, None)
        result_q.put((rank, [g.tolist() for g in bk.global_ids], out.tolist(), lse.tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_step_gloo_equals_unsharded(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, 91, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, q_emb, emb, qq, K, V = _problem(91)
    for rank, gids, out, lse in results:
        for b in range(w.B):
            ids, ref_o, ref_l, _ = oracle.decode_step(q_emb[b], emb[b], qq[b], K[b], V[b], w.k[b], w.C,
                                                     1.0 / math.sqrt(128))
            np.testing.assert_array_equal(gids[b], ids)
            np.testing.assert_allclose(np.array(out[b]), ref_o, rtol=0, atol=1e-12)
            np.testing.assert_allclose(np.array(lse[b]), ref_l, rtol=0, atol=1e-12)


def test_split_chunks():
    parts = sharded.split_chunks([10, 7], 3)
    assert [p[0] for p in parts] == [[3, 2], [3, 2], [4, 3]]
    assert [p[1] for p in parts] == [[0, 0], [3, 2], [6, 4]]
    with pytest.raises(ValueError):
        sharded.split_chunks([2], 3)
