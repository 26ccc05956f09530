"""The chunk-sharded step with real collectives and the CUDA kernels: two ranks as two processes
that share the one GPU, exchanging over a gloo process group (host memory). Each rank runs its
own shard through the library (score, local top-k, candidates, global select, attention over its
kept chunks, merge); the ranks' kernels never wait on one another, only the host collectives
do. Every rank must end with the unsharded fused step's kept ids, and its output and lse."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

CASE = dict(B=2, N=(300, 181), k=(40, 17), E=128, H=16, C=64, emb_dtype="bf16", kv_dtype="bf16", seed=77)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard_inputs(dw, w, go, ln):
    off = w.chunk_offsets
    emb = torch.cat([dw.chunk_emb[off[b] + go[b]:off[b] + go[b] + ln[b]] for b in range(w.B)]).contiguous()
    K = torch.cat([dw.K[(off[b] + go[b]) * w.C:(off[b] + go[b] + ln[b]) * w.C] for b in range(w.B)]).contiguous()
    V = torch.cat([dw.V[(off[b] + go[b]) * w.C:(off[b] + go[b] + ln[b]) * w.C] for b in range(w.B)]).contiguous()
    return emb, K, V


def _rank(rank, world, port, result_q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import datagen
        import learned_sparse_kv_decode_b200 as lsa
        from learned_sparse_kv_decode_b200 import sharded
        from tests import _gpu as G
        torch.cuda.set_device(0)
        w = datagen.small_workload(**CASE)
        dw = G.DeviceWorkload(w, lsa)
        ln, go = sharded.split_chunks(w.N, world)[rank]
        plan = sharded.ShardPlan(w.B, w.Q, w.E, w.H, w.C, world, rank, w.k, ln, go, w.emb_dtype, w.kv_dtype)
        bk = sharded.CudaShardBackend(plan)
        emb, K, V = _shard_inputs(dw, w, go, ln)
        out, lse = sharded.run_distributed(bk, dw.q_emb, emb, dw.q, K, V)
        torch.cuda.synchronize()
        status = (lsa.lsa_get_device_status(bk.ws_local), lsa.lsa_get_device_status(bk.ws_global))
        result_q.put((rank, bk.global_ids.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy(), status))
    finally:
        dist.destroy_process_group()


def test_sharded_step_two_ranks_gloo_cuda():
    import multiprocessing as mp
    sys.path.insert(0, ROOT)
    import datagen
    import learned_sparse_kv_decode_b200 as lsa
    from tests import _gpu as G
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        results = [q.get(timeout=300) for _ in range(world)]
    finally:
        for p in procs:
            p.join(timeout=120)
    for p in procs:
        assert p.exitcode == 0
    # the unsharded fused step on the same inputs, in this process
    w = datagen.small_workload(**CASE)
    dw = G.DeviceWorkload(w, lsa)
    lsa.lsa_decode_step(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, dw.ids, dw.out, dw.lse, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    ids, ref_out, ref_lse = dw.ids.cpu().numpy(), dw.out.cpu().numpy(), dw.lse.cpu().numpy()
    for rank, gids, out, lse, status in results:
        assert status == (lsa.LSA_OK, lsa.LSA_OK), (rank, status)
        np.testing.assert_array_equal(gids, ids)  # the same fp32 scores select the same ids
        np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-4)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-4)
