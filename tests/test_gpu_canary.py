"""Out-of-bounds writes, caught without a sanitizer: every output buffer of every entry point,
and the workspace, is a view into a larger allocation whose guard bands (64 KiB on each side)
hold a fill pattern. After the call the bands must be unchanged. The shapes are small and
ragged (partial tiles, single-chunk sequences, the largest window), where an index slip at a
boundary would land just outside a buffer."""
import numpy as np
import pytest
import torch

import datagen
from learned_sparse_kv_decode_b200 import sharded
from tests import _gpu as G

pytestmark = pytest.mark.gpu

GUARD = 64 * 1024
FILL = 0xA5


@pytest.fixture(scope="module")
def lsa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import learned_sparse_kv_decode_b200 as m
    return m


class Guards:
    """Allocates guarded tensors and checks every band at once."""

    def __init__(self):
        self.bufs = []

    def __call__(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((2 * GUARD + ((n + 255) // 256) * 256,), FILL, dtype=torch.uint8, device="cuda")
        t = raw[GUARD:GUARD + n].view(dtype).view(shape)
        if fill is not None:
            t.fill_(fill)
        self.bufs.append((raw, n))
        return t

    def workspace(self, lsa, dims):
        ws = self(lsa.lsa_workspace_size(dims), torch.uint8)
        lsa.lsa_workspace_init(ws)
        return ws

    def check(self):
        torch.cuda.synchronize()
        for raw, n in self.bufs:
            lo, hi = raw[:GUARD], raw[GUARD + n:]
            assert bool((lo == FILL).all()) and bool((hi == FILL).all()), "a guard band was overwritten"


CASES = [
    dict(B=3, N=(40, 1, 72), k=(5, 1, 9), E=64, H=4, C=16, emb_dtype="f32", kv_dtype="f32"),
    dict(B=2, N=(130, 257), k=(18, 35), E=128, Q=64, H=4, C=64, emb_dtype="bf16", kv_dtype="bf16"),
    dict(B=2, N=(33, 9), k=(7, 9), E=256, Q=3, H=8, C=32, emb_dtype="bf16", kv_dtype="bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}-Q{c.get('Q', 1)}-C{c['C']}-{c['kv_dtype']}")
def test_no_write_outside_outputs(lsa, case):
    w = datagen.small_workload(seed=71, **dict(case))
    dw = G.DeviceWorkload(w, lsa)
    g = Guards()
    ws = g.workspace(lsa, dw.dims)
    kt = G.tdtype(w.kv_dtype)
    f32, i32 = torch.float32, torch.int32

    scores = g((w.total_chunks,), f32)
    lsa.lsa_score_chunks(dw.dims, dw.q_emb, dw.chunk_emb, scores, ws)
    ids = g((w.total_kept,), i32)
    lsa.lsa_topk_select(dw.dims, scores, ids, ws)
    K_res = g((w.total_kept * w.C, w.H, w.Dh), kt)
    V_res = g((w.total_kept * w.C, w.H, w.Dh), kt)
    lsa.lsa_gather_kv(dw.dims, dw.K, dw.V, ids, K_res, V_res, ws)
    out, lse = g((w.B, w.H, w.Dh), f32), g((w.B, w.H), f32)
    lsa.lsa_sparse_decode_attn(dw.dims, dw.q, dw.K, dw.V, ids, out, lse, ws)
    lsa.lsa_sparse_decode_attn(dw.dims, dw.q, K_res, V_res, None, out, lse, ws)
    ids2 = g((w.total_kept,), i32)
    lsa.lsa_decode_step(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, ids2, out, lse, ws)
    counts = g((w.B,), i32)
    tau = float(torch.quantile(scores.float(), 0.9))
    lsa.lsa_threshold_select(dw.dims, scores, tau, 1, ids2, counts, ws)
    lsa.lsa_decode_step_threshold(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, tau, 1, ids2, counts,
                                  out, lse, ws)
    lsa.lsa_sparse_decode_attn_counts(dw.dims, dw.q, dw.K, dw.V, ids2, counts, out, lse, ws)
    slots = g((w.total_kept,), i32, fill=-1)
    Kr, Vr = g((w.total_kept * w.C, w.H, w.Dh), kt, fill=0), g((w.total_kept * w.C, w.H, w.Dh), kt, fill=0)
    moved = g((w.B,), i32)
    lsa.lsa_refresh_resident(dw.dims, dw.q_emb, dw.chunk_emb, dw.K, dw.V, slots, Kr, Vr, moved, ws)
    lsa.lsa_sparse_decode_attn_noalloc(dw.dims, dw.q, dw.K, dw.V, ids, out, lse)
    if w.kv_dtype == "bf16":
        q_la = G.to_device(datagen.make_lookahead_queries(w), "bf16")
        out_la, lse_la = g((w.B, w.Q, w.H, w.Dh), f32), g((w.B, w.Q, w.H), f32)
        lsa.lsa_sparse_decode_attn_lookahead(dw.dims, q_la, dw.K, dw.V, ids, out_la, lse_la, ws)
        lsa.lsa_sparse_decode_attn_lookahead(dw.dims, q_la, K_res, V_res, None, out_la, lse_la, ws)
        lsa.lsa_decode_step_lookahead(dw.dims, dw.q_emb, dw.chunk_emb, q_la, dw.K, dw.V, ids2, out_la, lse_la, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK
    g.check()


def test_no_write_outside_fp8_indexer(lsa):
    w = datagen.small_workload(B=2, N=(130, 3), k=(9, 3), E=lsa.LSA_INDEX_DIM, H=4, C=64, emb_dtype="bf16",
                               kv_dtype="bf16", seed=72)
    x = G.IndexerInputs(w, layers=3, heads=32)
    dw = G.DeviceWorkload(w, lsa)
    dims = lsa.Dims(w.B, 1, lsa.LSA_INDEX_DIM, w.H, w.C, chunk_offsets=w.chunk_offsets.tolist(), k_per_seq=w.k,
                    emb_dtype="bf16", kv_dtype="bf16")
    g = Guards()
    ws = g.workspace(lsa, dims)
    scores = g((w.total_chunks,), torch.float32)
    lsa.lsa_indexer_score_fp8(dims, 3, 32, lsa.LSA_ENSEMBLE_MAX, x.ck, x.q8, x.qs, x.hw, scores, ws)
    ids = g((w.total_kept,), torch.int32)
    out, lse = g((w.B, w.H, w.Dh), torch.float32), g((w.B, w.H), torch.float32)
    lsa.lsa_decode_step_fp8(dims, 3, 32, lsa.LSA_ENSEMBLE_MEAN, x.ck, x.q8, x.qs, x.hw, dw.q, dw.K, dw.V, ids, out,
                            lse, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK
    g.check()


def test_no_write_outside_sharded_step(lsa):
    # two emulated ranks: every buffer of the sharded phases is a guarded view
    n_chunks, k, H, C, E, G_ = [90, 41], [12, 7], 4, 16, 64, 2
    w = datagen.small_workload(B=2, N=tuple(n_chunks), k=tuple(k), E=E, H=H, C=C, emb_dtype="bf16",
                               kv_dtype="bf16", seed=73)
    dw = G.DeviceWorkload(w, lsa)
    g = Guards()
    backends = []
    parts = sharded.split_chunks(n_chunks, G_)
    for r, (ln, go) in enumerate(parts):
        plan = sharded.ShardPlan(B=2, Q=1, E=E, H=H, C=C, G=G_, rank=r, k=k, local_n=ln, global_offset=go)
        bk = sharded.CudaShardBackend(plan)
        for name in ("scores", "local_cand", "cand_s", "cand_i", "seq_s", "seq_i", "global_ids", "local_ids",
                     "local_count", "out_g", "lse_g", "out", "lse"):
            t = getattr(bk, name)
            setattr(bk, name, g(tuple(t.shape), t.dtype))
        for name, dims in (("ws_local", bk.local_dims), ("ws_global", bk.global_dims)):
            setattr(bk, name, g.workspace(lsa, dims))
        backends.append(bk)
    # each rank's chunk embeddings and K/V rows are its contiguous share of every sequence
    emb_off, tok_off = w.chunk_offsets, w.chunk_offsets * C
    chunk_embs, Ks, Vs = [], [], []
    for ln, go in parts:
        rows = np.concatenate([np.arange(emb_off[b] + go[b], emb_off[b] + go[b] + ln[b]) for b in range(2)])
        toks = np.concatenate([np.arange(tok_off[b] + go[b] * C, tok_off[b] + (go[b] + ln[b]) * C) for b in range(2)])
        rows_t, toks_t = torch.from_numpy(rows).cuda(), torch.from_numpy(toks).cuda()
        chunk_embs.append(dw.chunk_emb.index_select(0, rows_t).contiguous())
        Ks.append(dw.K.index_select(0, toks_t).contiguous())
        Vs.append(dw.V.index_select(0, toks_t).contiguous())
    sharded.run_emulated(backends, dw.q_emb, chunk_embs, dw.q, Ks, Vs)
    for bk in backends:
        assert lsa.lsa_get_device_status(bk.ws_local) == lsa.LSA_OK
        assert lsa.lsa_get_device_status(bk.ws_global) == lsa.LSA_OK
    g.check()
