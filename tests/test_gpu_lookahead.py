"""GPU parity of the lookahead-window attention (every window query over the kept tokens) and
of the fused lookahead step, against the float64 oracle on the same seeded inputs.

Tolerance (bf16 K/V, 2e-2 absolute on the output, as for the single-query path): the kernel
rounds each softmax weight p to bf16 for the P.V product (relative error <= 2^-9) and divides
by the fp32 sum of the unrounded weights, so the output is off by at most
2^-9 * sum_t p_t |V_t| / sum_t p_t <= 2^-9 * max|V| (~0.009 for these N(0,1) caches). The lse
comes from fp32 scores and fp32 sums only: 1e-4 absolute."""
import math

import numpy as np
import pytest
import torch

import datagen
import oracle
from tests import _gpu as G

pytestmark = pytest.mark.gpu

OUT_ATOL = 2e-2
LSE_ATOL = 1e-4


@pytest.fixture(scope="module")
def lsa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import learned_sparse_kv_decode_b200 as m
    return m


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


class Window:
    """A workload on the device plus its window queries [B, Q, H, Dh] and output buffers."""

    def __init__(self, w, lsa):
        self.dw = G.DeviceWorkload(w, lsa)
        self.q_host = datagen.make_lookahead_queries(w)
        self.q = G.to_device(self.q_host, w.kv_dtype)
        self.out = torch.full((w.B, w.Q, w.H, w.Dh), float("nan"), dtype=torch.float32, device="cuda")
        self.lse = torch.full((w.B, w.Q, w.H), float("nan"), dtype=torch.float32, device="cuda")

    def random_ids(self, seed):
        rng = np.random.default_rng(seed)
        w = self.dw.w
        return [np.sort(rng.choice(w.N[b], size=w.k[b], replace=False)).astype(np.int32) for b in range(w.B)]

    def oracle(self, b, ids, heads=None, queries=None):
        w = self.dw.w
        heads = np.arange(w.H) if heads is None else np.asarray(heads)
        queries = np.arange(w.Q) if queries is None else np.asarray(queries)
        tok = oracle.kept_tokens(ids, w.C)
        K = self.dw.kv_f("K", b, tok, heads)
        V = self.dw.kv_f("V", b, tok, heads)
        q = datagen.as_f32(self.q_host[b], w.kv_dtype)[queries][:, heads]
        return oracle.lookahead_attention(q, K, V, 1.0 / math.sqrt(w.Dh))


def _compare(win, b, ids, heads=None, queries=None):
    ref_o, ref_l = win.oracle(b, ids, heads, queries)
    w = win.dw.w
    heads = np.arange(w.H) if heads is None else np.asarray(heads)
    queries = np.arange(w.Q) if queries is None else np.asarray(queries)
    got_o = win.out[b].cpu().numpy()[queries][:, heads]
    got_l = win.lse[b].cpu().numpy()[queries][:, heads]
    assert np.isfinite(got_o).all() and np.isfinite(got_l).all()
    np.testing.assert_allclose(got_o, ref_o, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(got_l, ref_l, rtol=0, atol=LSE_ATOL)
    return float(np.abs(got_o - ref_o).max())


ATTN_CASES = [
    dict(B=2, N=(40, 72), k=(5, 9), C=64, Q=64, H=4),       # runs of 5 and 9 tiles
    dict(B=2, N=(40, 72), k=(5, 9), C=16, Q=64, H=4),       # 4 chunks a tile; ragged last tiles
    dict(B=2, N=(30, 50), k=(7, 3), C=32, Q=64, H=2),
    dict(B=2, N=(12, 20), k=(3, 5), C=128, Q=64, H=2),      # one tile a chunk
    dict(B=2, N=(9, 6), k=(4, 1), C=256, Q=64, H=2),        # 2 tiles a chunk
    dict(B=1, N=(5,), k=(3,), C=1024, Q=40, H=2),           # 8 tiles a chunk
    dict(B=2, N=(64, 40), k=(11, 1), C=8, Q=64, H=2),       # 8 chunks a tile; a 1-chunk sequence
    dict(B=2, N=(40, 72), k=(5, 9), C=64, Q=13, H=4),       # a partial window
    dict(B=1, N=(40,), k=(6,), C=64, Q=1, H=8),             # a single query
    dict(B=1, N=(2048,), k=(1024,), C=64, Q=64, H=1),       # one run split across every CTA
    dict(B=8, N=(256,) * 8, k=(20,) * 8, C=64, Q=64, H=16),  # 128 runs: most wholly inside a CTA
    dict(B=3, N=(300, 7, 129), k=(77, 7, 1), C=32, Q=64, H=8),
]


@pytest.mark.parametrize("case", ATTN_CASES,
                         ids=lambda c: f"B{c['B']}-C{c['C']}-Q{c['Q']}-H{c['H']}-k{c['k'][0]}")
def test_lookahead_attention_parity(lsa, case):
    case = dict(case)
    w = datagen.small_workload(E=64, kv_dtype="bf16", emb_dtype="bf16", seed=61, **case)
    win = Window(w, lsa)
    ids = win.random_ids(7)
    ids_d = torch.from_numpy(np.concatenate(ids)).cuda()
    lsa.lsa_sparse_decode_attn_lookahead(win.dw.dims, win.q, win.dw.K, win.dw.V, ids_d, win.out, win.lse,
                                         win.dw.ws)
    assert lsa.lsa_get_device_status(win.dw.ws) == lsa.LSA_OK
    # every sequence; all heads and queries, or a sample where the oracle would be slow
    big = w.Q * w.H * max(w.k) * w.C > 4_000_000
    for b in range(w.B):
        heads = sorted({0, w.H - 1}) if big else None
        queries = sorted({0, w.Q // 2, w.Q - 1}) if big else None
        _compare(win, b, ids[b], heads, queries)
    del win
    _free()


@pytest.mark.parametrize("C", [64, 16, 256])
def test_lookahead_bad_id_reported(lsa, C):
    # out-of-range ids are reported and masked: each sequence's window attends over its valid
    # ids only, including the sequences that hold the bad ids; no valid id: out 0, lse -inf
    w = datagen.small_workload(B=4, N=(4, 6, 9, 3), k=(2, 3, 4, 1), E=64, Q=64, H=2, C=C, kv_dtype="bf16",
                               emb_dtype="bf16", seed=63)
    win = Window(w, lsa)
    ids = np.array([0, 1,  2, -3, 5,  1, 9, 4, 8,  3], dtype=np.int32)
    valid = [np.array([0, 1]), np.array([2, 5]), np.array([1, 4, 8]), None]
    lsa.lsa_sparse_decode_attn_lookahead(win.dw.dims, win.q, win.dw.K, win.dw.V, torch.from_numpy(ids).cuda(),
                                         win.out, win.lse, win.dw.ws)
    assert lsa.lsa_get_device_status(win.dw.ws) == lsa.LSA_ERR_BAD_ID
    for b, v in enumerate(valid):
        if v is None:
            np.testing.assert_array_equal(win.out[b].cpu().numpy(), 0.0)
            assert np.isneginf(win.lse[b].cpu().numpy()).all()
            continue
        _compare(win, b, v)
    del win
    _free()


def _random_window_case(seed):
    """A random window-attention shape: ragged N_b and k_b, chunk length 8 to 256 (several chunks
    per tile, or several tiles per chunk), a partial or full window of queries, 1 to 16 heads."""
    rng = np.random.default_rng(3000 + seed)
    B = int(rng.integers(1, 6))
    C = int(rng.choice([8, 16, 32, 64, 128, 256]))
    N = [int(rng.integers(1, 4096 // C + 2)) for _ in range(B)]
    k = [int(rng.integers(1, n + 1)) for n in N]
    return dict(B=B, N=tuple(N), k=tuple(k), C=C, Q=int(rng.integers(1, 65)),
                H=int(rng.choice([1, 2, 4, 8, 16])))


@pytest.mark.parametrize("seed", range(20))
def test_lookahead_attention_random_shapes(lsa, seed):
    w = datagen.small_workload(E=64, kv_dtype="bf16", emb_dtype="bf16", seed=4000 + seed,
                               **_random_window_case(seed))
    win = Window(w, lsa)
    ids = win.random_ids(seed)
    ids_d = torch.from_numpy(np.concatenate(ids)).cuda()
    lsa.lsa_sparse_decode_attn_lookahead(win.dw.dims, win.q, win.dw.K, win.dw.V, ids_d, win.out, win.lse,
                                         win.dw.ws)
    assert lsa.lsa_get_device_status(win.dw.ws) == lsa.LSA_OK
    big = w.Q * w.H * max(w.k) * w.C > 4_000_000
    for b in range(w.B):
        heads = sorted({0, w.H - 1}) if big else None
        queries = sorted({0, w.Q // 2, w.Q - 1}) if big else None
        _compare(win, b, ids[b], heads, queries)
    del win
    _free()


def test_lookahead_resident_equals_indexed(lsa):
    # the same tiles in the same order: the resident form gives bit-identical results
    w = datagen.small_workload(B=2, N=(40, 72), k=(5, 9), C=16, E=64, Q=64, H=4, kv_dtype="bf16",
                               emb_dtype="bf16", seed=62)
    win = Window(w, lsa)
    ids = torch.from_numpy(np.concatenate(win.random_ids(3))).cuda()
    lsa.lsa_sparse_decode_attn_lookahead(win.dw.dims, win.q, win.dw.K, win.dw.V, ids, win.out, win.lse, win.dw.ws)
    a_o, a_l = win.out.clone(), win.lse.clone()
    rows = int(sum(w.k)) * w.C
    K_res = torch.empty((rows, w.H, w.Dh), dtype=torch.bfloat16, device="cuda")
    V_res = torch.empty_like(K_res)
    lsa.lsa_gather_kv(win.dw.dims, win.dw.K, win.dw.V, ids, K_res, V_res, win.dw.ws)
    win.out.fill_(float("nan"))
    lsa.lsa_sparse_decode_attn_lookahead(win.dw.dims, win.q, K_res, V_res, None, win.out, win.lse, win.dw.ws)
    assert lsa.lsa_get_device_status(win.dw.ws) == lsa.LSA_OK
    assert torch.equal(a_o, win.out) and torch.equal(a_l, win.lse)


def test_lookahead_one_query_matches_single_query_path(lsa):
    # Q = 1: the window attention is the ordinary decode attention (fp32 path) up to the
    # bf16 rounding of the softmax weights
    w = datagen.small_workload(B=2, N=(40, 72), k=(5, 9), C=64, E=64, Q=1, H=8, kv_dtype="bf16",
                               emb_dtype="bf16", seed=63)
    win = Window(w, lsa)
    ids = torch.from_numpy(np.concatenate(win.random_ids(5))).cuda()
    lsa.lsa_sparse_decode_attn_lookahead(win.dw.dims, win.q, win.dw.K, win.dw.V, ids, win.out, win.lse, win.dw.ws)
    q1 = win.q[:, 0].contiguous()
    out1 = torch.empty((w.B, w.H, w.Dh), dtype=torch.float32, device="cuda")
    lse1 = torch.empty((w.B, w.H), dtype=torch.float32, device="cuda")
    lsa.lsa_sparse_decode_attn(win.dw.dims, q1, win.dw.K, win.dw.V, ids, out1, lse1, win.dw.ws)
    assert lsa.lsa_get_device_status(win.dw.ws) == lsa.LSA_OK
    torch.testing.assert_close(win.out[:, 0], out1, rtol=0, atol=OUT_ATOL)
    torch.testing.assert_close(win.lse[:, 0], lse1, rtol=0, atol=LSE_ATOL)


def test_lookahead_deterministic(lsa):
    w = datagen.small_workload(B=1, N=(2048,), k=(300,), C=64, E=64, Q=64, H=2, kv_dtype="bf16",
                               emb_dtype="bf16", seed=64)
    win = Window(w, lsa)
    ids = torch.from_numpy(np.concatenate(win.random_ids(9))).cuda()
    lsa.lsa_sparse_decode_attn_lookahead(win.dw.dims, win.q, win.dw.K, win.dw.V, ids, win.out, win.lse, win.dw.ws)
    a = (win.out.clone(), win.lse.clone())
    for _ in range(3):
        lsa.lsa_sparse_decode_attn_lookahead(win.dw.dims, win.q, win.dw.K, win.dw.V, ids, win.out, win.lse,
                                             win.dw.ws)
        assert torch.equal(a[0], win.out) and torch.equal(a[1], win.lse)


STEP_CASES = [
    dict(B=1, N=(600,), k=(81,), E=256, Q=64, H=16, plant="copy_query"),
    dict(B=2, N=(130, 257), k=(18, 35), E=128, Q=64, H=4, plant="copy_query"),
    dict(B=3, N=(40, 72, 5), k=(5, 9, 5), E=64, Q=24, H=4),
]


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: f"B{c['B']}-E{c['E']}-Q{c['Q']}-H{c['H']}")
def test_decode_step_lookahead(lsa, case):
    w = datagen.small_workload(emb_dtype="bf16", kv_dtype="bf16", seed=65, **dict(case))
    win = Window(w, lsa)
    dw = win.dw
    lsa.lsa_decode_step_lookahead(dw.dims, dw.q_emb, dw.chunk_emb, win.q, dw.K, dw.V, dw.ids, win.out, win.lse,
                                  dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    got = dw.ids.cpu().numpy()
    for b in range(w.B):
        ref_s = oracle.chunk_scores(dw.q_emb_f(b), dw.emb_f(b))
        gids = got[w.k_offsets[b]:w.k_offsets[b + 1]]
        G.check_ids(gids, oracle.topk(ref_s, w.k[b]), ref_s, w.k[b])
        _compare(win, b, gids)


@pytest.mark.parametrize("seed", range(12))
def test_decode_step_lookahead_random_shapes(lsa, seed):
    # the fused window step over random ragged batches: kept ids, then every query and head
    rng = np.random.default_rng(8000 + seed)
    B = int(rng.integers(1, 5))
    N = tuple(int(rng.integers(1, 300)) for _ in range(B))
    k = tuple(int(rng.integers(1, min(n, 60) + 1)) for n in N)
    case = dict(B=B, N=N, k=k, E=int(rng.choice([64, 128, 256])), Q=int(rng.integers(1, 65)),
                H=int(rng.choice([1, 2, 4, 8, 16])), C=int(rng.choice([16, 32, 64, 128])), plant="copy_query")
    w = datagen.small_workload(emb_dtype="bf16", kv_dtype="bf16", seed=8100 + seed, **case)
    win = Window(w, lsa)
    dw = win.dw
    lsa.lsa_decode_step_lookahead(dw.dims, dw.q_emb, dw.chunk_emb, win.q, dw.K, dw.V, dw.ids, win.out, win.lse,
                                  dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    got = dw.ids.cpu().numpy()
    big = w.Q * w.H * max(w.k) * w.C > 4_000_000
    for b in range(w.B):
        ref_s = oracle.chunk_scores(dw.q_emb_f(b), dw.emb_f(b))
        gids = got[w.k_offsets[b]:w.k_offsets[b + 1]]
        G.check_ids(gids, oracle.topk(ref_s, w.k[b]), ref_s, w.k[b])
        _compare(win, b, gids, sorted({0, w.H - 1}) if big else None, sorted({0, w.Q // 2, w.Q - 1}) if big else None)
    del win, dw
    _free()


def test_decode_step_lookahead_full_size_1m(lsa):
    # the 1M lookahead workload in the launch configuration the benchmark times: all kept ids,
    # sampled (head, query) outputs
    w = datagen.workload("1m")
    win = Window(w, lsa)
    dw = win.dw
    lsa.lsa_decode_step_lookahead(dw.dims, dw.q_emb, dw.chunk_emb, win.q, dw.K, dw.V, dw.ids, win.out, win.lse,
                                  dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    ref_s = oracle.chunk_scores(dw.q_emb_f(0), dw.emb_f(0))
    gids = dw.ids.cpu().numpy()
    G.check_ids(gids, oracle.topk(ref_s, w.k[0]), ref_s, w.k[0])
    assert set(datagen.planted_positions(w, 0).tolist()) <= set(gids.tolist())
    _compare(win, 0, gids, heads=[3, 12], queries=[0, 21, 63])
    del win, dw
    _free()


def test_lookahead_argument_errors(lsa):
    w = datagen.small_workload(B=1, N=(40,), k=(5,), C=64, E=64, Q=64, H=4, kv_dtype="f32", emb_dtype="bf16")
    dw = G.DeviceWorkload(w, lsa)
    q = torch.zeros((1, 64, 4, 128), dtype=torch.float32, device="cuda")
    out = torch.empty((1, 64, 4, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_sparse_decode_attn_lookahead(dw.dims, q, dw.K, dw.V, dw.ids, out, None, dw.ws)
    assert e.value.status == lsa.LSA_ERR_UNSUPPORTED  # fp32 K/V: the tensor-core path is bf16
    w2 = datagen.small_workload(B=1, N=(40,), k=(5,), C=64, E=64, Q=65, H=4, kv_dtype="bf16", emb_dtype="bf16")
    dw2 = G.DeviceWorkload(w2, lsa)
    q2 = torch.zeros((1, 65, 4, 128), dtype=torch.bfloat16, device="cuda")
    out2 = torch.empty((1, 65, 4, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_sparse_decode_attn_lookahead(dw2.dims, q2, dw2.K, dw2.V, dw2.ids, out2, None, dw2.ws)
    assert e.value.status == lsa.LSA_ERR_UNSUPPORTED  # more than 64 window queries


def test_lookahead_max_batch_many_runs_per_cta(lsa):
    # 256 short ragged sequences (C = 16, so ragged last tiles) and 2 heads: 564 tiles over the
    # CTAs, up to four (sequence, head) runs in one CTA (first split, whole ones, last split)
    rng = np.random.default_rng(3)
    N = tuple(int(x) for x in rng.integers(4, 13, size=256))
    k = tuple(int(rng.integers(1, n + 1)) for n in N)
    w = datagen.small_workload(B=256, N=N, k=k, E=64, Q=7, H=2, C=16, emb_dtype="bf16", kv_dtype="bf16", seed=66)
    win = Window(w, lsa)
    ids = win.random_ids(11)
    ids_d = torch.from_numpy(np.concatenate(ids)).cuda()
    lsa.lsa_sparse_decode_attn_lookahead(win.dw.dims, win.q, win.dw.K, win.dw.V, ids_d, win.out, win.lse, win.dw.ws)
    assert lsa.lsa_get_device_status(win.dw.ws) == lsa.LSA_OK
    for b in range(w.B):
        _compare(win, b, ids[b])
    del win
    _free()
