"""GPU parity: every C-ABI call against the float64 oracle on the same seeded inputs.

Small cases are compared element by element (several tiles and ragged tails);
the full-size decode workloads are run in the same launch configuration the
benchmark times and compared on all chunk ids and on sampled (sequence, head)
outputs, which the oracle recomputes from regenerated K/V rows."""

import numpy as np
import pytest
import torch

import datagen
import oracle
from datagen import device as dgdev
from tests import _gpu as G
from tests import _gpu as GPU  # the same module, for tests where G is a rank count

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from learned_sparse_kv_decode_b200 import build
    build.build()
    import learned_sparse_kv_decode_b200 as m
    return m


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ input generator
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_device_generator_matches_host(dt):
    n, first = 100_003, 12_345_678_901
    t = torch.empty(n, dtype=G.tdtype(dt), device="cuda")
    dgdev.fill_normal(t, 7, 4, first)
    host = datagen.normal_f32(7, 4, np.arange(first, first + n, dtype=np.uint64))
    if dt == "bf16":
        got = t.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got, datagen.bf16_bits(host))
    else:
        np.testing.assert_array_equal(t.cpu().numpy(), host)


# ------------------------------------------------------------------ scores
SCORE_CASES = [
    dict(name="f32-E64", emb_dtype="f32", E=64, Q=1, N=(40, 72, 1)),
    dict(name="f32-E128", emb_dtype="f32", E=128, Q=1, N=(300, 1, 77)),
    dict(name="f32-E256", emb_dtype="f32", E=256, Q=1, N=(129, 64)),
    dict(name="bf16-E128", emb_dtype="bf16", E=128, Q=1, N=(2048, 5, 333)),
    dict(name="bf16-E256", emb_dtype="bf16", E=256, Q=1, N=(1000, 17)),
    dict(name="bf16-E1024", emb_dtype="bf16", E=1024, Q=1, N=(70, 3)),
    dict(name="f32-Q3", emb_dtype="f32", E=128, Q=3, N=(90, 31)),
    dict(name="umma-Q64-E256", emb_dtype="bf16", E=256, Q=64, N=(300, 129, 128, 1)),
    dict(name="umma-Q64-E128", emb_dtype="bf16", E=128, Q=64, N=(513, 7)),
    dict(name="umma-Q3-E64", emb_dtype="bf16", E=64, Q=3, N=(260,)),
    dict(name="umma-Q200-E128", emb_dtype="bf16", E=128, Q=200, N=(140, 120)),
    dict(name="umma-Q256-E256", emb_dtype="bf16", E=256, Q=256, N=(200, 3)),   # largest swizzled tiles
    dict(name="umma16-Q5-E32", emb_dtype="bf16", E=32, Q=5, N=(150, 9)),      # E not a multiple of 64:
    dict(name="umma16-Q16-E16", emb_dtype="bf16", E=16, Q=16, N=(77,)),       # 16-byte-column tiles
]


@pytest.mark.parametrize("case", SCORE_CASES, ids=lambda c: c["name"])
def test_score_chunks_parity(lsa, case):
    N = case["N"]
    w = datagen.small_workload(B=len(N), N=N, E=case["E"], Q=case["Q"], k=[1] * len(N), H=4,
                               emb_dtype=case["emb_dtype"], seed=21, plant="copy_query" if case["Q"] > 1 else "copy")
    dw = G.DeviceWorkload(w, lsa, with_kv=False)
    lsa.lsa_score_chunks(dw.dims, dw.q_emb, dw.chunk_emb, dw.scores, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    got = dw.scores.cpu().numpy()
    off = w.chunk_offsets
    for b in range(w.B):
        qf, ef = dw.q_emb_f(b), dw.emb_f(b)
        ref = oracle.chunk_scores(qf, ef)
        G.check_scores(got[off[b]:off[b + 1]], ref, G.score_tolerance(qf, ef))


@pytest.mark.parametrize("seed", range(24))
def test_score_chunks_random_shapes(lsa, seed):
    # random ragged batches over every scorer: one query (staged stream), several queries on the
    # CUDA cores (fp32) or on the tensor cores (bf16, E a multiple of 16), up to 256 queries
    rng = np.random.default_rng(5000 + seed)
    emb_dtype = str(rng.choice(["f32", "bf16"]))
    E = int(rng.choice([16, 32, 64, 128, 256] if emb_dtype == "bf16" else [64, 128, 256]))
    Q = int(rng.choice([1, 1, 2, 5, 16, 64, 200, 256]))
    if emb_dtype == "f32":  # the CUDA-core scorer holds the queries in shared memory (<= 200 KiB)
        Q = min(Q, 200 * 1024 // (4 * E))
    B = int(rng.integers(1, 9))
    N = tuple(int(rng.integers(1, 700)) for _ in range(B))
    w = datagen.small_workload(B=B, N=N, E=E, Q=Q, k=[1] * B, H=4, emb_dtype=emb_dtype, seed=5100 + seed,
                               plant="copy_query" if Q > 1 else "copy")
    dw = G.DeviceWorkload(w, lsa, with_kv=False)
    lsa.lsa_score_chunks(dw.dims, dw.q_emb, dw.chunk_emb, dw.scores, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    got = dw.scores.cpu().numpy()
    off = w.chunk_offsets
    for b in range(w.B):
        qf, ef = dw.q_emb_f(b), dw.emb_f(b)
        G.check_scores(got[off[b]:off[b + 1]], oracle.chunk_scores(qf, ef), G.score_tolerance(qf, ef))


@pytest.mark.parametrize("seed", range(24))
def test_topk_and_threshold_random(lsa, seed):
    # random ragged sequences of continuous or tie-heavy scores, random k, and a random threshold
    rng = np.random.default_rng(6000 + seed)
    B = int(rng.integers(1, 9))
    N = tuple(int(rng.integers(1, 40000 if seed % 4 == 0 else 3000)) for _ in range(B))
    k = tuple(int(rng.integers(1, n + 1)) for n in N)
    w = datagen.small_workload(B=B, N=N, k=k, E=64)
    dims = G.dims_of(w, lsa)
    ws = lsa.alloc_workspace(dims)
    s = np.concatenate([_tie_scores(n, 6100 + 10 * seed + i, levels=float(rng.choice([4.0, 1e6])))
                        for i, n in enumerate(N)])
    sd = torch.from_numpy(s).cuda()
    ids = torch.empty(w.total_kept, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_select(dims, sd, ids, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK
    got = ids.cpu().numpy()
    off, koff = w.chunk_offsets, w.k_offsets
    for b in range(w.B):
        np.testing.assert_array_equal(got[koff[b]:koff[b + 1]], oracle.topk(s[off[b]:off[b + 1]].astype(np.float64), k[b]))
    tau = np.float32(np.quantile(s, rng.uniform(0.5, 0.99)))
    k_min = int(rng.integers(1, 5))
    cnt = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    lsa.lsa_threshold_select(dims, sd, tau, k_min, ids, cnt, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK
    got, got_cnt = ids.cpu().numpy(), cnt.cpu().numpy()
    for b in range(w.B):
        ref = oracle.threshold_select(s[off[b]:off[b + 1]].astype(np.float64), tau, k_min, k[b])
        assert got_cnt[b] == len(ref)
        np.testing.assert_array_equal(got[koff[b]:koff[b] + len(ref)], ref)
        assert (got[koff[b] + len(ref):koff[b + 1]] == -1).all()


# ------------------------------------------------------------------ top-k
def _tie_scores(n, seed, levels=4.0):
    x = datagen.normal_f32(seed, 1, np.arange(n))
    return (np.round(x * levels) / levels).astype(np.float32)  # many exact ties


@pytest.mark.parametrize("N,k", [((1,), (1,)), ((7, 64), (3, 64)), ((300, 500), (40, 499)),
                                 ((1000, 999), (1, 998)),
                                 ((5000, 16384), (700, 2212)),
                                 ((30000, 17000), (4000, 2)),   # 16 keys per thread in an 8-CTA cluster
                                 ((60000,), (6000,)),
                                 ((120_000,), (16_000,)),       # per-CTA slices in shared memory
                                 ((400_000, 3), (54_000, 2))])  # slices too big for shared memory
def test_topk_bit_exact_with_ties(lsa, N, k):
    w = datagen.small_workload(B=len(N), N=N, k=k, E=64)
    dims = G.dims_of(w, lsa)
    ws = lsa.alloc_workspace(dims)
    s = np.concatenate([_tie_scores(n, 100 + i) for i, n in enumerate(N)])
    s[::17] = -s[::17]
    ids = torch.empty(w.total_kept, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_select(dims, torch.from_numpy(s).cuda(), ids, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK
    got = ids.cpu().numpy()
    off, koff = w.chunk_offsets, w.k_offsets
    for b in range(w.B):
        ref = oracle.topk(s[off[b]:off[b + 1]].astype(np.float64), k[b])
        np.testing.assert_array_equal(got[koff[b]:koff[b + 1]], ref)


def test_topk_signed_zero_and_all_equal(lsa):
    w = datagen.small_workload(B=3, N=(8, 10, 6), k=(7, 4, 6), E=64)
    dims = G.dims_of(w, lsa)
    ws = lsa.alloc_workspace(dims)
    s = np.array([3, 7, 7, 1, 7, -0.0, 0.0, 5] + [2.5] * 10 + [-1, -2, -3, -0.0, -5, -6], np.float32)
    ids = torch.empty(w.total_kept, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_select(dims, torch.from_numpy(s).cuda(), ids, ws)
    got = ids.cpu().numpy()
    np.testing.assert_array_equal(got[:7], [0, 1, 2, 3, 4, 5, 7])
    np.testing.assert_array_equal(got[7:11], [0, 1, 2, 3])
    np.testing.assert_array_equal(got[11:], [0, 1, 2, 3, 4, 5])


@pytest.mark.parametrize("k", [1, 17, 150, 299])
def test_topk_subnormal_scores(lsa, k):
    # subnormals of both signs, the smallest normals and +-0, repeated (ties): the
    # order-preserving key map must order them as floats do, with no flush to zero
    sub = np.array([1, 2, 3, 7, 1000, 2**22 - 1], np.uint32).view(np.float32)
    tiny = np.finfo(np.float32).tiny
    base = np.concatenate([sub, -sub, np.array([tiny, -tiny, 2 * tiny, -3 * tiny, 0.0, -0.0], np.float32)])
    rng = np.random.default_rng(31)
    s = rng.permutation(np.tile(base, 25)).astype(np.float32)   # 450 scores
    w = datagen.small_workload(B=1, N=(len(s),), k=(k,), E=64)
    dims = G.dims_of(w, lsa)
    ws = lsa.alloc_workspace(dims)
    ids = torch.empty(k, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_select(dims, torch.from_numpy(s).cuda(), ids, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK
    np.testing.assert_array_equal(ids.cpu().numpy(), oracle.topk(s.astype(np.float64), k))


def test_topk_nonfinite_reported(lsa):
    w = datagen.small_workload(B=1, N=(50,), k=(10,), E=64)
    dims = G.dims_of(w, lsa)
    ws = lsa.alloc_workspace(dims)
    s = _tie_scores(50, 3)
    s[11] = np.nan
    ids = torch.empty(10, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_select(dims, torch.from_numpy(s).cuda(), ids, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_ERR_NONFINITE
    got = ids.cpu().numpy()
    assert got.min() >= 0 and got.max() < 50 and 11 not in got
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK  # the word was cleared


# ------------------------------------------------------------------ read-stream utility
def test_read_stream_runs(lsa):
    # the measurement utility reads a buffer with a ragged tail (not a multiple of the unrolled
    # stride) and leaves the context usable; an unaligned view is rejected on the host
    buf = torch.empty((64 << 20) + 48, dtype=torch.uint8, device="cuda")
    lsa.lsa_read_stream(buf)
    torch.cuda.synchronize()
    with pytest.raises(lsa.LsaError):
        lsa.lsa_read_stream(buf[8:8 + 1024])
    torch.cuda.synchronize()


# ------------------------------------------------------------------ gather
@pytest.mark.parametrize("kv_dtype,H,C", [("f32", 8, 64), ("bf16", 16, 64), ("bf16", 2, 32), ("f32", 1, 8)])
def test_gather_bit_exact(lsa, kv_dtype, H, C):
    w = datagen.small_workload(B=3, N=(9, 4, 13), k=(3, 4, 5), E=64, H=H, C=C, kv_dtype=kv_dtype)
    dw = G.DeviceWorkload(w, lsa)
    rng = np.random.default_rng(5)
    ids = np.concatenate([np.sort(rng.permutation(n)[:k]) for n, k in zip(w.N, w.k)]).astype(np.int32)
    Kr = torch.empty((w.total_kept * C, H, w.Dh), dtype=G.tdtype(kv_dtype), device="cuda")
    Vr = torch.empty_like(Kr)
    lsa.lsa_gather_kv(dw.dims, dw.K, dw.V, torch.from_numpy(ids).cuda(), Kr, Vr, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    koff = w.k_offsets
    Kg, Vg = Kr.float().cpu().numpy(), Vr.float().cpu().numpy()
    for b in range(w.B):
        tok = oracle.kept_tokens(ids[koff[b]:koff[b + 1]], C)
        rows = slice(koff[b] * C, koff[b + 1] * C)
        np.testing.assert_array_equal(Kg[rows], dw.kv_f("K", b, tok))
        np.testing.assert_array_equal(Vg[rows], dw.kv_f("V", b, tok))


@pytest.mark.parametrize("seed", range(16))
def test_gather_random_shapes(lsa, seed):
    # random ragged batches, heads, chunk lengths and kept sets: every gathered row bit-exact
    rng = np.random.default_rng(7000 + seed)
    kv_dtype = str(rng.choice(["f32", "bf16"]))
    H = int(rng.choice([1, 2, 4, 8, 16]))
    C = int(rng.choice([8, 16, 32, 64, 128]))
    B = int(rng.integers(1, 7))
    N = tuple(int(rng.integers(1, 80)) for _ in range(B))
    k = tuple(int(rng.integers(1, n + 1)) for n in N)
    w = datagen.small_workload(B=B, N=N, k=k, E=64, H=H, C=C, kv_dtype=kv_dtype, seed=7100 + seed)
    dw = G.DeviceWorkload(w, lsa)
    ids = np.concatenate([np.sort(rng.permutation(n)[:kk]) for n, kk in zip(N, k)]).astype(np.int32)
    Kr = torch.empty((w.total_kept * C, H, w.Dh), dtype=G.tdtype(kv_dtype), device="cuda")
    Vr = torch.empty_like(Kr)
    lsa.lsa_gather_kv(dw.dims, dw.K, dw.V, torch.from_numpy(ids).cuda(), Kr, Vr, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    koff = w.k_offsets
    Kg, Vg = Kr.float().cpu().numpy(), Vr.float().cpu().numpy()
    for b in range(w.B):
        tok = oracle.kept_tokens(ids[koff[b]:koff[b + 1]], C)
        rows = slice(koff[b] * C, koff[b + 1] * C)
        np.testing.assert_array_equal(Kg[rows], dw.kv_f("K", b, tok))
        np.testing.assert_array_equal(Vg[rows], dw.kv_f("V", b, tok))
    del dw
    _free()


def test_gather_bad_id_reported(lsa):
    w = datagen.small_workload(B=1, N=(5,), k=(2,), E=64, H=2)
    dw = G.DeviceWorkload(w, lsa)
    Kr = torch.zeros((2 * w.C, 2, w.Dh), dtype=torch.float32, device="cuda")
    Vr = torch.zeros_like(Kr)
    lsa.lsa_gather_kv(dw.dims, dw.K, dw.V, torch.tensor([1, 5], dtype=torch.int32, device="cuda"), Kr, Vr, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_ERR_BAD_ID
    np.testing.assert_array_equal(Kr[:w.C].cpu().numpy(), dw.kv_f("K", 0, np.arange(w.C, 2 * w.C)))
    assert float(Kr[w.C:].abs().max()) == 0.0


# ------------------------------------------------------------------ sparse attention
ATTN_CASES = [
    dict(kv_dtype="f32", H=8, C=64, N=(20, 9), k=(6, 9)),
    dict(kv_dtype="bf16", H=16, C=64, N=(30, 3, 11), k=(10, 1, 11)),
    dict(kv_dtype="bf16", H=8, C=64, N=(12, 40), k=(12, 5)),
    dict(kv_dtype="bf16", H=32, C=64, N=(6,), k=(4,)),
    dict(kv_dtype="bf16", H=1, C=16, N=(50, 2), k=(33, 2)),
    dict(kv_dtype="f32", H=2, C=8, N=(64,), k=(17,)),
    dict(kv_dtype="f32", H=16, C=32, N=(10, 10), k=(3, 7)),
    dict(kv_dtype="bf16", H=4, C=128, N=(7, 5, 9, 1), k=(2, 5, 9, 1)),
]


@pytest.mark.parametrize("mode", ["indexed", "resident"])
@pytest.mark.parametrize("case", ATTN_CASES, ids=lambda c: f"{c['kv_dtype']}-H{c['H']}-C{c['C']}-B{len(c['N'])}")
def test_sparse_attention_parity(lsa, case, mode):
    w = datagen.small_workload(B=len(case["N"]), N=case["N"], k=case["k"], E=64, H=case["H"], C=case["C"],
                               kv_dtype=case["kv_dtype"], seed=33)
    dw = G.DeviceWorkload(w, lsa)
    rng = np.random.default_rng(7)
    ids = np.concatenate([np.sort(rng.permutation(n)[:k]) for n, k in zip(w.N, w.k)]).astype(np.int32)
    ids_d = torch.from_numpy(ids).cuda()
    if mode == "indexed":
        lsa.lsa_sparse_decode_attn(dw.dims, dw.q, dw.K, dw.V, ids_d, dw.out, dw.lse, dw.ws)
    else:
        Kr = torch.empty((w.total_kept * w.C, w.H, w.Dh), dtype=G.tdtype(w.kv_dtype), device="cuda")
        Vr = torch.empty_like(Kr)
        lsa.lsa_gather_kv(dw.dims, dw.K, dw.V, ids_d, Kr, Vr, dw.ws)
        lsa.lsa_sparse_decode_attn(dw.dims, dw.q, Kr, Vr, None, dw.out, dw.lse, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    out, lse = dw.out.cpu().numpy(), dw.lse.cpu().numpy()
    koff = w.k_offsets
    for b in range(w.B):
        ref_o, ref_l = G.oracle_attention(dw, b, ids[koff[b]:koff[b + 1]])
        np.testing.assert_allclose(out[b], ref_o, rtol=0, atol=G.ATTN_ATOL[w.kv_dtype])
        np.testing.assert_allclose(out[b], ref_o, rtol=0, atol=1e-4)   # fp32 arithmetic on exact inputs
        np.testing.assert_allclose(lse[b], ref_l, rtol=0, atol=1e-4)


@pytest.mark.parametrize("kv_dtype,C", [("f32", 64), ("bf16", 64), ("bf16", 16)])
def test_attention_bad_id_reported(lsa, kv_dtype, C):
    # out-of-range ids are reported and skipped: each sequence attends over its valid ids only,
    # including the sequences that hold the bad ids; a sequence with no valid id gets out 0, lse -inf
    w = datagen.small_workload(B=4, N=(4, 6, 9, 3), k=(2, 3, 4, 1), E=64, H=8, C=C, kv_dtype=kv_dtype)
    dw = G.DeviceWorkload(w, lsa)
    ids = np.array([0, 1,  2, -3, 5,  1, 9, 4, 8,  3], dtype=np.int32)
    valid = [np.array([0, 1]), np.array([2, 5]), np.array([1, 4, 8]), None]
    lsa.lsa_sparse_decode_attn(dw.dims, dw.q, dw.K, dw.V, torch.from_numpy(ids).cuda(), dw.out, dw.lse, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_ERR_BAD_ID
    out, lse = dw.out.cpu().numpy(), dw.lse.cpu().numpy()
    for b, v in enumerate(valid):
        if v is None:
            np.testing.assert_array_equal(out[b], 0.0)
            assert np.isneginf(lse[b]).all()
            continue
        ref_o, ref_l = G.oracle_attention(dw, b, v)
        np.testing.assert_allclose(out[b], ref_o, rtol=0, atol=1e-4)
        np.testing.assert_allclose(lse[b], ref_l, rtol=0, atol=1e-4)


# ------------------------------------------------------------------ fused decode step
def _run_step(lsa, dw):
    lsa.lsa_decode_step(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, dw.ids, dw.out, dw.lse, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK


def _check_step(dw, seqs=None, heads_per_seq=None):
    w = dw.w
    got_ids, out, lse = dw.ids.cpu().numpy(), dw.out.cpu().numpy(), dw.lse.cpu().numpy()
    koff = w.k_offsets
    seqs = range(w.B) if seqs is None else seqs
    exempt = 0
    for b in range(w.B):
        ref_s = oracle.chunk_scores(dw.q_emb_f(b), dw.emb_f(b))
        ref_ids = oracle.topk(ref_s, w.k[b])
        gids = got_ids[koff[b]:koff[b + 1]]
        exempt += G.check_ids(gids, ref_ids, ref_s, w.k[b])
        if b not in seqs:
            continue
        heads = None if heads_per_seq is None else heads_per_seq(b)
        ref_o, ref_l = G.oracle_attention(dw, b, gids, heads)
        got_o = out[b] if heads is None else out[b][heads]
        got_l = lse[b] if heads is None else lse[b][heads]
        np.testing.assert_allclose(got_o, ref_o, rtol=0, atol=G.ATTN_ATOL[w.kv_dtype])
        np.testing.assert_allclose(got_o, ref_o, rtol=0, atol=1e-4)
        np.testing.assert_allclose(got_l, ref_l, rtol=0, atol=1e-4)
    return exempt


def test_decode_step_tiny_full(lsa):
    dw = G.DeviceWorkload(datagen.workload("tiny"), lsa)
    _run_step(lsa, dw)
    assert _check_step(dw) == 0
    planted = datagen.planted_positions(dw.w, 0)
    assert set(planted.tolist()) <= set(dw.ids.cpu().numpy().tolist())


STEP_CASES = [
    dict(B=3, N=(40, 72, 5), k=(5, 9, 5), E=64, H=4, emb_dtype="f32", kv_dtype="f32"),
    dict(B=2, N=(300, 129), k=(40, 1), E=128, H=16, emb_dtype="bf16", kv_dtype="bf16"),
    dict(B=4, N=(33, 65, 1, 200), k=(33, 8, 1, 27), E=256, H=8, emb_dtype="bf16", kv_dtype="bf16"),
    dict(B=1, N=(600,), k=(81,), E=256, Q=64, H=16, emb_dtype="bf16", kv_dtype="bf16", plant="copy_query"),
    dict(B=2, N=(130, 257), k=(18, 35), E=128, Q=64, H=16, emb_dtype="bf16", kv_dtype="bf16", plant="copy_query"),
]


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: f"B{c['B']}-E{c['E']}-Q{c.get('Q', 1)}-H{c['H']}-{c['kv_dtype']}")
def test_decode_step_small(lsa, case):
    case = dict(case)
    w = datagen.small_workload(seed=44, **case)
    dw = G.DeviceWorkload(w, lsa)
    _run_step(lsa, dw)
    _check_step(dw)


# Small problems run the whole step in one launch (k_decode_small): one query per sequence, at most
# 48 (sequence, head) pairs, at most 256 chunks per sequence, rows <= 512 B, kept K/V <= 16 MB;
# with k_b <= 8 everywhere the partials are merged inside a cluster, otherwise through the workspace.
ONE_LAUNCH_CASES = [
    dict(B=1, N=(256,), k=(256,), E=64, H=2, C=8, emb_dtype="f32", kv_dtype="f32"),       # k = N = 256
    dict(B=3, N=(1, 37, 256), k=(1, 5, 19), E=128, H=16, C=16, emb_dtype="bf16", kv_dtype="bf16"),
    dict(B=2, N=(9, 20), k=(2, 3), E=256, H=2, C=1024, emb_dtype="bf16", kv_dtype="f32"),  # 1024-token chunks
    dict(B=6, N=(64, 3, 17, 100, 8, 50), k=(8, 3, 1, 12, 8, 7), E=128, H=8, C=64, emb_dtype="f32", kv_dtype="bf16"),
    # k_b <= 8 everywhere: the CTAs of a (sequence, head) merge inside a thread-block cluster
    dict(B=5, N=(8, 1, 30, 64, 3), k=(8, 1, 2, 5, 3), E=64, H=4, C=32, emb_dtype="bf16", kv_dtype="bf16"),
    dict(B=3, N=(200, 9, 40), k=(7, 8, 1), E=128, H=8, C=128, emb_dtype="f32", kv_dtype="f32"),
]


@pytest.mark.parametrize("case", ONE_LAUNCH_CASES, ids=lambda c: f"B{c['B']}-C{c['C']}-{c['emb_dtype']}-{c['kv_dtype']}")
def test_decode_step_one_launch(lsa, case):
    w = datagen.small_workload(seed=47, **case)
    dw = G.DeviceWorkload(w, lsa)
    for _ in range(3):  # the arrival counters are back at zero after every call
        dw.out.fill_(float("nan"))
        _run_step(lsa, dw)
        _check_step(dw)
    a = (dw.ids.clone(), dw.out.clone(), dw.lse.clone())
    _run_step(lsa, dw)  # deterministic whichever CTA merges
    assert torch.equal(a[0], dw.ids) and torch.equal(a[1], dw.out) and torch.equal(a[2], dw.lse)


@pytest.mark.parametrize("small", [True, False], ids=["one-launch", "four-kernels"])
def test_decode_step_nonfinite_reported(lsa, small):
    # a NaN chunk embedding gives a NaN score: reported as LSA_ERR_NONFINITE, never kept, and
    # the step still attends over valid ids only (both the one-launch and the four-kernel path)
    N = (40, 72) if small else (300, 129)
    w = datagen.small_workload(B=2, N=N, k=(5, 9), E=64, H=4, emb_dtype="f32", kv_dtype="f32", seed=48)
    dw = G.DeviceWorkload(w, lsa)
    bad_row = 7
    dw.chunk_emb[bad_row, 3] = float("nan")
    lsa.lsa_decode_step(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, dw.ids, dw.out, dw.lse, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_ERR_NONFINITE
    got = dw.ids.cpu().numpy()
    koff = w.k_offsets
    for b in range(w.B):
        mine = got[koff[b]:koff[b + 1]]
        assert np.all(np.diff(mine) > 0) and mine.min() >= 0 and mine.max() < w.N[b]
        if b == 0:
            assert bad_row not in mine
        ref_o, _ = G.oracle_attention(dw, b, mine)
        np.testing.assert_allclose(dw.out[b].cpu().numpy(), ref_o, rtol=0, atol=1e-4)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK  # the word was cleared


def test_decode_step_max_batch(lsa):
    # LSA_MAX_BATCH sequences, ragged lengths and keep counts, in one call
    rng = np.random.default_rng(21)
    N = tuple(int(x) for x in rng.integers(1, 40, size=256))
    k = tuple(int(rng.integers(1, n + 1)) for n in N)
    w = datagen.small_workload(B=256, N=N, k=k, E=64, H=2, C=16, emb_dtype="bf16", kv_dtype="bf16", seed=45)
    dw = G.DeviceWorkload(w, lsa)
    _run_step(lsa, dw)
    _check_step(dw)
    del dw
    _free()


def _fuzz_case(seed):
    """A random valid fused-step shape: ragged N_b and k_b, dtypes, heads, chunk length, queries
    (Q = 1 takes the CUDA-core scorer or, when small, the one-launch step; Q > 1 with bf16
    embeddings the tensor-core scorer), with the full K/V cache kept under 512 MB."""
    rng = np.random.default_rng(1000 + seed)
    while True:
        B = int(rng.integers(1, 7))
        emb_dtype = str(rng.choice(["f32", "bf16"]))
        kv_dtype = str(rng.choice(["f32", "bf16"]))
        E = int(rng.choice([64, 128] if emb_dtype == "f32" else [64, 128, 256]))
        Q = int(rng.choice([1, 1, 3, 64])) if emb_dtype == "bf16" else int(rng.choice([1, 1, 3]))
        H = int(rng.choice([1, 2, 4, 8, 16, 32]))
        C = int(rng.choice([8, 16, 32, 64, 128]))
        N = [int(rng.integers(1, 260)) for _ in range(B)]
        k = [int(rng.integers(1, min(n, 70) + 1)) for n in N]
        kv_bytes = sum(N) * C * H * 128 * (2 if kv_dtype == "bf16" else 4) * 2
        if kv_bytes <= (512 << 20):
            return dict(B=B, N=tuple(N), k=tuple(k), E=E, Q=Q, H=H, C=C, emb_dtype=emb_dtype,
                        kv_dtype=kv_dtype, seed=2000 + seed)


@pytest.mark.parametrize("seed", range(48))
def test_decode_step_random_shapes(lsa, seed):
    # every sequence and head against the oracle: ids (near-tie rule) and attention on them
    w = datagen.small_workload(**_fuzz_case(seed))
    dw = G.DeviceWorkload(w, lsa)
    _run_step(lsa, dw)
    _check_step(dw)
    del dw
    _free()


def test_decode_step_deterministic(lsa):
    w = datagen.small_workload(B=2, N=(300, 129), k=(40, 7), E=128, H=16, emb_dtype="bf16", kv_dtype="bf16")
    dw = G.DeviceWorkload(w, lsa)
    _run_step(lsa, dw)
    a = (dw.ids.clone(), dw.out.clone(), dw.lse.clone())
    for _ in range(3):
        _run_step(lsa, dw)
        assert torch.equal(a[0], dw.ids) and torch.equal(a[1], dw.out) and torch.equal(a[2], dw.lse)


def test_decode_step_keep_all_is_dense_attention(lsa):
    # k = N: the LSA step is plain dense decode attention (checked against torch SDPA in float64)
    w = datagen.small_workload(B=2, N=(12, 7), k=(12, 7), E=64, H=8, kv_dtype="f32")
    dw = G.DeviceWorkload(w, lsa)
    _run_step(lsa, dw)
    for b in range(w.B):
        L = w.L[b]
        K = torch.from_numpy(dw.kv_f("K", b, np.arange(L)).astype(np.float64)).permute(1, 0, 2)
        V = torch.from_numpy(dw.kv_f("V", b, np.arange(L)).astype(np.float64)).permute(1, 0, 2)
        q = torch.from_numpy(dw.q_f(b).astype(np.float64))[:, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(q, K, V)[:, 0, :].numpy()
        np.testing.assert_allclose(dw.out[b].cpu().numpy(), ref, rtol=0, atol=1e-4)


# ------------------------------------------------------------------ full-size workloads
@pytest.mark.parametrize("name", ["128k", "500k", "1m", "mixed"])
def test_decode_step_full_size(lsa, name):
    w = datagen.workload(name)
    dw = G.DeviceWorkload(w, lsa)
    _run_step(lsa, dw)
    rng = np.random.default_rng(1)
    seqs = sorted(rng.permutation(w.B)[:2].tolist())
    _check_step(dw, seqs=seqs)  # every chunk id of every sequence; all heads of two sequences
    if w.plant == "copy":
        got = dw.ids.cpu().numpy()
        for b in range(w.B):
            kept = set(got[w.k_offsets[b]:w.k_offsets[b + 1]].tolist())
            assert set(datagen.planted_positions(w, b).tolist()) <= kept
    del dw
    _free()


# ------------------------------------------------------------------ argument errors
def test_argument_errors(lsa):
    w = datagen.small_workload(B=1, N=(8,), k=(2,), E=64, H=4)
    dw = G.DeviceWorkload(w, lsa)
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_decode_step(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, dw.ids, dw.out, dw.lse, dw.ws[:64])
    assert e.value.status == lsa.LSA_ERR_WORKSPACE
    raw = torch.empty(dw.scores.numel() + 4, dtype=torch.float32, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_score_chunks(dw.dims, dw.q_emb, dw.chunk_emb, raw[1:], dw.ws)  # 4-byte offset: misaligned
    assert e.value.status == lsa.LSA_ERR_INVALID_ARG
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_sparse_decode_attn(dw.dims, None, dw.K, dw.V, dw.ids, dw.out, None, dw.ws)
    assert e.value.status == lsa.LSA_ERR_INVALID_ARG


# ------------------------------------------------------------------ resident refresh (retrieval cycle)
REFRESH_CASES = [
    dict(B=2, N=(40, 72), k=(6, 11), E=64, H=8, kv_dtype="f32", emb_dtype="f32"),
    dict(B=3, N=(300, 129, 64), k=(40, 17, 64), E=128, H=16, kv_dtype="bf16", emb_dtype="bf16"),
    dict(B=1, N=(600,), k=(81,), E=256, Q=64, H=16, kv_dtype="bf16", emb_dtype="bf16", plant="copy_query"),
]


def _random_refresh_case(seed):
    rng = np.random.default_rng(9000 + seed)
    B = int(rng.integers(1, 6))
    N = tuple(int(rng.integers(1, 400)) for _ in range(B))
    dt = str(rng.choice(["f32", "bf16"]))
    return dict(B=B, N=N, k=tuple(int(rng.integers(1, n + 1)) for n in N), E=int(rng.choice([64, 128])),
                H=int(rng.choice([1, 2, 4, 8])), C=int(rng.choice([16, 32, 64])), kv_dtype=dt, emb_dtype=dt)


REFRESH_CASES += [_random_refresh_case(i) for i in range(8)]  # seeded random ragged shapes


def _check_resident(dw, slots, Kr, Vr, skip=None):
    w = dw.w
    Kg, Vg = Kr.float().cpu().numpy(), Vr.float().cpu().numpy()
    for b in range(w.B):
        for j in range(w.k[b]):
            g = int(w.k_offsets[b]) + j
            if skip is not None and g in skip:
                continue
            tok = oracle.kept_tokens([slots[g]], w.C)
            rows = slice(g * w.C, (g + 1) * w.C)
            np.testing.assert_array_equal(Kg[rows], dw.kv_f("K", b, tok))
            np.testing.assert_array_equal(Vg[rows], dw.kv_f("V", b, tok))


@pytest.mark.parametrize("case", REFRESH_CASES, ids=lambda c: f"B{c['B']}-Q{c.get('Q', 1)}-{c['kv_dtype']}")
def test_refresh_resident_cycles(lsa, case):
    w = datagen.small_workload(seed=55, **case)
    dw = G.DeviceWorkload(w, lsa)
    koff = w.k_offsets
    slots = torch.full((w.total_kept,), -1, dtype=torch.int32, device="cuda")
    Kr = torch.zeros((w.total_kept * w.C, w.H, w.Dh), dtype=G.tdtype(w.kv_dtype), device="cuda")
    Vr = torch.zeros_like(Kr)
    moved = torch.zeros(w.B, dtype=torch.int32, device="cuda")

    def oracle_ids(q_emb_host):
        out = []
        for b in range(w.B):
            qf = datagen.as_f32(q_emb_host[b], w.emb_dtype)
            s = oracle.chunk_scores(qf, dw.emb_f(b))
            out.append((oracle.topk(s, w.k[b]), s))
        return out

    # cycle 1: cold start (all slots empty)
    lsa.lsa_refresh_resident(dw.dims, dw.q_emb, dw.chunk_emb, dw.K, dw.V, slots, Kr, Vr, moved, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    got = slots.cpu().numpy()
    for b, (ids, s) in enumerate(oracle_ids(dw.host["q_emb"])):
        mine = got[koff[b]:koff[b + 1]]
        G.check_ids(np.sort(mine), ids, s, w.k[b])
        exp, _ = oracle.refresh_resident([-1] * w.k[b], ids, w.N[b])
        np.testing.assert_array_equal(mine, exp)
    np.testing.assert_array_equal(moved.cpu().numpy(), w.k)
    _check_resident(dw, got, Kr, Vr)

    # cycle 2: another query; slots whose chunk stays are poisoned first and must not be rewritten
    v = datagen.make_query_variant(w, 1)
    q_emb2 = G.to_device(v["q_emb"], w.emb_dtype)
    new = oracle_ids(v["q_emb"])
    old = got.copy()
    staying = set()
    expected = np.empty_like(old)
    n_copies = []
    for b, (ids, s) in enumerate(new):
        exp, copies = oracle.refresh_resident(old[koff[b]:koff[b + 1]], ids, w.N[b])
        expected[koff[b]:koff[b + 1]] = exp
        n_copies.append(len(copies))
        kept = set(ids.tolist())
        for j, c in enumerate(old[koff[b]:koff[b + 1]]):
            if c in kept:
                staying.add(int(koff[b]) + j)
    for g in staying:
        Kr[g * w.C:(g + 1) * w.C] = 7.0
        Vr[g * w.C:(g + 1) * w.C] = -7.0
    lsa.lsa_refresh_resident(dw.dims, q_emb2, dw.chunk_emb, dw.K, dw.V, slots, Kr, Vr, moved, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    np.testing.assert_array_equal(slots.cpu().numpy(), expected)
    np.testing.assert_array_equal(moved.cpu().numpy(), n_copies)
    assert sum(n_copies) < w.total_kept or not staying
    _check_resident(dw, expected, Kr, Vr, skip=staying)
    for g in staying:  # untouched: still the poison
        assert float(Kr[g * w.C:(g + 1) * w.C].float().min()) == 7.0
        assert float(Vr[g * w.C:(g + 1) * w.C].float().max()) == -7.0

    # attention over the resident buffer (slot order) equals attention over the kept set
    for g in staying:  # restore the poisoned slots from the cache first
        b = int(np.searchsorted(koff, g, side="right") - 1)
        tok = oracle.kept_tokens([expected[g]], w.C)
        Kr[g * w.C:(g + 1) * w.C] = torch.from_numpy(dw.kv_f("K", b, tok)).to(Kr.dtype).cuda()
        Vr[g * w.C:(g + 1) * w.C] = torch.from_numpy(dw.kv_f("V", b, tok)).to(Vr.dtype).cuda()
    lsa.lsa_sparse_decode_attn(dw.dims, dw.q, Kr, Vr, None, dw.out, dw.lse, dw.ws)
    out = dw.out.cpu().numpy()
    for b, (ids, _) in enumerate(new):
        ref_o, _ = G.oracle_attention(dw, b, ids)
        np.testing.assert_allclose(out[b], ref_o, rtol=0, atol=1e-4)


# ------------------------------------------------------------------ threshold keep mask
@pytest.mark.parametrize("N,kmax", [((64,), (64,)), ((7, 2048), (7, 300)), ((5000, 16384), (900, 2500)),
                                    ((60000,), (9000,))])
@pytest.mark.parametrize("tau_kind", ["cap", "mid", "floor", "tie"])
def test_threshold_select_bit_exact(lsa, N, kmax, tau_kind):
    w = datagen.small_workload(B=len(N), N=N, k=kmax, E=64)
    dims = G.dims_of(w, lsa)
    ws = lsa.alloc_workspace(dims)
    s = np.concatenate([_tie_scores(n, 300 + i) for i, n in enumerate(N)])
    tau = {"cap": -100.0, "mid": 0.75, "floor": 100.0, "tie": float(s[3])}[tau_kind]
    k_min = 3
    ids = torch.full((w.total_kept,), 12345, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    lsa.lsa_threshold_select(dims, torch.from_numpy(s).cuda(), np.float32(tau), k_min, ids, cnt, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK
    got, got_cnt = ids.cpu().numpy(), cnt.cpu().numpy()
    off, koff = w.chunk_offsets, w.k_offsets
    for b in range(w.B):
        ref = oracle.threshold_select(s[off[b]:off[b + 1]].astype(np.float64), np.float32(tau), k_min, kmax[b])
        assert got_cnt[b] == len(ref)
        np.testing.assert_array_equal(got[koff[b]:koff[b] + len(ref)], ref)
        assert (got[koff[b] + len(ref):koff[b + 1]] == -1).all()


@pytest.mark.parametrize("case", STEP_CASES[:4], ids=lambda c: f"B{c['B']}-E{c['E']}-Q{c.get('Q', 1)}-H{c['H']}")
def test_decode_step_threshold(lsa, case):
    w = datagen.small_workload(seed=66, **dict(case))
    dw = G.DeviceWorkload(w, lsa)
    # tau between the scores: about a third of each sequence's chunks pass (capacity k_b)
    all_s = [oracle.chunk_scores(dw.q_emb_f(b), dw.emb_f(b)) for b in range(w.B)]
    tau = np.float32(np.median(np.concatenate(all_s)) + 0.5 * np.std(np.concatenate(all_s)))
    k_min = 1
    cnt = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    lsa.lsa_decode_step_threshold(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, tau, k_min, dw.ids, cnt,
                                  dw.out, dw.lse, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    got, got_cnt, out = dw.ids.cpu().numpy(), cnt.cpu().numpy(), dw.out.cpu().numpy()
    koff = w.k_offsets
    for b in range(w.B):
        s = all_s[b]
        absdot = G.score_tolerance(dw.q_emb_f(b), dw.emb_f(b))
        ref = oracle.threshold_select(s, tau, k_min, w.k[b])
        k_eff = int(got_cnt[b])
        mine = got[koff[b]:koff[b] + k_eff]
        assert (got[koff[b] + k_eff:koff[b + 1]] == -1).all()
        if k_eff != len(ref):
            # only scores within their own tolerance of tau may flip the count: k_eff must lie
            # between the counts of the chunks that surely pass and those that may pass
            tol = G.SCORE_RTOL * np.maximum(np.abs(s), absdot)
            lo = np.count_nonzero(s - tol >= float(tau))
            hi = np.count_nonzero(s + tol >= float(tau))
            floor = min(k_min, w.k[b])
            assert min(max(lo, floor), w.k[b]) <= k_eff <= min(max(hi, floor), w.k[b]), (k_eff, lo, hi)
        # the kept set is the top-k_eff by (score desc, index asc), near-ties at its edge exempt
        G.check_ids(mine, oracle.topk(s, k_eff), s, k_eff)
        ref_o, _ = G.oracle_attention(dw, b, mine)
        np.testing.assert_allclose(out[b], ref_o, rtol=0, atol=1e-4)


# ------------------------------------------------------------------ FP8 compressed-K indexer score
FP8_CASES = [
    dict(B=2, N=(300, 129), L=3, Hn=128, mean=False),
    dict(B=1, N=(64,), L=1, Hn=16, mean=True),
    dict(B=3, N=(257, 1, 128), L=2, Hn=64, mean=False),
    dict(B=2, N=(130, 400), L=3, Hn=256, mean=True),
]


def _random_fp8_case(seed):
    rng = np.random.default_rng(9500 + seed)
    B = int(rng.integers(1, 6))
    return dict(B=B, N=tuple(int(rng.integers(1, 700)) for _ in range(B)), L=int(rng.integers(1, 4)),
                Hn=16 * int(rng.integers(1, 17)), mean=bool(rng.integers(0, 2)))


FP8_CASES += [_random_fp8_case(i) for i in range(8)]  # seeded random shapes


@pytest.mark.parametrize("case", FP8_CASES, ids=lambda c: f"B{c['B']}-L{c['L']}-H{c['Hn']}-{'mean' if c['mean'] else 'max'}")
def test_indexer_score_fp8_parity(lsa, case):
    w = datagen.small_workload(B=case["B"], N=case["N"], k=[1] * case["B"], E=128, emb_dtype="bf16",
                               kv_dtype="bf16", seed=77)
    ix = G.IndexerInputs(w, case["L"], case["Hn"], case["mean"])
    dims = G.dims_of(w, lsa)
    ws = lsa.alloc_workspace(dims)
    sc = torch.empty(w.total_chunks, dtype=torch.float32, device="cuda")
    lsa.lsa_indexer_score_fp8(dims, case["L"], case["Hn"], int(case["mean"]), ix.ck, ix.q8, ix.qs, ix.hw, sc, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK
    got = sc.cpu().numpy().astype(np.float64)
    off = w.chunk_offsets
    worst = 0.0
    for b in range(w.B):
        ref, tol = ix.oracle_scores(b), ix.tolerance(b)
        err = np.abs(got[off[b]:off[b + 1]] - ref)
        worst = max(worst, float((err / tol).max()))
        assert (err <= tol).all(), f"max err {err.max()} vs tol {tol[err.argmax()]}"
    print(f"fp8 indexer: worst error / tolerance = {worst:.3g}")


def test_indexer_fp8_full_size_1m(lsa):
    # the 1M-context shape: 16384 chunks, 3 layers, 128 heads
    w = datagen.Workload("1m-idx", 1, [16384], 128, 1, [2212], 16, seed=3, plant="copy", plant_count=[164])
    ix = G.IndexerInputs(w, 3, 128)
    dims = G.dims_of(w, lsa)
    ws = lsa.alloc_workspace(dims)
    sc = torch.empty(w.total_chunks, dtype=torch.float32, device="cuda")
    lsa.lsa_indexer_score_fp8(dims, 3, 128, lsa.LSA_ENSEMBLE_MAX, ix.ck, ix.q8, ix.qs, ix.hw, sc, ws)
    ids = torch.empty(2212, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_select(dims, sc, ids, ws)
    assert lsa.lsa_get_device_status(ws) == lsa.LSA_OK
    ref, tol = ix.oracle_scores(0), ix.tolerance(0)
    got = sc.cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= tol).all()
    G.check_ids(ids.cpu().numpy(), oracle.topk(ref, 2212), ref, 2212, band=float(tol.max()))
    assert set(datagen.planted_positions(w, 0).tolist()) <= set(ids.cpu().numpy().tolist())


def test_decode_step_fp8(lsa):
    w = datagen.small_workload(B=2, N=(300, 129), k=(40, 13), E=128, H=16, emb_dtype="bf16", kv_dtype="bf16",
                               seed=78)
    dw = G.DeviceWorkload(w, lsa)
    ix = G.IndexerInputs(w, 3, 128)
    lsa.lsa_decode_step_fp8(dw.dims, 3, 128, lsa.LSA_ENSEMBLE_MAX, ix.ck, ix.q8, ix.qs, ix.hw, dw.q, dw.K, dw.V,
                            dw.ids, dw.out, dw.lse, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    got, out = dw.ids.cpu().numpy(), dw.out.cpu().numpy()
    for b in range(w.B):
        ref, tol = ix.oracle_scores(b), ix.tolerance(b)
        mine = got[w.k_offsets[b]:w.k_offsets[b + 1]]
        G.check_ids(mine, oracle.topk(ref, w.k[b]), ref, w.k[b], band=float(tol.max()))
        ref_o, _ = G.oracle_attention(dw, b, mine)
        np.testing.assert_allclose(out[b], ref_o, rtol=0, atol=1e-4)


# ------------------------------------------------------------------ chunk-sharded step (emulated ranks)
SHARD_CASES = [
    dict(B=2, N=(300, 129), k=(40, 13), E=128, H=16, emb_dtype="bf16", kv_dtype="bf16", G=2),
    dict(B=2, N=(300, 129), k=(40, 13), E=128, H=16, emb_dtype="bf16", kv_dtype="bf16", G=4),
    dict(B=1, N=(600,), k=(81,), E=256, Q=64, H=16, emb_dtype="bf16", kv_dtype="bf16", plant="copy_query", G=3),
    dict(B=2, N=(64, 90), k=(1, 1), E=64, H=8, emb_dtype="f32", kv_dtype="f32", G=4),  # most ranks keep nothing
]


@pytest.mark.parametrize("case", SHARD_CASES, ids=lambda c: f"G{c['G']}-B{c['B']}-Q{c.get('Q', 1)}-k{c['k'][0]}")
def test_sharded_step_emulated(lsa, case):
    from learned_sparse_kv_decode_b200 import sharded
    case = dict(case)
    G = case.pop("G")
    w = datagen.small_workload(seed=88, **case)
    dw = GPU.DeviceWorkload(w, lsa)
    off = w.chunk_offsets
    backends, embs, Ks, Vs = [], [], [], []
    for g, (ln, go) in enumerate(sharded.split_chunks(w.N, G)):
        plan = sharded.ShardPlan(w.B, w.Q, w.E, w.H, w.C, G, g, w.k, ln, go, w.emb_dtype, w.kv_dtype)
        backends.append(sharded.CudaShardBackend(plan))
        embs.append(torch.cat([dw.chunk_emb[off[b] + go[b]:off[b] + go[b] + ln[b]] for b in range(w.B)]).contiguous())
        Ks.append(torch.cat([dw.K[(off[b] + go[b]) * w.C:(off[b] + go[b] + ln[b]) * w.C] for b in range(w.B)]).contiguous())
        Vs.append(torch.cat([dw.V[(off[b] + go[b]) * w.C:(off[b] + go[b] + ln[b]) * w.C] for b in range(w.B)]).contiguous())
    results, gids = sharded.run_emulated(backends, dw.q_emb, embs, dw.q, Ks, Vs)
    # the unsharded fused step on the same inputs
    lsa.lsa_decode_step(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, dw.ids, dw.out, dw.lse, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    for bk in backends:
        assert lsa.lsa_get_device_status(bk.ws_local) == lsa.LSA_OK
        assert lsa.lsa_get_device_status(bk.ws_global) == lsa.LSA_OK
    np.testing.assert_array_equal(gids.cpu().numpy(), dw.ids.cpu().numpy())  # identical fp32 scores
    ref_out = dw.out.cpu().numpy()
    for out, lse in results:
        np.testing.assert_allclose(out.cpu().numpy(), ref_out, rtol=0, atol=1e-4)
        np.testing.assert_allclose(lse.cpu().numpy(), dw.lse.cpu().numpy(), rtol=0, atol=1e-4)
    got = gids.cpu().numpy()
    for b in range(w.B):
        ref_s = oracle.chunk_scores(dw.q_emb_f(b), dw.emb_f(b))
        mine = got[w.k_offsets[b]:w.k_offsets[b + 1]]
        GPU.check_ids(mine, oracle.topk(ref_s, w.k[b]), ref_s, w.k[b])
        ref_o, _ = GPU.oracle_attention(dw, b, mine)
        np.testing.assert_allclose(results[0][0][b].cpu().numpy(), ref_o, rtol=0, atol=1e-4)
