"""Pins for the float64 oracle: hand-worked fixtures, closed forms, brute force
and an independent library routine. Each test would fail for a plausible slip
in the oracle (dropped term, wrong sign or index, transposed operand, wrong
tie rule, unkept tokens leaking into the softmax)."""
import itertools
import math

import numpy as np
import pytest
import torch

import datagen
import oracle
from tests._golden import load


# ---------------------------------------------------------------- scores
def test_scores_golden_one_query():
    g = load("scores_tiny.txt")
    np.testing.assert_array_equal(oracle.chunk_scores(g["q1"], g["emb"]), g["s1"])


def test_scores_golden_two_queries_max():
    g = load("scores_tiny.txt")
    np.testing.assert_array_equal(oracle.chunk_scores(g["q2"], g["emb"]), g["s2"])


def test_scores_unit_vectors_pick_coordinates():
    # chunk i is the unit vector along axis d_i, so its score is q[d_i]
    rng = np.random.default_rng(0)
    E = 16
    q = rng.standard_normal(E)
    d = rng.permutation(E)[:10]
    emb = np.eye(E)[d]
    np.testing.assert_array_equal(oracle.chunk_scores(q, emb), q[d])


def test_scores_exact_on_integers():
    # integer inputs: the float64 result is exact; int64 matmul is an independent exact reference
    rng = np.random.default_rng(1)
    for Q in (1, 3, 64):
        q = rng.integers(-20, 21, size=(Q, 48))
        e = rng.integers(-20, 21, size=(37, 48))
        ref = (e @ q.T).max(axis=1).astype(np.float64)
        np.testing.assert_array_equal(oracle.chunk_scores(q, e), ref)


def test_scores_negative_and_mixed_sign():
    q = np.array([[-1.0, 0.0], [0.0, -1.0]])
    e = np.array([[2.0, 3.0], [-4.0, -1.0]])
    # chunk 0: max(-2, -3) = -2 ; chunk 1: max(4, 1) = 4
    np.testing.assert_array_equal(oracle.chunk_scores(q, e), [-2.0, 4.0])


# ---------------------------------------------------------------- top-k
@pytest.mark.parametrize("k", [1, 2, 4, 6, 7, 8])
def test_topk_golden_ties(k):
    g = load("topk_ties.txt")
    ids = oracle.topk(g["scores"], int(g[f"k{k}"]))
    np.testing.assert_array_equal(ids, np.atleast_1d(g[f"ids{k}"]).astype(np.int32))


def _valid_topk_sets(s, k):
    """All k-subsets S with: for i in S, j not in S, s_i > s_j or (s_i == s_j and i < j)."""
    n = len(s)
    out = []
    for S in itertools.combinations(range(n), k):
        inS = set(S)
        ok = all((s[i] > s[j]) or (s[i] == s[j] and i < j)
                 for i in S for j in range(n) if j not in inS)
        if ok:
            out.append(list(S))
    return out


def test_topk_brute_force_characterisation():
    rng = np.random.default_rng(2)
    for trial in range(300):
        n = int(rng.integers(1, 11))
        s = rng.integers(-3, 4, size=n).astype(np.float64)  # many ties
        k = int(rng.integers(1, n + 1))
        valid = _valid_topk_sets(s, k)
        assert len(valid) == 1, (s, k, valid)
        np.testing.assert_array_equal(oracle.topk(s, k), valid[0])


def test_topk_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.topk([1.0, float("nan"), 2.0], 1)
    with pytest.raises(ValueError):
        oracle.topk([1.0, float("inf")], 1)
    with pytest.raises(ValueError):
        oracle.topk([1.0, 2.0], 0)
    with pytest.raises(ValueError):
        oracle.topk([1.0, 2.0], 3)


def test_topk_permutation_equivariance_and_scale_invariance():
    rng = np.random.default_rng(3)
    s = rng.standard_normal(200)  # distinct almost surely
    k = 17
    ids = oracle.topk(s, k)
    perm = rng.permutation(200)           # new position p holds old chunk perm[p]
    ids_p = oracle.topk(s[perm], k)
    np.testing.assert_array_equal(np.sort(perm[ids_p]), ids)
    np.testing.assert_array_equal(oracle.topk(3.5 * s, k), ids)


def test_topk_keeps_the_largest():
    s = np.array([0.5, -1.0, 9.0, 2.0, 8.0, 3.0])
    np.testing.assert_array_equal(oracle.topk(s, 3), [2, 4, 5])
    np.testing.assert_array_equal(oracle.topk(-s, 2), [0, 1])  # sign matters: the two smallest of s


# ---------------------------------------------------------------- attention
def test_attention_golden_two_tokens():
    g = load("attention_two_tokens.txt")
    out, lse = oracle.attention(g["q"][None, :], g["K"][:, None, :], g["V"][:, None, :])
    np.testing.assert_allclose(out[0], g["out"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], g["lse"], rtol=0, atol=1e-15)


def _sdpa(q, K, V, mask=None):
    """torch float64 scaled_dot_product_attention (an independent library routine)."""
    qt = torch.from_numpy(np.asarray(q, np.float64))[:, None, :]          # [H, 1, Dh]
    Kt = torch.from_numpy(np.asarray(K, np.float64)).permute(1, 0, 2)     # [H, T, Dh]
    Vt = torch.from_numpy(np.asarray(V, np.float64)).permute(1, 0, 2)
    m = None if mask is None else torch.from_numpy(mask)[None, None, :].expand(qt.shape[0], 1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=m)
    return o[:, 0, :].numpy()


def test_attention_dense_matches_library_sdpa():
    rng = np.random.default_rng(4)
    T, H, Dh = 300, 4, 128
    q, K, V = rng.standard_normal((H, Dh)), rng.standard_normal((T, H, Dh)), rng.standard_normal((T, H, Dh))
    out, _ = oracle.attention(q, K, V)
    np.testing.assert_allclose(out, _sdpa(q, K, V), rtol=0, atol=1e-13)


def test_sparse_attention_equals_masked_dense():
    # attention over the kept chunks == dense attention with every unkept token masked out
    rng = np.random.default_rng(5)
    n, C, H, Dh, k = 12, 8, 2, 128, 4
    L = n * C
    q, K, V = rng.standard_normal((H, Dh)), rng.standard_normal((L, H, Dh)), rng.standard_normal((L, H, Dh))
    ids = np.sort(rng.permutation(n)[:k]).astype(np.int32)
    out, _ = oracle.attention(q, oracle.gather(K, ids, C), oracle.gather(V, ids, C))
    mask = np.zeros(L, dtype=bool)
    mask[oracle.kept_tokens(ids, C)] = True
    np.testing.assert_allclose(out, _sdpa(q, K, V, mask), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- lookahead window attention
def test_lookahead_golden_two_queries():
    g = load("lookahead_two_queries.txt")
    q = g["q"].reshape(2, 2, 4)
    K, V = g["K"].reshape(2, 2, 4), g["V"].reshape(2, 2, 4)
    out, lse = oracle.lookahead_attention(q, K, V)
    np.testing.assert_allclose(out.reshape(4, 4), g["out"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse.reshape(4), g["lse"], rtol=0, atol=1e-15)


def test_lookahead_matches_library_multi_query_sdpa():
    # every window query over every kept token, no mask between the queries: one library
    # call with a query length of Q
    rng = np.random.default_rng(9)
    Qw, T, H, Dh = 64, 200, 3, 128
    q = rng.standard_normal((Qw, H, Dh))
    K, V = rng.standard_normal((T, H, Dh)), rng.standard_normal((T, H, Dh))
    out, lse = oracle.lookahead_attention(q, K, V)
    qt = torch.from_numpy(q).permute(1, 0, 2)                       # [H, Q, Dh]
    Kt, Vt = torch.from_numpy(K).permute(1, 0, 2), torch.from_numpy(V).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)
    z = torch.einsum("hqd,htd->hqt", qt, Kt) / math.sqrt(Dh)
    np.testing.assert_allclose(lse, torch.logsumexp(z, dim=-1).permute(1, 0).numpy(), rtol=0, atol=1e-12)


def test_lookahead_equivariance():
    rng = np.random.default_rng(10)
    Qw, T, H, Dh = 7, 50, 2, 16
    q = rng.standard_normal((Qw, H, Dh))
    K, V = rng.standard_normal((T, H, Dh)), rng.standard_normal((T, H, Dh))
    out, lse = oracle.lookahead_attention(q, K, V)
    pq, pt = rng.permutation(Qw), rng.permutation(T)
    out2, lse2 = oracle.lookahead_attention(q[pq], K[pt], V[pt])
    np.testing.assert_allclose(out2, out[pq], rtol=0, atol=1e-13)   # queries permute the rows
    np.testing.assert_allclose(lse2, lse[pq], rtol=0, atol=1e-13)   # tokens do not matter in order


def test_lookahead_step_with_one_query_is_the_decode_step():
    rng = np.random.default_rng(11)
    n, E, H, Dh, C, k = 30, 16, 2, 8, 4, 6
    q_emb, emb = rng.standard_normal((1, E)), rng.standard_normal((n, E))
    q = rng.standard_normal((H, Dh))
    K, V = rng.standard_normal((n * C, H, Dh)), rng.standard_normal((n * C, H, Dh))
    ids, out, lse, s = oracle.decode_step(q_emb, emb, q, K, V, k, C)
    ids2, out2, lse2, s2 = oracle.decode_step_lookahead(q_emb, emb, q[None], K, V, k, C)
    np.testing.assert_array_equal(ids, ids2)
    np.testing.assert_array_equal(out, out2[0])
    np.testing.assert_array_equal(lse, lse2[0])


def test_attention_single_token_returns_v():
    rng = np.random.default_rng(6)
    q, K, V = rng.standard_normal((3, 128)), rng.standard_normal((1, 3, 128)), rng.standard_normal((1, 3, 128))
    out, lse = oracle.attention(q, K, V)
    np.testing.assert_allclose(out, V[0], rtol=0, atol=1e-15)
    z = np.einsum("hd,hd->h", q, K[0]) / math.sqrt(128)
    np.testing.assert_allclose(lse, z, rtol=0, atol=1e-13)


def test_attention_equal_keys_average_values():
    rng = np.random.default_rng(7)
    T, H, Dh = 50, 2, 128
    q = rng.standard_normal((H, Dh))
    K = np.broadcast_to(rng.standard_normal((1, H, Dh)), (T, H, Dh)).copy()
    V = rng.standard_normal((T, H, Dh))
    out, lse = oracle.attention(q, K, V)
    np.testing.assert_allclose(out, V.mean(axis=0), rtol=0, atol=1e-13)
    z = np.einsum("hd,hd->h", q, K[0]) / math.sqrt(Dh)
    np.testing.assert_allclose(lse, z + math.log(T), rtol=0, atol=1e-12)


def test_attention_weights_sum_to_one():
    rng = np.random.default_rng(8)
    T, H, Dh = 77, 3, 128
    q, K, V = 3 * rng.standard_normal((H, Dh)), rng.standard_normal((T, H, Dh)), rng.standard_normal((T, H, Dh))
    _, lse = oracle.attention(q, K, V)
    z = np.einsum("hd,thd->th", q, K) / math.sqrt(Dh)     # independent score computation
    np.testing.assert_allclose(np.exp(z - lse[None, :]).sum(axis=0), 1.0, rtol=0, atol=1e-12)


def test_attention_split_merge_is_associative():
    # attention over a token set split into parts, recombined with the log-sum-exp rule, equals
    # attention over the whole set (the split-K identity the GPU kernels rely on); this also
    # pins the lse the oracle returns
    rng = np.random.default_rng(12)
    T, H, Dh = 300, 4, 128
    q, K, V = 2 * rng.standard_normal((H, Dh)), rng.standard_normal((T, H, Dh)), rng.standard_normal((T, H, Dh))
    out, lse = oracle.attention(q, K, V)
    for cuts in ([0, 1, 300], [0, 100, 101, 250, 300], [0, 37, 74, 111, 148, 185, 222, 259, 300]):
        parts = [oracle.attention(q, K[a:b], V[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
        M = np.max([l for _, l in parts], axis=0)
        wts = [np.exp(l - M) for _, l in parts]
        L = np.sum(wts, axis=0)
        merged = np.sum([w[:, None] * o for w, (o, _) in zip(wts, parts)], axis=0) / L[:, None]
        np.testing.assert_allclose(merged, out, rtol=0, atol=1e-13)
        np.testing.assert_allclose(M + np.log(L), lse, rtol=0, atol=1e-13)


def test_attention_scale_is_one_over_sqrt_dh():
    # with scale = 1/sqrt(Dh) by default, doubling Dh-normalised logits must match an explicit scale
    rng = np.random.default_rng(9)
    q, K, V = rng.standard_normal((1, 128)), rng.standard_normal((9, 1, 128)), rng.standard_normal((9, 1, 128))
    a, _ = oracle.attention(q, K, V)
    b, _ = oracle.attention(q, K, V, scale=1.0 / math.sqrt(128.0))
    c, _ = oracle.attention(q / math.sqrt(128.0), K, V, scale=1.0)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_allclose(a, c, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- gather + whole step
def test_gather_identity_and_order():
    L, C = 24, 4
    K = np.arange(L * 2 * 3, dtype=np.float64).reshape(L, 2, 3)
    np.testing.assert_array_equal(oracle.gather(K, np.arange(L // C), C), K)
    g = oracle.gather(K, np.array([5, 1]), C)
    np.testing.assert_array_equal(g[:C], K[20:24])
    np.testing.assert_array_equal(g[C:], K[4:8])


def test_decode_step_golden():
    g = load("decode_step_tiny.txt")
    K = g["K"][:, None, :]
    V = g["V"][:, None, :]
    ids, out, lse, s = oracle.decode_step(g["q_emb"], g["emb"], g["q"][None, :], K, V, int(g["k"]), 2)
    np.testing.assert_array_equal(s, g["scores"])
    np.testing.assert_array_equal(ids, g["ids"])
    np.testing.assert_allclose(out[0], g["out"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], g["lse"], rtol=0, atol=1e-15)
    assert oracle.footprint(int(g["k"]), 2, 8) == g["footprint"]


def test_full_keep_equals_dense_attention():
    # k = every chunk: the LSA step reduces to ordinary dense decode attention
    rng = np.random.default_rng(10)
    n, C, E, H, Dh = 6, 4, 8, 2, 128
    L = n * C
    q_emb, emb = rng.standard_normal(E), rng.standard_normal((n, E))
    q, K, V = rng.standard_normal((H, Dh)), rng.standard_normal((L, H, Dh)), rng.standard_normal((L, H, Dh))
    ids, out, _, _ = oracle.decode_step(q_emb, emb, q, K, V, n, C)
    np.testing.assert_array_equal(ids, np.arange(n))
    np.testing.assert_allclose(out, _sdpa(q, K, V), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- footprint
@pytest.mark.parametrize("name,expect", [
    ("tiny", 0.125), ("128k", 0.125), ("500k", 819 / 8192), ("1m", 2212 / 16384)])
def test_footprint_of_workloads(name, expect):
    w = datagen.workload(name)
    assert oracle.footprint(w.k[0], w.C, w.L[0]) == expect


def test_footprint_matches_pages_headline():
    # the pages' average physical footprint is 13.5% of the full context; the 1M workload keeps
    # round(0.135 * 16384) = 2212 chunks, i.e. 13.50% resident, an 86.5% cut
    w = datagen.workload("1m")
    f = oracle.footprint(w.k[0], w.C, w.L[0])
    assert abs(f - 0.135) < 1e-4
    # the 500K workload keeps about 10%, the pages' "over 90% reduction at 500K"
    w = datagen.workload("500k")
    assert 1.0 - oracle.footprint(w.k[0], w.C, w.L[0]) > 0.90


# ---------------------------------------------------------------- planted structure
def test_planted_chunks_recovered_tiny():
    w = datagen.workload("tiny")
    x = datagen.make_inputs(w)
    s = oracle.chunk_scores(x["q_emb"][0], x["chunk_emb"])
    ids = oracle.topk(s, w.k[0])
    planted = datagen.planted_positions(w, 0)
    assert len(planted) == 4
    assert set(planted.tolist()) <= set(ids.tolist())


def test_planted_chunks_recovered_128k():
    # every sequence of the 128K workload plants 32 chunks near its query embedding; all 32
    # must be among the 256 kept
    w = datagen.workload("128k")
    x = datagen.make_inputs(w)
    off = w.chunk_offsets
    for b in range(w.B):
        s = oracle.chunk_scores(datagen.as_f32(x["q_emb"][b], w.emb_dtype),
                                datagen.as_f32(x["chunk_emb"][off[b]:off[b + 1]], w.emb_dtype))
        ids = oracle.topk(s, w.k[b])
        planted = datagen.planted_positions(w, b)
        assert len(planted) == 32
        assert set(planted.tolist()) <= set(ids.tolist())


# ---------------------------------------------------------------- resident refresh
def test_refresh_golden():
    g = load("refresh_slots.txt")
    slots, copies = oracle.refresh_resident(g["old"].astype(int), g["new"].astype(int), 12)
    np.testing.assert_array_equal(slots, g["slots"].astype(np.int32))
    assert copies == [tuple(int(x) for x in r) for r in g["copies"]]


def test_refresh_properties():
    rng = np.random.default_rng(12)
    for _ in range(200):
        n = int(rng.integers(1, 40))
        k = int(rng.integers(1, n + 1))
        old = rng.permutation(n)[:k].astype(int)
        old[rng.random(k) < 0.2] = -1                 # some empty slots
        new = np.sort(rng.permutation(n)[:k])
        slots, copies = oracle.refresh_resident(old, new, n)
        assert sorted(slots.tolist()) == new.tolist()          # exactly the kept set
        for j, c in enumerate(old):                            # kept chunks never move
            if c in set(new.tolist()):
                assert slots[j] == c
        moved = {c for c, _ in copies}
        assert moved == set(new.tolist()) - set(old.tolist())  # only entering chunks are copied
        assert [c for c, _ in copies] == sorted(moved)         # ascending chunks ...
        assert [j for _, j in copies] == sorted(j for _, j in copies)  # ... into ascending slots
    # cold start: every slot empty -> the slots list the kept chunks in ascending order
    s, c = oracle.refresh_resident([-1] * 4, [9, 3, 5, 0], 10)
    assert s.tolist() == [0, 3, 5, 9] and len(c) == 4
    # duplicates in a corrupt table: the chunk stays in its first slot only
    s, _ = oracle.refresh_resident([3, 3, -1], [1, 3, 7], 8)
    assert s.tolist() == [3, 1, 7]


# ---------------------------------------------------------------- threshold keep mask
@pytest.mark.parametrize("case", [1, 2, 3, 4, 5])
def test_threshold_golden(case):
    g = load("threshold_select.txt")
    ids = oracle.threshold_select(g["scores"], g[f"tau{case}"], int(g[f"kmin{case}"]), int(g[f"kmax{case}"]))
    np.testing.assert_array_equal(ids, np.atleast_1d(g[f"ids{case}"]).astype(np.int32))


def test_threshold_properties():
    rng = np.random.default_rng(13)
    for _ in range(200):
        n = int(rng.integers(1, 60))
        s = np.round(rng.standard_normal(n) * 3) / 2  # ties
        tau = float(rng.choice(s)) if rng.random() < 0.5 else float(rng.standard_normal())
        k_max = int(rng.integers(1, n + 1))
        k_min = int(rng.integers(1, k_max + 1))
        ids = oracle.threshold_select(s, tau, k_min, k_max)
        passing = np.flatnonzero(s >= tau)
        assert k_min <= len(ids) <= k_max
        if k_min <= len(passing) <= k_max:       # the threshold alone decides
            np.testing.assert_array_equal(ids, passing)
        elif len(passing) < k_min:              # fallback: every passing chunk is kept, plus the best others
            assert set(passing.tolist()) <= set(ids.tolist())
        else:                                    # cap: all kept chunks pass
            assert (s[ids] >= tau).all()
        np.testing.assert_array_equal(ids, oracle.topk(s, len(ids)))  # always a top-k set


# ---------------------------------------------------------------- FP8 indexer score
def test_indexer_golden():
    g = load("indexer_score.txt")
    k = g["k"].reshape(2, 2, 2)
    q = g["q"].reshape(2, 2, 2)
    for mean, key in ((False, "s_max"), (True, "s_mean")):
        s = oracle.indexer_scores(k, g["ks"], q, g["qs"], g["w"], mean=mean)
        np.testing.assert_allclose(s, g[key], rtol=0, atol=1e-15)


def test_e4m3_decode_matches_library():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    np.testing.assert_array_equal(ours[~np.isnan(ours)], ref[~np.isnan(ref)])
    assert oracle.e4m3_decode([0x7E])[0] == 448.0 and oracle.e4m3_decode([0x01])[0] == 2.0 ** -9


def test_compressed_k_split():
    row = np.zeros((1, 132), dtype=np.uint8)
    row[0, :3] = [0x38, 0xC0, 0x01]                      # 1.0, -2.0, 2^-9
    row[0, 128:] = np.array([0.75], dtype="<f4").view(np.uint8)
    keys, scales = oracle.split_compressed_k(row)
    np.testing.assert_array_equal(keys[0, :4], [1.0, -2.0, 2.0 ** -9, 0.0])
    assert scales[0] == 0.75


def test_indexer_reduces_to_dot_product():
    # one layer, one head, weight 1, unit scales, a positive dot: s = sigmoid(q . k)
    rng = np.random.default_rng(14)
    q, k = rng.standard_normal((1, 1, 8)), rng.standard_normal((1, 5, 8))
    k[0] *= np.sign(k[0] @ q[0, 0])[:, None]              # make every dot positive
    s = oracle.indexer_scores(k, np.ones((1, 5)), q, np.ones((1, 1)), np.ones((1, 1)))
    np.testing.assert_allclose(s, 1.0 / (1.0 + np.exp(-(k[0] @ q[0, 0]))), rtol=0, atol=1e-15)
    # ReLU: a negative head contributes nothing
    s0 = oracle.indexer_scores(-k, np.ones((1, 5)), q, np.ones((1, 1)), np.ones((1, 1)))
    np.testing.assert_allclose(s0, 0.5, rtol=0, atol=0)
