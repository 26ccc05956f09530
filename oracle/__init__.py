"""Float64 CPU oracle of the LSA decode step (FlashMemory-DeepSeek-V4).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this package; the product path never
does. It shares no code with the CUDA path. The arithmetic lives in plain C
(``lsa_oracle.c``, float64, loops in the order the definitions give); this file
only widens inputs to float64 and loops over the sequences of a batch.

What it computes, per sequence (review of FlashMemory-DeepSeek-V4 on
dimensionstp.github.io, section 3-2 (2)-(3); arXiv abstract):

1. chunk scores  s_i = max_j <q_emb[j], chunk_emb[i]>   (dual-encoder inner product;
   the max over the 64 lookahead queries, as the per-layer ensemble is a max);
2. top-k keep mask: order by (score desc, index asc), keep k, report ascending;
3. gather: the kept chunks' K/V rows, in kept order (a compaction);
4. exact softmax attention of the decode query over the kept tokens only,
   scale 1/sqrt(Dh), returning the output and the log-sum-exp per head;
5. footprint = k * chunk_len / L;
6. the retrieval cycle's resident refresh (review section 3-1 "retrieval interval" and
   section 3-2 (3) step 7): the slot table after a cycle, written out as its rule;
7. the threshold keep mask with a fallback floor (section 3-2 (3) step 5);
8. the indexer score on FP8 compressed-K chunks (section 3-2 (1)-(2)), decoding the
   132-byte chunk format and float8_e4m3 from their definitions;
9. the lookahead window's attention: every one of the window's queries attends over the
   same kept tokens (section 3-2 (3)), one ordinary decode attention per query.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(hand-worked fixtures in ``tests/golden/``, closed forms, a brute-force
characterisation of top-k, and torch's float64 scaled-dot-product attention
as an independent library reference).
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, dp, ip = ctypes.c_int64, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int32)
        lib.lsa_oracle_chunk_scores.argtypes = [i64, i64, i64, dp, dp, dp]
        lib.lsa_oracle_chunk_scores.restype = None
        lib.lsa_oracle_topk.argtypes = [i64, dp, i64, ip]
        lib.lsa_oracle_topk.restype = ctypes.c_int
        lib.lsa_oracle_attention.argtypes = [i64, i64, i64, ctypes.c_double, dp, dp, dp, dp, dp, dp]
        lib.lsa_oracle_attention.restype = None
        lib.lsa_oracle_footprint.argtypes = [i64, i64, i64]
        lib.lsa_oracle_footprint.restype = ctypes.c_double
        lib.lsa_oracle_indexer_scores.argtypes = [i64, i64, i64, i64, ctypes.c_int, dp, dp, dp, dp, dp, dp]
        lib.lsa_oracle_indexer_scores.restype = None
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def chunk_scores(q_emb, chunk_emb) -> np.ndarray:
    """s[i] = max_j sum_d q_emb[j, d] * chunk_emb[i, d]   (q_emb [Q, E] or [E]; chunk_emb [n, E])."""
    q = _f64(q_emb)
    if q.ndim == 1:
        q = q[None, :]
    e = _f64(chunk_emb)
    n, E = e.shape
    assert q.shape[1] == E
    s = np.empty(n, dtype=np.float64)
    _load().lsa_oracle_chunk_scores(n, q.shape[0], E, _dp(q), _dp(e), _dp(s))
    return s


def topk(scores, k: int) -> np.ndarray:
    """Kept chunk indices (int32, ascending): the k best by (score desc, index asc)."""
    s = _f64(scores)
    ids = np.empty(max(int(k), 0), dtype=np.int32)
    rc = _load().lsa_oracle_topk(s.shape[0], _dp(s), int(k),
                                 ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    if rc != 0:
        raise ValueError("top-k rejected its input (non-finite score, or k outside 1..n)")
    return ids


def attention(q, K, V, scale: float | None = None):
    """Exact softmax attention of one decode query. q [H, Dh]; K, V [T, H, Dh].

    Returns (out [H, Dh], lse [H]) in float64; scale defaults to 1/sqrt(Dh)."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    T, H, Dh = K.shape
    assert q.shape == (H, Dh) and V.shape == K.shape and T >= 1
    if scale is None:
        scale = 1.0 / math.sqrt(Dh)
    out = np.empty((H, Dh), dtype=np.float64)
    lse = np.empty(H, dtype=np.float64)
    z = np.empty(T, dtype=np.float64)
    _load().lsa_oracle_attention(T, H, Dh, float(scale), _dp(q), _dp(K), _dp(V),
                                 _dp(out), _dp(lse), _dp(z))
    return out, lse


def lookahead_attention(q, K, V, scale: float | None = None):
    """Attention of every query of the lookahead window over the same kept tokens.

    The indexer keeps the chunks that the next ~64 tokens will attend to, and until the next
    retrieval cycle each of those tokens attends over the kept chunks (review on
    dimensionstp.github.io, section 3-2 (3), lookahead window and steps 6-7). Read plainly:
    query j of the window is an ordinary decode query over the kept set, with no mask
    between the window's queries. q [Q, H, Dh]; K, V [T, H, Dh].
    Returns (out [Q, H, Dh], lse [Q, H]); row j is ``attention(q[j], K, V, scale)``."""
    q = _f64(q)
    assert q.ndim == 3
    outs, lses = [], []
    for j in range(q.shape[0]):
        o, l = attention(q[j], K, V, scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def kept_tokens(ids, chunk_len: int) -> np.ndarray:
    """Token positions (within the sequence) covered by the kept chunks, in kept order."""
    ids = np.asarray(ids, dtype=np.int64)
    return (ids[:, None] * chunk_len + np.arange(chunk_len)[None, :]).reshape(-1)


def gather(cache, ids, chunk_len: int) -> np.ndarray:
    """Resident buffer of one sequence: row j*C + t is row ids[j]*C + t of ``cache`` [L, ...]."""
    return np.asarray(cache)[kept_tokens(ids, chunk_len)]


def footprint(k: int, chunk_len: int, context_len: int) -> float:
    """Resident KV footprint: k * chunk_len / L."""
    return _load().lsa_oracle_footprint(int(k), int(chunk_len), int(context_len))


def decode_step(q_emb, chunk_emb, q, K, V, k: int, chunk_len: int, scale: float | None = None):
    """One sequence's full step: scores -> top-k -> gather -> attention.

    K and V are the full caches [L, H, Dh] of the sequence (or callables that
    return the rows of given token positions). Returns (ids, out, lse, scores)."""
    s = chunk_scores(q_emb, chunk_emb)
    ids = topk(s, k)
    tok = kept_tokens(ids, chunk_len)
    Kk = K(tok) if callable(K) else np.asarray(K)[tok]
    Vk = V(tok) if callable(V) else np.asarray(V)[tok]
    out, lse = attention(q, Kk, Vk, scale)
    return ids, out, lse, s


def decode_step_lookahead(q_emb, chunk_emb, q, K, V, k: int, chunk_len: int, scale: float | None = None):
    """One sequence's step for the whole lookahead window: scores (max over the Q query
    embeddings) -> top-k -> gather -> every window query's attention over the kept tokens.
    q is [Q, H, Dh]. Returns (ids, out [Q, H, Dh], lse [Q, H], scores)."""
    s = chunk_scores(q_emb, chunk_emb)
    ids = topk(s, k)
    tok = kept_tokens(ids, chunk_len)
    Kk = K(tok) if callable(K) else np.asarray(K)[tok]
    Vk = V(tok) if callable(V) else np.asarray(V)[tok]
    out, lse = lookahead_attention(q, Kk, Vk, scale)
    return ids, out, lse, s


def refresh_resident(old_slots, new_ids, n: int):
    """Resident slot table after a retrieval cycle, and the copies it needs.

    Review of FlashMemory-DeepSeek-V4, section 3-1 (re-score about every 64 decode
    steps) and section 3-2 (3) step 7 (attend over the kept chunks until the next
    cycle); only the kept chunks stay resident (abstract). The rule: a slot whose chunk
    (valid, 0 <= c < n) is still kept keeps it (a chunk listed twice stays in its first
    slot); every other slot is freed; the entering chunks in ascending order fill the
    freed slots in ascending order. Returns (slots, copies) with copies a list of
    (chunk, slot) pairs, the only chunks whose rows move."""
    new = sorted(int(c) for c in new_ids)
    new_set = set(new)
    slots = [int(c) for c in old_slots]
    staying = set()
    freed = []
    for j, c in enumerate(slots):
        if 0 <= c < n and c in new_set and c not in staying:
            staying.add(c)
        else:
            freed.append(j)
    entering = [c for c in new if c not in staying]
    assert len(entering) == len(freed)
    copies = []
    for c, j in zip(entering, freed):
        slots[j] = c
        copies.append((c, j))
    return np.array(slots, dtype=np.int32), copies


def threshold_select(scores, tau: float, k_min: int, k_max: int) -> np.ndarray:
    """Threshold keep mask with a fallback floor (review section 3-2 (3) step 5, "top-k or
    threshold"; section 4-3: precise-needle tasks need a threshold fallback). The pages give
    no rule; the one taken: k_eff = clamp(#{s >= tau}, min(k_min, k_max), k_max), and the kept
    set is the top-k_eff (score desc, index asc), reported ascending."""
    s = _f64(scores)
    count = int(np.count_nonzero(s >= float(tau)))
    k_eff = min(max(count, min(int(k_min), int(k_max))), int(k_max))
    return topk(s, k_eff)


def e4m3_decode(codes) -> np.ndarray:
    """float8_e4m3 (the "fn" variant: no infinities) bit patterns -> exact float64.

    1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is subnormal
    (m/8 * 2^-6); the all-ones exponent with mantissa 7 is NaN, the other codes with
    exponent 15 are normal numbers (up to 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7 == 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.power(2.0, e - 7)
    sub = (m / 8.0) * 2.0 ** -6
    val = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, val)


def split_compressed_k(rows) -> tuple:
    """132-byte compressed-K rows (review section 3-2 (1)): bytes 0..127 are e4m3 key values,
    bytes 128..131 a little-endian float32 dequant scale. Returns (keys float64, scales float64)."""
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.uint8))
    assert r.shape[-1] == 132
    keys = e4m3_decode(r[..., :128])
    scales = r[..., 128:132].copy().view("<f4")[..., 0].astype(np.float64)
    return keys, scales


def indexer_scores(k, ks, q, qs, w, mean: bool = False) -> np.ndarray:
    """s_i = ens_l sigmoid(sum_h w_lh ReLU(ks_li qs_lh q_lh . k_li)) for one sequence.
    k [L][n][D], ks [L][n], q [L][H][D], qs [L][H], w [L][H] (float64 values)."""
    k, ks, q, qs, w = _f64(k), _f64(ks), _f64(q), _f64(qs), _f64(w)
    L, n, D = k.shape
    H = q.shape[1]
    s = np.empty(n, dtype=np.float64)
    _load().lsa_oracle_indexer_scores(n, L, H, D, 1 if mean else 0, _dp(k), _dp(ks), _dp(q), _dp(qs),
                                      _dp(w), _dp(s))
    return s
