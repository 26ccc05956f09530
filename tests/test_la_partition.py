"""CPU checks of the lookahead attention's tile split (lsa_lookahead_partition, host code of
the C library): every CTA gets one contiguous, non-empty range of the (sequence, head) tile
list, and the ranges follow the documented cost rule exactly."""
import numpy as np
import pytest

from learned_sparse_kv_decode_b200 import build as lsa_build

lsa_build.build()
import learned_sparse_kv_decode_b200 as lsa  # noqa: E402

TILE = 128


def _dims(k, C, H, N=None, Q=64):
    N = N or [max(kb, 1) * 2 for kb in k]
    off = np.concatenate([[0], np.cumsum(N)]).tolist()
    return lsa.Dims(len(k), Q, 64, H, C, chunk_offsets=off, k_per_seq=list(k), emb_dtype="bf16", kv_dtype="bf16")


def _expected(k, C, H, max_ctas):
    """The rule written out over an explicit tile list: tile costs 1, a run start 4 more;
    CTA c takes the costs in [ceil(c F / G), ceil((c + 1) F / G)); even split if a CTA
    would be empty."""
    runs = [(b, h) for b in range(len(k)) for h in range(H)]
    tiles_of_run = [-(-k[b] * C // TILE) for b, _ in runs]
    S = sum(tiles_of_run)
    G = min(S, max_ctas, 256)
    run_of = np.repeat(np.arange(len(runs)), tiles_of_run)
    for W in (4, 0):
        cost = np.arange(S) + W * run_of  # cost(s) = s + W * run(s)
        F = S + W * (len(runs) - 1)
        starts = []
        for c in range(G + 1):
            T = -(-c * F // G)
            idx = np.nonzero(cost >= T)[0]
            starts.append(int(idx[0]) if len(idx) else S)
        if all(starts[c] < starts[c + 1] for c in range(G)) or W == 0:
            return starts, W
    raise AssertionError


CASES = [
    ([2212], 64, 16, 148),        # the 1M window shape: 16 runs of 1106 tiles
    ([2212], 64, 1, 148),         # one run over every CTA
    ([5], 64, 2, 148),            # fewer tiles than CTAs
    ([40, 1, 72], 16, 4, 148),    # ragged, C below a box
    ([256] * 8, 64, 16, 148),     # the 128k batch shape
    ([819] * 4, 64, 16, 148),     # 500k
    ([1, 2, 3, 1000], 1024, 8, 20),
    ([7] * 256, 8, 128, 148),     # the largest batch, many tiny runs
    ([3000, 5], 64, 2, 300),      # max_ctas above the 256 cap
]


@pytest.mark.parametrize("k,C,H,G", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_split_follows_the_cost_rule(k, C, H, G):
    starts = lsa.lsa_lookahead_partition(_dims(k, C, H), G)
    exp, _ = _expected(k, C, H, G)
    assert starts == exp
    assert starts[0] == 0 and starts[-1] == sum(H * -(-kb * C // TILE) for kb in k)
    assert all(a < b for a, b in zip(starts, starts[1:])), "a CTA without tiles"


def test_random_shapes():
    rng = np.random.default_rng(5)
    for _ in range(60):
        B = int(rng.integers(1, 12))
        C = int(2 ** rng.integers(3, 11))
        H = int(2 ** rng.integers(0, 6))
        k = [int(x) for x in rng.integers(1, 300, B)]
        G = int(rng.integers(1, 300))
        starts = lsa.lsa_lookahead_partition(_dims(k, C, H), G)
        assert starts == _expected(k, C, H, G)[0], (k, C, H, G)


def test_run_starts_take_fewer_tiles():
    # 1M window shape: CTAs that open a run carry its cost; every CTA gets 116..120 tiles
    starts = np.array(lsa.lsa_lookahead_partition(_dims([2212], 64, 16), 148))
    n = np.diff(starts)
    assert n.min() >= 116 and n.max() <= 120
    run_start = np.array([any(s0 < r * 1106 <= s1 - 1 or (s0 == r * 1106 and s0 > 0) for r in range(16))
                          for s0, s1 in zip(starts[:-1], starts[1:])])
    assert n[run_start].mean() < n[~run_start].mean()


@pytest.mark.parametrize("kw,status", [
    (dict(max_ctas=0), lsa.LSA_ERR_INVALID_ARG),
    (dict(kv_dtype="f32"), lsa.LSA_ERR_UNSUPPORTED),
    (dict(Q=65), lsa.LSA_ERR_UNSUPPORTED),
])
def test_rejects(kw, status):
    Q = kw.get("Q", 64)
    d = lsa.Dims(1, Q, 64, 4, 64, N=10, k=5, emb_dtype="bf16", kv_dtype=kw.get("kv_dtype", "bf16"))
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_lookahead_partition(d, kw.get("max_ctas", 148))
    assert e.value.status == status


def _slots_written(starts, run_tiles):
    """Slots the lookahead CTAs write for split runs: CTA c walks its tiles in order; a run it does
    not hold whole goes to slot 2c if it is the CTA's first run, else 2c + 1."""
    run_start = np.concatenate([[0], np.cumsum(run_tiles)])
    written = {}
    for c in range(len(starts) - 1):
        s0, s1 = starts[c], starts[c + 1]
        r = int(np.searchsorted(run_start, s0, side="right") - 1)
        first = True
        while r < len(run_tiles) and run_start[r] < s1:
            whole = run_start[r] >= s0 and run_start[r + 1] <= s1
            if not whole:
                slot = 2 * c + (0 if first else 1)
                assert slot not in written, "two pieces share a slot"
                written[slot] = r
            first = False
            r += 1
    return written, run_start


def _slots_read(starts, run_start, r):
    """Slots the merge kernel reads for run r: CTAs c0..c1 hold its pieces; piece 0 is c0's first
    run only if c0 starts exactly at the run, and every later piece is that CTA's first run."""
    cta_of = lambda s: int(np.searchsorted(starts[:-1], s, side="right") - 1)  # noqa: E731
    ts, te = run_start[r], run_start[r + 1]
    c0, c1 = cta_of(ts), cta_of(te - 1)
    if c0 == c1:
        return []
    return [2 * c0 + (0 if starts[c0] == ts else 1)] + [2 * (c0 + i) for i in range(1, c1 - c0 + 1)]


def _check_slots(starts, k, C, H):
    run_tiles = [-(-kb * C // TILE) for kb in k for _ in range(H)]
    written, run_start = _slots_written(starts, run_tiles)
    read = {}
    for r in range(len(run_tiles)):
        for slot in _slots_read(starts, run_start, r):
            assert slot not in read
            read[slot] = r
    assert read == written
    assert all(slot < 2 * (len(starts) - 1) for slot in written)  # the workspace holds 2 slots per CTA


@pytest.mark.parametrize("k,C,H,G", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_partial_slots_written_are_the_slots_merged(k, C, H, G):
    _check_slots(lsa.lsa_lookahead_partition(_dims(k, C, H), G), k, C, H)


def test_partial_slots_random_shapes():
    rng = np.random.default_rng(9)
    for _ in range(60):
        B = int(rng.integers(1, 10))
        C = int(2 ** rng.integers(3, 11))
        H = int(2 ** rng.integers(0, 5))
        k = [int(x) for x in rng.integers(1, 200, B)]
        _check_slots(lsa.lsa_lookahead_partition(_dims(k, C, H), int(rng.integers(1, 200))), k, C, H)
