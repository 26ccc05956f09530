"""The id checks the GPU parity tests rely on, exercised on the CPU with planted mistakes:
under the near-tie exemption a set that drops a clearly top-scoring chunk, or keeps a chunk
below the tie band, must still fail."""
import numpy as np
import pytest

import oracle
from tests import _gpu as G


def _scores():
    # chunk 0 clearly first, chunks 1 and 2 tie within 1e-5 relative at the k = 2 boundary,
    # chunk 3 clearly last
    return np.array([10.0, 5.0, 5.0 + 1e-6, -3.0])


def test_exact_match_is_not_exempt():
    s = _scores()
    ref = oracle.topk(s, 2)
    assert G.check_ids(ref.astype(np.int32), ref, s, 2) is False


def test_near_tie_choice_is_exempt():
    s = _scores()
    ref = oracle.topk(s, 2)                 # [0, 2]
    other = np.array([0, 1], np.int32)      # the other member of the tie band
    assert G.check_ids(other, ref, s, 2) is True


def test_near_tie_cannot_hide_a_dropped_top_chunk():
    s = _scores()
    ref = oracle.topk(s, 2)
    with pytest.raises(AssertionError, match="above the tie band"):
        G.check_ids(np.array([1, 2], np.int32), ref, s, 2)   # chunk 0 dropped


def test_near_tie_cannot_keep_a_chunk_below_the_band():
    s = np.array([10.0, 5.0, 5.0 + 1e-6, 5.0 - 1e-6, -3.0])
    ref = oracle.topk(s, 3)                 # [0, 1, 2]; chunk 3 is inside the band
    assert G.check_ids(np.array([0, 2, 3], np.int32), ref, s, 3) is True
    with pytest.raises(AssertionError):
        G.check_ids(np.array([0, 2, 4], np.int32), ref, s, 3)   # chunk 4 far below


def test_clear_mismatch_fails():
    s = np.array([4.0, 3.0, 2.0, 1.0])
    with pytest.raises(AssertionError, match="differ"):
        G.check_ids(np.array([0, 2], np.int32), oracle.topk(s, 2), s, 2)
