"""Host-side logic of the GPU tests, checked on the CPU: the reference kept set
the selection check compares against, and the full-size row plan."""
import numpy as np

from gpu_util import assert_selection_ok, reference_set
from test_gpu_fullsize import oracle_rows


def _brute_set(r, K):
    """Top-K of (score descending, position ascending) by a full sort."""
    order = sorted(range(r.shape[0]), key=lambda s: (-r[s], s))
    return np.sort(np.asarray(order[:K], np.int64))


def test_reference_set_equals_the_sorted_total_order():
    rng = np.random.default_rng(5)
    for trial in range(400):
        n = int(rng.integers(1, 90))
        K = int(rng.integers(1, 100))
        kind = trial % 4
        if kind == 0:
            r = rng.standard_normal(n)
        elif kind == 1:
            r = rng.integers(0, 4, n).astype(np.float64)          # heavy ties
        elif kind == 2:
            r = np.full(n, 0.5)                                   # all tied
        else:
            r = np.round(rng.standard_normal(n), 1)
        ref, kth = reference_set(r, min(K, n))
        np.testing.assert_array_equal(ref, _brute_set(r, min(K, n)))
        if K < n:
            assert kth == sorted(r, reverse=True)[K - 1]


def test_selection_check_accepts_band_swaps_and_rejects_real_misses():
    r = np.array([[5.0, 1.0, 3.0, 3.0005, 0.0, 2.0]])
    n = np.array([6])
    # oracle keeps {0, 2, 3} for K = 3; swapping 2 <-> 3 is not possible (both kept),
    # swapping 3 for 1 is a real miss (gap 2.0005 > 1e-3 * 5)
    assert_selection_ok(np.array([[0, 2, 3]]), r, n, 3)
    try:
        assert_selection_ok(np.array([[0, 1, 2]]), r, n, 3)
        raise RuntimeError("a real miss passed")
    except AssertionError:
        pass
    # a swap inside the band: scores 3.0 and 3.0005 around the cut of K = 2 -> kth = 3.0005
    assert_selection_ok(np.array([[0, 2]]), r, n, 2)
    # invalid lists: not ascending, bad padding
    for bad in (np.array([[3, 0, -1, -1, -1, -1, -1]]), np.array([[0, 3, 2]])):
        try:
            assert_selection_ok(bad, r, n, bad.shape[1])
            raise RuntimeError("an invalid list passed")
        except AssertionError:
            pass


def test_oracle_row_plan_covers_the_stated_rows():
    assert oracle_rows(0, 4) == [0, 1, 2, 3]
    assert oracle_rows(1, 64) == list(range(64))
    assert oracle_rows(3, 32) == list(range(32))
    for cfg, T in ((2, 32768), (4, 8192)):
        r = oracle_rows(cfg, T)
        assert len(r) == 256 and len(set(r)) == 256 and r == sorted(r)
        assert {0, 1, 2047, 2048, T - 1} <= set(r)
        assert max(r) < T
