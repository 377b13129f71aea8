"""The parity checker itself (CPU): it must accept a valid top-k that differs from the oracle only
inside the tie tolerance, and reject selections that a faulty kernel could produce on rows under the
gap waiver (the best entry dropped for the (k+1)-th, an entry far below the k-th taken)."""
import numpy as np
import pytest

from tests._helpers import GAP_REL, check_selection


def _row(n=40, k=8, seed=0, close=True):
    """One row of distinct scores whose k-th and (k+1)-th are closer than the waiver (close=True)."""
    r = np.random.default_rng(seed)
    s = np.sort(r.uniform(1.0, 2.0, n))[::-1].copy()
    if close:
        s[k] = s[k - 1] * (1 - GAP_REL / 4)        # (k+1)-th within the waiver of the k-th
    perm = r.permutation(n)
    scores = np.empty(n)
    scores[perm] = s                                # rank i sits at index perm[i]
    return scores, perm


def _sel(idx, k):
    out = np.full((1, k), -1, np.int32)
    v = np.sort(np.asarray(idx))
    out[0, :len(v)] = v
    return out


def _ref(scores, perm, k):
    return _sel(perm[:k], k), np.array([(scores[perm[k - 1]] - scores[perm[k]]) / abs(scores[perm[k - 1]])])


def test_checker_accepts_oracle_and_tie_swap():
    k = 8
    scores, perm = _row(k=k)
    ref, gap = _ref(scores, perm, k)
    assert gap[0] < GAP_REL
    nv = np.array([len(scores)])
    assert check_selection(ref, ref, gap, scores[None], nv, k, exact=False) == 1
    swapped = _sel(list(perm[:k - 1]) + [perm[k]], k)     # k-th and (k+1)-th exchanged: within eps
    check_selection(swapped, ref, gap, scores[None], nv, k, exact=False)


def test_checker_rejects_dropping_the_best_entry_on_a_waived_row():
    k = 8
    scores, perm = _row(k=k)
    ref, gap = _ref(scores, perm, k)
    bad = _sel(list(perm[1:k]) + [perm[k]], k)            # top-1 left out, (k+1)-th taken
    with pytest.raises(AssertionError, match="left out an entry far above"):
        check_selection(bad, ref, gap, scores[None], np.array([len(scores)]), k, exact=False)


def test_checker_rejects_a_low_entry_on_a_waived_row():
    k = 8
    scores, perm = _row(k=k)
    ref, gap = _ref(scores, perm, k)
    bad = _sel(list(perm[:k - 1]) + [perm[-1]], k)        # the worst entry instead of the k-th
    with pytest.raises(AssertionError):
        check_selection(bad, ref, gap, scores[None], np.array([len(scores)]), k, exact=False)


def test_checker_requires_the_exact_set_outside_the_waiver():
    k = 8
    scores, perm = _row(k=k, close=False)
    ref, gap = _ref(scores, perm, k)
    assert gap[0] >= GAP_REL
    swapped = _sel(list(perm[:k - 1]) + [perm[k]], k)
    with pytest.raises(AssertionError):
        check_selection(swapped, ref, gap, scores[None], np.array([len(scores)]), k, exact=False)


def test_checker_rejects_padding_order_and_range_errors():
    k = 8
    scores, perm = _row(k=k, close=False)
    ref, gap = _ref(scores, perm, k)
    nv = np.array([len(scores)])
    for bad in (ref[:, ::-1].copy(),                              # descending
                np.where(np.arange(k) == k - 1, len(scores), ref),  # beyond the visible range
                np.where(np.arange(k) == k - 1, -1, ref)):          # padding where k are visible
        with pytest.raises(AssertionError):
            check_selection(bad.astype(np.int32), ref, gap, scores[None], nv, k, exact=False)
