"""Pins of the top-k selection oracle (oracle/topk.py) against what the page
and the stated readings fix, independently of the oracle's own sort.

Page "GLM-5.3-FLASH" (dimsnsums.com), section "How can a layer search the
whole history selectively?": every past token gets a score, the 2,048
highest are kept.  Readings: equal scores rank the lower index first, -0 and
+0 are equal, the list is best first, -1 fills the slots past n.
"""
import os

import numpy as np
import pytest

from oracle.topk import topk_indices

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "topk_cases.txt")


def golden_cases():
    cases = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            head, scores, expect = (p.strip() for p in line.split("|"))
            _, name, kk = head.split()
            cases.append((name, int(kk.split("=")[1]), [float(x) for x in scores.split()],
                          [int(x) for x in expect.split()]))
    return cases


@pytest.mark.parametrize("name,k,scores,expect", golden_cases(), ids=[c[0] for c in golden_cases()])
def test_hand_built_cases(name, k, scores, expect):
    got = topk_indices(np.array([scores]), k)[0]
    assert got.tolist() == expect


def better(s, i, j):
    """Token i ranks above token j: a higher score, or an equal score and a lower index."""
    return s[i] > s[j] or (s[i] == s[j] and i < j)


def check_selection(s, k, got):
    """The selection rule restated as properties (no sorting): every kept
    token ranks above every dropped one, the list is best first, and its
    length is min(n, k) followed by -1."""
    n = len(s)
    m = min(n, k)
    kept = [int(x) for x in got[:m]]
    assert all(x == -1 for x in got[m:])
    assert len(set(kept)) == m and all(0 <= x < n for x in kept)
    dropped = np.setdiff1d(np.arange(n), kept)
    if len(dropped):
        # the weakest kept token still ranks above the strongest dropped one
        worst = kept[-1]
        best_dropped = max(dropped, key=lambda j: (s[j], -j))
        assert better(s, worst, best_dropped)
    for a, b in zip(kept, kept[1:]):
        assert better(s, a, b)


@pytest.mark.parametrize("seed,n,k,levels", [(0, 50, 7, None), (1, 300, 64, 5), (2, 1000, 1000, 3),
                                             (3, 64, 100, None), (4, 5000, 2048, 40), (5, 4097, 2048, None)])
def test_selection_properties_on_random_rows(seed, n, k, levels):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal(n)
    if levels:   # coarse values: many ties, some at the cut
        s = np.round(s * levels) / levels
    got = topk_indices(s[None, :], k)[0]
    check_selection(s, k, got)


def test_rows_are_independent_and_lengths_cut_rows():
    rng = np.random.default_rng(7)
    s = np.round(rng.standard_normal((3, 400)) * 4)
    lengths = [400, 17, 0]
    got = topk_indices(s, 32, lengths)
    for r in range(3):
        check_selection(s[r, :lengths[r]], 32, got[r])
        np.testing.assert_array_equal(got[r], topk_indices(s[r:r + 1, :lengths[r]], 32)[0])


def test_wrong_tie_rule_is_caught():
    # the same rule with the HIGHER index winning ties gives a different answer
    # on the hand-built tie cases; the property check rejects it
    s = np.array([1.0, 7.0, 4.0, 7.0, 4.0, 4.0])
    wrong = np.array([3, 1, 5])
    with pytest.raises(AssertionError):
        check_selection(s, 3, wrong)


def test_nan_is_rejected():
    with pytest.raises(ValueError):
        topk_indices(np.array([[1.0, np.nan]]), 1)
