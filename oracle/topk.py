"""Top-k token selection of the lightning indexer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` and the benchmark's CPU-baseline leg may import this module;
the library's product path never does, and it shares no code with the CUDA
implementation.

What it computes: page "GLM-5.3-FLASH" (dimsnsums.com), section "How can a
layer search the whole history selectively?": the lightning indexer of a
sparse layer scores all earlier tokens and passes only the best 2,048 on to
full attention.  The page defines neither the score nor what happens on
equal scores, so the selection is stated here on caller-given scores, with
these readings:

* per row (one query), among the row's n scores, the k largest are kept;
  when n <= k every token is kept;
* equal scores (-0.0 and +0.0 are equal) are ranked by index: the lower index
  counts as the larger, so the kept set is unique;
* the kept indices are listed best first, i.e. by descending score and, for
  equal scores, ascending index; slots past n (when n < k) hold -1;
* scores must not be NaN.

The definition written out: sort the row's indices by the key (-score,
index) and keep the first min(n, k).  ``numpy.lexsort`` is the sort.
"""
from __future__ import annotations

import numpy as np


def topk_indices(scores, k: int, lengths=None) -> np.ndarray:
    """scores: [rows, ld] array (any float dtype, no NaN); lengths: optional
    per-row token counts (default: all ld).  Returns int64 [rows, k]."""
    s = np.asarray(scores, dtype=np.float64)
    if s.ndim != 2:
        raise ValueError("scores must be [rows, n]")
    if np.isnan(s).any():
        raise ValueError("scores must not be NaN")
    rows, ld = s.shape
    out = np.full((rows, k), -1, dtype=np.int64)
    for r in range(rows):
        n = ld if lengths is None else int(lengths[r])
        row = s[r, :n] + 0.0            # -0.0 + 0.0 = +0.0: the two zeros compare equal
        idx = np.arange(n)
        order = np.lexsort((idx, -row))  # primary key -score, then index
        m = min(n, k)
        out[r, :m] = order[:m]
    return out
