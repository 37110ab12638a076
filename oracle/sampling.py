"""Seeded choice of query rows for checking large problems row by row.

TEST INFRASTRUCTURE ONLY.  Holds no arithmetic of the method: it only decides
which rows the oracle evaluates in full.
"""

from __future__ import annotations

import numpy as np


def sample_rows(n: int, n_sample: int, seed: int, must_include=()) -> np.ndarray:
    """Sorted unique row indices in [0, n): ``must_include`` (clipped to range),
    rows 0 and n-1, then uniform rows without replacement until ``n_sample``."""
    rng = np.random.default_rng(seed)
    fixed = {0, n - 1}
    fixed.update(int(i) for i in must_include if 0 <= int(i) < n)
    fixed = sorted(fixed)
    if n <= n_sample:
        return np.arange(n, dtype=np.int64)
    rest = np.setdiff1d(np.arange(n, dtype=np.int64), np.asarray(fixed, dtype=np.int64))
    k = max(0, n_sample - len(fixed))
    pick = rng.choice(rest, size=min(k, rest.size), replace=False)
    return np.unique(np.concatenate([np.asarray(fixed, dtype=np.int64), pick]))
