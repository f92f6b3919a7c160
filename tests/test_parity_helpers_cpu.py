"""The all-unit parity checker's kept-set test (no sort) agrees with the
set comparison of the sampled checker (oracle select, then the tie band)."""
import numpy as np

from oracle import rkv_oracle as ora
from parity import SEL_BAND, _kept_set_valid


def _by_set_comparison(s, got, c, budget):
    want = set(ora.select(s, c, 0, budget)[:budget].tolist())
    diff = set(got.tolist()) ^ want
    sb = np.sort(s)[::-1][budget - 1]
    band = SEL_BAND * np.max(np.abs(s))
    return all(abs(s[i] - sb) <= band for i in diff)


def test_kept_set_check_matches_set_comparison():
    rng = np.random.default_rng(5)
    agree = {True: 0, False: 0}
    for trial in range(400):
        c = int(rng.integers(2, 60))
        budget = int(rng.integers(1, c))
        s = rng.standard_normal(c)
        if trial % 3 == 0:                        # ties and near ties
            s = np.round(s, 1)
        if trial % 5 == 0:
            s[rng.integers(0, c, size=c // 2)] += 1e-9
        got = np.sort(np.lexsort((np.arange(c), -s))[:budget])
        if trial % 2:                             # a perturbed kept set
            out = rng.choice(np.setdiff1d(np.arange(c), got))
            got = np.sort(np.concatenate([np.delete(got, rng.integers(0, budget)), [out]]))
        want = _by_set_comparison(s, got, c, budget)
        assert _kept_set_valid(s, got, c, budget) == want, (trial, s, got)
        agree[want] += 1
    assert agree[True] > 50 and agree[False] > 50
