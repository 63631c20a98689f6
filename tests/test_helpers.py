"""The test helpers that decide pass or fail, checked on CPU against the oracle."""
import numpy as np
import pytest

from helpers import assert_exact_topk


def test_assert_exact_topk_accepts_the_oracle_and_rejects_mistakes(orc):
    rng = np.random.default_rng(7)
    s = rng.integers(-3, 4, 500).astype(np.float32)          # many ties
    s[10] = -0.0
    k = 37
    good = orc.topk(s, k)
    assert_exact_topk(s, good, k)
    assert_exact_topk(s[:20], orc.topk(s[:20], 30), 30)       # fewer entries than k: -1 padding
    bad_swap = good.copy()                                     # a tie given to a higher index
    v = s[good].min()
    hi = np.nonzero(s == v)[0]
    free = [j for j in hi if j not in set(good.tolist())]
    bad_swap[np.nonzero(good == hi[0])[0][0]] = free[-1]
    bad_swap.sort()
    with pytest.raises(AssertionError):
        assert_exact_topk(s, bad_swap, k)
    bad_low = good.copy()                                      # a lower score in place of a higher one
    lowest = int(np.argmin(s))
    bad_low[0] = lowest
    bad_low.sort()
    with pytest.raises(AssertionError):
        assert_exact_topk(s, bad_low, k)
    with pytest.raises(AssertionError):                        # not ascending
        assert_exact_topk(s, good[::-1], k)
