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


def test_assert_close_stored_bf16_allows_exactly_the_storage_rounding():
    import torch
    from helpers import assert_close_stored_bf16, bf16_half_ulp, rms
    rng = np.random.default_rng(3)
    ref = rng.standard_normal(4000) * np.where(rng.random(4000) < 0.01, 40.0, 1.0)
    slack = 2e-2 * rms(ref)
    # a kernel value within the arithmetic tolerance, then stored in bf16: accepted
    v = ref + rng.uniform(-slack, slack, ref.size)
    stored = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.max(np.abs(stored - ref)) > slack               # the storage rounding alone exceeds rel x RMS here
    assert_close_stored_bf16(stored, ref)
    # half an ulp is the most RNE moves a value
    assert np.all(np.abs(stored - v) <= bf16_half_ulp(v) * (1 + 1e-12))
    # an error beyond the tolerance plus the rounding: rejected
    bad = stored.copy()
    j = int(np.argmax(np.abs(ref)))
    bad[j] += 2 * (slack + bf16_half_ulp(abs(ref[j]) + slack))
    with pytest.raises(AssertionError):
        assert_close_stored_bf16(bad, ref)
