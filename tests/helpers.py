"""Shared test helpers: seeded inputs on the chosen device and parity checks."""
import numpy as np
import torch

from long_context_sparse_06_b200 import synth


def randn(name, shape, std=1.0, dtype=torch.float32, device="cpu"):
    return torch.from_numpy(synth.normal(name, shape, std=std).astype(np.float32)).to(dtype).to(device)


def rms(x):
    x = np.asarray(x, np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def assert_close_rel_rms(got, ref, rel=2e-2, what=""):
    """bf16 / FP8 outputs: max-abs error within rel * RMS(ref) (the stated bf16 / FP8 tolerance)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    bound = rel * rms(ref)
    assert err <= bound, f"{what}: max-abs error {err:.3e} > {bound:.3e} (= {rel} x RMS)"
    return err, bound


def assert_close_abs(got, ref, tol=1e-4, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert err <= tol, f"{what}: max-abs error {err:.3e} > {tol:.1e}"
    return err


def oracle_pool(fn, items):
    """Runs fn over items on all host cores (the oracle's C calls release the GIL)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    n = max(1, min(len(items), len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(max_workers=n) as ex:
        return list(ex.map(fn, items))


def selection_against_oracle(orc, s_gpu, idx, ref, bound, k, what):
    """Level 3 of the selection rule for scores the tensor cores computed: every GPU score
    lies within `bound` of the oracle's; when the GPU selection differs from the oracle's,
    the oracle's k-th and (k+1)-th scores must lie within twice the largest actual score
    difference (a near-tie), and the GPU selection must still be a top-k of the oracle's
    scores up to that difference.  Returns (oracle selection, near_tie)."""
    s_gpu = np.asarray(s_gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.abs(s_gpu - ref) <= bound), f"{what}: scores outside the rounding bound"
    ref_idx = orc.topk(ref, k)
    if np.array_equal(idx, ref_idx):
        return ref_idx, False
    diff = float(np.max(np.abs(s_gpu - ref)))
    srt = np.sort(ref)[::-1]
    assert srt.size > k and srt[k - 1] - srt[k] <= 2 * diff, f"{what}: selection differs beyond a near-tie"
    sel = idx[idx >= 0]
    mask = np.zeros(ref.size, bool)
    mask[sel] = True
    assert ref[sel].min() + 2 * diff >= ref[~mask].max(), f"{what}: selection not a top-k within the difference"
    return ref_idx, True


def bf16_score_bound(qI, w, kI):
    """|GPU - oracle| bound per key for bf16 index scores: each per-head dot from the
    tensor cores carries at most (d_I/16 + 1) fp32 roundings (or truncations) of partial
    sums bounded by sum|q||k|; the head chain adds H roundings."""
    qa, ka = np.abs(qI), np.abs(kI)
    sabs = ka @ qa.T                                   # [N, H]
    dI = qI.shape[1]
    dot_err = (dI // 16 + 1) * 2.0 ** -23 * sabs
    relu_abs = sabs                                    # |relu(dot)| <= sum|q||k|
    return dot_err @ np.abs(w) * 1.01 + relu_abs @ np.abs(w) * (w.size + 2) * 2.0 ** -24


def assert_exact_topk(scores, idx, k, what=""):
    """idx (ascending, -1 padded) selects the k largest of `scores` by (score desc, index
    asc): a property of any size, checked on the scores the kernels computed."""
    s = np.asarray(scores, np.float32)
    idx = np.asarray(idx)
    n = s.size
    t = min(k, n)
    sel = idx[:t]
    assert np.all(idx[t:] == -1), f"{what}: padding"
    assert sel.size == 0 or (np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() < n), f"{what}: order/range"
    if t == n or t == 0:
        return
    mask = np.zeros(n, bool)
    mask[sel] = True
    v = s[sel].min()
    assert s[~mask].max() <= v, f"{what}: an unselected score exceeds the selection's minimum"
    tie_uns = np.nonzero(~mask & (s == v))[0]
    if tie_uns.size:
        tie_sel = sel[s[sel] == v]
        assert tie_sel.max() < tie_uns.min(), f"{what}: a tie at the threshold went to a higher index"
