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


def topk_gap_ok(oracle_scores, k, bound):
    """True when the oracle's k-th and (k+1)-th best scores differ by more than 2*bound
    (the selection is then decided by the scores, not by rounding)."""
    s = np.sort(np.asarray(oracle_scores, np.float64))[::-1]
    if s.size <= k:
        return True
    return (s[k - 1] - s[k]) > 2 * bound
