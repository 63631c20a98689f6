"""csa_attend_noalloc: the allocation-free attention entry point.

It runs csa_attend's kernels on a fixed library-owned scratch array instead of a
caller workspace.  The GPU test compares two calls in a row with csa_attend on
the same inputs (bf16 tolerance: max-abs 2e-2 x RMS) and checks the device
status each call reports.  The file is named so that pytest collects it last:
it must pass alone in a fresh process and after every other test.
"""
import math

import pytest
import torch

from helpers import assert_close_rel_rms, randn

DEV = "cuda"


def test_noalloc_declared_limits_without_device():
    """No device: a well-formed call fails loudly; a bad one is rejected first."""
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    import long_context_sparse_06_b200 as L
    lib = L.lib()
    P = 4096   # a fake, aligned, never-dereferenced address
    assert lib.csa_attend_noalloc(P, L.BF16, P, P, L.BF16, 2, 1, 1000, 128, P, 512, None, None, 128, 64, 576, 512,
                                  0.05, P, L.BF16, None, None, None) == -3
    assert lib.csa_attend_noalloc(P, L.BF16, P, P, L.BF16, 2, 1, 1000, 128, None, 512, None, None, 128, 64, 576, 512,
                                  0.05, P, L.BF16, None, None, None) == -1
    assert lib.lcs_error_string(-7).startswith(b"problem needs more scratch")


@pytest.mark.gpu
@pytest.mark.parametrize("B,N_c,k", [(4, 3000, 512), (32, 32768, 512)])
def test_noalloc_matches_csa_attend(B, N_c, k):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_sparse_06_b200 as L
    H, D, dv, Tw = 64, 576, 512, 128
    scale = 1 / math.sqrt(D)
    q = randn(f"na.q{B}", (B, 1, H, D), dtype=torch.bfloat16).to(DEV)
    comp = randn(f"na.c{B}", (B, N_c, D), dtype=torch.bfloat16).to(DEV)
    win = randn(f"na.w{B}", (B, Tw, D), dtype=torch.bfloat16).to(DEV)
    g = torch.Generator().manual_seed(B)
    idx = torch.stack([torch.randperm(N_c, generator=g)[:k] for _ in range(B)]).int().view(B, 1, k)
    idx[0, 0, k - 7:] = -1                       # a shorter selection: -1 padding ends it
    idx = idx.to(DEV)
    ref = L.csa_attend(q, comp, win, idx, dv, scale).float()
    status = torch.full((1,), -99, dtype=torch.int32, device=DEV)
    for call in range(2):
        out = torch.empty((B, 1, H, dv), dtype=torch.bfloat16, device=DEV)
        L.csa_attend_noalloc(q, comp, win, idx, dv, scale, out=out, status_out=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        assert_close_rel_rms(out.float().cpu().numpy(), ref.cpu().numpy(), 2e-2, f"noalloc call {call}")
        status.fill_(-99)
