"""Failure detection without a GPU fault: the bounded waits of the pipelined kernels.

A kernel that waits on an mbarrier nothing completes must give up after its budget,
record LCS_ERR_TIMEOUT with where it waited, and return normally; a later wait in the
same grid must give up at once; the context must stay usable.  lcs_selftest_wait runs
that wait with the waiting code every pipelined kernel uses, on a short budget.
"""
import pytest
import torch

DEV = "cuda"


def test_selftest_wait_rejects_bad_arguments_without_device():
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    import long_context_sparse_06_b200 as L
    lib = L.lib()
    P = 4096   # a fake, never-dereferenced address
    assert lib.lcs_selftest_wait(1000, None, 256, P, None) == L.LCS_ERR_INVALID
    assert lib.lcs_selftest_wait(1000, P, 255, P, None) == L.LCS_ERR_INVALID   # smaller than the status word
    assert lib.lcs_selftest_wait(0, P, 256, P, None) == L.LCS_ERR_INVALID
    assert lib.lcs_selftest_wait(2000000, P, 256, P, None) == L.LCS_ERR_INVALID
    assert lib.lcs_selftest_wait(1000, P, 256, P, None) == L.LCS_ERR_CUDA      # well-formed: no device


@pytest.mark.gpu
def test_wait_runs_out_reports_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_sparse_06_b200 as L
    ws = L.workspace(256)
    out = torch.full((4,), -1, dtype=torch.int64, device=DEV)
    budget_us = 20000
    L.lcs_selftest_wait(budget_us, ws, out)
    torch.cuda.synchronize()
    code, detail = ws[:8].view(torch.int32).tolist()
    assert (code, detail) == (L.LCS_ERR_TIMEOUT, 901)
    ok1, ns1, ok2, ns2 = out.tolist()
    assert ok1 == 0 and budget_us * 1000 <= ns1 < budget_us * 1000 + 50_000_000, ns1
    assert ok2 == 0 and ns2 < 1_000_000, ns2          # gave up at once: the status was set
    assert L.lcs_status(ws) == L.LCS_ERR_TIMEOUT     # reported once, then cleared
    assert L.lcs_status(ws) == 0
    # the context is usable: a regular call runs and is right
    x = torch.ones((4, 576), dtype=torch.float32, device=DEV)
    rows = L.lcs_quant_kv_fp8(x)
    torch.cuda.synchronize()
    assert rows.shape == (4, 656) and int(rows[0, 0]) != 0
