"""Context parallelism for long requests ("DeepSeek V4 深度解析" §2, CSA steps 2-3, split over
shards of the compressed entries), with the ranks emulated in one process on one GPU: each
rank's phases run on its own shard, and the all-gathers are stacks in rank order.

* fp32 keys and KV (the tiny config's shapes): the split selection equals the oracle's
  unsplit selection bit for bit, and the merged output is within max-abs 1e-4 of the oracle's
  unsplit attention;
* bf16 keys and KV on the tensor cores (the 128K decode shapes at a smaller context): the
  split selection equals the unsplit GPU selection bit for bit (per-entry scores do not
  depend on the shard), and against the oracle's own selection up to counted near-ties; the
  merged output within 2e-2 x RMS of the oracle's attention wherever the selections agree;
* the 1M config's formats (FP8 KV rows, FP4 index keys, bf16 scores, k = 1024): the split
  selection equals the oracle's unsplit selection bit for bit, and the merged output is
  within 2e-2 x RMS of the oracle's attention.
"""
import math

import numpy as np
import pytest
import torch

from helpers import assert_close_abs, assert_close_rel_rms, bf16_score_bound, randn, selection_against_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_sparse_06_b200 as lcs
    lcs.lib()
    return lcs


def _split_step(L, q, comp, win, qI, w, kI, k, shards, d_v, scale, ops=None, shard_keys=None):
    """The CP step with every rank's phases run here; returns (out fp32, idx_global).
    shard_keys(off, S) gives a rank's index keys (default: a slice of kI)."""
    from long_context_sparse_06_b200 import cp
    ops = ops or cp.LibOps()
    shard_keys = shard_keys or (lambda off, S: kI[:, off:off + S].contiguous())
    cands = []
    for off, S in shards:
        cands.append(cp.local_candidates(ops, qI, w, shard_keys(off, S), k, off, S))
    cs = torch.stack([c[0] for c in cands])
    ci = torch.stack([c[1] for c in cands])
    parts, idx_g = [], None
    for r, (off, S) in enumerate(shards):
        wr = win if r == len(shards) - 1 else None        # the last rank holds the window
        ig, o, lse = cp.local_attention(ops, q, comp[:, off:off + S].contiguous(), wr, cs, ci, off, S, d_v, scale)
        if idx_g is None:
            idx_g = ig
        assert torch.equal(ig, idx_g), "ranks disagree on the selection"
        parts.append((o, lse))
    out = ops.merge(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]), torch.float32)
    return out, idx_g


def test_cp_fp32_exact_selection(L, orc):
    B, H, D, dv, HI, DI, Nc, k, Tw = 2, 8, 64, 48, 4, 32, 3000, 64, 128
    q = randn("cp.f.q", (B, H, D))
    comp = randn("cp.f.c", (B, Nc, D))
    win = randn("cp.f.w", (B, Tw, D))
    qI = randn("cp.f.qi", (B, HI, DI))
    w = randn("cp.f.wi", (B, HI), std=0.5)
    kI = randn("cp.f.k", (B, Nc, DI))
    shards = [(0, 1000), (1000, 1100), (2100, 900)]
    out, idx = _split_step(L, q.to(DEV), comp.to(DEV), win.to(DEV), qI.to(DEV), w.to(DEV), kI.to(DEV), k, shards, dv,
                           1 / 8)
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    for b in range(B):
        s = orc.index_scores_f32(qI[b].numpy(), w[b].numpy(), kI[b].numpy())
        ref_idx = orc.topk(s, k)
        np.testing.assert_array_equal(idx[b], ref_idx)
        o, _ = orc.csa_attend(q[b].double().numpy(), comp[b].double().numpy(), ref_idx, win[b].double().numpy(), 0,
                              -1, Tw, dv, 1 / 8)
        assert_close_abs(out[b], o, 1e-4, f"cp fp32 b {b}")


def test_cp_bf16_tensor_cores(L, orc):
    B, H, D, dv, HI, DI, Nc, k, Tw = 2, 64, 576, 512, 64, 128, 12000, 512, 128
    scale = 1 / math.sqrt(576)
    bf = torch.bfloat16
    q = randn("cp.b.q", (B, H, D), dtype=bf)
    comp = randn("cp.b.c", (B, Nc, D), dtype=bf)
    win = randn("cp.b.w", (B, Tw, D), dtype=bf)
    qI = randn("cp.b.qi", (B, HI, DI), dtype=bf)
    w = randn("cp.b.wi", (B, HI), std=1 / 8)
    kI = randn("cp.b.k", (B, Nc, DI), dtype=bf)
    shards = [(0, 4000), (4000, 4000), (8000, 4000)]
    qd, cd, wd, qid, wid, kid = (t.to(DEV) for t in (q, comp, win, qI, w, kI))
    out, idx = _split_step(L, qd, cd, wd, qid, wid, kid, k, shards, dv, scale)
    # the unsplit GPU selection
    idx_u = L.csa_index_topk(qid.view(B, 1, HI, DI), wid.view(B, 1, HI), kid, k)[:, 0]
    assert torch.equal(idx, idx_u), "the split selection differs from the unsplit one"
    sc = L.csa_index_topk(qid.view(B, 1, HI, DI), wid.view(B, 1, HI), kid, k, want_scores=True)[1][:, 0]
    out, idx, sc = out.cpu().numpy(), idx.cpu().numpy(), sc.cpu().numpy()
    near = []
    for b in range(B):
        qb, kb, wb = qI[b].double().numpy(), kI[b].double().numpy(), w[b].numpy()
        ref = orc.index_scores_bf16(qb, wb, kb)
        ref_idx, nt = selection_against_oracle(orc, sc[b], idx[b], ref, bf16_score_bound(qb, wb, kb), k, f"cp b {b}")
        if nt:
            near.append(b)
            continue
        o, _ = orc.csa_attend(q[b].double().numpy(), comp[b].double().numpy(), ref_idx, win[b].double().numpy(), 0,
                              -1, Tw, dv, scale)
        assert_close_rel_rms(out[b], o, 2e-2, f"cp bf16 b {b}")
    assert len(near) <= 1


def test_cp_mixed_fp8_rows_fp4_keys(L, orc):
    """The 1M config's formats split over three ranks: FP8 KV rows (E4M3 with a power-of-two
    scale per 128 dims, bf16 RoPE dims), FP4 index keys (E2M1 with an E4M3 scale per 32),
    bf16 scores, k = 1024, heavy-tailed values (1 % of elements x 20)."""
    from long_context_sparse_06_b200 import cp, synth
    B, H, D, dv, Nc, k, Tw = 2, 64, 576, 512, 6000, 1024, 128
    scale = 1 / math.sqrt(576)
    q = randn("cp.m.q", (B, H, D), dtype=torch.bfloat16)
    comp32 = synth.with_outliers("cp.m.c", synth.normal("cp.m.c", (B, Nc, D))).astype(np.float32)
    win32 = synth.with_outliers("cp.m.w", synth.normal("cp.m.w", (B, Tw, D))).astype(np.float32)
    k32 = synth.with_outliers("cp.m.k", synth.normal("cp.m.k", (B, Nc, 128))).astype(np.float32)
    comp_g = L.lcs_quant_kv_fp8(torch.from_numpy(comp32).to(DEV)).view(B, Nc, -1)
    win_g = L.lcs_quant_kv_fp8(torch.from_numpy(win32).to(DEV)).view(B, Tw, -1)
    qI = randn("cp.m.qi", (B, 64, 128), dtype=torch.bfloat16)
    w = randn("cp.m.wi", (B, 64), std=1 / 8)
    kp, ks = orc.quant_fp4(k32.reshape(B * Nc, 128))
    kp, ks = kp.reshape(B, Nc, 64), ks.reshape(B, Nc, 4)

    def shard_keys(off, S):   # a rank's FP4 planes: packed codes, then scales
        return torch.from_numpy(np.concatenate([kp[:, off:off + S].reshape(-1), ks[:, off:off + S].reshape(-1)])).to(DEV)

    ops = cp.LibOps(kv_dtype=L.KV_FP8, kI_dtype=L.FP4, score_dtype=L.BF16)
    shards = [(0, 2000), (2000, 2500), (4500, 1500)]
    out, idx = _split_step(L, q.to(DEV), comp_g, win_g, qI.to(DEV), w.to(DEV), None, k, shards, dv, scale, ops=ops,
                           shard_keys=shard_keys)
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    comp_d = orc.dequant_kv_fp8(orc.quant_kv_fp8(comp32))
    win_d = orc.dequant_kv_fp8(orc.quant_kv_fp8(win32))
    for b in range(B):
        ref_s = orc.index_scores_fp4(qI[b].float().numpy(), w[b].numpy(), kp[b], ks[b])
        ref_idx = orc.topk(ref_s.astype(np.float32), k)
        np.testing.assert_array_equal(idx[b], ref_idx, err_msg=f"cp mixed b {b}")
        o, _ = orc.csa_attend(q[b].double().numpy(), comp_d[b], ref_idx, win_d[b], 0, -1, Tw, dv, scale)
        assert_close_rel_rms(out[b], o, 2e-2, f"cp mixed b {b}")
