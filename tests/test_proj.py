"""Compressor and lightning indexer with their input projections fused in, at the tiny
prefill's sizes ("DeepSeek V4 深度解析" §2, CSA steps 1-2: rows, pooling logits, index
queries and head weights are linear in the token's hidden state; hidden 256).

The oracle projects with its fp32 chain (project_f32, the order both sides define) and then
runs its compressor and indexer on those values:
  * compressor: max-abs 1e-4 (fp32 entries), chunked with a tail and from the sequence start,
    KV rows with RoPE and index keys without; bf16 hidden states: the bf16 output is exactly
    the fp32 output rounded, and the fp32 output within 1e-4 of the oracle on the same bf16
    values;
  * indexer: scores and the causal top-k selection bit-exact.
"""
import math

import numpy as np
import pytest
import torch

from helpers import assert_close_abs, randn

pytestmark = pytest.mark.gpu

DEV = "cuda"
HID = 256


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_sparse_06_b200 as lcs
    lcs.lib()
    return lcs


@pytest.mark.parametrize("d,dr,pos0,tail", [(64, 16, 0, False), (64, 16, 1024, True), (32, 0, 0, False)])
def test_compress_proj(L, orc, d, dr, pos0, tail):
    B, T = 2, 1024
    sw = 1 / math.sqrt(HID)
    h = randn(f"pj.c.h{d}{pos0}", (B, T, HID))
    ht = randn(f"pj.c.ht{d}{pos0}", (B, 2, HID)) if tail else None
    Wx = randn(f"pj.c.w{d}", (HID, d), std=sw)
    wz = randn(f"pj.c.z{d}", (HID,), std=sw)
    bias = randn(f"pj.c.b{d}", (6,))
    out = L.lcs_compress_proj(h.to(DEV), Wx.to(DEV), wz.to(DEV), bias.to(DEV), m=4, overlap=2, d_rope=dr, pos0=pos0,
                              h_tail=ht.to(DEV) if tail else None).cpu().numpy()
    for b in range(B):
        x = orc.project_f32(h[b].numpy(), Wx.numpy())
        z = orc.project_f32(h[b].numpy(), wz.numpy()[:, None])[:, 0]
        xt = orc.project_f32(ht[b].numpy(), Wx.numpy()) if tail else None
        zt = orc.project_f32(ht[b].numpy(), wz.numpy()[:, None])[:, 0] if tail else None
        ref, _ = orc.compress(x, z, bias.numpy(), 4, 2, d_rope=dr, pos0=pos0, x_tail=xt, z_tail=zt)
        assert_close_abs(out[b], ref, 1e-4, f"compress_proj b {b}")


def test_compress_proj_bf16(L, orc):
    B, T, d = 2, 512, 64
    bf = torch.bfloat16
    h = randn("pj.cb.h", (B, T, HID), dtype=bf)
    Wx = randn("pj.cb.w", (HID, d), std=1 / 16, dtype=bf)
    wz = randn("pj.cb.z", (HID,), std=1 / 16)
    bias = randn("pj.cb.b", (6,))
    args = (h.to(DEV), Wx.to(DEV), wz.to(DEV), bias.to(DEV))
    o32 = L.lcs_compress_proj(*args, m=4, overlap=2, d_rope=16, out_dtype=torch.float32)
    o16 = L.lcs_compress_proj(*args, m=4, overlap=2, d_rope=16, out_dtype=bf)
    assert torch.equal(o16, o32.to(bf))
    o32 = o32.cpu().numpy()
    for b in range(B):
        hb = h[b].float().numpy()
        x = orc.project_f32(hb, Wx.float().numpy())
        z = orc.project_f32(hb, wz.numpy()[:, None])[:, 0]
        ref, _ = orc.compress(x, z, bias.numpy(), 4, 2, d_rope=16)
        assert_close_abs(o32[b], ref, 1e-4, f"compress_proj bf16 b {b}")


def test_index_topk_proj_bit_exact(L, orc):
    B, Q, HI, DI, Nc, k = 2, 160, 4, 32, 256, 64
    sw = 1 / math.sqrt(HID)
    h = randn("pj.i.h", (B, Q, HID))
    WqI = randn("pj.i.wq", (HID, HI * DI), std=sw)
    Ww = randn("pj.i.ww", (HID, HI), std=sw)
    kI = randn("pj.i.k", (B, Nc, DI))
    q_pos = (torch.arange(Q, dtype=torch.int64) * 6 + 1).reshape(1, Q).repeat(B, 1)
    q_pos[1] += 3
    idx, sc = L.csa_index_topk_proj(h.to(DEV), WqI.to(DEV), Ww.to(DEV), kI.to(DEV), k, HI, q_pos=q_pos.to(DEV), m=4,
                                    want_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    for b in range(B):
        qI = orc.project_f32(h[b].numpy(), WqI.numpy()).reshape(Q, HI, DI)
        w = orc.project_f32(h[b].numpy(), Ww.numpy())
        for t in range(Q):
            n = orc.n_avail(int(q_pos[b, t]), 4, Nc)
            ref = orc.index_scores_f32(qI[t], w[t], kI[b, :n].numpy())
            np.testing.assert_array_equal(sc[b, t, :n], ref, err_msg=f"b {b} q {t}")
            np.testing.assert_array_equal(idx[b, t], orc.topk(ref, k), err_msg=f"b {b} q {t}")
