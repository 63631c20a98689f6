"""Decode-time cache update against the oracle's CacheState ("DeepSeek V4 深度解析" §4, the
KV cache of the mixed attention: the state cache and the compressed cache).

Three requests stream tokens one call at a time; request b's first token arrives at call
offsets[b], so the requests sit at different positions in every call and emit their CSA
entries (every 4 tokens) and HCA entries (every 128) at different calls.  Each gets at
least 300 tokens.  Checks:
  * fp32 storage: every CSA entry, index key and HCA entry, and the window rows, within
    max-abs 1e-4 of CacheState (the whole-sequence compressor's entries, emitted as soon
    as their last token arrives); entries not yet due are still untouched;
  * FP8 KV rows and FP4 index keys: the stored bytes are exactly the library's cache
    writers (pinned bit-exact to the oracle's quantisers) applied to the fp32 entries;
  * bf16 inputs and storage: within 1e-4 of CacheState on the bf16 inputs with fp32
    storage, and the bf16 caches are exactly those values rounded;
  * the decode loop: a fused CSA decode step (k covering the whole compressed cache) and a
    fused HCA decode step run directly on the appended bf16 caches, against the oracle's
    attention over CacheState's entries (rounded to bf16, unwritten slots zero), within
    2e-2 x RMS.
"""
import math

import numpy as np
import pytest
import torch

from helpers import assert_close_abs, assert_close_rel_rms, randn

pytestmark = pytest.mark.gpu

DEV = "cuda"
B, D, DR, DI = 3, 576, 64, 128
OFFSETS = (0, 1, 5)
STEPS = 305
NC, NH = STEPS // 4 + 1, STEPS // 128 + 1


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_sparse_06_b200 as lcs
    lcs.lib()
    return lcs


def _inputs():
    from long_context_sparse_06_b200 import synth
    return dict(x=synth.normal("cu.x", (B, STEPS, D)).astype(np.float32),
                kx=synth.normal("cu.kx", (B, STEPS, DI)).astype(np.float32),
                z=synth.normal("cu.z", (B, STEPS)).astype(np.float32),
                zI=synth.normal("cu.zi", (B, STEPS)).astype(np.float32),
                zh=synth.normal("cu.zh", (B, STEPS)).astype(np.float32),
                bias=synth.normal("cu.b", 6).astype(np.float32),
                biasI=synth.normal("cu.bi", 6).astype(np.float32),
                biash=synth.normal("cu.bh", 128).astype(np.float32))


def _stream(L, inp, x_dtype, kv, win_dtype, kI_kind):
    """Runs the whole stream; returns the caches (device tensors)."""
    row = {"f32": (D, torch.float32), "bf16": (D, torch.bfloat16), "fp8": (656, torch.uint8)}
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)        # noqa: E731
    raw = torch.zeros((B, 128, D + DI), dtype=x_dtype, device=DEV)
    logits = torch.zeros((B, 3, 128), dtype=torch.float32, device=DEV)
    win = torch.zeros((B, 128, row[win_dtype][0]), dtype=row[win_dtype][1], device=DEV)
    comp = torch.zeros((B, NC, row[kv][0]), dtype=row[kv][1], device=DEV)
    hca = torch.zeros((B, NH, row[kv][0]), dtype=row[kv][1], device=DEV)
    if kI_kind == "fp4":
        kI = torch.zeros(B * NC * DI // 2 + B * NC * DI // 32, dtype=torch.uint8, device=DEV)
    else:
        kI = torch.zeros((B, NC, DI), dtype=row[kI_kind][1], device=DEV)
    x = f(inp["x"]).to(x_dtype)
    kx = f(inp["kx"]).to(x_dtype)
    z, zI, zh = f(inp["z"]), f(inp["zI"]), f(inp["zh"])
    bias, biasI, biash = f(inp["bias"]), f(inp["biasI"]), f(inp["biash"])
    ws = L.workspace(256, DEV)
    for s in range(STEPS):
        pos = torch.tensor([s - o if s >= o else -1 for o in OFFSETS], dtype=torch.int64, device=DEV)
        tok = torch.tensor([max(s - o, 0) for o in OFFSETS], device=DEV)
        sel = torch.arange(B, device=DEV)
        L.lcs_cache_append(pos, x[sel, tok].contiguous(), kx[sel, tok].contiguous(), z[sel, tok].contiguous(),
                           zI[sel, tok].contiguous(), zh[sel, tok].contiguous(), bias, biasI, biash, raw, logits,
                           win, comp, kI, hca, d_rope=DR, ws=ws)
    torch.cuda.synchronize()
    assert L.lcs_status(ws) == 0
    return dict(win=win, comp=comp, kI=kI, hca=hca)


def _oracle_states(orc, inp, bf16_inputs):
    sts = []
    for b in range(B):
        cs = orc.CacheState(inp["bias"], inp["biasI"], inp["biash"], d_rope=DR)
        x, kx = inp["x"][b], inp["kx"][b]
        if bf16_inputs:
            x = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
            kx = torch.from_numpy(kx).to(torch.bfloat16).double().numpy()
        for t in range(STEPS - OFFSETS[b]):
            cs.append(x[t], kx[t], inp["z"][b, t], inp["zI"][b, t], inp["zh"][b, t])
        sts.append(cs)
    return sts


def _check_against_states(g, sts, what):
    for b, cs in enumerate(sts):
        nc, nh = len(cs.csa), len(cs.hca)
        assert nc == (STEPS - OFFSETS[b]) // 4 and nh == (STEPS - OFFSETS[b]) // 128
        assert_close_abs(g["comp"][b, :nc].double().cpu().numpy(), np.array(cs.csa), 1e-4, f"{what} CSA b{b}")
        assert_close_abs(g["kI"][b, :nc].double().cpu().numpy(), np.array(cs.csa_keys), 1e-4, f"{what} keys b{b}")
        assert_close_abs(g["hca"][b, :nh].double().cpu().numpy(), np.array(cs.hca), 1e-4, f"{what} HCA b{b}")
        # entries not due yet are untouched
        assert torch.count_nonzero(g["comp"][b, nc:]) == 0 and torch.count_nonzero(g["hca"][b, nh:]) == 0
        for p, rowv in cs.window:
            assert_close_abs(g["win"][b, p % 128].double().cpu().numpy(), rowv, 1e-4, f"{what} window b{b} pos {p}")


def test_cache_update_stream(L, orc):
    inp = _inputs()
    # fp32 inputs: fp32 storage against the oracle
    g32 = _stream(L, inp, torch.float32, "f32", "f32", "f32")
    _check_against_states(g32, _oracle_states(orc, inp, False), "fp32")
    # quantise-on-write: FP8 KV rows and FP4 keys are the cache writers applied to the fp32 entries
    g8 = _stream(L, inp, torch.float32, "fp8", "fp8", "fp4")
    assert torch.equal(g8["win"], L.lcs_quant_kv_fp8(g32["win"]))
    packed = g8["kI"][:B * NC * DI // 2].view(B, NC, DI // 2)
    scales = g8["kI"][B * NC * DI // 2:].view(B, NC, DI // 32)
    for b in range(B):
        nc, nh = (STEPS - OFFSETS[b]) // 4, (STEPS - OFFSETS[b]) // 128
        assert torch.equal(g8["comp"][b, :nc], L.lcs_quant_kv_fp8(g32["comp"][b, :nc].contiguous()))
        assert torch.equal(g8["hca"][b, :nh], L.lcs_quant_kv_fp8(g32["hca"][b, :nh].contiguous()))
        q4 = L.lcs_quant_fp4(g32["kI"][b, :nc].contiguous())
        assert torch.equal(packed[b, :nc], q4[:nc * DI // 2].view(nc, DI // 2))
        assert torch.equal(scales[b, :nc], q4[nc * DI // 2:].view(nc, DI // 32))
        assert torch.count_nonzero(packed[b, nc:]) == 0 and torch.count_nonzero(scales[b, nc:]) == 0
    # bf16 inputs: fp32 storage against the oracle on the same bf16 values; bf16 storage
    # is exactly those entries rounded
    gb32 = _stream(L, inp, torch.bfloat16, "f32", "f32", "f32")
    _check_against_states(gb32, _oracle_states(orc, inp, True), "bf16 inputs")
    gb16 = _stream(L, inp, torch.bfloat16, "bf16", "bf16", "bf16")
    for k in ("comp", "kI", "hca", "win"):
        assert torch.equal(gb16[k], gb32[k].to(torch.bfloat16)), k


def test_decode_on_appended_caches(L, orc):
    inp = _inputs()
    g = _stream(L, inp, torch.bfloat16, "bf16", "bf16", "bf16")
    sts = _oracle_states(orc, inp, True)
    bf = torch.bfloat16
    scale = 1 / math.sqrt(D)
    q = randn("cu.dq", (B, 64, D), dtype=bf)
    qI = randn("cu.dqi", (B, 64, DI), dtype=bf)
    w = randn("cu.dw", (B, 64), std=1 / 8)
    idx = torch.empty((B, NC), dtype=torch.int32, device=DEV)
    out_c = L.decode_fused(L.MODE_CSA, q.to(DEV), g["comp"], g["win"], 512, scale, qI=qI.to(DEV), w=w.to(DEV),
                           kI=g["kI"], k=NC, idx_out=idx, out_dtype=torch.float32).cpu().numpy()
    out_h = L.decode_fused(L.MODE_HCA, q.to(DEV), g["hca"], g["win"], 512, scale,
                           out_dtype=torch.float32).cpu().numpy()
    assert torch.equal(idx.cpu(), torch.arange(NC, dtype=torch.int32).repeat(B, 1))   # k covers every slot
    r16 = lambda a: torch.from_numpy(np.asarray(a, np.float64)).to(bf).double().numpy()   # noqa: E731
    for b, cs in enumerate(sts):
        comp_o = np.zeros((NC, D))
        comp_o[:len(cs.csa)] = r16(cs.csa)
        hca_o = np.zeros((NH, D))
        hca_o[:len(cs.hca)] = r16(cs.hca)
        win_o = np.zeros((128, D))
        for p, rowv in cs.window:
            win_o[p % 128] = r16(rowv)
        qb = q[b].double().numpy()
        o, _ = orc.csa_attend(qb, comp_o, np.arange(NC, dtype=np.int32), win_o, 0, -1, 128, 512, scale)
        assert_close_rel_rms(out_c[b], o, 2e-2, f"CSA decode on the appended caches b{b}")
        o, _ = orc.csa_attend(qb, hca_o, np.arange(NH, dtype=np.int32), win_o, 0, -1, 128, 512, scale)
        assert_close_rel_rms(out_h[b], o, 2e-2, f"HCA decode on the appended caches b{b}")
