"""Parity at the benchmark's full sizes, in the launch configuration bench.py times.

Each test builds one bench.py workload (the same seeded inputs, made on the device) and
runs its step: the call sequence and launch shapes the benchmark times.  Every request
or query is then checked through properties that hold at any size (the step is
deterministic, its selection is the exact top-k of the scores the kernels computed), and
sampled requests / queries element by element against the oracle.

The oracle never takes a value the CUDA path produced.  Quantised rows and keys are made
again by the oracle's own quantisers from the regenerated fp32 values (and compared with
the device's bytes); attention is checked with the oracle's own selection; the prefill's
index and attention stages run on seeded entries after the compressor has been checked.

Tolerances: bf16-key scores within the derived rounding bound; FP4 scores and selections
bit-exact.  The benchmark stores attention outputs and compressed entries in bf16, so
each element must lie within 2e-2 x RMS of the oracle plus the storage rounding, half a
bf16 ulp (heavy-tailed outputs reach |o| ~ 64, where that half ulp alone is 0.125).
"""
import numpy as np
import pytest
import torch

from helpers import assert_close_stored_bf16, assert_exact_topk, bf16_score_bound, topk_gap_ok

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_sparse_06_b200 as lcs
    lcs.lib()
    return lcs


def _workload(L, name):
    """bench.py's workload `name`, built and stepped once (as the benchmark does)."""
    import bench
    wl = bench.WORKLOADS[name](L, DEV, 0)
    wl.build()
    wl.step(torch.cuda.current_stream())
    torch.cuda.synchronize()
    return wl


def _np(t):
    return t.double().cpu().numpy()


def _selection_against_oracle(orc, s_gpu, idx, ref, bound, k, what):
    """The GPU scores lie within `bound` of the oracle's; the GPU selection equals the
    oracle's when the oracle's k-th score gap exceeds the rounding, else it is a valid
    top-k up to that bound.  Returns the oracle's selection when the two are equal."""
    assert np.all(np.abs(s_gpu - ref) <= bound), f"{what}: scores outside the rounding bound"
    ref_idx = orc.topk(ref, k)
    if topk_gap_ok(ref, k, float(bound.max())):
        np.testing.assert_array_equal(idx, ref_idx, err_msg=what)
        return ref_idx
    sel = idx[idx >= 0]
    mask = np.zeros(ref.size, bool)
    mask[sel] = True
    if mask.all():
        return ref_idx
    assert ref[sel].min() + 2 * bound.max() >= ref[~mask].max(), f"{what}: selection not a top-k within the bound"
    return ref_idx if np.array_equal(idx, ref_idx) else None


# ---------------------------------------------------------------- CSA decode
@pytest.mark.parametrize("name", ["csa_decode_bf16_128k", "csa_decode_mixed_1m"])
def test_full_csa_decode(L, orc, name):
    import bench
    from long_context_sparse_06_b200 import synth
    wl = _workload(L, name)
    B, NC, K = wl.B, wl.NC, wl.K
    H, D, DV, HI, DI, TW, SCALE = bench.H, bench.D, bench.DV, bench.HI, bench.DI, bench.TW, bench.SCALE
    # the scores and selection behind the step (same kernels and launch shapes), and the
    # step again with its selection exported: the same output, the same selection
    idx, scores = L.csa_index_topk(wl.qI.view(B, 1, HI, DI), wl.w.view(B, 1, HI), wl.kI, K, N_c=NC,
                                   kI_dtype=wl.kI_dtype, score_dtype=wl.score_dtype, want_scores=True)
    out2 = torch.empty_like(wl.out)
    idx2 = torch.empty((B, K), dtype=torch.int32, device=DEV)
    L.decode_fused(L.MODE_CSA, wl.q, wl.comp, wl.win, DV, SCALE, kv_dtype=wl.kv_dtype, qI=wl.qI, w=wl.w, kI=wl.kI,
                   kI_dtype=wl.kI_dtype, k=K, score_dtype=wl.score_dtype, out=out2, idx_out=idx2, ws=wl.ws)
    torch.cuda.synchronize()
    assert torch.equal(out2, wl.out), "the step is not deterministic"
    assert torch.equal(idx2, idx[:, 0]), "decode_fused and csa_index_topk select differently"
    idx = idx[:, 0].cpu().numpy()
    s_gpu = scores[:, 0].float().cpu().numpy()
    out = wl.out.float().cpu().numpy()
    for b in range(B):
        assert_exact_topk(s_gpu[b], idx[b], K, f"{name} request {b}")
    checked = 0
    if not wl.mixed:
        for b in (0, B // 2 + 1, B - 1):
            qI, w, kI = _np(wl.qI[b]), wl.w[b].cpu().numpy(), _np(wl.kI[b])
            ref = orc.index_scores_bf16(qI, w, kI)
            ref_idx = _selection_against_oracle(orc, s_gpu[b], idx[b], ref, bf16_score_bound(qI, w, kI), K,
                                                f"{name} request {b}")
            if ref_idx is None:
                continue
            o, _ = orc.csa_attend(_np(wl.q[b]), _np(wl.comp[b]), ref_idx, _np(wl.win[b]), 0, -1, TW, DV, SCALE)
            assert_close_stored_bf16(out[b], o, 2e-2, f"{name} request {b}")
            checked += 1
    else:
        # the fp32 values the benchmark quantised, made again from the same streams
        f32 = torch.float32
        kraw = synth.with_outliers_t(wl.tag("kI"), synth.normal_t(wl.tag("kI"), (B, NC, DI), dtype=f32, device=DEV))
        comp32 = synth.with_outliers_t(wl.tag("comp"), synth.normal_t(wl.tag("comp"), (B, NC, D), dtype=f32,
                                                                        device=DEV))
        win32 = synth.with_outliers_t(wl.tag("win"), synth.normal_t(wl.tag("win"), (B, TW, D), dtype=f32,
                                                                      device=DEV))
        planes = wl.kI.cpu().numpy()
        tot = B * NC
        gp, gs = planes[:tot * 64].reshape(B, NC, 64), planes[tot * 64:].reshape(B, NC, 4)
        for b, whole in ((0, True), (B - 1, False)):
            kp, ks = orc.quant_fp4(kraw[b].cpu().numpy())
            np.testing.assert_array_equal(gp[b], kp)
            np.testing.assert_array_equal(gs[b], ks)
            qf, w = wl.qI[b].float().cpu().numpy(), wl.w[b].cpu().numpy()
            if whole:
                # every score of the request, bit for bit, and so the selection
                ref = orc.index_scores_fp4(qf, w, kp, ks)
                np.testing.assert_array_equal(s_gpu[b], ref.astype(np.float32))
                ref_idx = orc.topk(ref, K)
                np.testing.assert_array_equal(idx[b], ref_idx)
                sel = torch.from_numpy(ref_idx.astype(np.int64)).to(DEV)
                rows = orc.quant_kv_fp8(comp32[b, sel].cpu().numpy())
                wrows = orc.quant_kv_fp8(win32[b].cpu().numpy())
                np.testing.assert_array_equal(wl.comp[b, sel].cpu().numpy(), rows)
                np.testing.assert_array_equal(wl.win[b].cpu().numpy(), wrows)
                o, _ = orc.csa_attend(_np(wl.q[b]), orc.dequant_kv_fp8(rows), np.arange(K, dtype=np.int32),
                                      orc.dequant_kv_fp8(wrows), 0, -1, TW, DV, SCALE)
                assert_close_stored_bf16(out[b], o, 2e-2, f"{name} request {b}")
                checked += 1
            else:
                # a random sample of keys plus the selected ones, bit for bit
                rng = np.random.default_rng(1234 + b)
                pick = np.unique(np.concatenate([rng.choice(NC, 4096, replace=False), idx[b]]))
                ref = orc.index_scores_fp4(qf, w, kp[pick], ks[pick])
                np.testing.assert_array_equal(s_gpu[b][pick], ref.astype(np.float32))
    assert checked >= 1


# ---------------------------------------------------------------- HCA decode
@pytest.mark.parametrize("name", ["hca_decode_bf16_1m", "hca_decode_fp8_1m"])
def test_full_hca_decode(L, orc, name):
    import bench
    from long_context_sparse_06_b200 import synth
    wl = _workload(L, name)
    B, NC = wl.B, wl.NC
    D, DV, TW, SCALE = bench.D, bench.DV, bench.TW, bench.SCALE
    fp8 = name.endswith("fp8_1m")
    kvd = L.KV_FP8 if fp8 else None
    out2 = torch.empty_like(wl.out)
    L.decode_fused(L.MODE_HCA, wl.q, wl.comp, wl.win, DV, SCALE, kv_dtype=kvd, out=out2, ws=wl.ws)
    torch.cuda.synchronize()
    assert torch.equal(out2, wl.out), "the step is not deterministic"
    out = wl.out.float().cpu().numpy()
    if fp8:
        comp32 = synth.normal_t(wl.tag("comp"), (B, NC, D), dtype=torch.float32, device=DEV)
        win32 = synth.normal_t(wl.tag("win"), (B, TW, D), dtype=torch.float32, device=DEV)
    for b in (0, B - 1):
        if fp8:
            rows = orc.quant_kv_fp8(comp32[b].cpu().numpy())
            wrows = orc.quant_kv_fp8(win32[b].cpu().numpy())
            np.testing.assert_array_equal(wl.comp[b].cpu().numpy(), rows)
            np.testing.assert_array_equal(wl.win[b].cpu().numpy(), wrows)
            comp, win = orc.dequant_kv_fp8(rows), orc.dequant_kv_fp8(wrows)
        else:
            comp, win = _np(wl.comp[b]), _np(wl.win[b])
        o, _ = orc.hca_attend(_np(wl.q[b]), comp, 128, win, 0, -1, TW, DV, SCALE)
        assert_close_stored_bf16(out[b], o, 2e-2, f"{name} request {b}")


# ------------------------------------------------------------- CSA prefill
def test_full_csa_prefill(L, orc):
    import bench
    from long_context_sparse_06_b200 import synth
    wl = _workload(L, "csa_prefill_bf16_8k")
    Q, NC, K, P0 = wl.Q, wl.NC, wl.K, wl.P0
    D, DV, HI, DI, TW, SCALE = bench.D, bench.DV, bench.HI, bench.DI, bench.TW, bench.SCALE
    n0 = P0 // 4
    # 1. the chunk's compressed KV entries and index keys against the oracle's compressor
    ref_c, _ = orc.compress(_np(wl.x[0]), _np(wl.z[0]), _np(wl.bias), 4, 2, d_rope=64, pos0=P0,
                            x_tail=_np(wl.x_tail[0]), z_tail=_np(wl.z_tail[0]))
    assert_close_stored_bf16(wl.comp[0, n0:].float().cpu().numpy(), ref_c, 2e-2, "prefill compressed KV")
    ref_k, _ = orc.compress(_np(wl.kx[0]), _np(wl.zI[0]), _np(wl.biasI), 4, 2, d_rope=0, pos0=P0,
                            x_tail=_np(wl.kx_tail[0]), z_tail=_np(wl.zI_tail[0]))
    assert_close_stored_bf16(wl.kI[0, n0:].float().cpu().numpy(), ref_k, 2e-2, "prefill compressed index keys")
    # 2. index, top-k and attention stages as the benchmark launches them, on seeded
    # entries in place of the compressor's (the oracle takes no value the device made)
    bf = torch.bfloat16
    wl.comp[:, n0:] = synth.normal_t("full.prefill.comp", (1, NC - n0, D), dtype=bf, device=DEV)
    wl.kI[:, n0:] = synth.normal_t("full.prefill.kI", (1, NC - n0, DI), dtype=bf, device=DEV)
    stream = torch.cuda.current_stream()
    wl.stage("index", stream)
    wl.stage("attend", stream)
    torch.cuda.synchronize()
    idx_g = wl.idx[0].cpu().numpy()
    out = wl.out[0].float().cpu().numpy()
    idx_s, scores = L.csa_index_topk(wl.qI, wl.w, wl.kI, K, q_pos=wl.q_pos, want_scores=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx_s[0].cpu().numpy(), idx_g)
    kI = _np(wl.kI[0])
    comp = _np(wl.comp[0])
    win = _np(wl.win[0])
    checked = 0
    for t in (0, Q // 3, 2 * Q // 3, Q - 1):
        pos = P0 + t
        na = min(NC, (pos + 1) // 4)
        s_gpu = scores[0, t, :na].float().cpu().numpy()
        assert_exact_topk(s_gpu, idx_g[t], K, f"prefill query {t}")
        qI, w = _np(wl.qI[0, t]), wl.w[0, t].cpu().numpy()
        ref = orc.index_scores_bf16(qI, w, kI[:na])
        ref_idx = _selection_against_oracle(orc, s_gpu, idx_g[t], ref, bf16_score_bound(qI, w, kI[:na]), K,
                                            f"prefill query {t}")
        if ref_idx is None:
            continue
        o, _ = orc.csa_attend(_np(wl.q[0, t]), comp, ref_idx, win, P0 - 127, pos, TW, DV, SCALE)
        assert_close_stored_bf16(out[t], o, 2e-2, f"prefill query {t}")
        checked += 1
    assert checked >= 1


# ------------------------------------------------------------ compressor stream
def test_full_compress_stream(L, orc):
    wl = _workload(L, "compress_stream_1m")
    T = wl.T
    passes = (("CSA KV", wl.x, wl.z, wl.bias, wl.csa, 4, 2, 64),
              ("CSA index keys", wl.kx, wl.zI, wl.biasI, wl.csaI, 4, 2, 0),
              ("HCA KV", wl.x, wl.zh, wl.biash, wl.hca, 128, 0, 64))
    for what, x, z, bias, out, m, ov, dr in passes:
        n = T // m
        span = 256 if m == 4 else 16
        for j0 in (0, n // 2 - span // 2, n - span):
            t0, t1 = j0 * m, (j0 + span) * m
            tail = (_np(x[0, t0 - ov:t0]), _np(z[0, t0 - ov:t0])) if (ov and t0 > 0) else (None, None)
            ref, _ = orc.compress(_np(x[0, t0:t1]), _np(z[0, t0:t1]), _np(bias), m, ov, d_rope=dr, pos0=t0,
                                  x_tail=tail[0], z_tail=tail[1])
            assert_close_stored_bf16(out[0, j0:j0 + span].float().cpu().numpy(), ref, 2e-2, f"{what} entries {j0}..")
