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

Tolerances: bf16-key scores within the derived rounding bound, and the selection equal
to the oracle's for every request or query whose oracle k-th score gap exceeds twice that
bound (the others, near-ties, are counted and printed); FP4 scores and selections
bit-exact.  Attention is checked on the oracle's own selection, with fp32 output, at
max-abs 2e-2 x RMS of the oracle; the bf16 output the benchmark stores must be exactly
that fp32 output rounded to bf16.
"""
import numpy as np
import pytest
import torch

from helpers import assert_close_rel_rms, assert_exact_topk, bf16_score_bound, oracle_pool, selection_against_oracle

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
    return selection_against_oracle(orc, s_gpu, idx, ref, bound, k, what)


def _check_fp32_and_stored(out32, out16, ref, what):
    """fp32 output within 2e-2 x RMS of the oracle; the bf16 output is that value rounded."""
    assert torch.equal(out16, out32.to(torch.bfloat16)), f"{what}: bf16 output is not the rounded fp32 output"
    assert_close_rel_rms(out32.double().cpu().numpy(), ref, 2e-2, what)


# ---------------------------------------------------------------- CSA decode
@pytest.mark.parametrize("name", ["csa_decode_bf16_128k", "csa_decode_mixed_1m"])
def test_full_csa_decode(L, orc, name):
    import bench
    from long_context_sparse_06_b200 import synth
    wl = _workload(L, name)
    B, NC, K = wl.B, wl.NC, wl.K
    H, D, DV, HI, DI, TW, SCALE = bench.H, bench.D, bench.DV, bench.HI, bench.DI, bench.TW, bench.SCALE
    # the scores and selection behind the step (same kernels and launch shapes), and the
    # step again with its selection exported and fp32 output: the same selection, and the
    # bf16 output the benchmark stored is that fp32 output rounded
    idx, scores = L.csa_index_topk(wl.qI.view(B, 1, HI, DI), wl.w.view(B, 1, HI), wl.kI, K, N_c=NC,
                                   kI_dtype=wl.kI_dtype, score_dtype=wl.score_dtype, want_scores=True)
    out32 = torch.empty(wl.out.shape, dtype=torch.float32, device=DEV)
    idx2 = torch.empty((B, K), dtype=torch.int32, device=DEV)
    L.decode_fused(L.MODE_CSA, wl.q, wl.comp, wl.win, DV, SCALE, kv_dtype=wl.kv_dtype, qI=wl.qI, w=wl.w, kI=wl.kI,
                   kI_dtype=wl.kI_dtype, k=K, score_dtype=wl.score_dtype, out=out32, idx_out=idx2, ws=wl.ws)
    torch.cuda.synchronize()
    assert torch.equal(idx2, idx[:, 0]), "decode_fused and csa_index_topk select differently"
    assert torch.equal(wl.out, out32.to(torch.bfloat16)), "the stored bf16 output is not the rounded fp32 output"
    idx_np = idx[:, 0].cpu().numpy()
    s_gpu = scores[:, 0].float().cpu().numpy()
    for b in range(B):
        assert_exact_topk(s_gpu[b], idx_np[b], K, f"{name} request {b}")

    # every request against the oracle (on all host cores)
    if not wl.mixed:
        def one(b):
            qI, w, kI = _np(wl.qI[b]), wl.w[b].cpu().numpy(), _np(wl.kI[b])
            ref = orc.index_scores_bf16(qI, w, kI)
            return _selection_against_oracle(orc, s_gpu[b], idx_np[b], ref, bf16_score_bound(qI, w, kI), K,
                                             f"{name} request {b}")
        res = oracle_pool(one, list(range(B)))
        ref_idx = np.stack([r[0] for r in res])
        near = [b for b, r in enumerate(res) if r[1]]
        comp_f = lambda b: _np(wl.comp[b])                       # noqa: E731
        win_f = lambda b: _np(wl.win[b])                          # noqa: E731
    else:
        # the fp32 values the benchmark quantised, made again from the same streams; the
        # oracle quantises them itself and its bytes must equal the device's
        f32 = torch.float32
        kraw = synth.with_outliers_t(wl.tag("kI"), synth.normal_t(wl.tag("kI"), (B, NC, DI), dtype=f32, device=DEV))
        comp32 = synth.with_outliers_t(wl.tag("comp"), synth.normal_t(wl.tag("comp"), (B, NC, D), dtype=f32,
                                                                        device=DEV))
        win32 = synth.with_outliers_t(wl.tag("win"), synth.normal_t(wl.tag("win"), (B, TW, D), dtype=f32,
                                                                      device=DEV))
        planes = wl.kI.cpu().numpy()
        tot = B * NC
        gp, gs = planes[:tot * 64].reshape(B, NC, 64), planes[tot * 64:].reshape(B, NC, 4)
        kraw_np = [kraw[b].cpu().numpy() for b in range(B)]
        comp_np = comp32.cpu().numpy()
        win_np = win32.cpu().numpy()
        del kraw, comp32, win32

        def one(b):
            kp, ks = orc.quant_fp4(kraw_np[b])
            np.testing.assert_array_equal(gp[b], kp)
            np.testing.assert_array_equal(gs[b], ks)
            # every score of the request, bit for bit, and so the selection
            ref = orc.index_scores_fp4(wl.qI[b].float().cpu().numpy(), wl.w[b].cpu().numpy(), kp, ks)
            np.testing.assert_array_equal(s_gpu[b], ref.astype(np.float32))
            ri = orc.topk(ref, K)
            np.testing.assert_array_equal(idx_np[b], ri)
            return ri
        ref_idx = np.stack(oracle_pool(one, list(range(B))))
        near = []
        rows_q = {}

        def quant_rows(b):
            rows_q[b] = (orc.quant_kv_fp8(comp_np[b][ref_idx[b]]), orc.quant_kv_fp8(win_np[b]))
        oracle_pool(quant_rows, list(range(B)))
        for b in range(B):
            sel = torch.from_numpy(ref_idx[b].astype(np.int64)).to(DEV)
            np.testing.assert_array_equal(wl.comp[b, sel].cpu().numpy(), rows_q[b][0])
            np.testing.assert_array_equal(wl.win[b].cpu().numpy(), rows_q[b][1])
    print(f"\n{name}: {B} requests against the oracle, {len(near)} near-ties (k-th gap within twice the "
          f"score bound): {near}")

    # attention on the oracle's selection, in the step's launch configuration, fp32 output
    sel_t = torch.from_numpy(ref_idx).to(DEV).view(B, 1, K).contiguous()
    att32 = L.csa_attend(wl.q.view(B, 1, H, D), wl.comp, wl.win, sel_t, DV, SCALE, kv_dtype=wl.kv_dtype,
                         out_dtype=torch.float32)
    att16 = L.csa_attend(wl.q.view(B, 1, H, D), wl.comp, wl.win, sel_t, DV, SCALE, kv_dtype=wl.kv_dtype,
                         out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    for b in range(B):
        if b not in near:   # same selection, same kernels and split plan: the step's own output
            assert torch.equal(att32[b, 0], out32[b]), f"{name} request {b}: step output differs"

    def ref_att(b):
        if wl.mixed:
            c, wrows = orc.dequant_kv_fp8(rows_q[b][0]), orc.dequant_kv_fp8(rows_q[b][1])
            return orc.csa_attend(_np(wl.q[b]), c, np.arange(K, dtype=np.int32), wrows, 0, -1, TW, DV, SCALE)[0]
        return orc.csa_attend(_np(wl.q[b]), comp_f(b), ref_idx[b], win_f(b), 0, -1, TW, DV, SCALE)[0]
    refs = oracle_pool(ref_att, list(range(B)))
    for b in range(B):
        _check_fp32_and_stored(att32[b, 0], att16[b, 0], refs[b], f"{name} request {b}")


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
    out32 = torch.empty(wl.out.shape, dtype=torch.float32, device=DEV)
    L.decode_fused(L.MODE_HCA, wl.q, wl.comp, wl.win, DV, SCALE, kv_dtype=kvd, out=out32, ws=wl.ws)
    torch.cuda.synchronize()
    if fp8:
        comp32 = synth.normal_t(wl.tag("comp"), (B, NC, D), dtype=torch.float32, device=DEV).cpu().numpy()
        win32 = synth.normal_t(wl.tag("win"), (B, TW, D), dtype=torch.float32, device=DEV).cpu().numpy()

    def one(b):
        if fp8:
            rows = orc.quant_kv_fp8(comp32[b])
            wrows = orc.quant_kv_fp8(win32[b])
            np.testing.assert_array_equal(wl.comp[b].cpu().numpy(), rows)
            np.testing.assert_array_equal(wl.win[b].cpu().numpy(), wrows)
            comp, win = orc.dequant_kv_fp8(rows), orc.dequant_kv_fp8(wrows)
        else:
            comp, win = _np(wl.comp[b]), _np(wl.win[b])
        return orc.hca_attend(_np(wl.q[b]), comp, 128, win, 0, -1, TW, DV, SCALE)[0]
    refs = oracle_pool(one, list(range(B)))
    for b in range(B):   # every request
        _check_fp32_and_stored(out32[b], wl.out[b], refs[b], f"{name} request {b}")


# ------------------------------------------------------------- CSA prefill
def _compress_fp32_and_stored(L, orc, stored, ref, x, z, bias, m, ov, dr, pos0, x_tail, z_tail, what):
    """The compressor run again with fp32 output on the same inputs and launch shape: within
    2e-2 x RMS of the oracle, and the stored bf16 entries are exactly those values rounded."""
    out32 = torch.empty(stored.shape, dtype=torch.float32, device=DEV)
    L.csa_compress(x, z, bias, m=m, overlap=ov, d_rope=dr, pos0=pos0, x_tail=x_tail, z_tail=z_tail, out=out32)
    torch.cuda.synchronize()
    assert torch.equal(stored, out32.to(torch.bfloat16)), f"{what}: stored entries are not the rounded fp32 ones"
    assert_close_rel_rms(out32.double().cpu().numpy(), ref, 2e-2, what)


def test_full_csa_prefill(L, orc):
    import bench
    from long_context_sparse_06_b200 import synth
    wl = _workload(L, "csa_prefill_bf16_8k")
    Q, NC, K, P0 = wl.Q, wl.NC, wl.K, wl.P0
    D, DV, H, HI, DI, TW, SCALE = bench.D, bench.DV, bench.H, bench.HI, bench.DI, bench.TW, bench.SCALE
    n0 = P0 // 4
    # 1. the chunk's compressed KV entries and index keys against the oracle's compressor
    ref_c, _ = orc.compress(_np(wl.x[0]), _np(wl.z[0]), _np(wl.bias), 4, 2, d_rope=64, pos0=P0,
                            x_tail=_np(wl.x_tail[0]), z_tail=_np(wl.z_tail[0]))
    _compress_fp32_and_stored(L, orc, wl.comp[:, n0:], ref_c, wl.x, wl.z, wl.bias, 4, 2, 64, P0, wl.x_tail,
                              wl.z_tail, "prefill compressed KV")
    ref_k, _ = orc.compress(_np(wl.kx[0]), _np(wl.zI[0]), _np(wl.biasI), 4, 2, d_rope=0, pos0=P0,
                            x_tail=_np(wl.kx_tail[0]), z_tail=_np(wl.zI_tail[0]))
    _compress_fp32_and_stored(L, orc, wl.kI[:, n0:], ref_k, wl.kx, wl.zI, wl.biasI, 4, 2, 0, P0, wl.kx_tail,
                              wl.zI_tail, "prefill compressed index keys")
    # 2. index, top-k and attention stages as the benchmark launches them, on seeded
    # entries in place of the compressor's (the oracle takes no value the device made)
    bf = torch.bfloat16
    wl.comp[:, n0:] = synth.normal_t("full.prefill.comp", (1, NC - n0, D), dtype=bf, device=DEV)
    wl.kI[:, n0:] = synth.normal_t("full.prefill.kI", (1, NC - n0, DI), dtype=bf, device=DEV)
    stream = torch.cuda.current_stream()
    wl.stage("index", stream)
    torch.cuda.synchronize()
    idx_g = wl.idx[0].cpu().numpy()
    idx_s, scores = L.csa_index_topk(wl.qI, wl.w, wl.kI, K, q_pos=wl.q_pos, want_scores=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx_s[0].cpu().numpy(), idx_g)
    # every query: its selection is the exact top-k of the scores the kernels computed
    sc_all = scores[0]
    for t in range(Q):
        na = min(NC, (P0 + t + 1) // 4)
        if t % 512 == 0 or t == Q - 1:
            assert_exact_topk(sc_all[t, :na].float().cpu().numpy(), idx_g[t], K, f"prefill query {t}")
    # 40 queries against the oracle: the first 8, the last 8 and 24 strided between
    sample = sorted(set(list(range(8)) + list(range(Q - 8, Q)) + [8 + i * (Q - 16) // 24 for i in range(24)]))
    kI = _np(wl.kI[0])

    def one(t):
        na = min(NC, (P0 + t + 1) // 4)
        s_gpu = sc_all[t, :na].float().cpu().numpy()
        assert_exact_topk(s_gpu, idx_g[t], K, f"prefill query {t}")
        qI, w = _np(wl.qI[0, t]), wl.w[0, t].cpu().numpy()
        ref = orc.index_scores_bf16(qI, w, kI[:na])
        return _selection_against_oracle(orc, s_gpu, idx_g[t], ref, bf16_score_bound(qI, w, kI[:na]), K,
                                         f"prefill query {t}")
    res = oracle_pool(one, sample)
    near = [t for t, r in zip(sample, res) if r[1]]
    print(f"\ncsa_prefill_bf16_8k: {len(sample)} queries against the oracle, {len(near)} near-ties: {near}")
    # attention on the oracle's selection for the sampled queries (the GPU's elsewhere), in
    # the benchmark's launch configuration, fp32 and bf16 output
    idx_ref = wl.idx.clone()
    for t, r in zip(sample, res):
        idx_ref[0, t] = torch.from_numpy(r[0]).to(DEV)
    args = (wl.q, wl.comp, wl.win, idx_ref, DV, SCALE)
    kw = dict(q_pos=wl.q_pos, win_pos0=wl.win_pos0, W=TW)
    out32 = L.csa_attend(*args, out_dtype=torch.float32, ws=wl.ws_a, **kw)
    out16 = L.csa_attend(*args, out_dtype=torch.bfloat16, ws=wl.ws_a, **kw)
    torch.cuda.synchronize()
    comp = _np(wl.comp[0])
    win = _np(wl.win[0])

    def ref_att(ir):
        t, r = ir
        return orc.csa_attend(_np(wl.q[0, t]), comp, r[0], win, P0 - 127, P0 + t, TW, DV, SCALE)[0]
    refs = oracle_pool(ref_att, list(zip(sample, res)))
    for t, o in zip(sample, refs):
        _check_fp32_and_stored(out32[0, t], out16[0, t], o, f"prefill query {t}")


# ------------------------------------------------------------ compressor stream
def test_full_compress_stream(L, orc):
    wl = _workload(L, "compress_stream_1m")
    T = wl.T
    passes = (("CSA KV", wl.x, wl.z, wl.bias, wl.csa, 4, 2, 64),
              ("CSA index keys", wl.kx, wl.zI, wl.biasI, wl.csaI, 4, 2, 0),
              ("HCA KV", wl.x, wl.zh, wl.biash, wl.hca, 128, 0, 64))
    for what, x, z, bias, out, m, ov, dr in passes:
        # the pass again with fp32 output: the stored bf16 entries are those values rounded
        out32 = torch.empty(out.shape, dtype=torch.float32, device=DEV)
        if m == 128:
            L.hca_compress(x, z, bias, m=m, d_rope=dr, out=out32)
        else:
            L.csa_compress(x, z, bias, m=m, overlap=ov, d_rope=dr, out=out32)
        torch.cuda.synchronize()
        assert torch.equal(out, out32.to(torch.bfloat16)), f"{what}: stored entries are not the rounded fp32 ones"
        n = T // m
        span = 256 if m == 4 else 16
        for j0 in (0, n // 2 - span // 2, n - span):
            t0, t1 = j0 * m, (j0 + span) * m
            tail = (_np(x[0, t0 - ov:t0]), _np(z[0, t0 - ov:t0])) if (ov and t0 > 0) else (None, None)
            ref, _ = orc.compress(_np(x[0, t0:t1]), _np(z[0, t0:t1]), _np(bias), m, ov, d_rope=dr, pos0=t0,
                                  x_tail=tail[0], z_tail=tail[1])
            assert_close_rel_rms(out32[0, j0:j0 + span].double().cpu().numpy(), ref, 2e-2, f"{what} entries {j0}..")
