"""GPU parity: every kernel of the hot path against the CPU oracle on seeded inputs.

Sizes are small enough for the oracle to finish in seconds while spanning several
tiles and a ragged tail.  Tolerances: integer / byte / index work bit-exact;
fp32 outputs max-abs 1e-4; bf16 / FP8 outputs max-abs 2e-2 x RMS(oracle).
"""
import math
import zlib

import numpy as np
import pytest
import torch

from helpers import assert_close_abs, assert_close_rel_rms, randn, selection_against_oracle
from helpers import bf16_score_bound as _bf16_score_bound

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import long_context_sparse_06_b200 as lcs
    lcs.lib()
    return lcs


def both_outputs(run):
    """Runs an attention call with fp32 and with bf16 output.  The bf16 output must be
    exactly the fp32 one rounded to bf16 (same arithmetic, one final rounding); the fp32
    one is returned for the comparison with the oracle, so that the 2e-2 x RMS bound
    measures the kernel's arithmetic rather than the bf16 storage step."""
    o32 = run(torch.float32)
    o16 = run(torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16)), "bf16 output is not the rounded fp32 output"
    return o32


# ------------------------------------------------------------- codecs / RoPE
def test_quant_kv_fp8_bit_exact(L, orc):
    from long_context_sparse_06_b200 import synth
    x = synth.with_outliers("g.kv8", synth.normal("g.kv8", (777, 576))).astype(np.float32)
    gpu = L.lcs_quant_kv_fp8(torch.from_numpy(x).to(DEV)).cpu().numpy()
    np.testing.assert_array_equal(gpu, orc.quant_kv_fp8(x))


def test_quant_fp4_bit_exact(L, orc):
    from long_context_sparse_06_b200 import synth
    x = synth.with_outliers("g.fp4", synth.normal("g.fp4", (513, 128))).astype(np.float32)
    x[5] = 0.0                                   # an all-zero vector: scale 1
    x[6, :32] = 1e-9                             # a block whose amax/6 underflows E4M3
    gpu = L.lcs_quant_fp4(torch.from_numpy(x).to(DEV)).cpu().numpy()
    p, s = orc.quant_fp4(x)
    np.testing.assert_array_equal(gpu[:513 * 64].reshape(513, 64), p)
    np.testing.assert_array_equal(gpu[513 * 64:].reshape(513, 4), s)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_rope(L, orc, dtype):
    x = randn("g.rope", (300, 64), dtype=dtype)
    pos = torch.arange(300, dtype=torch.int64) * 3497 + 11
    g = L.lcs_rope(x.to(DEV).clone(), pos.to(DEV), 16).float().cpu().numpy()
    ref = orc.rope(x.double().numpy(), pos.numpy(), 16)
    if dtype == torch.float32:
        assert_close_abs(g, ref, 1e-5, "rope fp32")
    else:
        assert_close_rel_rms(g, ref, 1e-2, "rope bf16")


# ------------------------------------------------------------------ compress
@pytest.mark.parametrize("case", ["c1_f32", "csa_bf16_tail", "csa_bf16_notail", "hca_bf16", "m1_identity"])
def test_compress(L, orc, case):
    if case == "c1_f32":
        B, T, d, m, ov, dr, dt, pos0 = 2, 1024, 64, 4, 2, 16, torch.float32, 0
    elif case == "csa_bf16_tail":
        B, T, d, m, ov, dr, dt, pos0 = 2, 260, 576, 4, 2, 64, torch.bfloat16, 131072
    elif case == "csa_bf16_notail":   # 3 requests: the first window of each starts before its sequence
        B, T, d, m, ov, dr, dt, pos0 = 3, 200, 128, 4, 2, 0, torch.bfloat16, 0
    elif case == "hca_bf16":
        B, T, d, m, ov, dr, dt, pos0 = 2, 128 * 5, 576, 128, 0, 64, torch.bfloat16, 0
    else:
        B, T, d, m, ov, dr, dt, pos0 = 1, 96, 64, 1, 0, 0, torch.float32, 0
    x = randn(f"g.cx.{case}", (B, T, d), dtype=dt)
    z = randn(f"g.cz.{case}", (B, T))
    bias = randn(f"g.cb.{case}", (m + ov,))
    tail = zt = None
    if case == "csa_bf16_tail":
        tail = randn("g.ct", (B, ov, d), dtype=dt)
        zt = randn("g.czt", (B, ov))
    if m == 128:
        out = L.hca_compress(x.to(DEV), z.to(DEV), bias.to(DEV), m=m, d_rope=dr, pos0=pos0)
    else:
        out = L.csa_compress(x.to(DEV), z.to(DEV), bias.to(DEV), m=m, overlap=ov, d_rope=dr, pos0=pos0,
                             x_tail=None if tail is None else tail.to(DEV), z_tail=None if zt is None else zt.to(DEV))
    g = out.float().cpu().numpy()
    for b in range(B):
        ref, _ = orc.compress(x[b].double().numpy(), z[b].double().numpy(), bias.double().numpy(), m, ov,
                              d_rope=dr, pos0=pos0,
                              x_tail=None if tail is None else tail[b].double().numpy(),
                              z_tail=None if zt is None else zt[b].double().numpy())
        if case == "m1_identity":
            np.testing.assert_array_equal(g[b], x[b].numpy())
        elif dt == torch.float32:
            assert_close_abs(g[b], ref, 1e-4, case)
        else:
            assert_close_rel_rms(g[b], ref, 2e-2, case)


# --------------------------------------------------------------------- top-k
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N", [3000, 2999])   # 2999: rows after the first start off 16-byte alignment
def test_topk_bit_exact_on_same_scores(L, orc, dtype, N):
    rows = 7
    s = randn("g.tk", (1, rows, N), std=4.0)
    s[0, 1] = torch.round(s[0, 1])                 # heavy ties
    s[0, 2] = 0.0
    s[0, 2, ::7] = -0.0                            # signed zeros tie with +0
    s[0, 3, 100:] = -1e30                          # almost all equal below the top
    s = s.to(dtype)
    for k in (1, 64, 512, 1024, 2999, 3000, 4000):
        idx = L.lcs_topk(s.to(DEV), k).cpu().numpy()
        for r in range(rows):
            ref = orc.topk(s[0, r].float().numpy(), k)
            np.testing.assert_array_equal(idx[0, r], ref, err_msg=f"row {r} k {k}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N", [8192, 32768, 40000, 65536, 65537])   # 1, 4, 5 and 8 CTAs per row; one more
def test_topk_register_rows(L, orc, dtype, N):
    """Rows at the register-resident limit: ties at the threshold, all-equal rows, monotone
    rows, +-0, a threshold bin crowded to its last bits, and causal availability."""
    rows = 8
    s = randn(f"g.tkr{N}", (1, rows, N), std=3.0)
    s[0, 1] = torch.round(s[0, 1] * 2) / 2                        # heavy ties
    s[0, 2] = 1.5                                                 # all equal
    s[0, 3] = torch.arange(N, dtype=torch.float32)                # increasing
    s[0, 4] = -torch.arange(N, dtype=torch.float32)               # decreasing
    s[0, 5] = 0.0
    s[0, 5, ::3] = -0.0
    s[0, 5, ::97] = 2.0
    s[0, 6] = 1.0 + torch.arange(N, dtype=torch.float32) * 2.0 ** -22 * (torch.arange(N) % 5 == 0)   # one bin
    s[0, 7, : N // 2] = -1e30
    s = s.to(dtype)
    for k in (1, 512, 1024, 4096):
        idx = L.lcs_topk(s.to(DEV), k).cpu().numpy()
        for r in range(rows):
            np.testing.assert_array_equal(idx[0, r], orc.topk(s[0, r].float().numpy(), k), err_msg=f"row {r} k {k}")
    q_pos = torch.tensor([[2, 3, 2047, 4100, 65535, 4 * N + 8, 40000, 131070]], dtype=torch.int64)
    idx = L.lcs_topk(s.to(DEV), 512, q_pos=q_pos.to(DEV), m=4).cpu().numpy()
    for r in range(rows):
        n = orc.n_avail(int(q_pos[0, r]), 4, N)
        np.testing.assert_array_equal(idx[0, r], orc.topk(s[0, r, :n].float().numpy(), 512), err_msg=f"causal {r}")


def test_topk_large_rows_and_causal(L, orc):
    # rows longer than the shared-memory cache; causal availability per query
    s = randn("g.tkl", (1, 5, 70000), std=3.0)
    s[0, 1] = torch.round(s[0, 1] * 4) / 4
    s[0, 2] = 1.5                                   # all equal: the sampled bound keeps every element
    s[0, 3, :] = torch.arange(70000, dtype=torch.float32)      # strictly increasing row
    s[0, 4, :] = -torch.arange(70000, dtype=torch.float32)
    idx = L.lcs_topk(s.to(DEV), 1024).cpu().numpy()
    for r in range(5):
        np.testing.assert_array_equal(idx[0, r], orc.topk(s[0, r].numpy(), 1024))
    q_pos = torch.tensor([[0, 3, 4, 100, 4095, 20000]], dtype=torch.int64)
    s2 = randn("g.tkc", (1, 6, 5000))
    idx = L.lcs_topk(s2.to(DEV), 64, q_pos=q_pos.to(DEV), m=4).cpu().numpy()
    for r in range(6):
        n = orc.n_avail(int(q_pos[0, r]), 4, 5000)
        np.testing.assert_array_equal(idx[0, r], orc.topk(s2[0, r, :n].numpy(), 64))


def test_topk_few_long_rows_run_as_clusters(L, orc):
    """Four rows of 262144 bf16 scores (the 1M decode's shape): exact, and each row split over
    a cluster.  One CTA per row gives the same selection about 30x slower (0.8 ms against
    25 us per launch), so the launch time tells the two forms apart."""
    rows, N, k = 4, 262144, 1024
    s = randn("g.tkf", (1, rows, N), std=3.0).to(torch.bfloat16)
    sd = s.to(DEV)
    idx = L.lcs_topk(sd, k).cpu().numpy()
    for r in range(rows):
        np.testing.assert_array_equal(idx[0, r], orc.topk(s[0, r].float().numpy(), k), err_msg=f"row {r}")
    ws = L.workspace(L.lcs_workspace_size(L.OP_TOPK), sd.device)
    st = torch.cuda.current_stream()
    for _ in range(3):
        L.lcs_topk(sd, k, ws=ws, stream=st)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(20):
        L.lcs_topk(sd, k, ws=ws, stream=st)
    e1.record(st)
    torch.cuda.synchronize()
    per_us = e0.elapsed_time(e1) / 20 * 1e3
    assert per_us < 300, f"{per_us:.0f} us per launch: the rows did not run as clusters"


# ------------------------------------------------------------------- indexer
def test_index_f32_bit_exact(L, orc):
    """C1 indexer shape: 4 heads x 32 dims, causal over 256 entries."""
    B, Q, H, dI, Nc, k = 1, 200, 4, 32, 256, 64
    qI = randn("g.i32.q", (B, Q, H, dI))
    w = randn("g.i32.w", (B, Q, H), std=0.5)
    kI = randn("g.i32.k", (B, Nc, dI))
    q_pos = (torch.arange(Q, dtype=torch.int64) * 5 + 3).reshape(B, Q)
    idx, sc = L.csa_index_topk(qI.to(DEV), w.to(DEV), kI.to(DEV), k, q_pos=q_pos.to(DEV), m=4, want_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    for q in range(Q):
        n = orc.n_avail(int(q_pos[0, q]), 4, Nc)
        ref = orc.index_scores_f32(qI[0, q].numpy(), w[0, q].numpy(), kI[0, :n].numpy())
        np.testing.assert_array_equal(sc[0, q, :n], ref)
        np.testing.assert_array_equal(idx[0, q], orc.topk(ref, k))


def test_index_bf16_tensor_cores(L, orc):
    B, H, dI, Nc, k = 6, 64, 128, 1500, 128           # 12 tiles per request, ragged last tile
    qI = randn("g.ib.q", (B, 1, H, dI), dtype=torch.bfloat16)
    w = randn("g.ib.w", (B, 1, H), std=1 / 8)
    kI = randn("g.ib.k", (B, Nc, dI), dtype=torch.bfloat16)
    idx, sc = L.csa_index_topk(qI.to(DEV), w.to(DEV), kI.to(DEV), k, want_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    near = []
    for b in range(B):
        qd, kd, wd = qI[b, 0].double().numpy(), kI[b].double().numpy(), w[b, 0].numpy()
        ref = orc.index_scores_bf16(qd, wd, kd)
        bound = _bf16_score_bound(qd, wd, kd)
        err = np.abs(sc[b, 0].astype(np.float64) - ref)
        assert np.all(err <= bound), f"b={b}: max err/bound {np.max(err / bound):.3f}"
        # level 1: the selection on the GPU's own scores is the oracle's selection
        np.testing.assert_array_equal(idx[b, 0], orc.topk(sc[b, 0], k))
        # level 3: equal to the oracle's selection unless a near-tie explains the difference
        if selection_against_oracle(orc, sc[b, 0], idx[b, 0], ref, bound, k, f"b={b}")[1]:
            near.append(b)
    print(f"\nbf16 indexer: {B} rows, near-ties {near}")
    assert len(near) <= 1, f"near-ties {near}"


def test_index_bf16_dot_rounding(L, orc):
    """How the tensor cores round a 128-long bf16 dot (kind::f16, fp32 accumulation):
    with a one-hot head weight the score is exactly ReLU of one head's dot, which the
    oracle defines as the exact dot rounded once to fp32.  Every GPU dot must lie within
    the derived bound of it; the share that equals it is reported (when it is all of them,
    bf16-key selections are bit-exact end to end)."""
    B, H, dI, Nc = 64, 64, 128, 2048
    qI = randn("g.ir.q", (B, 1, H, dI), dtype=torch.bfloat16)
    kI = randn("g.ir.k", (B, Nc, dI), dtype=torch.bfloat16)
    w = torch.zeros((B, 1, H))
    for b in range(B):
        w[b, 0, b % H] = 1.0                       # request b tests head b's accumulator column
    tot = eq = 0
    worst = 0.0
    for sign in (1.0, -1.0):                       # the negated query turns the other half positive
        q_s = (qI * sign).contiguous()
        _, sc = L.csa_index_topk(q_s.to(DEV), w.to(DEV), kI.to(DEV), 1, want_scores=True)
        sc = sc.cpu().numpy()[:, 0]
        for b in range(B):
            qd, kd = q_s[b, 0].double().numpy(), kI[b].double().numpy()
            ref = orc.index_scores_bf16(qd, w[b, 0].numpy(), kd).astype(np.float64)
            pos = ref > 0
            g = sc[b].astype(np.float64)
            bound = (dI // 16 + 1) * 2.0 ** -23 * (np.abs(kd) @ np.abs(qd[b % H]))
            assert np.all(np.abs(g - ref) <= bound), f"b={b}: a dot outside the bound"
            tot += int(pos.sum())
            eq += int((g[pos] == ref[pos]).sum())
            worst = max(worst, float(np.max(np.abs(g - ref)[pos] / bound[pos])))
    print(f"\nkind::f16 128-dot: {eq}/{tot} equal to the correctly rounded dot "
          f"({100.0 * eq / tot:.2f} %), largest error {worst:.3f} of the bound")
    assert tot > B * Nc // 2


@pytest.mark.parametrize("B,Q", [(1, 40), (2, 38)])   # 38: the last group of four queries is ragged
def test_index_bf16_causal_prefill(L, orc, B, Q):
    H, dI, Nc, k = 64, 128, 700, 64
    qI = randn(f"g.ic.q{B}", (B, Q, H, dI), dtype=torch.bfloat16)
    w = randn(f"g.ic.w{B}", (B, Q, H), std=1 / 8)
    kI = randn(f"g.ic.k{B}", (B, Nc, dI), dtype=torch.bfloat16)
    q_pos = (torch.arange(Q, dtype=torch.int64) * 71 + 2).reshape(1, Q).repeat(B, 1)
    q_pos[B - 1] += 5
    idx, sc = L.csa_index_topk(qI.to(DEV), w.to(DEV), kI.to(DEV), k, q_pos=q_pos.to(DEV), m=4, want_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    for b in range(B):
        for q in range(Q):
            n = orc.n_avail(int(q_pos[b, q]), 4, Nc)
            qd, kd, wd = qI[b, q].double().numpy(), kI[b, :n].double().numpy(), w[b, q].numpy()
            ref = orc.index_scores_bf16(qd, wd, kd)
            if n:
                assert np.all(np.abs(sc[b, q, :n] - ref) <= _bf16_score_bound(qd, wd, kd))
            np.testing.assert_array_equal(idx[b, q], orc.topk(sc[b, q, :n], k))


# ----------------------------------------------------------------- attention
def test_attend_f32_c1(L, orc):
    """C1 attention shape: 8 heads, D = 64 (48 + 16), d_v = 48, k = 64, window 128, causal."""
    B, Q, H, D, dv, Nc, k, W = 1, 160, 8, 64, 48, 256, 64, 128
    T = 1024
    q = randn("g.a32.q", (B, Q, H, D))
    comp = randn("g.a32.c", (B, Nc, D))
    win = randn("g.a32.w", (B, T, D))
    q_pos = (torch.arange(Q, dtype=torch.int64) * 6 + 5).reshape(B, Q)
    rng = np.random.default_rng(0)
    idx = np.full((B, Q, k), -1, np.int32)
    for q_ in range(Q):
        n = orc.n_avail(int(q_pos[0, q_]), 4, Nc)
        take = min(k, n)
        if take:
            idx[0, q_, :take] = np.sort(rng.choice(n, take, replace=False))
    wp0 = torch.zeros(B, dtype=torch.int64)
    out, lse = L.csa_attend(q.to(DEV), comp.to(DEV), win.to(DEV), torch.from_numpy(idx).to(DEV), dv, 1 / 8,
                            q_pos=q_pos.to(DEV), win_pos0=wp0.to(DEV), W=W, want_lse=True)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for q_ in range(Q):
        o, l = orc.csa_attend(q[0, q_].double().numpy(), comp[0].double().numpy(), idx[0, q_],
                              win[0].double().numpy(), 0, int(q_pos[0, q_]), W, dv, 1 / 8)
        assert_close_abs(out[0, q_], o, 1e-4, f"q {q_}")
        assert_close_abs(lse[0, q_], l, 1e-4, f"lse q {q_}")


def _rand_sel(name, B, Q, k, navail):
    rng = np.random.default_rng(zlib.crc32(name.encode()))   # str hash() is salted per process
    idx = np.full((B, Q, k), -1, np.int32)
    for b in range(B):
        for q in range(Q):
            n = navail[b][q] if isinstance(navail, list) else navail
            t = min(k, n)
            if t:
                idx[b, q, :t] = np.sort(rng.choice(n, t, replace=False))
    return idx


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_csa_attend_decode_tc(L, orc, kv):
    B, H, D, dv, Nc, k, Tw = 5, 64, 576, 512, 3000, 512, 128
    scale = 1 / math.sqrt(576)
    q = randn(f"g.ad.q.{kv}", (B, 1, H, D), dtype=torch.bfloat16)
    comp32 = randn(f"g.ad.c.{kv}", (B, Nc, D))
    win32 = randn(f"g.ad.w.{kv}", (B, Tw, D))
    idx = _rand_sel(f"sel.{kv}", B, 1, k, Nc)
    idx[1, 0, 300:] = -1                         # a short selection
    idx[2, 0, :] = -1                            # window only
    if kv == "bf16":
        comp, win = comp32.to(torch.bfloat16), win32.to(torch.bfloat16)
        comp_g, win_g, kvd = comp.to(DEV), win.to(DEV), L.BF16
        comp_d, win_d = comp.double().numpy(), win.double().numpy()
    else:
        comp_g = L.lcs_quant_kv_fp8(comp32.to(DEV))
        win_g = L.lcs_quant_kv_fp8(win32.to(DEV))
        kvd = L.KV_FP8
        comp_d = orc.dequant_kv_fp8(orc.quant_kv_fp8(comp32.numpy()))
        win_d = orc.dequant_kv_fp8(orc.quant_kv_fp8(win32.numpy()))
    idx_g = torch.from_numpy(idx).to(DEV)
    out = both_outputs(lambda od: L.csa_attend(q.to(DEV), comp_g, win_g, idx_g, dv, scale, kv_dtype=kvd,
                                               out_dtype=od)).cpu().numpy()
    _, lse = L.csa_attend(q.to(DEV), comp_g, win_g, idx_g, dv, scale, kv_dtype=kvd, want_lse=True)
    lse = lse.cpu().numpy()
    for b in range(B):
        o, l = orc.csa_attend(q[b, 0].double().numpy(), comp_d[b], idx[b, 0], win_d[b], 0, -1, 128, dv, scale)
        assert_close_rel_rms(out[b, 0], o, 2e-2, f"{kv} b {b}")
        assert_close_abs(lse[b, 0], l, 2e-2, f"{kv} lse b {b}")


def test_hca_attend_decode_tc(L, orc):
    B, H, D, dv, Nc, Tw = 3, 64, 576, 512, 1100, 128     # many chunks, several splits
    scale = 1 / math.sqrt(576)
    q = randn("g.h.q", (B, 1, H, D), dtype=torch.bfloat16)
    comp = randn("g.h.c", (B, Nc, D), dtype=torch.bfloat16)
    win = randn("g.h.w", (B, Tw, D), dtype=torch.bfloat16)
    out = both_outputs(lambda od: L.hca_attend(q.to(DEV), comp.to(DEV), win.to(DEV), dv, scale,
                                               out_dtype=od)).cpu().numpy()
    _, lse = L.hca_attend(q.to(DEV), comp.to(DEV), win.to(DEV), dv, scale, want_lse=True)
    lse = lse.cpu().numpy()
    for b in range(B):
        o, l = orc.hca_attend(q[b, 0].double().numpy(), comp[b].double().numpy(), 128, win[b].double().numpy(), 0,
                              -1, 128, dv, scale)
        assert_close_rel_rms(out[b, 0], o, 2e-2, f"hca b {b}")
        assert_close_abs(lse[b, 0], l, 2e-2, f"hca lse b {b}")


def test_hca_attend_decode_fp8(L, orc):
    """HCA over FP8 rows (content E4M3 with a power-of-two scale per 128, RoPE dims bf16),
    heavy-tailed values: the 1M-context row format applied to dense attention."""
    from long_context_sparse_06_b200 import synth
    B, H, D, dv, Nc, Tw = 3, 64, 576, 512, 1100, 128
    scale = 1 / math.sqrt(576)
    q = randn("g.h8.q", (B, 1, H, D), dtype=torch.bfloat16)
    comp32 = synth.with_outliers("g.h8.c", synth.normal("g.h8.c", (B, Nc, D))).astype(np.float32)
    win32 = synth.with_outliers("g.h8.w", synth.normal("g.h8.w", (B, Tw, D))).astype(np.float32)
    comp_g = L.lcs_quant_kv_fp8(torch.from_numpy(comp32).to(DEV))
    win_g = L.lcs_quant_kv_fp8(torch.from_numpy(win32).to(DEV))
    out = both_outputs(lambda od: L.hca_attend(q.to(DEV), comp_g, win_g, dv, scale, kv_dtype=L.KV_FP8,
                                               out_dtype=od)).cpu().numpy()
    comp_d = orc.dequant_kv_fp8(orc.quant_kv_fp8(comp32))
    win_d = orc.dequant_kv_fp8(orc.quant_kv_fp8(win32))
    for b in range(B):
        o, _ = orc.hca_attend(q[b, 0].double().numpy(), comp_d[b], 128, win_d[b], 0, -1, 128, dv, scale)
        assert_close_rel_rms(out[b, 0], o, 2e-2, f"hca fp8 b {b}")


@pytest.mark.parametrize("case", ["hca_full_chunks", "csa_gathered", "hca_partial_chunks"])
def test_attend_fp8_widening_exact(L, orc, case):
    """FP8 rows reach the tensor cores exactly widened to bf16.  With q = 0 every score is 0,
    every softmax weight exactly 1; every row is the same row and the number of rows is a
    power of two, so o = V of that row, bit for bit, in fp32.  The row holds all 254
    finite E4M3 codes (subnormals, +-0 included) under block scales 2^-117, 2^-3, 2^15 and
    2^20.  Cases: whole 64-row chunks (TMA, widened in shared memory), gathered selected
    rows, partial chunks (row-by-row loads)."""
    H, D, dv = 64, 576, 512
    codes = [c for c in range(256) if c not in (0x7F, 0xFF)]
    codes = np.array((codes * 3)[:512], np.uint8)
    rope = torch.from_numpy(synth_normal("g.fp8x.r", (64,))).to(torch.bfloat16).view(torch.int16).numpy()
    scales = np.array([2.0 ** -117, 2.0 ** -3, 2.0 ** 15, 2.0 ** 20], np.float32)
    row = np.concatenate([codes, rope.view(np.uint8), scales.view(np.uint8)])
    assert row.size == 656
    n_c, tw, idx = {"hca_full_chunks": (64, 64, None), "csa_gathered": (100, 64, list(range(3, 67))),
                    "hca_partial_chunks": (37, 27, None)}[case]
    comp = torch.from_numpy(np.tile(row, (1, n_c, 1))).to(DEV)
    win = torch.from_numpy(np.tile(row, (1, tw, 1))).to(DEV)
    q = torch.zeros((1, 1, H, D), dtype=torch.bfloat16, device=DEV)   # every score exactly 0
    if idx is None:
        out = L.hca_attend(q, comp, win, dv, 1 / 24, kv_dtype=L.KV_FP8, out_dtype=torch.float32)
    else:
        sel = torch.tensor(idx, dtype=torch.int32).view(1, 1, -1).to(DEV)
        out = L.csa_attend(q, comp, win, sel, dv, 1 / 24, kv_dtype=L.KV_FP8, out_dtype=torch.float32)
    want = orc.dequant_kv_fp8(row)[:dv]
    got = out[0, 0].double().cpu().numpy()
    bad = np.nonzero(got != want[None, :])
    assert bad[0].size == 0, f"{bad[0].size} outputs differ, first at head {bad[0][0]} dim {bad[1][0]}: " \
                             f"{got[bad[0][0], bad[1][0]]!r} vs {want[bad[1][0]]!r}"


def synth_normal(name, shape):
    from long_context_sparse_06_b200 import synth
    return synth.normal(name, shape).astype(np.float32)


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_attend_rows_outside_range_unread(L, orc, kv):
    """Rows outside a query's row set (compressed entries >= n_avail, window rows outside
    [t-W+1, t], rows a partial 64-row chunk spans past its end) may hold anything: a cache
    fills as the sequence grows.  Here they are all NaN; HCA and CSA must still equal the
    oracle on the defined rows (partial window chunks of 6 and 21 rows, compressed tails
    of 37, 37 and 8 rows)."""
    from long_context_sparse_06_b200 import synth
    B, H, D, dv, Nc, Tw, W, m, k = 3, 64, 576, 512, 260, 128, 128, 128, 96
    scale = 1 / math.sqrt(576)
    avail, nwin = [37, 101, 200], [70, 128, 21]
    t = [m * a + 5 for a in avail]                     # n_avail = floor((t+1)/m) = avail
    wp0 = [t[b] - (nwin[b] - 1) for b in range(B)]     # window rows 0..nwin-1 in range
    q = randn(f"g.nan.{kv}.q", (B, 1, H, D), dtype=torch.bfloat16)
    comp32 = synth.normal(f"g.nan.{kv}.c", (B, Nc, D)).astype(np.float32)
    win32 = synth.normal(f"g.nan.{kv}.w", (B, Tw, D)).astype(np.float32)
    if kv == "bf16":
        comp_g = torch.from_numpy(comp32).to(torch.bfloat16)
        win_g = torch.from_numpy(win32).to(torch.bfloat16)
        comp_o, win_o = comp_g.double().numpy(), win_g.double().numpy()
        poison = float("nan")
        kvd = None
    else:
        comp_g = L.lcs_quant_kv_fp8(torch.from_numpy(comp32).to(DEV)).cpu()
        win_g = L.lcs_quant_kv_fp8(torch.from_numpy(win32).to(DEV)).cpu()
        comp_o = orc.dequant_kv_fp8(orc.quant_kv_fp8(comp32))
        win_o = orc.dequant_kv_fp8(orc.quant_kv_fp8(win32))
        poison = 0xFF                                  # NaN codes, NaN scales, NaN RoPE dims
        kvd = L.KV_FP8
    for b in range(B):
        comp_g[b, avail[b]:] = poison
        win_g[b, nwin[b]:] = poison
    q_pos = torch.tensor(t, dtype=torch.int64).reshape(B, 1).to(DEV)
    win_pos0 = torch.tensor(wp0, dtype=torch.int64).to(DEV)
    qd, cd, wd = q.to(DEV), comp_g.to(DEV), win_g.to(DEV)
    outh = both_outputs(lambda od: L.hca_attend(qd, cd, wd, dv, scale, kv_dtype=kvd, q_pos=q_pos, win_pos0=win_pos0,
                                                m=m, W=W, out_dtype=od)).cpu().numpy()
    idx = _rand_sel(f"sel.nan.{kv}", B, 1, k, [[a] for a in avail])
    outc = both_outputs(lambda od: L.csa_attend(qd, cd, wd, torch.from_numpy(idx).to(DEV), dv, scale, kv_dtype=kvd,
                                                q_pos=q_pos, win_pos0=win_pos0, W=W, out_dtype=od)).cpu().numpy()
    assert np.isfinite(outh).all() and np.isfinite(outc).all()
    for b in range(B):
        qb = q[b, 0].double().numpy()
        comp_b = comp_o[b, :avail[b]]
        o, _ = orc.hca_attend(qb, comp_b, m, win_o[b], wp0[b], t[b], W, dv, scale)
        assert_close_rel_rms(outh[b, 0], o, 2e-2, f"hca b {b}")
        o, _ = orc.csa_attend(qb, comp_b, idx[b, 0], win_o[b, :nwin[b]], wp0[b], t[b], W, dv, scale)
        assert_close_rel_rms(outc[b, 0], o, 2e-2, f"csa b {b}")


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_attend_degenerate_row_sets(L, orc, kv):
    """Degenerate row sets: a selection that is all -1 (the window alone), no window at
    all (Tw = 0: the selection alone), and neither (R empty: o = 0, lse = -inf)."""
    from long_context_sparse_06_b200 import synth
    B, H, D, dv, Nc, k, Tw = 2, 64, 576, 512, 700, 200, 128
    scale = 1 / 24
    q = randn(f"g.dg.{kv}.q", (B, 1, H, D), dtype=torch.bfloat16)
    comp32 = synth.normal(f"g.dg.{kv}.c", (B, Nc, D)).astype(np.float32)
    win32 = synth.normal(f"g.dg.{kv}.w", (B, Tw, D)).astype(np.float32)
    if kv == "bf16":
        comp_g, win_g = torch.from_numpy(comp32).to(torch.bfloat16), torch.from_numpy(win32).to(torch.bfloat16)
        comp_o, win_o = comp_g.double().numpy(), win_g.double().numpy()
        comp_g, win_g, kvd = comp_g.to(DEV), win_g.to(DEV), None
    else:
        comp_g = L.lcs_quant_kv_fp8(torch.from_numpy(comp32).to(DEV))
        win_g = L.lcs_quant_kv_fp8(torch.from_numpy(win32).to(DEV))
        comp_o = orc.dequant_kv_fp8(orc.quant_kv_fp8(comp32))
        win_o = orc.dequant_kv_fp8(orc.quant_kv_fp8(win32))
        kvd = L.KV_FP8
    qd = q.to(DEV)
    sel = _rand_sel(f"sel.dg.{kv}", B, 1, k, Nc)
    none = np.full((B, 1, k), -1, np.int32)
    no_win = np.zeros((0, D))
    # the window alone
    out = both_outputs(lambda od: L.csa_attend(qd, comp_g, win_g, torch.from_numpy(none).to(DEV), dv, scale,
                                               kv_dtype=kvd, out_dtype=od)).cpu().numpy()
    for b in range(B):
        o, _ = orc.csa_attend(q[b, 0].double().numpy(), comp_o[b], none[b, 0], win_o[b], 0, -1, 128, dv, scale)
        assert_close_rel_rms(out[b, 0], o, 2e-2, f"window alone b {b}")
    # the selection alone
    out = both_outputs(lambda od: L.csa_attend(qd, comp_g, None, torch.from_numpy(sel).to(DEV), dv, scale,
                                               kv_dtype=kvd, out_dtype=od)).cpu().numpy()
    for b in range(B):
        o, _ = orc.csa_attend(q[b, 0].double().numpy(), comp_o[b], sel[b, 0], no_win, 0, -1, 128, dv, scale)
        assert_close_rel_rms(out[b, 0], o, 2e-2, f"selection alone b {b}")
    # nothing: the empty sum
    out, lse = L.csa_attend(qd, comp_g, None, torch.from_numpy(none).to(DEV), dv, scale, kv_dtype=kvd,
                            want_lse=True, out_dtype=torch.float32)
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


@pytest.mark.parametrize("tail", [127, 50])
def test_attend_prefill_tc_causal(L, orc, tail):
    """C4-shaped (smaller): queries at positions p0.., window from the chunk plus a prefix tail
    of `tail` raw rows (50: the first queries see partial windows of 51.. rows)."""
    B, Q, H, D, dv, k, W = 1, 24, 64, 576, 512, 256, 128
    p0 = 4000
    Nc = (p0 + Q) // 4
    Tw = tail + Q
    scale = 1 / math.sqrt(576)
    q = randn("g.ap.q", (B, Q, H, D), dtype=torch.bfloat16)
    comp = randn("g.ap.c", (B, Nc, D), dtype=torch.bfloat16)
    win = randn("g.ap.w", (B, Tw, D), dtype=torch.bfloat16)
    q_pos = (p0 + torch.arange(Q, dtype=torch.int64)).reshape(B, Q)
    wp0 = torch.tensor([p0 - tail], dtype=torch.int64)
    nav = [[orc.n_avail(int(t), 4, Nc) for t in q_pos[0]]]
    idx = _rand_sel("sel.pf", B, Q, k, nav)
    out = both_outputs(lambda od: L.csa_attend(q.to(DEV), comp.to(DEV), win.to(DEV), torch.from_numpy(idx).to(DEV),
                                               dv, scale, q_pos=q_pos.to(DEV), win_pos0=wp0.to(DEV),
                                               out_dtype=od)).cpu().numpy()
    for t in range(Q):
        o, _ = orc.csa_attend(q[0, t].double().numpy(), comp[0].double().numpy(), idx[0, t],
                              win[0].double().numpy(), p0 - tail, int(q_pos[0, t]), W, dv, scale)
        assert_close_rel_rms(out[0, t], o, 2e-2, f"prefill q {t}")
    # HCA causal with m' = 128 on the same queries
    Nh = (p0 + Q) // 128
    outh = both_outputs(lambda od: L.hca_attend(q.to(DEV), comp[:, :Nh].contiguous().to(DEV), win.to(DEV), dv, scale,
                                                q_pos=q_pos.to(DEV), win_pos0=wp0.to(DEV), m=128,
                                                out_dtype=od)).cpu().numpy()
    for t in range(0, Q, 5):
        o, _ = orc.hca_attend(q[0, t].double().numpy(), comp[0, :Nh].double().numpy(), 128, win[0].double().numpy(),
                              p0 - tail, int(q_pos[0, t]), W, dv, scale)
        assert_close_rel_rms(outh[0, t], o, 2e-2, f"hca prefill q {t}")


# -------------------------------------------------------------- fused decode
def test_decode_fused_csa_bf16(L, orc):
    B, H, D, dv, Nc, k, Tw, HI, dI = 4, 64, 576, 512, 2500, 256, 128, 64, 128
    scale = 1 / math.sqrt(576)
    q = randn("g.df.q", (B, H, D), dtype=torch.bfloat16)
    comp = randn("g.df.c", (B, Nc, D), dtype=torch.bfloat16)
    win = randn("g.df.w", (B, Tw, D), dtype=torch.bfloat16)
    qI = randn("g.df.qi", (B, HI, dI), dtype=torch.bfloat16)
    w = randn("g.df.wi", (B, HI), std=1 / 8)
    kI = randn("g.df.ki", (B, Nc, dI), dtype=torch.bfloat16)
    idx_out = torch.empty((B, k), dtype=torch.int32, device=DEV)
    out = both_outputs(lambda od: L.decode_fused(L.MODE_CSA, q.to(DEV), comp.to(DEV), win.to(DEV), dv, scale,
                                                 qI=qI.to(DEV), w=w.to(DEV), kI=kI.to(DEV), k=k, idx_out=idx_out,
                                                 out_dtype=od))
    out, idx = out.cpu().numpy(), idx_out.cpu().numpy()
    near = []
    ref_idx = np.zeros((B, k), np.int32)
    for b in range(B):
        qd, kd, wd = qI[b].double().numpy(), kI[b].double().numpy(), w[b].numpy()
        ref_s = orc.index_scores_bf16(qd, wd, kd)
        s_gpu = L.csa_index_topk(qI[b:b + 1, None].to(DEV), w[b:b + 1, None].to(DEV), kI[b:b + 1].to(DEV), k,
                                 want_scores=True)[1][0, 0].cpu().numpy()
        ref_idx[b], nt = selection_against_oracle(orc, s_gpu, idx[b], ref_s, _bf16_score_bound(qd, wd, kd), k,
                                                  f"fused b {b}")
        if nt:
            near.append(b)
    assert len(near) <= 1, f"near-ties {near}"
    # attention on the oracle's selection: the fused step's output where the selections
    # agree, else csa_attend given the oracle's selection
    att = both_outputs(lambda od: L.csa_attend(q.to(DEV).view(B, 1, H, D), comp.to(DEV), win.to(DEV),
                                               torch.from_numpy(ref_idx).to(DEV).view(B, 1, k), dv, scale,
                                               out_dtype=od)).cpu().numpy()[:, 0]
    for b in range(B):
        if b not in near:
            np.testing.assert_array_equal(out[b], att[b])
        o, _ = orc.csa_attend(q[b].double().numpy(), comp[b].double().numpy(), ref_idx[b],
                              win[b].double().numpy(), 0, -1, 128, dv, scale)
        assert_close_rel_rms(att[b], o, 2e-2, f"fused b {b}")


def test_decode_fused_hca(L, orc):
    B, H, D, dv, Nc, Tw = 2, 64, 576, 512, 900, 128
    scale = 1 / math.sqrt(576)
    q = randn("g.dh.q", (B, H, D), dtype=torch.bfloat16)
    comp = randn("g.dh.c", (B, Nc, D), dtype=torch.bfloat16)
    win = randn("g.dh.w", (B, Tw, D), dtype=torch.bfloat16)
    out = both_outputs(lambda od: L.decode_fused(L.MODE_HCA, q.to(DEV), comp.to(DEV), win.to(DEV), dv, scale,
                                                 out_dtype=od)).cpu().numpy()
    for b in range(B):
        o, _ = orc.hca_attend(q[b].double().numpy(), comp[b].double().numpy(), 128, win[b].double().numpy(), 0, -1,
                              128, dv, scale)
        assert_close_rel_rms(out[b], o, 2e-2, f"fused hca b {b}")


# --------------------------------------------------------- grouped projection
def test_group_oproj(L, orc):
    T, H, dv, G, dg, hidden = 300, 8, 48, 2, 64, 256
    o = randn("g.gp.o", (T, H, dv))
    Wg = randn("g.gp.g", (G, H // G * dv, dg), std=1 / math.sqrt(H // G * dv))
    Wo = randn("g.gp.w", (G * dg, hidden), std=1 / math.sqrt(G * dg))
    y = L.group_oproj(o.to(DEV), Wg.to(DEV), Wo.to(DEV)).cpu().numpy()
    for t in range(0, T, 7):
        assert_close_abs(y[t], orc.group_oproj(o[t].double().numpy(), Wg.double().numpy(), Wo.double().numpy()),
                         1e-4, f"t {t}")


# ------------------------------------------------- determinism and invariance
def test_determinism_and_batch_invariance(L):
    B, H, D, dv, Nc, k, Tw = 4, 64, 576, 512, 1800, 256, 128
    scale = 1 / math.sqrt(576)
    q = randn("g.di.q", (B, H, D), dtype=torch.bfloat16).to(DEV)
    comp = randn("g.di.c", (B, Nc, D), dtype=torch.bfloat16).to(DEV)
    win = randn("g.di.w", (B, Tw, D), dtype=torch.bfloat16).to(DEV)
    qI = randn("g.di.qi", (B, 64, 128), dtype=torch.bfloat16).to(DEV)
    w = randn("g.di.wi", (B, 64), std=1 / 8).to(DEV)
    kI = randn("g.di.ki", (B, Nc, 128), dtype=torch.bfloat16).to(DEV)
    args = dict(qI=qI, w=w, kI=kI, k=k)
    o1 = L.decode_fused(L.MODE_CSA, q, comp, win, dv, scale, **args)
    o2 = L.decode_fused(L.MODE_CSA, q, comp, win, dv, scale, **args)
    assert torch.equal(o1, o2)
    perm = torch.tensor([2, 0, 3, 1], device=DEV)
    o3 = L.decode_fused(L.MODE_CSA, q[perm].contiguous(), comp[perm].contiguous(), win[perm].contiguous(), dv, scale,
                        qI=qI[perm].contiguous(), w=w[perm].contiguous(), kI=kI[perm].contiguous(), k=k)
    assert torch.equal(o3, o1[perm])
    # the selection does not depend on the batch at all
    i1 = torch.empty((B, k), dtype=torch.int32, device=DEV)
    i4 = torch.empty((1, k), dtype=torch.int32, device=DEV)
    L.decode_fused(L.MODE_CSA, q, comp, win, dv, scale, idx_out=i1, **args)
    L.decode_fused(L.MODE_CSA, q[1:2].contiguous(), comp[1:2].contiguous(), win[1:2].contiguous(), dv, scale,
                   qI=qI[1:2].contiguous(), w=w[1:2].contiguous(), kI=kI[1:2].contiguous(), k=k, idx_out=i4)
    assert torch.equal(i4[0], i1[1])


# ------------------------------------------------------------- FP4 QK path
def _fp4_keys(L, orc, name, B, Nc):
    from long_context_sparse_06_b200 import synth
    raw = synth.with_outliers(name, synth.normal(name, (B, Nc, 128))).astype(np.float32)
    planes = L.lcs_quant_fp4(torch.from_numpy(raw).to(DEV))
    p, s = orc.quant_fp4(raw.reshape(B * Nc, 128))
    got = planes.cpu().numpy()
    np.testing.assert_array_equal(got[:B * Nc * 64].reshape(B * Nc, 64), p)
    np.testing.assert_array_equal(got[B * Nc * 64:].reshape(B * Nc, 4), s)
    return planes, p.reshape(B, Nc, 64), s.reshape(B, Nc, 4)


def test_index_fp4_bit_exact(L, orc):
    """FP4 keys and on-the-fly FP4 query: bf16 scores and the selection bit-exact."""
    B, H, Nc, k = 2, 64, 2000, 256
    qI = randn("g.i4.q", (B, 1, H, 128), dtype=torch.bfloat16)
    w = randn("g.i4.w", (B, 1, H), std=1 / 8)
    planes, kp, ks = _fp4_keys(L, orc, "g.i4.k", B, Nc)
    idx, sc = L.csa_index_topk(qI.to(DEV), w.to(DEV), planes, k, N_c=Nc, kI_dtype=L.FP4, want_scores=True)
    idx, sc = idx.cpu().numpy(), sc.float().cpu().numpy()
    for b in range(B):
        ref = orc.index_scores_fp4(qI[b, 0].float().numpy(), w[b, 0].numpy(), kp[b], ks[b])
        np.testing.assert_array_equal(sc[b, 0], ref)
        np.testing.assert_array_equal(idx[b, 0], orc.topk(ref.astype(np.float32), k))


@pytest.mark.parametrize("B,Q,Nc", [(2, 9, 1000), (3, 40, 130)])
def test_index_fp4_causal_groups(L, orc, B, Q, Nc):
    """FP4 index over several queries per request with causal availability: query groups
    change often (the per-group scale factors), tiles past a query's available entries are
    skipped by every role of the kernel alike, the last tile is ragged, and one query has no
    available entry.  Scores of the available entries and the selection bit-exact."""
    H, k = 64, 64
    qI = randn(f"g.i4c.q{Q}", (B, Q, H, 128), dtype=torch.bfloat16)
    w = randn(f"g.i4c.w{Q}", (B, Q, H), std=1 / 8)
    planes, kp, ks = _fp4_keys(L, orc, f"g.i4c.k{Q}", B, Nc)
    q_pos = (torch.arange(Q, dtype=torch.int64) * (4 * Nc // Q + 9) - 1).reshape(1, Q).repeat(B, 1)
    q_pos[:, 0] = 0                                   # n_avail = 0
    q_pos[B - 1] += 6
    idx, sc = L.csa_index_topk(qI.to(DEV), w.to(DEV), planes, k, q_pos=q_pos.to(DEV), m=4, N_c=Nc,
                               kI_dtype=L.FP4, want_scores=True)
    idx, sc = idx.cpu().numpy(), sc.float().cpu().numpy()
    for b in range(B):
        for q in range(Q):
            n = orc.n_avail(int(q_pos[b, q]), 4, Nc)
            ref = orc.index_scores_fp4(qI[b, q].float().numpy(), w[b, q].numpy(), kp[b, :n], ks[b, :n])
            np.testing.assert_array_equal(sc[b, q, :n], ref, err_msg=f"b {b} q {q}")
            np.testing.assert_array_equal(idx[b, q], orc.topk(ref.astype(np.float32), k), err_msg=f"b {b} q {q}")


def test_decode_fused_mixed_precision(L, orc):
    """The 1M-context config's formats at a small size: FP8 KV with bf16 RoPE dims,
    FP4 index keys, bf16 scores, k = 1024."""
    B, H, D, dv, Nc, k, Tw = 2, 64, 576, 512, 3000, 1024, 128
    from long_context_sparse_06_b200 import synth
    scale = 1 / math.sqrt(576)
    q = randn("g.c5.q", (B, H, D), dtype=torch.bfloat16)
    comp32 = synth.with_outliers("g.c5.c", synth.normal("g.c5.c", (B, Nc, D))).astype(np.float32)
    win32 = synth.with_outliers("g.c5.w", synth.normal("g.c5.w", (B, Tw, D))).astype(np.float32)
    comp_g = L.lcs_quant_kv_fp8(torch.from_numpy(comp32).to(DEV))
    win_g = L.lcs_quant_kv_fp8(torch.from_numpy(win32).to(DEV))
    qI = randn("g.c5.qi", (B, 64, 128), dtype=torch.bfloat16)
    w = randn("g.c5.wi", (B, 64), std=1 / 8)
    planes, kp, ks = _fp4_keys(L, orc, "g.c5.k", B, Nc)
    idx_out = torch.empty((B, k), dtype=torch.int32, device=DEV)
    out = both_outputs(lambda od: L.decode_fused(L.MODE_CSA, q.to(DEV), comp_g, win_g, dv, scale, kv_dtype=L.KV_FP8,
                                                 qI=qI.to(DEV), w=w.to(DEV), kI=planes, kI_dtype=L.FP4, k=k,
                                                 idx_out=idx_out, out_dtype=od)).cpu().numpy()
    idx = idx_out.cpu().numpy()
    comp_d = orc.dequant_kv_fp8(orc.quant_kv_fp8(comp32))
    win_d = orc.dequant_kv_fp8(orc.quant_kv_fp8(win32))
    for b in range(B):
        ref_s = orc.index_scores_fp4(qI[b].float().numpy(), w[b].numpy(), kp[b], ks[b])
        np.testing.assert_array_equal(idx[b], orc.topk(ref_s.astype(np.float32), k))
        o, _ = orc.csa_attend(q[b].double().numpy(), comp_d[b], idx[b], win_d[b], 0, -1, 128, dv, scale)
        assert_close_rel_rms(out[b], o, 2e-2, f"mixed-precision b {b}")
