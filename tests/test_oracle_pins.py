"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties an oracle function to a published format table, a library routine
(torch / numpy / scipy / Python's exact rationals), a closed form, an invariant
or brute force on tiny inputs -- chosen so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from long_context_sparse_06_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def round_fraction_f32(fr: Fraction) -> float:
    """Correctly rounded (nearest, ties to even) fp32 value of an exact rational."""
    if fr == 0:
        return 0.0
    f = np.float32(float(fr))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    def key(c):
        return (abs(Fraction(float(c)) - fr), int(np.array(c, np.float32).view(np.uint32)) & 1)
    return float(min(cands, key=key))


# ----------------------------------------------------------------- formats
def test_bf16_rounding_matches_torch(orc):
    x = synth.normal("pin.bf16", 20000) * np.exp(synth.normal("pin.bf16.e", 20000) * 4)
    x32 = x.astype(np.float32)
    # exact ties: bf16 values plus half an ulp
    b = torch.from_numpy(x32[:2000]).to(torch.bfloat16).float().numpy().astype(np.float64)
    half_ulp = 2.0 ** np.floor(np.log2(np.abs(b))) * 2.0 ** -8     # b != 0 for these draws
    ties = (b + half_ulp).astype(np.float32)
    allx = np.concatenate([x32, ties])
    ref = torch.from_numpy(allx).to(torch.bfloat16).float().numpy().astype(np.float64)
    got = orc.round_bf16(allx.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_e4m3_decode_matches_published_table_and_torch(orc):
    g = _gold("ofp_formats.json")
    codes = np.arange(256, dtype=np.uint8)
    dec = orc.e4m3_decode(codes)
    tor = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    nan = np.isnan(dec)
    assert sorted(np.nonzero(nan)[0].tolist()) == g["e4m3_nan_codes"]
    np.testing.assert_array_equal(np.isnan(tor), nan)
    np.testing.assert_array_equal(dec[~nan], tor[~nan])
    assert np.nanmax(dec) == g["e4m3_max_normal"]
    assert dec[8] == g["e4m3_min_normal"] and dec[1] == g["e4m3_min_subnormal"]
    # encode is the inverse of decode on every finite code
    fin = codes[~nan]
    np.testing.assert_array_equal(orc.e4m3_encode(dec[~nan]), fin)


def test_e4m3_rounding_matches_torch_in_range(orc):
    x = synth.normal("pin.e4m3", 30000) * np.exp(synth.normal("pin.e4m3.e", 30000) * 2.5)
    x = x[np.abs(x) < 460].astype(np.float32)
    # every exact midpoint between neighbouring E4M3 values
    vals = np.unique(orc.e4m3_decode(np.arange(0, 127, dtype=np.uint8)))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    allx = np.concatenate([x, mids, -mids])
    ref = torch.from_numpy(allx).to(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = orc.round_to(allx.astype(np.float64), orc.FMT_E4M3)
    np.testing.assert_array_equal(got, ref)
    # saturation (torch's cast is not saturating, so check separately)
    assert orc.round_to(np.array([500.0, -1e6, 464.0, 479.0]), orc.FMT_E4M3).tolist() == [448, -448, 448, 448]


def test_e2m1_table_and_rounding(orc):
    g = _gold("ofp_formats.json")
    codes = np.arange(16, dtype=np.uint8)
    dec = orc.e2m1_decode(codes)
    np.testing.assert_array_equal(dec, np.array(g["e2m1_values_by_code"]))
    np.testing.assert_array_equal(np.signbit(dec), np.signbit(np.array(g["e2m1_values_by_code"])))
    np.testing.assert_array_equal(orc.e2m1_encode(dec), codes)
    # midpoints go to the value with an even code (last mantissa bit 0)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    exp = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    assert orc.round_to(np.array(mids), orc.FMT_E2M1).tolist() == exp
    assert orc.round_to(-np.array(mids), orc.FMT_E2M1).tolist() == [-e for e in exp]
    assert orc.round_to(np.array([7.0, 100.0, -9.0]), orc.FMT_E2M1).tolist() == [6.0, 6.0, -6.0]
    # brute force: nearest of the 8 magnitudes, ties to even code
    mags = np.array(g["e2m1_values_by_code"][:8])
    for v in np.linspace(0, 8, 321):
        d = np.abs(mags - v)
        best = [i for i in range(8) if d[i] == d.min()]
        pick = [i for i in best if i % 2 == 0][0] if len(best) > 1 else best[0]
        assert orc.round_to(np.array([v]), orc.FMT_E2M1)[0] == mags[pick]


def test_fp4_to_fp8_is_exact_under_power_of_two_scales(orc):
    """"DeepSeek V4 深度解析" §4: FP4 -> FP8 is lossless because FP8 has two more
    exponent bits, as long as a block's range stays under a threshold.  With a
    power-of-two scale 2^e every E2M1 value times 2^e is an E4M3 value whenever
    the block's largest magnitude (6*2^e) is <= 448 and its finest step (0.5*2^e)
    is >= the E4M3 subnormal step 2^-9; and E2M1 x any E4M3 scale is exact in fp32."""
    e2 = orc.e2m1_decode(np.arange(16, dtype=np.uint8))
    e4 = orc.e4m3_decode(np.arange(256, dtype=np.uint8))
    e4 = e4[np.isfinite(e4)]
    prod = np.outer(e2, e4).ravel()
    np.testing.assert_array_equal(prod.astype(np.float32).astype(np.float64), prod)
    for e in range(-12, 8):
        blk = e2 * 2.0 ** e
        exact = np.array_equal(orc.round_to(blk, orc.FMT_E4M3), blk)
        cond = 6 * 2.0 ** e <= 448 and 0.5 * 2.0 ** e >= 2.0 ** -9
        assert exact == cond, e


def test_kv_fp8_quantiser(orc):
    x = synth.with_outliers("pin.kv8", synth.normal("pin.kv8", (64, 576))).astype(np.float32)
    rows = orc.quant_kv_fp8(x)
    assert rows.shape == (64, 656)
    deq = orc.dequant_kv_fp8(rows)
    # RoPE dims: bf16 of the value (torch's conversion)
    ref_r = torch.from_numpy(x[:, 512:]).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(deq[:, 512:], ref_r)
    sc = rows[:, 576 + 64:].copy().view(np.float32)          # [64, 4]
    for b in range(4):
        blk = x[:, b * 128:(b + 1) * 128].astype(np.float64)
        amax = np.abs(blk).max(axis=1)
        t = amax.astype(np.float32) / np.float32(448)
        # the scale is the smallest power of two >= amax/448
        assert np.all(np.log2(sc[:, b]) == np.round(np.log2(sc[:, b])))
        assert np.all(sc[:, b] >= t) and np.all(sc[:, b] / 2 < t)
        # every stored value is exactly a bf16 value (widening to bf16 is exact)
        blkq = deq[:, b * 128:(b + 1) * 128]
        np.testing.assert_array_equal(torch.from_numpy(blkq.astype(np.float32)).to(torch.bfloat16).double().numpy(),
                                      blkq)
        codes = rows[:, b * 128:(b + 1) * 128]
        assert np.all(np.abs(orc.e4m3_decode(codes & 0x7F)).max(axis=1) * sc[:, b] >= amax * (1 - 2.0 ** -4))
        err = np.abs(deq[:, b * 128:(b + 1) * 128] - blk)
        assert np.all(err <= (2.0 ** -4) * np.abs(blk) + 2.0 ** -10 * sc[:, b:b + 1] + 1e-12)


def test_fp4_quantiser(orc):
    x = synth.normal("pin.fp4", (200, 128)).astype(np.float32)
    p, s = orc.quant_fp4(x)
    assert p.shape == (200, 64) and s.shape == (200, 4)
    deq = orc.dequant_fp4(p, s)
    sc = orc.e4m3_decode(s)
    for b in range(4):
        blk = x[:, b * 32:(b + 1) * 32].astype(np.float64)
        amax = np.abs(blk).max(axis=1)
        exp_sc = orc.round_to((amax.astype(np.float32) / np.float32(6)).astype(np.float64), orc.FMT_E4M3)
        np.testing.assert_array_equal(sc[:, b], np.where(exp_sc == 0, 1.0, exp_sc))
        q = deq[:, b * 32:(b + 1) * 32] / sc[:, b:b + 1]
        # codes are the E2M1 rounding of x/scale (x/scale in fp32)
        t = (blk.astype(np.float32) / sc[:, b:b + 1].astype(np.float32)).astype(np.float64)
        np.testing.assert_array_equal(q, orc.round_to(t, orc.FMT_E2M1))
    # packing: element 2j in the low nibble
    np.testing.assert_array_equal(orc.e2m1_decode(p[:, :1] & 15)[:, 0] * sc[:, 0], deq[:, 0])
    np.testing.assert_array_equal(orc.e2m1_decode(p[:, :1] >> 4)[:, 0] * sc[:, 0], deq[:, 1])


# --------------------------------------------------------------------- RoPE
def test_rope_against_complex_rotation(orc):
    d, dr = 64, 16
    x = synth.normal("pin.rope", (10, d))
    pos = np.arange(10) * 977 + 3
    got = orc.rope(x, pos, dr)
    np.testing.assert_array_equal(got[:, :d - dr], x[:, :d - dr])
    h = dr // 2
    z = x[:, d - dr:d - h] + 1j * x[:, d - h:]
    freq = 10000.0 ** (-np.arange(h) * 2.0 / dr)
    zr = z * np.exp(1j * pos[:, None] * freq[None, :])
    np.testing.assert_allclose(got[:, d - dr:d - h], zr.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[:, d - h:], zr.imag, rtol=0, atol=1e-12)
    # pair 0 has frequency 1: the unit vector turns by exactly pos radians
    e = np.zeros((1, d)); e[0, d - dr] = 1.0
    r = orc.rope(e, [1], dr)
    assert r[0, d - dr] == pytest.approx(math.cos(1.0), abs=1e-15)
    assert r[0, d - h] == pytest.approx(math.sin(1.0), abs=1e-15)
    np.testing.assert_array_equal(orc.rope(x, 0, dr), x)


def test_rope_relative_position(orc):
    d, dr = 32, 32
    a, b = synth.normal("pin.rope.a", d), synth.normal("pin.rope.b", d)
    def dot(pa, pb):
        return float(orc.rope(a[None], [pa], dr)[0] @ orc.rope(b[None], [pb], dr)[0])
    assert dot(5, 2) == pytest.approx(dot(1005, 1002), abs=1e-9)
    assert dot(5, 2) != pytest.approx(dot(5, 3), abs=1e-6)


# --------------------------------------------------------------- compressor
def test_compress_m1_identity(orc):
    x = synth.normal("pin.c.id", (40, 8))
    z = synth.normal("pin.c.idz", 40)
    e, pw = orc.compress(x, z, np.array([0.3]), m=1, overlap=0)
    np.testing.assert_array_equal(e, x)
    np.testing.assert_array_equal(pw, np.ones((40, 1)))


def test_compress_one_hot_selects_the_token(orc):
    x = synth.normal("pin.c.oh", (64, 8))
    z = synth.normal("pin.c.ohz", 64)
    for pos in range(6):
        bias = np.full(6, -1e4); bias[pos] = 0.0
        e, _ = orc.compress(x, z, bias, m=4, overlap=2)
        for j in range(16):
            t = 4 * j - 2 + pos
            if t >= 0:
                np.testing.assert_array_equal(e[j], x[t])


def test_compress_one_hot_logit_selects_its_token(orc):
    """The pooling logit of token t weights token t ("DeepSeek V4 深度解析" §2, CSA step 1:
    one learned weight per raw token).  With zero bias and one token's logit far above the
    rest, every entry whose window holds that token is exactly that token's row, and every
    other entry is the plain mean of its window.  Reading the logit of a neighbouring token
    (either direction) or a window shifted by one fails here."""
    T, d = 64, 8
    x = synth.normal("pin.c.zoh", (T, d))
    for m, ov in ((4, 2), (4, 0), (8, 3)):
        W = m + ov
        for hot in (0, 1, 5, 6, 30, 33, T - 1):
            z = np.zeros(T)
            z[hot] = 1e4                       # exp(-1e4) underflows to 0 in double
            e, pw = orc.compress(x, z, np.zeros(W), m=m, overlap=ov)
            for j in range(T // m):
                lo = m * j - ov
                ts = [t for t in range(lo, lo + W) if 0 <= t < T]
                if hot in ts:
                    np.testing.assert_array_equal(e[j], x[hot], err_msg=f"m={m} ov={ov} hot={hot} j={j}")
                    assert pw[j, hot - lo] == 1.0
                else:
                    np.testing.assert_allclose(e[j], x[ts].mean(axis=0), rtol=0, atol=1e-14)


def test_compress_weights_sum_to_one_and_mean(orc):
    x = synth.normal("pin.c.s", (256, 16))
    z = 3 * synth.normal("pin.c.sz", 256)
    b = synth.normal("pin.c.sb", 6)
    _, pw = orc.compress(x, z, b, m=4, overlap=2)
    assert np.all(np.abs(pw.sum(axis=1) - 1.0) <= 6 * 2.0 ** -52)
    assert np.all(pw >= 0)
    # first entry: the two positions before the sequence are left out
    assert pw[0, 0] == 0 and pw[0, 1] == 0
    # equal logits, zero bias: the plain mean of the window
    e, _ = orc.compress(x, np.full(256, 0.7), np.zeros(6), m=4, overlap=2)
    for j in range(1, 64):
        np.testing.assert_allclose(e[j], np.mean(x[4 * j - 2:4 * j + 4], axis=0), rtol=0, atol=1e-14)
    np.testing.assert_allclose(e[0], np.mean(x[0:4], axis=0), rtol=0, atol=1e-14)
    e128, _ = orc.compress(x, np.zeros(256), np.zeros(128), m=128, overlap=0)
    np.testing.assert_allclose(e128, x.reshape(2, 128, 16).mean(axis=1), rtol=0, atol=1e-14)


def test_compress_chunked_equals_whole(orc):
    """Compressing a chunk with its overlap tail equals compressing the whole sequence."""
    x = synth.normal("pin.c.ch", (128, 12))
    z = synth.normal("pin.c.chz", 128)
    b = synth.normal("pin.c.chb", 6)
    whole, _ = orc.compress(x, z, b, m=4, overlap=2, d_rope=4, pos0=1000)
    part, _ = orc.compress(x[64:], z[64:], b, m=4, overlap=2, d_rope=4, pos0=1064,
                           x_tail=x[62:64], z_tail=z[62:64])
    np.testing.assert_allclose(part, whole[16:], rtol=0, atol=1e-13)


def test_compress_is_causal_and_rope_at_last_token(orc):
    x = synth.normal("pin.c.ca", (64, 12))
    z = synth.normal("pin.c.caz", 64)
    b = synth.normal("pin.c.cab", 6)
    e, _ = orc.compress(x, z, b, m=4, overlap=2)
    x2 = x.copy(); x2[40:] += 100.0
    z2 = z.copy(); z2[40:] -= 50.0
    e2, _ = orc.compress(x2, z2, b, m=4, overlap=2)
    np.testing.assert_array_equal(e[:10], e2[:10])          # entries 0..9 end at token 39
    assert not np.allclose(e[10], e2[10])
    er, _ = orc.compress(x, z, b, m=4, overlap=2, d_rope=4, pos0=7)
    np.testing.assert_allclose(er, orc.rope(e, 7 + 4 * np.arange(16) + 3, 4), rtol=0, atol=1e-13)


# ------------------------------------------------------------------ indexer
def test_exact_dot_against_rationals(orc):
    rng_vals = []
    for i in range(300):
        n = 128 if i % 3 else 7
        a = synth.normal(f"pin.dot.a{i}", n)
        b = synth.normal(f"pin.dot.b{i}", n)
        if i % 2:   # wide exponent spread forces the big-integer path
            a = a * np.exp2(np.round(synth.normal(f"pin.dot.e{i}", n) * 30))
        a = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).double().numpy()
        b = torch.from_numpy(b.astype(np.float32)).to(torch.bfloat16).double().numpy()
        exact = sum((Fraction(float(p)) * Fraction(float(q)) for p, q in zip(a, b)), Fraction(0))
        rng_vals.append((orc.exact_dot_f32(a, b), round_fraction_f32(exact)))
    for got, ref in rng_vals:
        assert got == ref
    # 1 + n*2^-24 with a cancelling pair of tiny terms (forces the big-integer path):
    # odd n is an exact tie and must go to the neighbour with an even significand
    tiny = 2.0 ** -100
    for n_lo in range(-7, 8):
        a = np.array([1.0, 2.0 ** -12, tiny, -tiny])
        b = np.array([1.0, n_lo * 2.0 ** -12, tiny, tiny])
        exact = Fraction(1) + Fraction(n_lo, 2 ** 24)
        assert orc.exact_dot_f32(a, b) == round_fraction_f32(exact)
    a = np.array([1.0, 2.0 ** -12, tiny, -tiny]); b = np.array([1.0, 2.0 ** -12, tiny, tiny])
    assert orc.exact_dot_f32(a, b) == 1.0
    b[1] = 3 * 2.0 ** -12
    assert orc.exact_dot_f32(a, b) == 1.0 + 2.0 ** -22


def test_index_f32_chain_against_fp64(orc):
    H, dI, N = 4, 32, 300
    qI = synth.normal("pin.i.q", (H, dI)).astype(np.float32)
    w = synth.normal("pin.i.w", H, std=0.5).astype(np.float32)
    kI = synth.normal("pin.i.k", (N, dI)).astype(np.float32)
    s = orc.index_scores_f32(qI, w, kI)
    dots = kI.astype(np.float64) @ qI.astype(np.float64).T            # [N, H]
    ref = np.maximum(dots, 0) @ w.astype(np.float64)
    bound = (np.abs(kI).astype(np.float64) @ np.abs(qI).astype(np.float64).T) @ np.abs(w) * (dI + H + 2) * 2.0 ** -24
    assert np.all(np.abs(s - ref) <= bound)
    # a head with w_h = 0 and a head with all-negative dots contribute nothing
    w2 = w.copy(); w2[1] = 0
    s2 = orc.index_scores_f32(qI, w2, kI)
    ref2 = np.maximum(dots, 0) @ w2.astype(np.float64)
    assert np.all(np.abs(s2 - ref2) <= bound)


def test_index_bf16_against_fp64(orc):
    H, dI, N = 8, 128, 200
    qI = synth.bf16_tensor(synth.normal("pin.ib.q", (H, dI))).double().numpy()
    kI = synth.bf16_tensor(synth.normal("pin.ib.k", (N, dI))).double().numpy()
    w = synth.normal("pin.ib.w", H, std=0.125).astype(np.float32)
    s = orc.index_scores_bf16(qI, w, kI)
    dots = kI @ qI.T
    np.testing.assert_array_equal(orc.round_to(dots, orc.FMT_F32)[:5, 0],
                                  [orc.exact_dot_f32(qI[0], kI[i]) for i in range(5)])
    ref = np.maximum(dots, 0) @ w.astype(np.float64)
    bound = np.maximum(dots, 0) @ np.abs(w) * (H + 2) * 2.0 ** -23 + 1e-30
    assert np.all(np.abs(s - ref) <= bound)


def test_index_fp4_against_dequantised_fp64(orc):
    H, dI, N = 16, 128, 300
    qI = synth.bf16_tensor(synth.normal("pin.i4.q", (H, dI))).float().numpy()
    w = synth.normal("pin.i4.w", H, std=0.25).astype(np.float32)
    kraw = synth.with_outliers("pin.i4.k", synth.normal("pin.i4.k", (N, dI))).astype(np.float32)
    kp, ks = orc.quant_fp4(kraw)
    s = orc.index_scores_fp4(qI, w, kp, ks)
    qp, qs = orc.quant_fp4(qI)
    dots = orc.dequant_fp4(kp, ks) @ orc.dequant_fp4(qp, qs).T
    ref = np.maximum(dots, 0) @ w.astype(np.float64)
    # fp32 chain error plus one bf16 rounding
    bound = np.maximum(np.abs(dots), 0) @ np.abs(w) * (H + 6) * 2.0 ** -23 + np.abs(ref) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(s - ref) <= bound)
    np.testing.assert_array_equal(orc.round_bf16(s), s)
    # the fp32 sum before the bf16 rounding: the fp32 chain error alone
    s32 = orc.index_scores_fp4(qI, w, kp, ks, round_bf16=False)
    bound32 = np.maximum(np.abs(dots), 0) @ np.abs(w) * (H + 6) * 2.0 ** -23 + 1e-30
    assert np.all(np.abs(s32 - ref) <= bound32)
    np.testing.assert_array_equal(s32.astype(np.float32).astype(np.float64), s32)
    np.testing.assert_array_equal(orc.round_bf16(s32), s)
    # the block dots are exact multiples of 1/4 (checked through a one-block key)
    one = np.zeros((1, dI), np.float32); one[0, :32] = kraw[0, :32]
    p1, s1 = orc.quant_fp4(one)
    blk = (orc.dequant_fp4(p1, s1)[0, :32] / orc.e4m3_decode(s1[0, 0])) @ \
          (orc.dequant_fp4(qp, qs)[0, :32] / orc.e4m3_decode(qs[0, 0]))
    assert blk * 4 == round(blk * 4)


# -------------------------------------------------------------------- top-k
def _brute_topk(s, k):
    order = sorted(range(len(s)), key=lambda i: (-float(s[i]), i))[:k]
    return sorted(order) + [-1] * (k - min(k, len(s)))


def test_topk_brute_force_small(orc):
    for n in range(0, 7):
        for vals in itertools.product([-1.0, 0.0, 2.0], repeat=n):
            s = np.array(vals, np.float32)
            for k in range(0, 8):
                assert orc.topk(s, k).tolist() == _brute_topk(s, k)


def test_topk_random_with_ties(orc):
    for i in range(50):
        n = 1 + (i * 37) % 300
        s = np.round(synth.normal(f"pin.tk{i}", n) * 3).astype(np.float32)
        for k in (1, 7, 64, n, n + 5):
            assert orc.topk(s, k).tolist() == _brute_topk(s, k)
    s = np.array([0.0, -0.0, 0.0, -0.0], np.float32)
    assert orc.topk(s, 2).tolist() == [0, 1]
    s = np.array([-np.inf, 1.0, np.inf, -np.inf], np.float32)
    assert orc.topk(s, 3).tolist() == [0, 1, 2]


# ---------------------------------------------------------------- attention
def _sdpa(q, k, v, mask, scale):
    """torch's scaled_dot_product_attention in float64 (one batch, heads share K/V)."""
    qt = torch.from_numpy(q)[None]                      # [1, H, D]
    kt = torch.from_numpy(k)[None, None].expand(1, q.shape[0], *k.shape)
    vt = torch.from_numpy(v)[None, None].expand(1, q.shape[0], *v.shape)
    m = torch.from_numpy(mask)[None, None] if mask is not None else None
    o = torch.nn.functional.scaled_dot_product_attention(qt[:, :, None, :], kt, vt, attn_mask=m, scale=scale)
    return o[0, :, 0, :].numpy()


def test_window_only_equals_sliding_window_attention(orc):
    T, H, D, dv, W = 300, 4, 24, 16, 128
    kv = synth.normal("pin.swa.kv", (T, D))
    q = synth.normal("pin.swa.q", (T, H, D))
    scale = 1 / math.sqrt(D)
    comp = synth.normal("pin.swa.c", (8, D))
    for t in (0, 5, 127, 128, 200, 299):
        idx = np.full(16, -1, np.int32)                    # k = 0 selected
        o, _ = orc.csa_attend(q[t], comp, idx, kv, 0, t, W, dv, scale)
        mask = np.array([t - W < p <= t for p in range(T)])
        ref = _sdpa(q[t], kv, kv[:, :dv], mask, scale)
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_full_selection_equals_dense(orc):
    Nc, H, D, dv, W, m = 50, 4, 24, 16, 128, 4
    comp = synth.normal("pin.fs.c", (Nc, D))
    win = synth.normal("pin.fs.w", (128, D))
    q = synth.normal("pin.fs.q", (H, D))
    t = 4 * Nc - 1 + 1000
    o_h, l_h = orc.hca_attend(q, comp, m, win, t - 127, -1, W, dv, 0.2)
    for k in (Nc, Nc + 30):
        idx = np.full(k, -1, np.int32); idx[:Nc] = np.arange(Nc)
        o_c, l_c = orc.csa_attend(q, comp, idx, win, t - 127, -1, W, dv, 0.2)
        np.testing.assert_allclose(o_c, o_h, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l_c, l_h, rtol=0, atol=1e-13)


def test_union_equals_lse_merge(orc):
    H, D, dv = 8, 40, 32
    q = synth.normal("pin.um.q", (H, D))
    a = synth.normal("pin.um.a", (17, D)) * 2
    b = synth.normal("pin.um.b", (9, D)) * 2
    o, l = orc.mqa_rows(q, np.concatenate([a, b]), 0.3, dv)
    oa, la = orc.mqa_rows(q, a, 0.3, dv)
    ob, lb = orc.mqa_rows(q, b, 0.3, dv)
    mx = np.maximum(la, lb)
    wa, wb = np.exp(la - mx), np.exp(lb - mx)
    np.testing.assert_allclose(o, (oa * wa[:, None] + ob * wb[:, None]) / (wa + wb)[:, None], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l, mx + np.log(wa + wb), rtol=0, atol=1e-13)


def test_hca_m1_without_window_is_causal_mqa(orc):
    T, H, D, dv = 40, 4, 16, 12
    kv = synth.normal("pin.h1.kv", (T, D))
    q = synth.normal("pin.h1.q", (T, H, D))
    empty = np.zeros((0, D))
    for t in range(T):
        o, _ = orc.hca_attend(q[t], kv, 1, empty, 0, t, 128, dv, 0.25)
        mask = np.arange(T) <= t
        np.testing.assert_allclose(o, _sdpa(q[t], kv, kv[:, :dv], mask, 0.25), rtol=0, atol=1e-12)


def test_attention_closed_forms(orc):
    D, dv = 8, 4
    q = synth.normal("pin.cf.q", (3, D))
    row = synth.normal("pin.cf.r", (1, D))
    o, l = orc.mqa_rows(q, np.repeat(row, 5, axis=0), 0.5, dv)
    np.testing.assert_allclose(o, np.repeat(row[:, :dv], 3, axis=0), rtol=0, atol=1e-15)
    np.testing.assert_allclose(l, 0.5 * (q @ row[0]) + math.log(5), rtol=0, atol=1e-13)
    r2 = synth.normal("pin.cf.r2", (2, D))
    o, _ = orc.mqa_rows(q, r2, 0.5, dv)
    p1 = 1 / (1 + np.exp(0.5 * (q @ r2[0] - q @ r2[1])))      # sigmoid weight of row 1
    np.testing.assert_allclose(o, (1 - p1)[:, None] * r2[0, :dv] + p1[:, None] * r2[1, :dv], rtol=0, atol=1e-14)


def test_attention_empty_row_set(orc):
    """No selected entry and no window row: the empty sum, o = 0 and lse = log 0 = -inf,
    whether the set is empty by selection (-1 padding) or by an empty window."""
    D, dv = 576, 512
    q = synth.normal("pin.em.q", (4, D))
    comp = synth.normal("pin.em.c", (10, D))
    none = np.full(8, -1, np.int32)
    o, l = orc.csa_attend(q, comp, none, np.zeros((0, D)), 0, -1, 128, dv, 0.1)
    np.testing.assert_array_equal(o, np.zeros((4, dv)))
    assert np.all(np.isneginf(l))
    win = synth.normal("pin.em.w", (6, D))                    # window rows all after the query
    o, l = orc.csa_attend(q, comp, none, win, 100, 50, 128, dv, 0.1)
    np.testing.assert_array_equal(o, np.zeros((4, dv)))
    assert np.all(np.isneginf(l))


@pytest.mark.parametrize("T", [300, 130])
def test_cache_stream_equals_whole_sequence(orc, T):
    """Tokens appended one at a time emit, as each entry completes, exactly the entries the
    whole-sequence compressor makes (CSA KV, CSA index keys, HCA KV); the state cache then
    holds the uncompressed tail and the last W rows after RoPE at their own positions; the
    compressed cache holds whole blocks of lcm(4, 128) = 128 raw tokens."""
    D, DI, dr, W = 64, 32, 16, 128
    x = synth.normal(f"pin.cs{T}.x", (T, D))
    kx = synth.normal(f"pin.cs{T}.k", (T, DI))
    z, zI, zh = (synth.normal(f"pin.cs{T}.{n}", T) for n in ("z", "zI", "zh"))
    bias, biasI = synth.normal("pin.cs.b", 6), synth.normal("pin.cs.bI", 6)
    biash = synth.normal("pin.cs.bh", 128)
    st = orc.CacheState(bias, biasI, biash, dr, W=W)
    n_csa = []
    for t in range(T):
        st.append(x[t], kx[t], z[t], zI[t], zh[t])
        n_csa.append(len(st.csa))
    assert n_csa == [(t + 1) // 4 for t in range(T)]               # emitted as soon as complete
    csa, _ = orc.compress(x[:T // 4 * 4], z[:T // 4 * 4], bias, 4, 2, dr)
    keys, _ = orc.compress(kx[:T // 4 * 4], zI[:T // 4 * 4], biasI, 4, 2, 0)
    nh = T // 128
    hca, _ = orc.compress(x[:nh * 128], zh[:nh * 128], biash, 128, 0, dr)
    np.testing.assert_array_equal(np.array(st.csa), csa)
    np.testing.assert_array_equal(np.array(st.csa_keys), keys)
    np.testing.assert_array_equal(np.array(st.hca).reshape(nh, D), hca)
    pos = [p_ for p_, _ in st.window]
    assert pos == list(range(max(0, T - W), T))
    np.testing.assert_array_equal(np.array([r for _, r in st.window]),
                                  orc.rope(x[max(0, T - W):], np.arange(max(0, T - W), T), dr))
    keep = max(2 + T % 4, T % 128)
    assert len(st.raw) == keep
    np.testing.assert_array_equal(np.array(st.raw), x[T - keep:])
    assert st.blocks() == T // 128 and len(st.hca) == st.blocks() and len(st.csa) >= 32 * st.blocks()


def test_group_oproj_equals_block_diagonal(orc):
    from scipy.linalg import block_diag
    H, dv, G, dg, hidden = 8, 48, 2, 64, 256
    o = synth.normal("pin.gp.o", (H, dv))
    Wg = synth.normal("pin.gp.g", (G, H // G * dv, dg))
    Wo = synth.normal("pin.gp.w", (G * dg, hidden))
    y = orc.group_oproj(o, Wg, Wo)
    ref = o.reshape(-1) @ block_diag(*Wg) @ Wo
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-10)


def test_oracle_reentrant_under_threads(orc):
    """Tests and the CPU baseline run the oracle on several threads at once: concurrent
    top-k and score calls return exactly what sequential ones do."""
    from concurrent.futures import ThreadPoolExecutor
    rows = [synth.normal(f"pin.mt.{i}", 20000).astype(np.float32) for i in range(24)]
    ref = [orc.topk(r, 300) for r in rows]
    with ThreadPoolExecutor(8) as ex:
        got = list(ex.map(lambda r: orc.topk(r, 300), rows * 3))
    for i, g in enumerate(got):
        np.testing.assert_array_equal(g, ref[i % len(rows)])
    q = synth.normal("pin.mt.q", (4, 32)).astype(np.float32)
    w = synth.normal("pin.mt.w", 4).astype(np.float32)
    ks = [synth.normal(f"pin.mt.k{i}", (500, 32)).astype(np.float32) for i in range(8)]
    ref_s = [orc.index_scores_f32(q, w, k) for k in ks]
    with ThreadPoolExecutor(8) as ex:
        got_s = list(ex.map(lambda k: orc.index_scores_f32(q, w, k), ks * 3))
    for i, g in enumerate(got_s):
        np.testing.assert_array_equal(g, ref_s[i % len(ks)])


def test_project_f32_against_fp64_and_exact_integers(orc):
    """The fp32 projection: within the fp32 chain's error bound of the fp64 product, exact when
    every product and partial sum is representable, and each output a chain in input order
    (a reordered sum would round differently on the cancelling case)."""
    h = synth.normal("pin.pj.h", (40, 256)).astype(np.float32)
    W = (synth.normal("pin.pj.w", (256, 36)) / 16).astype(np.float32)
    got = orc.project_f32(h, W)
    ref = h.astype(np.float64) @ W.astype(np.float64)
    bound = 256 * 2.0 ** -24 * (np.abs(h).astype(np.float64) @ np.abs(W).astype(np.float64))
    assert np.all(np.abs(got - ref) <= bound)
    hi = np.round(synth.normal("pin.pj.hi", (12, 64)) * 8).astype(np.float32)
    Wi = np.round(synth.normal("pin.pj.wi", (64, 5)) * 8).astype(np.float32)
    np.testing.assert_array_equal(orc.project_f32(hi, Wi), (hi.astype(np.float64) @ Wi.astype(np.float64)))
    # order: 1 + 2^-24 + 2^-24 - 1 in sequence is 0 (each 2^-24 is lost against 1), not 2^-23
    hc = np.array([[1.0, 2.0 ** -24, 2.0 ** -24, -1.0]], np.float32)
    Wc = np.ones((4, 1), np.float32)
    assert orc.project_f32(hc, Wc)[0, 0] == 0.0
    assert orc.project_f32(hc[:, ::-1].copy(), Wc)[0, 0] == 2.0 ** -23
