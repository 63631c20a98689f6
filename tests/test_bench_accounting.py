"""The roofline numerators bench.py uses, against the algorithmic work of each workload
written out from its shapes (no device needed: the accounting is plain arithmetic).

Decode: per request, the index keys streamed once, the selected and window rows gathered
once, q / qI / w read, the output written.  Prefill: 2 FLOPs per multiply-add of the
indexer over every causal (query, entry) pair, plus the attention over k + W rows per
query.  Compressor: raw rows and logits read once, entries written once.
"""
import bench

H, D, DV, HI, DI, TW = 64, 576, 512, 64, 128, 128


def _decode(cls, row):
    wl = cls(None, "cpu", 0)
    wl.row = row
    return wl


def test_csa_decode_bytes():
    q_in = H * D * 2 + HI * DI * 2 + HI * 4                    # q bf16, qI bf16, w fp32: 90,368 B
    out = H * DV * 2                                           # 65,536 B
    keys = 32768 * DI * 2                                      # 8,388,608 B
    rows = (512 + TW) * D * 2                                  # 737,280 B
    wl = _decode(bench.CsaDecode, D * 2)
    assert keys + rows + q_in + out == 9_281_792
    assert wl.alg_bytes_per_step() == 32 * 9_281_792           # 297.0 MB per step
    assert wl.dominant_bytes() == 32 * (keys + HI * DI * 2 + HI * 4)


def test_mixed_decode_bytes():
    keys = 262144 * (DI // 2 + DI // 32)                        # FP4 codes + E4M3 scales: 17,825,792 B
    rows = (1024 + TW) * 656                                   # FP8 rows
    wl = _decode(bench.CsaDecodeMixed, 656)
    per = keys + rows + H * D * 2 + HI * DI * 2 + HI * 4 + H * DV * 2
    assert per == 18_737_408
    assert wl.alg_bytes_per_step() == 4 * per                  # 74.9 MB per step


def test_hca_decode_bytes():
    wl = bench.HcaDecode(None, "cpu", 0)
    per = (8192 + TW) * D * 2 + H * D * 2 + H * DV * 2
    assert per == 9_723_904
    assert wl.alg_bytes_per_step() == 16 * per                 # 155.6 MB per step
    fp8 = bench.HcaDecodeFp8(None, "cpu", 0)
    assert fp8.alg_bytes_per_step() == 16 * ((8192 + TW) * 656 + H * D * 2 + H * DV * 2)


def test_prefill_flops():
    wl = bench.CsaPrefill(None, "cpu", 0)
    wl.NC = (wl.P0 + wl.Q) // 4
    pairs = sum(min(wl.NC, (wl.P0 + i + 1) // 4) for i in range(wl.Q))
    assert pairs == 276_822_016
    assert wl.dominant_flops() == pairs * HI * DI * 2          # 4.535 TFLOP
    assert wl.alg_flops_per_step() == pairs * HI * DI * 2 + wl.Q * (1024 + TW) * H * (D + DV) * 2   # 5.850 TFLOP


def test_compress_stream_bytes():
    wl = bench.CompressStream(None, "cpu", 0)
    T = 1 << 20
    csa_kv = T * D * 2 + T * 4 + (T // 4) * D * 2              # rows + logits read, entries written
    csa_keys = T * DI * 2 + T * 4 + (T // 4) * DI * 2
    hca = T * D * 2 + T * 4 + (T // 128) * D * 2
    assert wl.alg_bytes_per_step() == csa_kv + csa_keys + hca
    assert wl.dominant_bytes() == csa_kv


def test_c1_attention_flops():
    """C1: QK (64 dims) and PV (48 dims) over each query's selected entries (up to 64 of
    its complete ones) and its causal window (up to 128 rows), 8 heads."""
    wl = bench.C1Prefill(None, "cpu", 0)
    sel = sum(min(64, (t + 1) // 4) for t in range(1024))
    win = sum(min(128, t + 1) for t in range(1024))
    assert sel == 57_280                                       # the selected (query, entry) pairs
    assert wl.attend_flops() == (sel + win) * 8 * (64 + 48) * 2


def test_rows_generator_matches_whole_tensor():
    """The reference arm makes only the selected compressed rows; they equal the same rows
    of the whole seeded tensor the GPU arm makes."""
    import torch
    from long_context_sparse_06_b200 import synth
    full = synth.normal_t("acct.rows", (3, 40, 576), dtype=torch.bfloat16)
    idx = torch.tensor([0, 39, 40, 77, 119])
    got = synth.normal_rows_t("acct.rows", (120, 576), idx, dtype=torch.bfloat16)
    assert torch.equal(got, full.reshape(120, 576)[idx])
