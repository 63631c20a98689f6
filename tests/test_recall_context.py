"""Recall of the BF16-score top-k against the fp32-score top-k (context only).

"V3 vs V4" page, section on why FP4 is lossless: the index scores drop to BF16, which
makes the top-k twice as fast, and the pages report the KV recall staying at 99.7 %.  On
the 1M-context mixed-precision decode shape (262144 FP4 index keys with an E4M3 scale
per 32, 64 index heads of 128 dims, k = 1024; values N(0,1) with 1 % of elements x20
before quantisation) this computes, with the oracle, the share of the entries selected
from the fp32 scores that the BF16 scores also select.  Synthetic inputs need not match
the pages' number; the test prints it and checks only what must hold.

By default it runs 65536 entries with k = 256 (the same selected share, 1/256, in about
20 s of oracle time); LCS_RECALL_FULL=1 runs the full 262144 entries with k = 1024.
"""
import os

import numpy as np

from long_context_sparse_06_b200 import synth


def test_bf16_score_topk_recall_mixed_1m_shape(orc):
    H, dI = 64, 128
    N, k = (262144, 1024) if os.environ.get("LCS_RECALL_FULL") == "1" else (65536, 256)
    qI = synth.bf16_tensor(synth.with_outliers("rc.q", synth.normal("rc.q", (H, dI)))).float().numpy()
    w = synth.normal("rc.w", H, std=1.0 / 8).astype(np.float32)
    kraw = synth.with_outliers("rc.k", synth.normal("rc.k", (N, dI))).astype(np.float32)
    kp, ks = orc.quant_fp4(kraw)
    s32 = orc.index_scores_fp4(qI, w, kp, ks, round_bf16=False)
    s16 = orc.round_bf16(s32)
    sel32 = set(orc.topk(s32, k).tolist())
    sel16 = set(orc.topk(s16, k).tolist())
    recall = len(sel32 & sel16) / k
    ties = int(np.sum(s16 == np.sort(s16)[-k]))
    print(f"\nBF16-score top-{k} recall vs fp32 scores over {N} entries: {recall:.4f} "
          f"({ties} entries share the k-th BF16 score)")
    assert len(sel32) == len(sel16) == k
    assert 0.0 < recall <= 1.0
