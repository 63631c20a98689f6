#!/usr/bin/env python3
"""Benchmark of the CSA / HCA compressed-attention hot path on B200.

Default workload (the headline): CSA decode, bf16 -- 32 requests with a 128K-token
context each: 32768 compressed entries (m = 4) of dim 576 (512 content + 64 RoPE),
64 query heads sharing the KV, lightning indexer 64 heads x 128 over bf16 keys,
top-512, a 128-row raw window; N(0,1) values, query scale 1/sqrt(576).  One step
= one decode token for every request = index scoring -> top-k -> sparse MQA
(decode_fused), captured once as a CUDA graph and replayed.

Other workloads (`--workload`) measure the remaining rows of the path:
  hca_decode_bf16_1m     16 requests x 8192 entries (1M tokens, m' = 128), dense MQA
  csa_decode_mixed_1m    4 requests x 262144 entries, FP8 KV + bf16 RoPE dims,
                         FP4 index keys, bf16 scores, top-1024
  csa_prefill_bf16_8k    8192 new tokens after a 131072-token prefix: compress the
                         chunk's KV and index keys, causal index + top-1024, attention
  compress_stream_1m     1M raw rows x 576 bf16: CSA (m=4, overlap 2) and HCA
                         (m'=128) compression of the KV, CSA of 128-dim index keys

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
  python bench.py --stage index|topk|attend|compress ...   (one stage alone, for ncu)

N > 1 is launched with torchrun: every rank runs its own copy of the workload on
its own GPU (requests are independent: no collective on the data path); the step
time is the max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA decode tok/s and achieved HBM GB/s vs roofline at 128K-1M ctx"
D, DV, H, HI, DI, TW = 576, 512, 64, 64, 128, 128
SCALE = 1.0 / math.sqrt(576.0)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


KERNEL_FILES = {
    "index_bf16_tc_kernel": ["long_context_sparse_06_b200/csrc/indexer.cu",
                             "long_context_sparse_06_b200/csrc/lcs_common.cuh"],
    "index_fp4_tc_kernel": ["long_context_sparse_06_b200/csrc/indexer_fp4.cu",
                            "long_context_sparse_06_b200/csrc/lcs_common.cuh"],
    "attend_tc_kernel": ["long_context_sparse_06_b200/csrc/attend.cu",
                         "long_context_sparse_06_b200/csrc/lcs_common.cuh"],
    "compress_tma_kernel": ["long_context_sparse_06_b200/csrc/compress.cu",
                            "long_context_sparse_06_b200/csrc/lcs_common.cuh"],
}


def recorded_traffic(kernel, workload):
    """dram bytes per launch from a committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(f"{kernel}@{workload}")
    if not d or d.get("source_hash") != kernel_source_hash(KERNEL_FILES[kernel]):
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            pci = getattr(props, "pci_bus_id", None)
            if pci is not None:
                dom = getattr(props, "pci_domain_id", 0)
                dev_id = getattr(props, "pci_device_id", 0)
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{pci:02x}:{dev_id:02x}.0")
            else:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                idx = int(vis.split(",")[device_index]) if vis else device_index
                self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
        except Exception:
            self._h = None

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            self._stop.wait(0.005)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------- workloads
class Workload:
    """One configuration of the path: inputs, the step, stages and accounting."""
    name = ""
    unit = "tok/s"
    bound = "hbm"
    stage_names = ()

    def __init__(self, lcs, dev, rank):
        self.lcs, self.dev, self.rank = lcs, dev, rank

    def tag(self, s):
        return f"bench.{self.name}.r{self.rank}.{s}"

    def dominant_stage(self):
        return 0


class CsaDecode(Workload):
    """CSA decode: decode_fused(MODE_CSA) over B requests."""
    name = "csa_decode_bf16_128k"
    B, NC, K = 32, 32768, 512
    mixed = False
    stage_names = ("index", "topk", "attend")
    dominant = "index_bf16_tc_kernel"

    def config(self):
        return dict(workload=self.name, requests=self.B, context_tokens=self.NC * 4, compressed_entries=self.NC, m=4,
                    kv_dim=D, d_v=DV, heads=H, index_heads=HI, index_dim=DI, topk=self.K, window=TW,
                    kv_format="fp8-e4m3 (pow2 scale per 128) + bf16 rope" if self.mixed else "bf16",
                    index_key_format="fp4-e2m1 + e4m3 scale per 32" if self.mixed else "bf16",
                    score_format="bf16" if self.mixed else "fp32")

    def build(self):
        import torch
        from long_context_sparse_06_b200 import synth
        L, dev, bf = self.lcs, self.dev, torch.bfloat16
        B, NC = self.B, self.NC
        self.q = synth.normal_t(self.tag("q"), (B, H, D), dtype=bf, device=dev)
        self.qI = synth.normal_t(self.tag("qI"), (B, HI, DI), dtype=bf, device=dev)
        self.w = synth.normal_t(self.tag("w"), (B, HI), std=1.0 / 8, device=dev)
        if self.mixed:
            f32 = torch.float32
            comp = synth.with_outliers_t(self.tag("comp"), synth.normal_t(self.tag("comp"), (B, NC, D), dtype=f32,
                                                                            device=dev))
            self.comp = L.lcs_quant_kv_fp8(comp)
            del comp
            win = synth.with_outliers_t(self.tag("win"), synth.normal_t(self.tag("win"), (B, TW, D), dtype=f32,
                                                                          device=dev))
            self.win = L.lcs_quant_kv_fp8(win)
            kraw = synth.with_outliers_t(self.tag("kI"), synth.normal_t(self.tag("kI"), (B, NC, DI), dtype=f32,
                                                                          device=dev))
            self.kI = L.lcs_quant_fp4(kraw)
            del kraw
            self.kv_dtype, self.kI_dtype, self.score_dtype, self.row = L.KV_FP8, L.FP4, L.BF16, 656
        else:
            self.comp = synth.normal_t(self.tag("comp"), (B, NC, D), dtype=bf, device=dev)
            self.win = synth.normal_t(self.tag("win"), (B, TW, D), dtype=bf, device=dev)
            self.kI = synth.normal_t(self.tag("kI"), (B, NC, DI), dtype=bf, device=dev)
            self.kv_dtype, self.kI_dtype, self.score_dtype, self.row = L.BF16, L.BF16, L.F32, 2 * D
        self.out = torch.empty((B, H, DV), dtype=bf, device=dev)
        self.ws = L.workspace(L.lcs_workspace_size(L.OP_DECODE, B, 1, NC, TW, self.K, H, DV, self.score_dtype), dev)
        torch.cuda.synchronize()

    def step(self, stream):
        L = self.lcs
        L.decode_fused(L.MODE_CSA, self.q, self.comp, self.win, DV, SCALE, kv_dtype=self.kv_dtype, qI=self.qI,
                       w=self.w, kI=self.kI, kI_dtype=self.kI_dtype, k=self.K, score_dtype=self.score_dtype,
                       out=self.out, ws=self.ws, stream=stream)

    def stage(self, name, stream):
        """One stage alone (for profiling); index and top-k run as csa_index_topk."""
        L = self.lcs
        if name in ("index", "topk"):
            L.csa_index_topk(self.qI.view(self.B, 1, HI, DI), self.w.view(self.B, 1, HI), self.kI, self.K,
                             N_c=self.NC, kI_dtype=self.kI_dtype, score_dtype=self.score_dtype, stream=stream)
        elif name == "attend":
            if not hasattr(self, "idx"):
                import torch
                self.idx = L.csa_index_topk(self.qI.view(self.B, 1, HI, DI), self.w.view(self.B, 1, HI), self.kI,
                                            self.K, N_c=self.NC, kI_dtype=self.kI_dtype,
                                            score_dtype=self.score_dtype).contiguous()
                torch.cuda.synchronize()
            L.csa_attend(self.q.view(self.B, 1, H, D), self.comp, self.win, self.idx, DV, SCALE,
                         kv_dtype=self.kv_dtype, stream=stream)

    def units_per_step(self):
        return self.B

    def key_bytes(self):
        return self.NC * (DI // 2 + DI // 32 if self.mixed else DI * 2)

    def alg_bytes_per_step(self):
        rows = (self.K + TW) * self.row
        qin = H * D * 2 + HI * DI * 2 + HI * 4
        return self.B * (self.key_bytes() + rows + qin + H * DV * 2)

    def dominant_bytes(self):
        return self.B * (self.key_bytes() + HI * DI * 2 + HI * 4)

    def dominant_ms(self, stream, K, torch):
        """The index scoring alone (csa_index_topk with k = 0 runs no selection), K launches
        back to back on the step's inputs and workspace."""
        L = self.lcs
        idx = torch.empty(1, dtype=torch.int32, device=self.dev)
        fn = lambda: L._call("csa_index_topk", L._ptr(self.qI), L.BF16, L._ptr(self.w), L._ptr(self.kI),
                             self.kI_dtype, self.B, 1, self.NC, HI, DI, None, 4, 0, self.score_dtype, L._ptr(idx),
                             None, L._ptr(self.ws), self.ws.numel(), L._stream(stream))
        return _time_launches(fn, stream, K, torch)

    def io_names(self):
        return ["q", "qI", "w"], "out"

    def cpu_prepare(self):
        """Host copies of the step's inputs; a unit is one request's whole path."""
        self._cpu = {k: getattr(self, k).cpu() for k in ("q", "qI", "w", "comp", "win")}
        if self.mixed:
            planes = self.kI.cpu().numpy()
            tot = self.B * self.NC
            self._cpu["kp"] = planes[:tot * 64].reshape(self.B, self.NC, 64)
            self._cpu["ks"] = planes[tot * 64:].reshape(self.B, self.NC, 4)
        else:
            self._cpu["kI"] = self.kI.cpu()
        return list(range(self.B)), (f"requests: index over all {self.NC} entries, top-{self.K}, attention over "
                                     f"{self.K}+{TW} rows")

    def cpu_unit(self, b):
        import torch
        from oracle import oracle as orc
        c = self._cpu
        if self.mixed:
            s = orc.index_scores_fp4(c["qI"][b].float().numpy(), c["w"][b].numpy(), c["kp"][b], c["ks"][b])
            idx = orc.topk(s.astype(np.float32), self.K)
            rows = orc.dequant_kv_fp8(c["comp"][b][torch.from_numpy(idx.astype(np.int64))].numpy())
            win = orc.dequant_kv_fp8(c["win"][b].numpy())
        else:
            s = orc.index_scores_bf16(c["qI"][b].double().numpy(), c["w"][b].numpy(), c["kI"][b].double().numpy())
            idx = orc.topk(s, self.K)
            rows = c["comp"][b][torch.from_numpy(idx.astype(np.int64))].double().numpy()
            win = c["win"][b].double().numpy()
        # the selected rows gathered first (harness marshalling); attention over them and the window
        orc.csa_attend(c["q"][b].double().numpy(), rows, np.arange(self.K, dtype=np.int32), win, 0, -1, TW, DV,
                       SCALE)
        return 1


def _time_launches(fn, stream, K, torch):
    """Average device time of K back-to-back launches of fn (after 3 untimed ones)."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / K


class CsaDecodeMixed(CsaDecode):
    name = "csa_decode_mixed_1m"
    B, NC, K = 4, 262144, 1024
    mixed = True
    dominant = "index_fp4_tc_kernel"


class HcaDecode(Workload):
    name = "hca_decode_bf16_1m"
    B, NC = 16, 8192
    stage_names = ("attend",)
    dominant = "attend_tc_kernel"
    row = 2 * D

    def config(self):
        return dict(workload=self.name, requests=self.B, context_tokens=self.NC * 128, compressed_entries=self.NC,
                    m=128, kv_dim=D, d_v=DV, heads=H, window=TW, kv_format="bf16")

    def build(self):
        import torch
        from long_context_sparse_06_b200 import synth
        L, dev, bf = self.lcs, self.dev, torch.bfloat16
        self.q = synth.normal_t(self.tag("q"), (self.B, H, D), dtype=bf, device=dev)
        self.comp = synth.normal_t(self.tag("comp"), (self.B, self.NC, D), dtype=bf, device=dev)
        self.win = synth.normal_t(self.tag("win"), (self.B, TW, D), dtype=bf, device=dev)
        self.out = torch.empty((self.B, H, DV), dtype=bf, device=dev)
        self.ws = L.workspace(L.lcs_workspace_size(L.OP_DECODE, self.B, 1, self.NC, TW, 0, H, DV), dev)

    def step(self, stream):
        L = self.lcs
        L.decode_fused(L.MODE_HCA, self.q, self.comp, self.win, DV, SCALE, out=self.out, ws=self.ws, stream=stream)

    def stage(self, name, stream):
        self.step(stream)

    def units_per_step(self):
        return self.B

    def alg_bytes_per_step(self):
        return self.B * ((self.NC + TW) * D * 2 + H * D * 2 + H * DV * 2)

    def dominant_bytes(self):
        return self.alg_bytes_per_step()

    def dominant_ms(self, stream, K, torch):
        """The attention alone (kernel and split combine), K launches back to back."""
        L = self.lcs
        fn = lambda: L._call("hca_attend", L._ptr(self.q), L.BF16, L._ptr(self.comp), L._ptr(self.win), L.BF16,
                             self.B, 1, self.NC, TW, None, None, 128, TW, H, D, DV, SCALE, L._ptr(self.out), L.BF16,
                             None, L._ptr(self.ws), self.ws.numel(), L._stream(stream))
        return _time_launches(fn, stream, K, torch)

    def io_names(self):
        return ["q"], "out"

    def cpu_prepare(self):
        self._cpu = {k: getattr(self, k).cpu() for k in ("q", "comp", "win")}
        return list(range(self.B)), f"requests: dense attention over {self.NC}+{TW} rows"

    def cpu_unit(self, b):
        from oracle import oracle as orc
        c = self._cpu
        if self.row == 656:
            comp, win = orc.dequant_kv_fp8(c["comp"][b].numpy()), orc.dequant_kv_fp8(c["win"][b].numpy())
        else:
            comp, win = c["comp"][b].double().numpy(), c["win"][b].double().numpy()
        orc.hca_attend(c["q"][b].double().numpy(), comp, 128, win, 0, -1, TW, DV, SCALE)
        return 1


class HcaDecodeFp8(HcaDecode):
    """HCA decode over FP8 rows (the 1M-context mixed-precision row format)."""
    name = "hca_decode_fp8_1m"
    row = 656

    def config(self):
        return dict(super().config(), workload=self.name,
                    kv_format="fp8-e4m3 (pow2 scale per 128) + bf16 rope")

    def build(self):
        import torch
        from long_context_sparse_06_b200 import synth
        L, dev = self.lcs, self.dev
        f32 = torch.float32
        self.q = synth.normal_t(self.tag("q"), (self.B, H, D), dtype=torch.bfloat16, device=dev)
        self.comp = L.lcs_quant_kv_fp8(synth.normal_t(self.tag("comp"), (self.B, self.NC, D), dtype=f32, device=dev))
        self.win = L.lcs_quant_kv_fp8(synth.normal_t(self.tag("win"), (self.B, TW, D), dtype=f32, device=dev))
        self.out = torch.empty((self.B, H, DV), dtype=torch.bfloat16, device=dev)
        self.ws = L.workspace(L.lcs_workspace_size(L.OP_DECODE, self.B, 1, self.NC, TW, 0, H, DV), dev)

    def step(self, stream):
        L = self.lcs
        L.decode_fused(L.MODE_HCA, self.q, self.comp, self.win, DV, SCALE, kv_dtype=L.KV_FP8, out=self.out,
                       ws=self.ws, stream=stream)

    def alg_bytes_per_step(self):
        return self.B * ((self.NC + TW) * self.row + H * D * 2 + H * DV * 2)

    def dominant_ms(self, stream, K, torch):
        L = self.lcs
        fn = lambda: L._call("hca_attend", L._ptr(self.q), L.BF16, L._ptr(self.comp), L._ptr(self.win), L.KV_FP8,
                             self.B, 1, self.NC, TW, None, None, 128, TW, H, D, DV, SCALE, L._ptr(self.out), L.BF16,
                             None, L._ptr(self.ws), self.ws.numel(), L._stream(stream))
        return _time_launches(fn, stream, K, torch)


class CsaPrefill(Workload):
    """Chunked prefill: 8192 new tokens after a 131072-token prefix."""
    name = "csa_prefill_bf16_8k"
    unit = "query-tok/s"
    bound = "tensor"
    P0, Q, K = 131072, 8192, 1024
    stage_names = ("compress", "index", "topk", "attend")
    dominant = "index_bf16_tc_kernel"

    def config(self):
        return dict(workload=self.name, requests=1, prefix_tokens=self.P0, new_tokens=self.Q, m=4, overlap=2,
                    compressed_entries=(self.P0 + self.Q) // 4, kv_dim=D, d_v=DV, heads=H, index_heads=HI,
                    index_dim=DI, topk=self.K, window=TW, kv_format="bf16", causal=True)

    def build(self):
        import torch
        from long_context_sparse_06_b200 import synth
        L, dev, bf = self.lcs, self.dev, torch.bfloat16
        Q, P0 = self.Q, self.P0
        self.NC = (P0 + Q) // 4
        n0 = P0 // 4
        self.comp = torch.empty((1, self.NC, D), dtype=bf, device=dev)
        self.comp[:, :n0] = synth.normal_t(self.tag("prefix_comp"), (1, n0, D), dtype=bf, device=dev)
        self.kI = torch.empty((1, self.NC, DI), dtype=bf, device=dev)
        self.kI[:, :n0] = synth.normal_t(self.tag("prefix_kI"), (1, n0, DI), dtype=bf, device=dev)
        self.x = synth.normal_t(self.tag("x"), (1, Q, D), dtype=bf, device=dev)           # raw chunk KV
        self.x_tail = synth.normal_t(self.tag("x_tail"), (1, 2, D), dtype=bf, device=dev)
        self.kx = synth.normal_t(self.tag("kx"), (1, Q, DI), dtype=bf, device=dev)        # raw index keys
        self.kx_tail = synth.normal_t(self.tag("kx_tail"), (1, 2, DI), dtype=bf, device=dev)
        self.z = synth.normal_t(self.tag("z"), (1, Q), device=dev)
        self.z_tail = synth.normal_t(self.tag("z_tail"), (1, 2), device=dev)
        self.zI = synth.normal_t(self.tag("zI"), (1, Q), device=dev)
        self.zI_tail = synth.normal_t(self.tag("zI_tail"), (1, 2), device=dev)
        self.bias = synth.normal_t(self.tag("bias"), (6,), device=dev)
        self.biasI = synth.normal_t(self.tag("biasI"), (6,), device=dev)
        self.win = synth.normal_t(self.tag("win"), (1, 127 + Q, D), dtype=bf, device=dev)  # post-RoPE rows
        self.win_pos0 = torch.tensor([P0 - 127], dtype=torch.int64, device=dev)
        self.q_pos = (P0 + torch.arange(Q, dtype=torch.int64, device=dev)).view(1, Q)
        self.q = synth.normal_t(self.tag("q"), (1, Q, H, D), dtype=bf, device=dev)
        self.qI = synth.normal_t(self.tag("qI"), (1, Q, HI, DI), dtype=bf, device=dev)
        self.w = synth.normal_t(self.tag("w"), (1, Q, HI), std=1.0 / 8, device=dev)
        self.idx = torch.empty((1, Q, self.K), dtype=torch.int32, device=dev)
        self.out = torch.empty((1, Q, H, DV), dtype=bf, device=dev)
        self.ws_i = L.workspace(L.lcs_workspace_size(L.OP_INDEX_TOPK, 1, Q, self.NC, 0, self.K), dev)
        self.ws_a = L.workspace(L.lcs_workspace_size(L.OP_ATTEND, 1, Q, self.NC, TW, self.K, H, DV), dev)
        torch.cuda.synchronize()

    def _compress(self, stream):
        L = self.lcs
        n0 = self.P0 // 4
        L.csa_compress(self.x, self.z, self.bias, m=4, overlap=2, d_rope=64, pos0=self.P0, x_tail=self.x_tail,
                       z_tail=self.z_tail, out=self.comp[:, n0:], stream=stream)
        L.csa_compress(self.kx, self.zI, self.biasI, m=4, overlap=2, d_rope=0, pos0=self.P0, x_tail=self.kx_tail,
                       z_tail=self.zI_tail, out=self.kI[:, n0:], stream=stream)

    def _index(self, stream):
        L = self.lcs
        L._call("csa_index_topk", L._ptr(self.qI), L.BF16, L._ptr(self.w), L._ptr(self.kI), L.BF16, 1, self.Q,
                self.NC, HI, DI, L._ptr(self.q_pos), 4, self.K, L.F32, L._ptr(self.idx), None, L._ptr(self.ws_i),
                self.ws_i.numel(), L._stream(stream))

    def _attend(self, stream):
        L = self.lcs
        L._call("csa_attend", L._ptr(self.q), L.BF16, L._ptr(self.comp), L._ptr(self.win), L.BF16, 1, self.Q,
                self.NC, self.win.shape[1], L._ptr(self.idx), self.K, L._ptr(self.q_pos), L._ptr(self.win_pos0),
                TW, H, D, DV, SCALE, L._ptr(self.out), L.BF16, None, L._ptr(self.ws_a), self.ws_a.numel(),
                L._stream(stream))

    def step(self, stream):
        self._compress(stream)
        self._index(stream)
        self._attend(stream)

    def stage(self, name, stream):
        {"compress": self._compress, "index": self._index, "topk": self._index, "attend": self._attend}[name](stream)

    def units_per_step(self):
        return self.Q

    def pairs(self):
        return sum(min(self.NC, (self.P0 + i + 1) // 4) for i in range(self.Q))

    def alg_flops_per_step(self):
        idx = self.pairs() * HI * DI * 2
        att = self.Q * (self.K + TW) * H * (D + DV) * 2
        return idx + att

    def dominant_flops(self):
        return self.pairs() * HI * DI * 2

    def io_names(self):
        return ["x", "kx", "z", "zI", "q", "qI", "w"], "out"

    def cpu_prepare(self):
        """Units are whole queries (index over their available entries, top-k, attention),
        the first and last queries of the chunk alternately; compression excluded."""
        self._cpu = {k: getattr(self, k)[0].cpu() for k in ("comp", "kI", "win", "qI", "w", "q")}
        self._cpu["kI64"] = self._cpu["kI"].double().numpy()
        order = [i // 2 if i % 2 == 0 else self.Q - 1 - i // 2 for i in range(self.Q)]
        return order, f"queries (index over their available entries, top-{self.K}, attention; compression excluded)"

    def cpu_unit(self, t):
        import torch
        from oracle import oracle as orc
        c = self._cpu
        pos = self.P0 + t
        na = min(self.NC, (pos + 1) // 4)
        s = orc.index_scores_bf16(c["qI"][t].double().numpy(), c["w"][t].numpy(), c["kI64"][:na])
        idx = orc.topk(s, self.K)
        nv = int((idx >= 0).sum())
        rows = c["comp"][torch.from_numpy(idx[:nv].astype(np.int64))].double().numpy()
        lo = pos - TW + 1 - (self.P0 - 127)
        win = c["win"][lo:lo + TW].double().numpy()
        orc.csa_attend(c["q"][t].double().numpy(), rows, np.arange(nv, dtype=np.int32), win, pos - TW + 1, pos, TW,
                       DV, SCALE)
        return 1


class CompressStream(Workload):
    """1M raw rows: CSA and HCA compression of the KV, CSA compression of the index keys."""
    name = "compress_stream_1m"
    unit = "tok/s"
    T = 1 << 20
    stage_names = ("csa_kv", "csa_index_keys", "hca_kv")
    dominant = "compress_tma_kernel"

    def config(self):
        return dict(workload=self.name, raw_tokens=self.T, kv_dim=D, index_dim=DI, csa_m=4, csa_overlap=2,
                    hca_m=128, d_rope=64, kv_format="bf16")

    def build(self):
        import torch
        from long_context_sparse_06_b200 import synth
        dev, bf = self.dev, torch.bfloat16
        T = self.T
        self.x = synth.normal_t(self.tag("x"), (1, T, D), dtype=bf, device=dev)
        self.kx = synth.normal_t(self.tag("kx"), (1, T, DI), dtype=bf, device=dev)
        self.z = synth.normal_t(self.tag("z"), (1, T), device=dev)
        self.zI = synth.normal_t(self.tag("zI"), (1, T), device=dev)
        self.zh = synth.normal_t(self.tag("zh"), (1, T), device=dev)
        self.bias = synth.normal_t(self.tag("bias"), (6,), device=dev)
        self.biasI = synth.normal_t(self.tag("biasI"), (6,), device=dev)
        self.biash = synth.normal_t(self.tag("biash"), (128,), device=dev)
        self.csa = torch.empty((1, T // 4, D), dtype=bf, device=dev)
        self.csaI = torch.empty((1, T // 4, DI), dtype=bf, device=dev)
        self.hca = torch.empty((1, T // 128, D), dtype=bf, device=dev)

    def _csa_kv(self, stream):
        self.lcs.csa_compress(self.x, self.z, self.bias, m=4, overlap=2, d_rope=64, out=self.csa, stream=stream)

    def _csa_keys(self, stream):
        self.lcs.csa_compress(self.kx, self.zI, self.biasI, m=4, overlap=2, d_rope=0, out=self.csaI, stream=stream)

    def _hca(self, stream):
        self.lcs.hca_compress(self.x, self.zh, self.biash, m=128, d_rope=64, out=self.hca, stream=stream)

    def step(self, stream):
        self._csa_kv(stream)
        self._csa_keys(stream)
        self._hca(stream)

    def stage(self, name, stream):
        {"compress": self._csa_kv, "csa_kv": self._csa_kv, "csa_index_keys": self._csa_keys,
         "hca_kv": self._hca}[name](stream)

    def units_per_step(self):
        return self.T

    def alg_bytes_per_step(self):
        T = self.T
        return 2 * T * D * 2 + T * DI * 2 + 3 * T * 4 + (T // 4) * (D + DI) * 2 + (T // 128) * D * 2

    def dominant_bytes(self):
        T = self.T
        return T * D * 2 + T * 4 + (T // 4) * D * 2

    def io_names(self):
        return ["z", "zI", "zh"], "hca"

    def cpu_prepare(self):
        """Units are slices of 4096 raw rows of the CSA KV compression (one of the three
        passes); each counts as the raw rows of the whole step that take the same share of
        the step's algorithmic bytes."""
        self._cpu = {k: getattr(self, k)[0].cpu() for k in ("x", "z")}
        self._cpu["bias"] = self.bias.double().cpu().numpy()
        return list(range(0, self.T, 4096)), "slices of 4096 raw rows of the CSA KV compression, rows scaled " \
                                              "by that pass's share of the step's bytes"

    def cpu_unit(self, n):
        from oracle import oracle as orc
        c = self._cpu
        x = c["x"][n:n + 4096].double().numpy()
        z = c["z"][n:n + 4096].double().numpy()
        tail = (c["x"][n - 2:n].double().numpy(), c["z"][n - 2:n].double().numpy()) if n else (None, None)
        orc.compress(x, z, c["bias"], 4, 2, d_rope=64, pos0=n, x_tail=tail[0], z_tail=tail[1])
        return 4096 * (self.T * D * 2) / self.alg_bytes_per_step()


class C1Prefill(Workload):
    """The tiny fp32 CSA prefill: seq 1024, hidden 256; compressors m = 4 / overlap 2 for the
    KV (64 = 48 + 16 RoPE) and the index keys (32), causal indexer 4 x 32 with top-64,
    8-head MQA with a 128-row window, grouped output projection 2 x 64 -> 256.  The
    projections from the hidden states are harness inputs, made once on the device; one
    step is the library chain: two compressions, index + top-k, attention, projection."""
    name = "c1_prefill_f32"
    unit = "query-tok/s"
    bound = "alu"
    T, HID, DKV, DR, DVc, HIc, DIc, Kc, Hc, G, DG = 1024, 256, 64, 16, 48, 4, 32, 64, 8, 2, 64
    stage_names = ("compress", "index", "attend", "oproj")
    dominant = "attend_f32_kernel"

    def config(self):
        return dict(workload=self.name, requests=1, seq_len=self.T, hidden=self.HID, m=4, overlap=2,
                    compressed_entries=self.T // 4, kv_dim=self.DKV, d_rope=self.DR, d_v=self.DVc,
                    heads=self.Hc, index_heads=self.HIc, index_dim=self.DIc, topk=self.Kc, window=TW,
                    groups=self.G, group_dim=self.DG, dtype="fp32", causal=True)

    def build(self):
        import torch
        from long_context_sparse_06_b200 import synth
        L, dev = self.lcs, self.dev
        T, HID = self.T, self.HID
        sw = 1.0 / math.sqrt(HID)
        r = lambda n, shape, std=1.0: synth.normal_t(self.tag(n), shape, std=std, device=dev)   # noqa: E731
        h = r("h", (T, HID))
        self.x = (h @ r("W_kv", (HID, self.DKV), sw)).view(1, T, self.DKV).contiguous()
        self.kx = (h @ r("W_ki", (HID, self.DIc), sw)).view(1, T, self.DIc).contiguous()
        self.z = (h @ r("w_z", (HID,), sw)).view(1, T).contiguous()
        self.zI = (h @ r("w_zi", (HID,), sw)).view(1, T).contiguous()
        self.qI = (h @ r("W_qi", (HID, self.HIc * self.DIc), sw)).view(1, T, self.HIc, self.DIc).contiguous()
        self.w = (h @ r("W_w", (HID, self.HIc), sw)).view(1, T, self.HIc).contiguous()
        self.q = (h @ r("W_q", (HID, self.Hc * self.DKV), sw)).view(1, T, self.Hc, self.DKV).contiguous()
        self.bias = r("bias", (6,))
        self.biasI = r("bias_i", (6,))
        self.Wg = r("Wg", (self.G, self.Hc // self.G * self.DVc, self.DG), 1.0 / math.sqrt(self.Hc // self.G * self.DVc))
        self.Wo = r("Wo", (self.G * self.DG, HID), 1.0 / math.sqrt(self.G * self.DG))
        self.q_pos = torch.arange(T, dtype=torch.int64, device=dev).view(1, T)
        self.win_pos0 = torch.zeros(1, dtype=torch.int64, device=dev)
        # post-RoPE queries and window rows (harness inputs, rotated once by the library)
        self.win = self.x.clone()
        L.lcs_rope(self.win, self.q_pos.view(-1), self.DR)
        L.lcs_rope(self.q, self.q_pos.view(-1).repeat_interleave(self.Hc), self.DR)
        self.comp = torch.empty((1, T // 4, self.DKV), dtype=torch.float32, device=dev)
        self.kI = torch.empty((1, T // 4, self.DIc), dtype=torch.float32, device=dev)
        self.idx = torch.empty((1, T, self.Kc), dtype=torch.int32, device=dev)
        self.o = torch.empty((1, T, self.Hc, self.DVc), dtype=torch.float32, device=dev)
        self.out = torch.empty((T, HID), dtype=torch.float32, device=dev)
        self.ws_i = L.workspace(L.lcs_workspace_size(L.OP_INDEX_TOPK, 1, T, T // 4, 0, self.Kc), dev)
        self.ws_a = L.workspace(L.lcs_workspace_size(L.OP_ATTEND, 1, T, T // 4, T, self.Kc, self.Hc, self.DVc), dev)
        torch.cuda.synchronize()

    def _compress(self, stream):
        L = self.lcs
        L.csa_compress(self.x, self.z, self.bias, m=4, overlap=2, d_rope=self.DR, out=self.comp, stream=stream)
        L.csa_compress(self.kx, self.zI, self.biasI, m=4, overlap=2, d_rope=0, out=self.kI, stream=stream)

    def _index(self, stream):
        L = self.lcs
        L._call("csa_index_topk", L._ptr(self.qI), L.F32, L._ptr(self.w), L._ptr(self.kI), L.F32, 1, self.T,
                self.T // 4, self.HIc, self.DIc, L._ptr(self.q_pos), 4, self.Kc, L.F32, L._ptr(self.idx), None,
                L._ptr(self.ws_i), self.ws_i.numel(), L._stream(stream))

    def _attend(self, stream):
        L = self.lcs
        L._call("csa_attend", L._ptr(self.q), L.F32, L._ptr(self.comp), L._ptr(self.win), L.F32, 1, self.T,
                self.T // 4, self.T, L._ptr(self.idx), self.Kc, L._ptr(self.q_pos), L._ptr(self.win_pos0), TW,
                self.Hc, self.DKV, self.DVc, 1.0 / math.sqrt(self.DKV), L._ptr(self.o), L.F32, None,
                L._ptr(self.ws_a), self.ws_a.numel(), L._stream(stream))

    def _oproj(self, stream):
        self.lcs.group_oproj(self.o.view(self.T, self.Hc, self.DVc), self.Wg, self.Wo, out=self.out, stream=stream)

    def step(self, stream):
        self._compress(stream)
        self._index(stream)
        self._attend(stream)
        self._oproj(stream)

    def stage(self, name, stream):
        {"compress": self._compress, "index": self._index, "topk": self._index, "attend": self._attend,
         "oproj": self._oproj}[name](stream)

    def units_per_step(self):
        return self.T

    def attend_flops(self):
        """QK and PV over each query's rows (selected entries plus its causal window)."""
        rows = 0
        for t in range(self.T):
            rows += min(self.Kc, min(self.T // 4, (t + 1) // 4)) + min(TW, t + 1)
        return rows * self.Hc * (self.DKV + self.DVc) * 2

    def dominant_flops(self):
        return self.attend_flops()

    def dominant_ms(self, stream, K, torch):
        return _time_launches(lambda: self._attend(stream), stream, K, torch)

    def io_names(self):
        return ["x", "kx", "z", "zI", "qI", "w", "q", "win"], "out"

    def cpu_unit(self, t):
        """The oracle's chain for query t (the compressed entries of the whole sequence are
        made once, outside the timed sample)."""
        from oracle import oracle as orc
        c = self._cpu_cache
        n = orc.n_avail(t, 4, self.T // 4)
        s = orc.index_scores_f32(c["qI"][t], c["w"][t], c["kI"][:n])
        idx = orc.topk(s, self.Kc)
        o, _ = orc.csa_attend(c["q"][t], c["comp"], idx, c["win"], 0, t, TW, self.DVc, 1.0 / math.sqrt(self.DKV))
        orc.group_oproj(o, c["Wg"], c["Wo"])
        return 1

    def cpu_prepare(self):
        from oracle import oracle as orc
        c = {k: getattr(self, k)[0].cpu().numpy() for k in ("qI", "w")}
        c["q"] = self.q[0].double().cpu().numpy()
        c["win"] = self.win[0].double().cpu().numpy()
        c["comp"] = orc.compress(self.x[0].cpu().numpy(), self.z[0].cpu().numpy(), self.bias.cpu().numpy(), 4, 2,
                                 d_rope=self.DR)[0]
        c["kI"] = orc.compress(self.kx[0].cpu().numpy(), self.zI[0].cpu().numpy(), self.biasI.cpu().numpy(), 4, 2,
                               d_rope=0)[0].astype(np.float32)
        c["Wg"], c["Wo"] = self.Wg.double().cpu().numpy(), self.Wo.double().cpu().numpy()
        self._cpu_cache = c
        return list(range(self.T)), "queries of the 1024-token sequence (index, top-64, attention, projection)"


WORKLOADS = {c.name: c for c in (CsaDecode, HcaDecode, HcaDecodeFp8, CsaDecodeMixed, CsaPrefill, CompressStream,
                                  C1Prefill)}
LAUNCHES_PER_STEP = {"csa_decode_bf16_128k": 4, "csa_decode_mixed_1m": 5, "hca_decode_bf16_1m": 2,
                     "hca_decode_fp8_1m": 2,
                     "csa_prefill_bf16_8k": 5, "compress_stream_1m": 3,
                     "c1_prefill_f32": 6}


# ------------------------------------------------------------- ranks (N > 1)
# One process per GPU; requests are independent, so every rank runs its own replica of the
# workload and the only cross-rank traffic is the timing: barriers around the timed region
# and the maximum of the per-rank step times.
def rank_env():
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world, device):
    """The largest of the ranks' values (the job's step time is that of its slowest rank)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, units_per_rank_step, ms_step):
    """Whole-job throughput: the units every rank processed per step over the step time."""
    return world * units_per_rank_step / (ms_step / 1e3)


# ------------------------------------------------------------- CPU baseline
def host_cores():
    return len(os.sched_getaffinity(0))


def cpu_baseline(wl, budget_s):
    """The oracle as it stands on this workload, on the host cores: first one thread over
    whole units until about a quarter of the budget, then a pool of threads over all cores
    (the oracle's C calls release the GIL) on as many units as fit the rest.  Units are the
    workload's independent pieces (requests, queries, row slices); each counts for its share
    of the metric."""
    from concurrent.futures import ThreadPoolExecutor
    units, what = wl.cpu_prepare()
    cores = host_cores()
    t0 = time.perf_counter()
    got1, i = 0.0, 0
    while i < len(units) and (i == 0 or time.perf_counter() - t0 < budget_s / 4):
        got1 += wl.cpu_unit(units[i])
        i += 1
    el1 = time.perf_counter() - t0
    per_unit = el1 / i
    n_par = int(min(len(units), max(cores, cores * (0.75 * budget_s) / per_unit)))
    threads = min(cores, n_par)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        t0 = time.perf_counter()
        got = sum(ex.map(wl.cpu_unit, units[:n_par]))
        el = time.perf_counter() - t0
    return {"value": round(got / el, 4), "unit": wl.unit, "cores": threads, "kind": "oracle",
            "sample": f"{n_par} of {len(units)} {what}; {threads} threads on {cores} host cores",
            "single_thread": {"value": round(got1 / el1, 4), "unit": wl.unit, "cores": 1,
                              "sample": f"{i} of {len(units)} {what}"}}


# ------------------------------------------------------------------- GPU arm
def capture(wl, dev, torch):
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        wl.step(torch.cuda.current_stream(dev))
    return graph


def e2e_leg(wl, graph, dev, stream, steps, warmup, world, torch):
    """The step through the public API with its inputs copied from pinned host memory and its
    result read back every step.  The copies run on their own streams with two sets of
    device inputs and outputs, so that step i+1's inputs and step i-1's result move while
    step i computes (each set is reused only after the step that read it has finished and
    its result has reached the host).  Returns (ms per step, H2D bytes, D2H bytes)."""
    in_names, out_name = wl.io_names()
    names = in_names + [out_name]
    set_a = {n: getattr(wl, n) for n in names}
    set_b = {n: t.clone() for n, t in set_a.items()}
    for n, t in set_b.items():
        setattr(wl, n, t)
    graph_b = capture(wl, dev, torch)
    for n, t in set_a.items():
        setattr(wl, n, t)
    sets, graphs = (set_a, set_b), (graph, graph_b)
    hosts = [set_a[n].cpu().pin_memory() for n in in_names]
    res = set_a[out_name]
    houts = [torch.empty(res.shape, dtype=res.dtype).pin_memory() for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        h2d_s.wait_stream(stream)
        for i in range(n):
            j = i & 1
            S = sets[j]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev_done[j])          # step i-2 has read set j's inputs
                for name, h in zip(in_names, hosts):
                    S[name].copy_(h, non_blocking=True)
                ev_in[j].record(h2d_s)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])              # step i-2's result has left set j
            graphs[j].replay()
            ev_done[j].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[j])
                houts[j].copy_(S[out_name], non_blocking=True)
                ev_out[j].record(d2h_s)
        stream.wait_stream(h2d_s)
        stream.wait_stream(d2h_s)

    run(max(3, warmup))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    del graph_b
    return ms, sum(h.numel() * h.element_size() for h in hosts), houts[0].numel() * houts[0].element_size()


def measure(wl, lcs, args, world, dev, torch, headline):
    """Builds and times one workload: K graph replays of the whole step (after W warm-up
    steps), the stage times, the dominant kernel alone, and for the headline the
    end-to-end leg and the CPU baseline."""
    wl.build()
    stream = torch.cuda.current_stream(dev)
    workspaces = [getattr(wl, a) for a in ("ws", "ws_i", "ws_a") if hasattr(wl, a)]
    for _ in range(args.warmup):
        wl.step(stream)
    torch.cuda.synchronize()
    for ws in workspaces:
        st = lcs.lcs_status(ws)
        if st != 0:
            raise RuntimeError(f"{wl.name}: device status after warm-up: {st}")
    # the step captured once as a CUDA graph and replayed: decode loops are launch-bound
    # on the host otherwise
    graph = capture(wl, dev, torch)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    # ---- timed region: K steps of the whole path (inputs larger than L2, except C1's)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_step = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    value = job_value(world, wl.units_per_step(), ms_step)

    # ---- stage times on the launching stream; stages then run without programmatic overlap
    stage_ms = time_stages(wl, lcs, stream, args.steps, torch)
    stage_ms = {k: max_over_ranks(v, world, dev) for k, v in stage_ms.items()}

    e2e = None
    if headline:
        e2e_ms, h2d, d2h = e2e_leg(wl, graph, dev, stream, args.steps, args.warmup, world, torch)
        e2e = {"value": round(job_value(world, wl.units_per_step(), e2e_ms), 1), "unit": wl.unit,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5),
               "inputs": "per-step inputs H2D from pinned host and the result D2H, on copy streams overlapping "
                         "the neighbouring steps (two device buffer sets); caches resident"}
    for ws in workspaces:
        st = lcs.lcs_status(ws)
        if st != 0:
            raise RuntimeError(f"{wl.name}: device status after timing: {st}")
    del graph

    hbm, tf_burst, tf_sust, peak_kind = load_peaks()
    if wl.bound == "tensor":
        dom_ms = stage_ms["index"]
        achieved = wl.dominant_flops() / (dom_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": wl.dominant, "achieved": round(achieved, 1), "peak": tf_burst,
                "unit": "TFLOP/s", "frac": round(achieved / tf_burst, 4), "peak_source": f"{peak_kind} bf16 burst",
                "frac_of_sustained": round(achieved / tf_sust, 4),
                "algorithmic_flops_per_launch": wl.dominant_flops(),
                "traffic": recorded_traffic(wl.dominant, wl.name)}
        step_flops = wl.alg_flops_per_step()
        step_roof = {"algorithmic_flops_per_step": step_flops,
                     "achieved_tflops": round(step_flops / (ms_step / 1e3) / 1e12, 1),
                     "frac": round(step_flops / (ms_step / 1e3) / 1e12 / tf_burst, 4)}
    elif wl.bound == "alu":
        dom_ms = max_over_ranks(wl.dominant_ms(stream, args.steps, torch), world, dev)
        achieved = wl.dominant_flops() / (dom_ms / 1e3) / 1e12
        peak = FP32_PEAK_TFLOPS
        roof = {"bound": "alu", "kernel": wl.dominant, "achieved": round(achieved, 3), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": "fp32 CUDA-core FMA: 148 SMs x 128 lanes x 2 flops x 1965 MHz",
                "kernel_ms": round(dom_ms, 5), "algorithmic_flops_per_launch": wl.dominant_flops(),
                "traffic": None}
        step_roof = {"note": "latency-bound parity size; query-tok/s is the figure of merit"}
    else:
        dom_ms = (wl.dominant_ms(stream, args.steps, torch) if hasattr(wl, "dominant_ms")
                  else list(stage_ms.values())[wl.dominant_stage()])
        dom_ms = max_over_ranks(dom_ms, world, dev)
        achieved = wl.dominant_bytes() / (dom_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": wl.dominant, "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "peak_source": f"{peak_kind} copy bandwidth",
                "kernel_ms": round(dom_ms, 5),
                "timing": "K back-to-back launches of the stage alone between CUDA events" if hasattr(wl, "dominant_ms")
                else "stage events inside the step",
                "algorithmic_bytes_per_launch": wl.dominant_bytes(),
                "traffic": recorded_traffic(wl.dominant, wl.name)}
        step_bytes = wl.alg_bytes_per_step()
        step_roof = {"algorithmic_bytes_per_step": step_bytes,
                     "achieved_gbs": round(step_bytes / (ms_step / 1e3) / 1e9, 1),
                     "frac": round(step_bytes / (ms_step / 1e3) / 1e9 / hbm, 4)}
    rec = {"value": round(value, 1), "unit": wl.unit, "ms_per_step": round(ms_step, 5),
           "config": dict(wl.config(), l2=("inputs smaller than L2 (parity size)" if wl.name == "c1_prefill_f32"
                                           else "inputs larger than L2 (126 MB) every step"),
                          parallelism=f"replicas x{world} (requests independent)"),
           "roofline": roof, "step_roofline": step_roof,
           "stage_ms": {k: round(v, 5) for k, v in stage_ms.items()},
           "gpu_launches": args.steps * LAUNCHES_PER_STEP[wl.name], "clocks": sampler.summary()}
    if e2e is not None:
        rec["e2e"] = e2e
    return rec


FP32_PEAK_TFLOPS = round(148 * 128 * 2 * 1.965e9 / 1e12, 1)


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import long_context_sparse_06_b200 as lcs

    world, rank, local = rank_env()
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lcs.lib()
    wl = WORKLOADS[args.workload](lcs, dev, rank)

    if args.stage:
        # one stage alone: warm-up, then K launches (for profilers; prints timing only)
        wl.build()
        stream = torch.cuda.current_stream(dev)
        for _ in range(args.warmup):
            wl.stage(args.stage, stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            wl.stage(args.stage, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        print(json.dumps({"workload": wl.name, "stage": args.stage, "ms": e0.elapsed_time(e1) / args.steps}))
        return None

    rec = measure(wl, lcs, args, world, dev, torch, headline=True)
    res = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_baseline(wl, args.cpu_budget)
        res = {"metric": METRIC, "value": rec["value"], "unit": wl.unit, "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "bf16" if wl.name != "c1_prefill_f32" else "f32",
               "data": "synthetic (seeded splitmix64 + Box-Muller)", "config": rec["config"],
               "roofline": rec["roofline"], "step_roofline": rec["step_roofline"], "stage_ms": rec["stage_ms"],
               "e2e": rec["e2e"], "gpu_launches": rec["gpu_launches"], "clocks": rec["clocks"],
               "cpu_baseline": cpu}
    del wl
    torch.cuda.empty_cache()
    # the other workloads, each timed the same way (one GPU only: every rank would hold all of
    # them otherwise); the headline figures above are the ones the line reports
    if world == 1 and not args.no_workloads and args.workload == "csa_decode_bf16_128k":
        nested = {}
        for name in NESTED:
            w2 = WORKLOADS[name](lcs, dev, rank)
            nested[name] = measure(w2, lcs, args, world, dev, torch, headline=False)
            del w2
            torch.cuda.empty_cache()
        res["workloads"] = nested
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return res


NESTED = ("hca_decode_bf16_1m", "hca_decode_fp8_1m", "csa_decode_mixed_1m", "csa_prefill_bf16_8k",
          "compress_stream_1m", "c1_prefill_f32")


def time_stages(wl, lcs, stream, steps, torch):
    names = wl.stage_names
    if isinstance(wl, (CsaDecode, HcaDecode)):
        # Back-to-back steps, each with its own set of events between the stages (the
        # library records them on the launching stream), read once after the last step.
        n_ev = len(names) + 1
        sets = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
        for es in sets:   # torch creates the CUDA event on its first record
            for e in es:
                e.record(stream)
        torch.cuda.synchronize()
        handles = [(lcs.C.c_void_p * n_ev)(*[e.cuda_event for e in es]) for es in sets]
        try:
            lcs.lib().lcs_set_stage_events(handles[0], n_ev)
            for _ in range(3):
                wl.step(stream)
            torch.cuda.synchronize()
            for i in range(steps):
                lcs.lib().lcs_set_stage_events(handles[i], n_ev)
                wl.step(stream)
            torch.cuda.synchronize()
        finally:
            lcs.lib().lcs_set_stage_events(None, 0)
        acc = [0.0] * len(names)
        for es in sets:
            for i in range(len(names)):
                acc[i] += es[i].elapsed_time(es[i + 1])
        return {n: a / steps for n, a in zip(names, acc)}
    if isinstance(wl, CsaPrefill):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        for e in evs:
            e.record(stream)
        torch.cuda.synchronize()
        handles = (lcs.C.c_void_p * 3)(*[e.cuda_event for e in evs])
        acc = {n: 0.0 for n in names}
        for _ in range(steps):
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            wl._compress(stream)
            a1.record(stream)
            lcs.lib().lcs_set_stage_events(handles, 3)
            try:
                wl._index(stream)
            finally:
                lcs.lib().lcs_set_stage_events(None, 0)
            b0.record(stream)
            wl._attend(stream)
            b1.record(stream)
            torch.cuda.synchronize()
            acc["compress"] += a0.elapsed_time(a1)
            acc["index"] += evs[0].elapsed_time(evs[1])
            acc["topk"] += evs[1].elapsed_time(evs[2])
            acc["attend"] += b0.elapsed_time(b1)
        return {n: v / steps for n, v in acc.items()}
    if isinstance(wl, C1Prefill):
        fns = {"compress": wl._compress, "index": wl._index, "attend": wl._attend, "oproj": wl._oproj}
    else:
        fns = {"csa_kv": wl._csa_kv, "csa_index_keys": wl._csa_keys, "hca_kv": wl._hca}
    acc = {n: 0.0 for n in names}
    for _ in range(steps):
        for n in names:
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            fns[n](stream)
            a1.record(stream)
            torch.cuda.synchronize()
            acc[n] += a0.elapsed_time(a1)
    return {n: v / steps for n, v in acc.items()}


# ------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle as the reference arm, on the host cores.  One step is the headline
    workload itself -- its 32 requests, each the whole path (index over all 32768 entries,
    top-512, attention over 512 + 128 rows) -- on a pool of threads over all cores, with the
    same seeded inputs as the GPU arm (made on the host: the keys whole, the compressed rows
    only where selected).  If the host is too small to finish K + W such steps in about four
    minutes, each step takes an equal share of the requests instead (said in the line).
    Under torchrun only rank 0 runs it; the other ranks return without work."""
    rank = rank_env()[1]
    if rank != 0:
        return None
    import torch
    from concurrent.futures import ThreadPoolExecutor
    from long_context_sparse_06_b200 import synth
    from oracle import oracle as orc
    if args.workload != "csa_decode_bf16_128k":
        return {"impl": "reference", "unavailable": "the reference arm is timed on the headline workload only"}
    B, NC, K = CsaDecode.B, CsaDecode.NC, CsaDecode.K
    tag = lambda s_: f"bench.csa_decode_bf16_128k.r0.{s_}"          # noqa: E731  (the GPU arm's rank-0 streams)
    bf = torch.bfloat16
    q = synth.normal_t(tag("q"), (B, H, D), dtype=bf)
    qI = synth.normal_t(tag("qI"), (B, HI, DI), dtype=bf)
    w = synth.normal_t(tag("w"), (B, HI), std=1.0 / 8)
    kI = synth.normal_t(tag("kI"), (B, NC, DI), dtype=bf)
    win = synth.normal_t(tag("win"), (B, TW, D), dtype=bf)

    def request(b):
        s_ = orc.index_scores_bf16(qI[b].double().numpy(), w[b].numpy(), kI[b].double().numpy())
        idx = orc.topk(s_, K)
        rows = synth.normal_rows_t(tag("comp"), (B * NC, D), b * NC + torch.from_numpy(idx.astype(np.int64)),
                                   dtype=bf).double().numpy()
        orc.csa_attend(q[b].double().numpy(), rows, np.arange(K, dtype=np.int32), win[b].double().numpy(), 0, -1,
                       TW, DV, SCALE)
        return 1

    cores = host_cores()
    threads = min(cores, B)
    t0 = time.perf_counter()
    request(0)
    t_req = time.perf_counter() - t0
    rounds = -(-B // threads)
    per_step = rounds * t_req * 1.2
    n_req = B
    if per_step * (args.steps + args.warmup) > 240.0:
        n_req = max(1, min(B, int(240.0 / (args.steps + args.warmup) / (t_req * 1.2)) * threads))
    pool = ThreadPoolExecutor(max_workers=min(threads, n_req))

    def one_step(i):
        reqs = [(i * n_req + j) % B for j in range(n_req)]
        t0 = time.perf_counter()
        done = sum(pool.map(request, reqs))
        return done, time.perf_counter() - t0

    for i in range(args.warmup):
        one_step(i)
    tot_n, tot_t = 0, 0.0
    for i in range(args.steps):
        n, t = one_step(args.warmup + i)
        tot_n += n
        tot_t += t
    pool.shutdown()
    value = tot_n / tot_t
    ms = tot_t / args.steps * 1e3
    same = n_req == B
    sample = (f"{n_req} of {B} requests per step, each the whole path (index over all {NC} entries, top-{K}, "
              f"attention over {K}+{TW} rows); {min(threads, n_req)} threads on {cores} host cores; "
              f"one request alone on one thread: {t_req:.3f} s")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tok/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (fp32 where the oracle fixes it)",
            "data": "synthetic (seeded splitmix64 + Box-Muller, N(0,1); the GPU arm's rank-0 streams)",
            "config": dict(CsaDecode.config(CsaDecode(None, None, 0)), requests_per_step=n_req,
                           same_as_gpu_arm=same),
            "cpu_baseline": {"kind": "oracle", "cores": min(threads, n_req), "sample": sample,
                             "value": round(value, 4), "unit": "tok/s",
                             "single_thread": {"value": round(1.0 / t_req, 4), "unit": "tok/s", "cores": 1}},
            "e2e": {"value": round(value, 4), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="lcs", choices=["lcs", "reference"])
    ap.add_argument("--workload", default="csa_decode_bf16_128k", choices=sorted(WORKLOADS))
    ap.add_argument("--stage", default=None, help="run one stage alone (profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="headline only, no nested workload records")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    args = ap.parse_args()
    if args.warmup < 3 and not args.stage:
        args.warmup = 3
    res = run_reference(args) if args.impl == "reference" else run_gpu(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
