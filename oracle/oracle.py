"""CPU oracle for the CSA / HCA compressed-attention hot path (DeepSeek-V4).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product package
never imports it, and it imports nothing from the product package: the two
share no code.  The arithmetic lives in ``lcs_oracle.c`` (plain scalar C, fp64
unless a step fixes fp32, built with ``-ffp-contract=off``); this file only
builds and loads that library and marshals numpy arrays.

Every function cites the page passage it follows (titles and sections of the
pages; the pages state the method in prose only):

* "DeepSeek V4 深度解析" section 2 -- CSA steps 1-3 (compress with position-biased
  softmax weights and overlapping blocks, lightning indexer + top-k, sliding
  window of 128 raw tokens joined with the selection), the HCA paragraph
  (m'=128, dense, shared-KV MQA, grouped output projection) and the
  mixed-precision KV sentence (RoPE dims bf16, the rest FP8).
* same page, section 4, "FP4量化感知訓練" -- the indexer's QK path is FP4.
* "V3 vs V4" page, inline headings "V4 改进一CSA 与 HCA" and "FP4 为什么能无损"
  -- the same method restated; index scores in BF16.
* podcast show-notes glossary, entries CSA (4:1, query picks entries) and HCA
  (128:1, no picking).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lcs_oracle.c")
_LIB = os.path.join(_HERE, "liblcs_oracle.so")

FMT_F32, FMT_BF16, FMT_E4M3, FMT_E2M1 = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile ``lcs_oracle.c`` with gcc into ``liblcs_oracle.so`` (in place)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_LIB)
        P = C.c_void_p
        I64, I, D = C.c_int64, C.c_int, C.c_double
        sig = {
            "orc_round_array": (None, [P, I64, I, P]),
            "orc_decode_array": (None, [P, I64, I, P]),
            "orc_encode_array": (None, [P, I64, I, P]),
            "orc_quant_kv_fp8": (None, [P, I64, I, I, P]),
            "orc_dequant_kv_fp8": (None, [P, I64, I, I, P]),
            "orc_quant_fp4": (None, [P, I64, I, P, P]),
            "orc_rope": (None, [P, P, I64, I, I, D]),
            "orc_compress": (I, [P, P, P, P, P, I64, I, I, I, I, D, I64, P, P]),
            "orc_index_scores_f32": (None, [P, P, P, I64, I, I, P]),
            "orc_index_scores_bf16": (None, [P, P, P, I64, I, I, P]),
            "orc_index_scores_fp4": (None, [P, P, P, P, P, I64, I, I, I, P]),
            "orc_exact_dot_f32": (C.c_float, [P, P, I]),
            "orc_topk": (None, [P, I64, I, P]),
            "orc_mqa_rows": (None, [P, P, I64, I, I, I, D, P, P]),
            "orc_csa_attend": (I64, [P, P, I64, P, I, P, I64, I64, I64, I, I, I, I, D, P, P]),
            "orc_hca_attend": (I64, [P, P, I64, I, P, I64, I64, I64, I, I, I, I, D, P, P]),
            "orc_group_oproj": (None, [P, P, P, I, I, I, I, I, P]),
            "orc_project_f32": (None, [P, P, I64, I, I, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


# ---------------------------------------------------------------- formats
def round_to(x, fmt):
    """Round doubles to fp32 / bf16 / E4M3 / E2M1 values, RNE (E4M3, E2M1 saturate)."""
    x = _f64(x)
    out = np.empty_like(x)
    lib().orc_round_array(_p(x), x.size, fmt, _p(out))
    return out


def round_bf16(x):
    return round_to(x, FMT_BF16)


def e4m3_decode(codes):
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_decode_array(_p(c), c.size, FMT_E4M3, _p(out))
    return out


def e2m1_decode(nibbles):
    c = np.ascontiguousarray(nibbles, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_decode_array(_p(c), c.size, FMT_E2M1, _p(out))
    return out


def e4m3_encode(values):
    v = _f64(values)
    out = np.empty(v.shape, np.uint8)
    lib().orc_encode_array(_p(v), v.size, FMT_E4M3, _p(out))
    return out


def e2m1_encode(values):
    v = _f64(values)
    out = np.empty(v.shape, np.uint8)
    lib().orc_encode_array(_p(v), v.size, FMT_E2M1, _p(out))
    return out


def bf16_bits(x):
    """bf16 codes (uint16) of values that are already bf16."""
    return (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b):
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------- storage quantisers
def kv_fp8_row_bytes(d_c=512, d_r=64):
    return d_c + 2 * d_r + 4 * (d_c // 128)


def quant_kv_fp8(x, d_c=512, d_r=64):
    """Mixed-precision KV rows ("DeepSeek V4 深度解析" §2, last paragraph: RoPE dims
    BF16, the rest FP8).  x [..., d_c+d_r] fp32 -> uint8 [..., row_bytes]."""
    x = _f32(x)
    lead = x.shape[:-1]
    n = int(np.prod(lead)) if lead else 1
    out = np.empty(lead + (kv_fp8_row_bytes(d_c, d_r),), np.uint8)
    lib().orc_quant_kv_fp8(_p(x), n, d_c, d_r, _p(out))
    return out


def dequant_kv_fp8(rows, d_c=512, d_r=64):
    rows = np.ascontiguousarray(rows, np.uint8)
    lead = rows.shape[:-1]
    n = int(np.prod(lead)) if lead else 1
    out = np.empty(lead + (d_c + d_r,), np.float64)
    lib().orc_dequant_kv_fp8(_p(rows), n, d_c, d_r, _p(out))
    return out


def quant_fp4(x):
    """FP4 E2M1 with an E4M3 scale per 32 elements ("DeepSeek V4 深度解析" §4,
    "FP4量化感知訓練").  x [..., d] fp32 -> (packed [..., d/2] u8, scales [..., d/32] u8)."""
    x = _f32(x)
    lead, d = x.shape[:-1], x.shape[-1]
    n = int(np.prod(lead)) if lead else 1
    packed = np.empty(lead + (d // 2,), np.uint8)
    scales = np.empty(lead + (d // 32,), np.uint8)
    lib().orc_quant_fp4(_p(x), n, d, _p(packed), _p(scales))
    return packed, scales


def dequant_fp4(packed, scales):
    packed = np.ascontiguousarray(packed, np.uint8)
    lo = e2m1_decode(packed & 15)
    hi = e2m1_decode(packed >> 4)
    vals = np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * 2,))
    sc = e4m3_decode(scales)
    return vals * np.repeat(sc, 32, axis=-1)


# ------------------------------------------------------------------ RoPE
def rope(rows, pos, d_rope, theta=10000.0):
    """Rotate-half RoPE of the last d_rope dims of each row at its position."""
    r = _f64(rows).copy()
    d = r.shape[-1]
    flat = r.reshape(-1, d)
    pos = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, np.int64), flat.shape[:1]))
    lib().orc_rope(_p(flat), _p(pos), flat.shape[0], d, d_rope, float(theta))
    return flat.reshape(r.shape)


# ------------------------------------------------------------- compressor
def compress(x, z, bias, m, overlap, d_rope=0, theta=10000.0, pos0=0, x_tail=None, z_tail=None):
    """Token compressor ("DeepSeek V4 深度解析" §2 CSA step 1; HCA paragraph for m'=128).

    x [T, d], z [T], bias [m+overlap]; optional x_tail [overlap, d], z_tail [overlap].
    Returns (entries [T/m, d] fp64 unrounded, pooling weights [T/m, m+overlap])."""
    x, z, bias = _f64(x), _f64(z), _f64(bias)
    T, d = x.shape
    xt = None if x_tail is None else _f64(x_tail)
    zt = None if z_tail is None else _f64(z_tail)
    out = np.empty((T // m, d), np.float64)
    pw = np.empty((T // m, m + overlap), np.float64)
    rc = lib().orc_compress(_p(x), _p(xt), _p(z), _p(zt), _p(bias), T, d, m, overlap, d_rope,
                            float(theta), int(pos0), _p(out), _p(pw))
    if rc != 0:
        raise ValueError("compress: T must be a multiple of m")
    return out, pw


# ----------------------------------------------------- decode-time cache update
class CacheState:
    """One request's caches as tokens arrive one at a time ("DeepSeek V4 深度解析" §4, the
    KV cache for mixed attention): a state cache holding the sliding window's rows and the
    raw tail not yet enough to compress, and a compressed cache of CSA and HCA entries in
    blocks that each cover lcm(m, m') raw tokens.

    append() takes token t's raw (un-rotated) KV row x, its index-key row kx and its three
    pooling logits; an entry is emitted as soon as its last token has arrived, pooled
    exactly as the whole-sequence compressor pools it.  The window keeps the last W rows
    after RoPE at their own positions (the rows attention reads)."""

    def __init__(self, bias, biasI, biash, d_rope, m=4, overlap=2, mh=128, W=128, theta=10000.0):
        self.bias, self.biasI, self.biash = _f64(bias), _f64(biasI), _f64(biash)
        self.d_rope, self.m, self.overlap, self.mh, self.W, self.theta = d_rope, m, overlap, mh, W, theta
        self.t = 0
        self.raw, self.kraw, self.z, self.zI, self.zh = [], [], [], [], []   # the uncompressed tails
        self.window = []                                                      # (position, rotated row)
        self.csa, self.csa_keys, self.hca = [], [], []

    def append(self, x, kx, z, zI, zh):
        t = self.t
        x, kx = _f64(x), _f64(kx)
        self.raw.append(x)
        self.kraw.append(kx)
        self.z.append(float(z))
        self.zI.append(float(zI))
        self.zh.append(float(zh))
        self.window.append((t, rope(x[None], t, self.d_rope, self.theta)[0]))
        self.window = self.window[-self.W:]
        m, ov = self.m, self.overlap
        if (t + 1) % m == 0:                       # CSA entry j = t // m: tokens m*j - ov .. t
            j = t // m
            have = min(ov, m * j)                  # overlap rows that exist before the entry
            rows = np.array(self.raw[-(m + have):])
            krows = np.array(self.kraw[-(m + have):])
            zz, zzI = np.array(self.z[-(m + have):]), np.array(self.zI[-(m + have):])
            tail = (rows[:have], zz[:have]) if have else (None, None)
            ktail = (krows[:have], zzI[:have]) if have else (None, None)
            e, _ = compress(rows[have:], zz[have:], self.bias, m, ov, self.d_rope, self.theta, m * j, tail[0], tail[1])
            k, _ = compress(krows[have:], zzI[have:], self.biasI, m, ov, 0, self.theta, m * j, ktail[0], ktail[1])
            self.csa.append(e[0])
            self.csa_keys.append(k[0])
        if (t + 1) % self.mh == 0:                 # HCA entry h = t // mh: tokens mh*h .. t
            h = t // self.mh
            rows = np.array(self.raw[-self.mh:])
            zz = np.array(self.zh[-self.mh:])
            e, _ = compress(rows, zz, self.biash, self.mh, 0, self.d_rope, self.theta, self.mh * h)
            self.hca.append(e[0])
        # the tail keeps what the next entries still need: the overlap rows and the rows of
        # the incomplete CSA entry, and the rows of the incomplete HCA entry
        keep = max(ov + (t + 1) % m, (t + 1) % self.mh)
        self.raw, self.kraw = self.raw[-keep:] if keep else [], self.kraw[-keep:] if keep else []
        self.z, self.zI, self.zh = (self.z[-keep:] if keep else [], self.zI[-keep:] if keep else [],
                                    self.zh[-keep:] if keep else [])
        self.t = t + 1

    def blocks(self):
        """Complete compressed-cache blocks: each covers lcm(m, m') raw tokens."""
        return self.t // np.lcm(self.m, self.mh)


# ---------------------------------------------------------------- indexer
def index_scores_f32(qI, w, kI):
    """fp32 lightning-indexer scores in the fixed fma order ("DeepSeek V4 深度解析" §2 step 2).
    qI [H, dI], w [H], kI [N, dI] (fp32) -> score [N] fp32."""
    qI, w, kI = _f32(qI), _f32(w), _f32(kI)
    H, dI = qI.shape
    out = np.empty(kI.shape[0], np.float32)
    lib().orc_index_scores_f32(_p(qI), _p(w), _p(kI), kI.shape[0], H, dI, _p(out))
    return out


def index_scores_bf16(qI, w, kI):
    """bf16 inputs: per-head dot exact then rounded once to fp32; fp32 fma chain over heads."""
    qI, kI, w = _f64(qI), _f64(kI), _f32(w)
    H, dI = qI.shape
    out = np.empty(kI.shape[0], np.float32)
    lib().orc_index_scores_bf16(_p(qI), _p(w), _p(kI), kI.shape[0], H, dI, _p(out))
    return out


def index_scores_fp4(qI, w, k_packed, k_scales, round_bf16=True):
    """FP4 QK path ("DeepSeek V4 深度解析" §4; "V3 vs V4" page "FP4 为什么能无损"):
    qI [H, dI] (bf16 values) is quantised like the keys; scores rounded to bf16 (the
    same page: index scores in BF16), or the fp32 sum before that rounding."""
    qp, qs = quant_fp4(_f32(qI))
    w = _f32(w)
    kp, ks = np.ascontiguousarray(k_packed, np.uint8), np.ascontiguousarray(k_scales, np.uint8)
    H, dI = np.asarray(qI).shape
    out = np.empty(kp.shape[0], np.float64)
    lib().orc_index_scores_fp4(_p(qp), _p(qs), _p(w), _p(kp), _p(ks), kp.shape[0], H, dI, int(bool(round_bf16)),
                               _p(out))
    return out


def exact_dot_f32(a, b):
    a, b = _f64(a), _f64(b)
    return float(lib().orc_exact_dot_f32(_p(a), _p(b), a.size))


def n_avail(t, m, n_c):
    """Entries usable by a query at absolute position t: entry j is complete once
    token m*j+m-1 <= t.  t < 0 means decode (all entries)."""
    return n_c if t < 0 else min(n_c, (t + 1) // m)


# ------------------------------------------------------------------ top-k
def topk(score, k):
    """k largest by (score desc, index asc), returned ascending, -1 padded."""
    s = _f32(score)
    out = np.empty(k, np.int32)
    lib().orc_topk(_p(s), s.size, k, _p(out))
    return out


# -------------------------------------------------------------- attention
def mqa_rows(q, rows, scale, dv):
    """Shared-KV MQA of H query heads over one row set (one joint softmax)."""
    q, rows = _f64(q), _f64(rows)
    H, D = q.shape
    out = np.empty((H, dv), np.float64)
    lse = np.empty(H, np.float64)
    lib().orc_mqa_rows(_p(q), _p(rows), rows.shape[0], H, D, dv, float(scale), _p(out), _p(lse))
    return out, lse


def csa_attend(q, comp, idx, win, win_pos0, t, W, dv, scale):
    """CSA attention of one query ("DeepSeek V4 深度解析" §2 step 3): selected compressed
    rows (idx != -1) together with the window rows at positions [t-W+1, t]
    (t < 0: every row of win).  q [H, D]; comp [Nc, D]; win [Tw, D] (fp64 values)."""
    q, comp, win = _f64(q), _f64(comp), _f64(win)
    idx = np.ascontiguousarray(idx, np.int32)
    H, D = q.shape
    out = np.empty((H, dv), np.float64)
    lse = np.empty(H, np.float64)
    R = lib().orc_csa_attend(_p(q), _p(comp), comp.shape[0], _p(idx), idx.size, _p(win), win.shape[0],
                             int(win_pos0), int(t), W, H, D, dv, float(scale), _p(out), _p(lse))
    if R < 0:
        raise ValueError("csa_attend: index out of range")
    return out, lse


def hca_attend(q, comp, m, win, win_pos0, t, W, dv, scale):
    """HCA attention of one query ("DeepSeek V4 深度解析" §2 HCA paragraph): all
    available compressed rows plus the window, no selection."""
    q, comp, win = _f64(q), _f64(comp), _f64(win)
    H, D = q.shape
    out = np.empty((H, dv), np.float64)
    lse = np.empty(H, np.float64)
    lib().orc_hca_attend(_p(q), _p(comp), comp.shape[0], m, _p(win), win.shape[0], int(win_pos0),
                         int(t), W, H, D, dv, float(scale), _p(out), _p(lse))
    return out, lse


def group_oproj(o, Wg, Wo):
    """Grouped output projection ("DeepSeek V4 深度解析" §2 HCA paragraph: 分組輸出投影).
    o [H, dv]; Wg [G, (H/G)*dv, dg]; Wo [G*dg, hidden] -> y [hidden]."""
    o, Wg, Wo = _f64(o), _f64(Wg), _f64(Wo)
    H, dv = o.shape
    G, _, dg = Wg.shape
    hidden = Wo.shape[1]
    y = np.empty(hidden, np.float64)
    lib().orc_group_oproj(_p(o), _p(Wg), _p(Wo), H, dv, G, dg, hidden, _p(y))
    return y


def project_f32(h, W):
    """fp32 projection of hidden states ("DeepSeek V4 深度解析" §2, CSA steps 1-2: rows, logits,
    index queries and head weights are linear in the hidden state): out[t, c] is the fp32
    fma chain over i of h[t, i] * W[i, c], in order.  h [T, n], W [n, d] -> [T, d] float32."""
    h, W = _f32(h), _f32(W)
    T, n = h.shape
    d = W.shape[1]
    out = np.empty((T, d), np.float32)
    lib().orc_project_f32(_p(h), _p(W), T, n, d, _p(out))
    return out
