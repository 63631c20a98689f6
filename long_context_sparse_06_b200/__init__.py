"""B200-native CSA / HCA compressed attention (DeepSeek-V4 hot path).

Thin Python binding over ``liblcs.so`` (the C ABI declared in ``include/lcs.h``).
Every function here only marshals arguments -- device pointers of torch
tensors, the current CUDA stream, workspace buffers -- and calls the library
function of the same name; all arithmetic runs in the library's CUDA kernels.
There is no CPU path: without the built library or a CUDA device every call
raises.
"""
from __future__ import annotations

import ctypes as C
import os

__all__ = [
    "F32", "BF16", "KV_FP8", "FP4", "MODE_CSA", "MODE_HCA", "LcsError", "lib",
    "csa_compress", "hca_compress", "lcs_compress_proj", "csa_index_topk", "csa_index_topk_proj", "lcs_topk", "csa_attend", "hca_attend",
    "decode_fused", "lcs_cache_append", "lcs_cp_candidates", "lcs_cp_select", "lcs_attn_merge", "group_oproj", "lcs_rope", "lcs_quant_kv_fp8", "lcs_quant_fp4",
    "lcs_workspace_size", "lcs_status", "lcs_clear_status", "lcs_selftest_wait", "workspace", "kv_fp8_row_bytes",
]

F32, BF16, KV_FP8, FP4 = 0, 1, 2, 3
MODE_CSA, MODE_HCA = 0, 1
OP_INDEX_TOPK, OP_ATTEND, OP_DECODE, OP_TOPK, OP_CP_SELECT = 1, 2, 3, 4, 5
# return codes (include/lcs.h)
LCS_OK, LCS_ERR_INVALID, LCS_ERR_UNSUPPORTED, LCS_ERR_CUDA = 0, -1, -2, -3
LCS_ERR_TIMEOUT, LCS_ERR_DEVICE, LCS_ERR_WORKSPACE, LCS_ERR_TOO_LARGE = -4, -5, -6, -7

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblcs.so")

_lib = None


class LcsError(RuntimeError):
    def __init__(self, name, code):
        msg = lib().lcs_error_string(code).decode() if _lib is not None else str(code)
        super().__init__(f"{name}: {msg} ({code})")
        self.code = code


def lib():
    """Load liblcs.so (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"liblcs.so not built ({LIB_PATH}); run __graft_entry__.build()")
        L = C.CDLL(LIB_PATH)
        P, I, I64, F, SZ = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t
        sig = {
            "csa_compress": [P, I, I64, I64, I, P, P, P, P, I, I, I, F, I64, P, I, P],
            "hca_compress": [P, I, I64, I64, I, P, P, I, I, F, I64, P, I, P],
            "csa_index_topk": [P, I, P, P, I, I64, I64, I64, I, I, P, I, I, I, P, P, P, SZ, P],
            "lcs_topk": [P, I, I64, I64, I64, P, I, I, P, P, SZ, P],
            "csa_attend": [P, I, P, P, I, I64, I64, I64, I64, P, I, P, P, I, I, I, I, F, P, I, P, P, SZ, P],
            "csa_attend_noalloc": [P, I, P, P, I, I64, I64, I64, I64, P, I, P, P, I, I, I, I, F, P, I, P, P, P],
            "hca_attend": [P, I, P, P, I, I64, I64, I64, I64, P, P, I, I, I, I, I, F, P, I, P, P, SZ, P],
            "lcs_cache_append": [I64, P, P, P, I, P, P, P, P, P, P, I, I, I, F, P, P, P, I, P, P, P, I64, I64, I, I,
                                 P, SZ, P],
            "lcs_cp_candidates": [P, I, I64, I64, P, I, I64, P, P, P],
            "lcs_compress_proj": [P, I, I64, I64, I, P, P, I, P, P, I, I, I, F, I64, P, I, P],
            "csa_index_topk_proj": [P, I, P, P, P, I64, I64, I64, I, I, P, I, I, P, P, P, SZ, P],
            "lcs_cp_select": [P, P, I, I64, I, I64, I64, P, P, P, SZ, P],
            "lcs_attn_merge": [P, P, I, I64, I, P, I, P, P],
            "decode_fused": [I, I64, P, I, P, P, I, I64, I64, I, I, I, F, P, I, P, P, I, I, I, I, I, P, I, P, P, P,
                             SZ, P],
            "group_oproj": [P, I64, I, I, P, I, I, P, I, P, P],
            "lcs_rope": [P, I, I64, I, I, F, P, P],
            "lcs_quant_kv_fp8": [P, I64, I, I, P, P],
            "lcs_quant_fp4": [P, I64, I, P, P],
            "lcs_status": [P, P],
            "lcs_clear_status": [P, P],
            "lcs_selftest_wait": [I, P, SZ, P, P],
            "lcs_set_stage_events": [P, I],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = I
        L.lcs_workspace_size.argtypes = [I, I64, I64, I64, I64, I, I, I, I]
        L.lcs_workspace_size.restype = I64
        L.lcs_error_string.argtypes = [I]
        L.lcs_error_string.restype = C.c_char_p
        _lib = L
    return _lib


def _torch():
    import torch
    return torch


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("liblcs takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("liblcs takes contiguous tensors only")
    return t.data_ptr()


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dt(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def _call(name, *args):
    rc = getattr(lib(), name)(*args)
    if rc != 0:
        raise LcsError(name, rc)


def kv_fp8_row_bytes(d_c=512, d_r=64):
    return d_c + 2 * d_r + 4 * (d_c // 128)


def lcs_workspace_size(op, B=0, Q=1, N_c=0, Tw=0, k=0, H=64, d_v=512, score_dtype=F32):
    n = lib().lcs_workspace_size(op, B, Q, N_c, Tw, k, H, d_v, score_dtype)
    if n < 0:
        raise ValueError("lcs_workspace_size: invalid sizes")
    return n


def workspace(nbytes, device="cuda"):
    """A zeroed, 256-byte-aligned device workspace of at least nbytes."""
    torch = _torch()
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def lcs_status(ws, stream=None):
    return lib().lcs_status(_ptr(ws), _stream(stream))


def lcs_clear_status(ws, stream=None):
    _call("lcs_clear_status", _ptr(ws), _stream(stream))


def lcs_selftest_wait(budget_us, ws, out, stream=None):
    """Runs the bounded-wait self-test; out is a 4-element int64 device tensor."""
    _call("lcs_selftest_wait", int(budget_us), _ptr(ws), ws.numel() * ws.element_size(), _ptr(out), _stream(stream))


# ---------------------------------------------------------------- compressor
def csa_compress(x, z, bias, m=4, overlap=2, d_rope=0, rope_theta=10000.0, pos0=0, x_tail=None, z_tail=None,
                 out_dtype=None, out=None, stream=None):
    """x [B,T,d] (fp32/bf16), z [B,T] fp32, bias [m+overlap] -> [B,T/m,d]."""
    torch = _torch()
    B, T, d = x.shape
    od = out_dtype if out_dtype is not None else x.dtype
    if out is None:
        out = torch.empty((B, T // m, d), dtype=od, device=x.device)
    _call("csa_compress", _ptr(x), _dt(x), B, T, d, _ptr(x_tail), _ptr(z_tail), _ptr(z), _ptr(bias), m, overlap,
          d_rope, rope_theta, pos0, _ptr(out), _dt(out), _stream(stream))
    return out


def hca_compress(x, z, bias, m=128, d_rope=0, rope_theta=10000.0, pos0=0, out_dtype=None, out=None, stream=None):
    torch = _torch()
    B, T, d = x.shape
    od = out_dtype if out_dtype is not None else x.dtype
    if out is None:
        out = torch.empty((B, T // m, d), dtype=od, device=x.device)
    _call("hca_compress", _ptr(x), _dt(x), B, T, d, _ptr(z), _ptr(bias), m, d_rope, rope_theta, pos0, _ptr(out),
          _dt(out), _stream(stream))
    return out


def lcs_compress_proj(h, Wx, wz, bias, m=4, overlap=2, d_rope=0, rope_theta=10000.0, pos0=0, h_tail=None,
                      out_dtype=None, out=None, stream=None):
    """h [B,T,hidden] (fp32/bf16), Wx [hidden,d] (h's dtype), wz [hidden] fp32 -> [B,T/m,d]."""
    torch = _torch()
    B, T, hidden = h.shape
    d = Wx.shape[1]
    if out is None:
        out = torch.empty((B, T // m, d), dtype=out_dtype or h.dtype, device=h.device)
    _call("lcs_compress_proj", _ptr(h), _dt(h), B, T, hidden, _ptr(h_tail), _ptr(Wx), d, _ptr(wz), _ptr(bias), m,
          overlap, d_rope, rope_theta, pos0, _ptr(out), _dt(out), _stream(stream))
    return out


# ------------------------------------------------------------------- indexer
def csa_index_topk_proj(h, W_qI, W_w, kI, k, H_I, q_pos=None, m=4, want_scores=False, ws=None, stream=None):
    """h [B,Q,hidden] fp32, W_qI [hidden,H_I*d_I], W_w [hidden,H_I], kI [B,N_c,d_I] fp32 ->
    idx [B,Q,k] (and the scores [B,Q,N_c])."""
    torch = _torch()
    B, Q, hidden = h.shape
    N_c, d_I = kI.shape[1], kI.shape[2]
    idx = torch.empty((B, Q, k), dtype=torch.int32, device=h.device)
    scores = torch.empty((B, Q, N_c), dtype=torch.float32, device=h.device) if want_scores else None
    if ws is None:
        ws = workspace(lcs_workspace_size(OP_INDEX_TOPK, B, Q, N_c, 0, k), h.device)
    _call("csa_index_topk_proj", _ptr(h), hidden, _ptr(W_qI), _ptr(W_w), _ptr(kI), B, Q, N_c, H_I, d_I, _ptr(q_pos), m,
          k, _ptr(idx), _ptr(scores), _ptr(ws), ws.numel(), _stream(stream))
    return (idx, scores) if want_scores else idx


def csa_index_topk(qI, w, kI, k, N_c=None, kI_dtype=None, q_pos=None, m=4, score_dtype=None, want_scores=False,
                   ws=None, stream=None):
    """qI [B,Q,H_I,d_I]; w [B,Q,H_I]; kI [B,N_c,d_I] (fp32/bf16) or FP4 planes (uint8).
    Returns idx [B,Q,k] int32 (and the scores [B,Q,N_c] if want_scores)."""
    torch = _torch()
    B, Q, H_I, d_I = qI.shape
    if kI_dtype is None:
        kI_dtype = _dt(kI)
    if N_c is None:
        N_c = kI.shape[1]
    if score_dtype is None:
        score_dtype = BF16 if kI_dtype == FP4 else F32
    idx = torch.empty((B, Q, k), dtype=torch.int32, device=qI.device)
    scores = None
    if want_scores:
        scores = torch.empty((B, Q, N_c), dtype=torch.bfloat16 if score_dtype == BF16 else torch.float32,
                             device=qI.device)
    if ws is None:
        ws = workspace(lcs_workspace_size(OP_INDEX_TOPK, B, Q, N_c, 0, k, score_dtype=score_dtype), qI.device)
    _call("csa_index_topk", _ptr(qI), _dt(qI), _ptr(w), _ptr(kI), kI_dtype, B, Q, N_c, H_I, d_I, _ptr(q_pos), m, k,
          score_dtype, _ptr(idx), _ptr(scores), _ptr(ws), ws.numel(), _stream(stream))
    return (idx, scores) if want_scores else idx


def lcs_topk(scores, k, q_pos=None, m=4, ws=None, stream=None):
    torch = _torch()
    B, Q, N_c = scores.shape
    idx = torch.empty((B, Q, k), dtype=torch.int32, device=scores.device)
    if ws is None:
        ws = workspace(lcs_workspace_size(OP_TOPK), scores.device)
    _call("lcs_topk", _ptr(scores), _dt(scores), B, Q, N_c, _ptr(q_pos), m, k, _ptr(idx), _ptr(ws), ws.numel(),
          _stream(stream))
    return idx


# ----------------------------------------------------------------- attention
def _attend_common(q, comp, win, kv_dtype, d_v):
    B, Q, H, D = q.shape
    if kv_dtype is None:
        kv_dtype = _dt(comp)
    N_c = comp.shape[1]
    Tw = win.shape[1] if win is not None else 0
    return B, Q, H, D, kv_dtype, N_c, Tw


def csa_attend(q, comp, win, idx, d_v, scale, kv_dtype=None, q_pos=None, win_pos0=None, W=128, want_lse=False,
               out_dtype=None, ws=None, stream=None):
    """q [B,Q,H,D]; comp [B,N_c,row]; win [B,Tw,row]; idx [B,Q,k] -> out [B,Q,H,d_v] (and lse)."""
    torch = _torch()
    B, Q, H, D, kv_dtype, N_c, Tw = _attend_common(q, comp, win, kv_dtype, d_v)
    k = idx.shape[-1]
    out = torch.empty((B, Q, H, d_v), dtype=out_dtype or q.dtype, device=q.device)
    lse = torch.empty((B, Q, H), dtype=torch.float32, device=q.device) if want_lse else None
    if ws is None:
        ws = workspace(lcs_workspace_size(OP_ATTEND, B, Q, N_c, Tw, k, H, d_v), q.device)
    _call("csa_attend", _ptr(q), _dt(q), _ptr(comp), _ptr(win), kv_dtype, B, Q, N_c, Tw, _ptr(idx), k, _ptr(q_pos),
          _ptr(win_pos0), W, H, D, d_v, scale, _ptr(out), _dt(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    return (out, lse) if want_lse else out


def csa_attend_noalloc(q, comp, win, idx, d_v, scale, kv_dtype=None, q_pos=None, win_pos0=None, W=128,
                       want_lse=False, out=None, out_dtype=None, status_out=None, stream=None):
    """csa_attend on the library's fixed per-device scratch: for callers that cannot give
    the library device memory (an engine whose HBM is all reserved for its KV-cache pool,
    a host program with no device allocator).  Pass `out` (and `status_out`, an int32
    device tensor of one element) to keep this wrapper allocation-free as well.  Calls
    that overlap in time on one device race on the shared scratch."""
    torch = _torch()
    B, Q, H, D, kv_dtype, N_c, Tw = _attend_common(q, comp, win, kv_dtype, d_v)
    k = idx.shape[-1]
    if out is None:
        out = torch.empty((B, Q, H, d_v), dtype=out_dtype or q.dtype, device=q.device)
    lse = torch.empty((B, Q, H), dtype=torch.float32, device=q.device) if want_lse else None
    _call("csa_attend_noalloc", _ptr(q), _dt(q), _ptr(comp), _ptr(win), kv_dtype, B, Q, N_c, Tw, _ptr(idx), k,
          _ptr(q_pos), _ptr(win_pos0), W, H, D, d_v, scale, _ptr(out), _dt(out), _ptr(lse), _ptr(status_out),
          _stream(stream))
    return (out, lse) if want_lse else out


def hca_attend(q, comp, win, d_v, scale, kv_dtype=None, q_pos=None, win_pos0=None, m=128, W=128, want_lse=False,
               out_dtype=None, ws=None, stream=None):
    torch = _torch()
    B, Q, H, D, kv_dtype, N_c, Tw = _attend_common(q, comp, win, kv_dtype, d_v)
    out = torch.empty((B, Q, H, d_v), dtype=out_dtype or q.dtype, device=q.device)
    lse = torch.empty((B, Q, H), dtype=torch.float32, device=q.device) if want_lse else None
    if ws is None:
        ws = workspace(lcs_workspace_size(OP_ATTEND, B, Q, N_c, Tw, 0, H, d_v), q.device)
    _call("hca_attend", _ptr(q), _dt(q), _ptr(comp), _ptr(win), kv_dtype, B, Q, N_c, Tw, _ptr(q_pos),
          _ptr(win_pos0), m, W, H, D, d_v, scale, _ptr(out), _dt(out), _ptr(lse), _ptr(ws), ws.numel(),
          _stream(stream))
    return (out, lse) if want_lse else out


def decode_fused(mode, q, comp, win, d_v, scale, kv_dtype=None, qI=None, w=None, kI=None, kI_dtype=None, k=0,
                 score_dtype=None, out=None, out_dtype=None, want_lse=False, idx_out=None, ws=None, stream=None):
    """One decode step (Q = 1 per request).  q [B,H,D]; comp [B,N_c,row]; win [B,Tw,row];
    CSA: qI [B,H_I,d_I], w [B,H_I], kI [B,N_c,d_I] or FP4 planes.  Returns out [B,H,d_v]."""
    torch = _torch()
    B, H, D = q.shape
    if kv_dtype is None:
        kv_dtype = _dt(comp)
    N_c = comp.shape[1]
    Tw = win.shape[1]
    H_I = d_I = 0
    qI_dt = F32
    if mode == MODE_CSA:
        H_I, d_I = qI.shape[-2], qI.shape[-1]
        qI_dt = _dt(qI)
        if kI_dtype is None:
            kI_dtype = _dt(kI)
        if score_dtype is None:
            score_dtype = BF16 if kI_dtype == FP4 else F32
    else:
        kI_dtype = kI_dtype if kI_dtype is not None else F32
        score_dtype = score_dtype if score_dtype is not None else F32
    if out is None:
        out = torch.empty((B, H, d_v), dtype=out_dtype or q.dtype, device=q.device)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if want_lse else None
    if ws is None:
        ws = workspace(lcs_workspace_size(OP_DECODE, B, 1, N_c, Tw, k, H, d_v, score_dtype), q.device)
    _call("decode_fused", mode, B, _ptr(q), _dt(q), _ptr(comp), _ptr(win), kv_dtype, N_c, Tw, H, D, d_v, scale,
          _ptr(qI), qI_dt, _ptr(w), _ptr(kI), kI_dtype, H_I, d_I, k, score_dtype, _ptr(out), _dt(out), _ptr(lse),
          _ptr(idx_out), _ptr(ws), ws.numel(), _stream(stream))
    return (out, lse) if want_lse else out


# ------------------------------------------------------- decode cache update
def lcs_cache_append(pos, x, kx, z, zI, zh, bias, biasI, biash, raw, logits, win, comp, kI, hca, d_rope=64,
                     rope_theta=10000.0, win_dtype=None, kv_dtype=None, kI_dtype=None, N_c=None, ws=None,
                     stream=None):
    """Appends one token per request (pos [B] int64; negative: no token for that request).
    x [B,D], kx [B,d_I] (fp32/bf16); z, zI, zh [B]; rings raw [B,128,D+d_I], logits
    [B,3,128]; caches win [B,128,row], comp [B,N_c,row], kI [B,N_c,d_I] or FP4 planes,
    hca [B,N_h,row].  The storage dtypes default to the tensors' own (uint8 rows: FP8 KV)."""
    B, D = x.shape
    d_I = kx.shape[1]
    u8 = _torch().uint8
    if kv_dtype is None:
        kv_dtype = KV_FP8 if comp.dtype == u8 else _dt(comp)
    if win_dtype is None:
        win_dtype = KV_FP8 if win.dtype == u8 else _dt(win)
    if kI_dtype is None:
        kI_dtype = FP4 if kI.dtype == u8 else _dt(kI)
    if N_c is None:
        N_c = comp.shape[1]
    if ws is None:
        ws = workspace(256, x.device)
    _call("lcs_cache_append", B, _ptr(pos), _ptr(x), _ptr(kx), _dt(x), _ptr(z), _ptr(zI), _ptr(zh), _ptr(bias),
          _ptr(biasI), _ptr(biash), D, d_rope, d_I, rope_theta, _ptr(raw), _ptr(logits), _ptr(win), win_dtype,
          _ptr(comp), _ptr(kI), _ptr(hca), N_c, hca.shape[1], kv_dtype, kI_dtype, _ptr(ws), ws.numel(),
          _stream(stream))
    return ws


# ------------------------------------------------- context parallelism (one long request)
def lcs_cp_candidates(scores, idx_local, offset, stream=None):
    """scores [B, S] (fp32/bf16), idx_local [B, k] -> (cand_score [B, k] fp32, cand_idx [B, k] int32)."""
    torch = _torch()
    B, S = scores.shape
    k = idx_local.shape[-1]
    cs = torch.empty((B, k), dtype=torch.float32, device=scores.device)
    ci = torch.empty((B, k), dtype=torch.int32, device=scores.device)
    _call("lcs_cp_candidates", _ptr(scores), _dt(scores), B, S, _ptr(idx_local), k, offset, _ptr(cs), _ptr(ci),
          _stream(stream))
    return cs, ci


def lcs_cp_select(cand_score, cand_idx, offset, S, ws=None, stream=None):
    """cand_score, cand_idx [G, B, k] -> (idx_global [B, k], idx_local [B, k])."""
    torch = _torch()
    G, B, k = cand_score.shape
    ig = torch.empty((B, k), dtype=torch.int32, device=cand_score.device)
    il = torch.empty((B, k), dtype=torch.int32, device=cand_score.device)
    if ws is None:
        ws = workspace(lcs_workspace_size(OP_CP_SELECT, B, G, 0, 0, k), cand_score.device)
    _call("lcs_cp_select", _ptr(cand_score), _ptr(cand_idx), G, B, k, offset, S, _ptr(ig), _ptr(il), _ptr(ws),
          ws.numel(), _stream(stream))
    return ig, il


def lcs_attn_merge(o, lse, out_dtype=None, want_lse=False, stream=None):
    """o [G, ..., d_v] fp32, lse [G, ...] fp32 -> out [..., d_v] (and the merged lse)."""
    torch = _torch()
    G = o.shape[0]
    d_v = o.shape[-1]
    rows = lse[0].numel()
    out = torch.empty(o.shape[1:], dtype=out_dtype or torch.float32, device=o.device)
    lo = torch.empty(lse.shape[1:], dtype=torch.float32, device=o.device) if want_lse else None
    _call("lcs_attn_merge", _ptr(o), _ptr(lse), G, rows, d_v, _ptr(out), _dt(out), _ptr(lo), _stream(stream))
    return (out, lo) if want_lse else out


# --------------------------------------------------------------------- misc
def group_oproj(o, Wg, Wo, out=None, stream=None):
    """o [T,H,d_v] fp32; Wg [G,(H/G)*d_v,d_g]; Wo [G*d_g,hidden] -> y [T,hidden]."""
    torch = _torch()
    T, H, d_v = o.shape
    G, _, d_g = Wg.shape
    hidden = Wo.shape[1]
    if out is None:
        out = torch.empty((T, hidden), dtype=torch.float32, device=o.device)
    _call("group_oproj", _ptr(o), T, H, d_v, _ptr(Wg), G, d_g, _ptr(Wo), hidden, _ptr(out), _stream(stream))
    return out


def lcs_rope(rows, pos, d_rope, rope_theta=10000.0, stream=None):
    """In-place RoPE of the last d_rope dims of rows [..., d] at positions pos [n] (int64)."""
    d = rows.shape[-1]
    n = rows.numel() // d
    _call("lcs_rope", _ptr(rows), _dt(rows), n, d, d_rope, rope_theta, _ptr(pos), _stream(stream))
    return rows


def lcs_quant_kv_fp8(x, d_c=512, d_r=64, out=None, stream=None):
    torch = _torch()
    lead = x.shape[:-1]
    n = x.numel() // (d_c + d_r)
    if out is None:
        out = torch.empty(tuple(lead) + (kv_fp8_row_bytes(d_c, d_r),), dtype=torch.uint8, device=x.device)
    _call("lcs_quant_kv_fp8", _ptr(x), n, d_c, d_r, _ptr(out), _stream(stream))
    return out


def lcs_quant_fp4(x, out=None, stream=None):
    """x [..., d] fp32 -> uint8 [n*d/2 + n*d/32] (packed plane, then scale plane)."""
    torch = _torch()
    d = x.shape[-1]
    n = x.numel() // d
    if out is None:
        out = torch.empty(n * d // 2 + n * d // 32, dtype=torch.uint8, device=x.device)
    _call("lcs_quant_fp4", _ptr(x), n, d, _ptr(out), _stream(stream))
    return out
