"""The C ABI without a GPU: the library builds, loads, exports every function that
include/lcs.h declares, and rejects bad arguments before touching the device."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lcs.h")


@pytest.fixture(scope="module")
def L():
    from long_context_sparse_06_b200 import build
    build.build()
    import long_context_sparse_06_b200 as lcs
    return lcs


def declared():
    txt = open(HEADER).read()
    return re.findall(r"LCS_API\s+(?:const\s+)?[a-z0-9_]+\**\s+\**([a-z_0-9]+)\s*\(", txt)


def test_header_declares_the_boundary():
    names = set(declared())
    for n in ("csa_compress", "hca_compress", "csa_index_topk", "csa_attend", "hca_attend", "decode_fused",
              "group_oproj", "lcs_workspace_size", "lcs_status"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    lib = C.CDLL(L.LIB_PATH)
    for n in declared():
        assert hasattr(lib, n), n


def test_validation_without_device(L):
    lib = L.lib()
    P = 4096   # a fake, aligned, never-dereferenced address
    # null pointers / bad shapes
    assert lib.csa_compress(None, L.BF16, 1, 8, 576, None, None, P, P, 4, 2, 64, 1e4, 0, P, L.BF16, None) == -1
    assert lib.csa_compress(P, L.BF16, 1, 10, 576, None, None, P, P, 4, 2, 64, 1e4, 0, P, L.BF16, None) == -1
    assert lib.csa_compress(P, 7, 1, 8, 576, None, None, P, P, 4, 2, 64, 1e4, 0, P, L.BF16, None) == -2
    assert lib.hca_compress(P, L.BF16, 1, 256, 576, P, P, 0, 0, 1e4, 0, P, L.BF16, None) == -1
    # indexer: Q > 1 needs positions; unsupported head counts on the tensor-core path
    assert lib.csa_index_topk(P, L.BF16, P, P, L.BF16, 1, 2, 100, 64, 128, None, 4, 8, L.F32, P, None, P, 1 << 20,
                              None) == -1
    assert lib.csa_index_topk(P, L.BF16, P, P, L.BF16, 1, 1, 100, 32, 128, None, 4, 8, L.F32, P, None, P, 1 << 20,
                              None) == -2
    # workspace too small
    assert lib.csa_index_topk(P, L.BF16, P, P, L.BF16, 1, 1, 100, 64, 128, None, 4, 8, L.F32, P, None, P, 16,
                              None) == -6
    # attention: tensor-core shapes only for bf16 / FP8
    assert lib.csa_attend(P, L.BF16, P, P, L.BF16, 1, 1, 10, 4, P, 4, None, None, 128, 32, 576, 512, 0.1, P, L.BF16,
                          None, P, 1 << 20, None) == -2
    assert lib.hca_attend(P, L.BF16, P, None, L.BF16, 1, 1, 10, 4, None, None, 128, 128, 64, 576, 512, 0.1, P,
                          L.BF16, None, P, 1 << 20, None) == -1
    # row buffers off a 16-byte boundary (TMA); more rows than int32 row coordinates reach
    for kv in (L.BF16, L.KV_FP8):
        assert lib.hca_attend(P, L.BF16, P + 8, P, kv, 1, 1, 10, 4, None, None, 128, 128, 64, 576, 512, 0.1, P,
                              L.BF16, None, P, 1 << 20, None) == -1
        assert lib.hca_attend(P, L.BF16, P, P + 8, kv, 1, 1, 10, 4, None, None, 128, 128, 64, 576, 512, 0.1, P,
                              L.BF16, None, P, 1 << 20, None) == -1
        assert lib.hca_attend(P, L.BF16, P, P, kv, 2, 1, 1 << 30, 4, None, None, 128, 128, 64, 576, 512, 0.1, P,
                              L.BF16, None, P, 1 << 20, None) == -2
        assert lib.csa_attend(P, L.BF16, P, P, kv, 1 << 20, 1, 1 << 11, 4, P, 4, None, None, 128, 64, 576, 512, 0.1,
                              P, L.BF16, None, P, 1 << 20, None) == -2
    assert lib.decode_fused(5, 1, P, L.BF16, P, P, L.BF16, 10, 4, 64, 576, 512, 0.1, P, L.BF16, P, P, L.BF16, 64, 128,
                            8, L.F32, P, L.BF16, None, None, P, 1 << 20, None) == -1
    assert lib.group_oproj(P, 4, 8, 48, P, 3, 64, P, 256, P, None) == -1
    assert lib.lcs_quant_fp4(P, 4, 48, P, None) == -1
    assert lib.lcs_workspace_size(99, 1, 1, 1, 1, 1, 64, 512, 0) == -1
    assert lib.lcs_workspace_size(L.OP_DECODE, 32, 1, 32768, 128, 512, 64, 512, L.F32) > 32 * 32768 * 4
    assert lib.lcs_error_string(-4) == b"device-side wait timed out"


def test_valid_call_without_device_fails_loudly(L):
    """No CPU fallback: a well-formed call on a machine without an sm_100 device
    returns LCS_ERR_CUDA."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    lib = L.lib()
    P = 4096
    assert lib.lcs_quant_fp4(P, 4, 64, P, None) == -3
    assert lib.csa_compress(P, L.BF16, 1, 8, 576, None, None, P, P, 4, 2, 64, 1e4, 0, P, L.BF16, None) == -3


def _header_arg_counts():
    """Parameter count of every declaration in include/lcs.h (comments stripped)."""
    txt = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"LCS_API\s+(?:const\s+)?[a-z0-9_]+\**\s+\**([a-z_0-9]+)\s*\(([^)]*)\)", txt):
        params = [p for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        out[m.group(1)] = len(params)
    return out


def _ctype_of(param):
    """The ctypes type a C parameter declaration needs (x86-64: a 32-bit int passed for an
    int64_t leaves the register's upper half undefined)."""
    p = param.strip()
    if "*" in p or p.startswith("cudaStream_t"):
        return C.c_void_p
    kind = p.split()[0] if not p.startswith("const ") else p.split()[1]
    return {"int64_t": C.c_int64, "int": C.c_int, "float": C.c_float, "size_t": C.c_size_t}[kind]


def test_binding_signatures_match_the_header(L):
    """Every function the Python binding declares to ctypes takes the arguments of its C
    declaration, in number and in kind: a mismatch would corrupt the call silently."""
    lib = L.lib()
    counts = _header_arg_counts()
    assert len(counts) == len(declared())
    txt = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    checked = 0
    for m in re.finditer(r"LCS_API\s+(?:const\s+)?[a-z0-9_]+\**\s+\**([a-z_0-9]+)\s*\(([^)]*)\)", txt):
        name, params = m.group(1), [q for q in m.group(2).split(",") if q.strip() and q.strip() != "void"]
        fn = getattr(lib, name)
        assert fn.argtypes is not None, f"{name} is not bound"
        assert len(fn.argtypes) == counts[name], f"{name}: binding has {len(fn.argtypes)} arguments, header {counts[name]}"
        for i, (q, t) in enumerate(zip(params, fn.argtypes)):
            assert t == _ctype_of(q), f"{name} argument {i} ({q.strip()}): binding {t.__name__}"
        checked += 1
    assert checked == len(counts)
