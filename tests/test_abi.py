"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/csa.h declares, and host validation rejects bad
arguments before any launch."""
import ctypes
import os
import re

import pytest

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return csa.load()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(csa_\w+)\s*\(", text)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "csa_compress" in names and "csa_decode_step" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(csa.EXPORTS) <= set(names)


def test_exports_are_c_symbols():
    out = os.popen(f"nm -D --defined-only {csa.LIB_PATH}").read()
    for n in declared_functions():
        assert re.search(rf"\bT {n}$", out, flags=re.M), f"{n} is not an extern \"C\" text symbol"


def _t(ptr=16, dtype=csa.CSA_BF16, scale=None, group=0):
    return csa.Tensor(ptr, scale, dtype, group)


def test_compress_rejects_bad_arguments(lib):
    C, Z, out = _t(), _t(), _t()
    st = lib.csa_compress(ctypes.byref(C), ctypes.byref(Z), 1, 64, 100, 4, ctypes.byref(out), 16, None, 0, None, None)
    assert st == 1 and b"d=100" in lib.csa_last_error() or b"shape" in lib.csa_last_error()
    bad = _t(ptr=18)  # not 16-byte aligned
    st = lib.csa_compress(ctypes.byref(bad), ctypes.byref(Z), 1, 64, 128, 4, ctypes.byref(out), 16, None, 0, None, None)
    assert st == 1 and b"aligned" in lib.csa_last_error()
    fp8_out = _t(dtype=csa.CSA_FP8_E4M3, scale=32, group=32)
    st = lib.csa_compress(ctypes.byref(C), ctypes.byref(Z), 1, 64, 128, 4, ctypes.byref(fp8_out), 16, None, 0, None,
                          None)
    assert st == 1 and b"scale_group" in lib.csa_last_error()
    st = lib.csa_compress(ctypes.byref(C), ctypes.byref(Z), 1, 64, 128, 4, ctypes.byref(out), 8, None, 0, None, None)
    assert st == 1 and b"out_rows" in lib.csa_last_error()


def test_index_topk_rejects_bad_arguments(lib):
    p = csa.params(4, 512, 128, 64, 64, 0, 128, 128)
    q, k = _t(), _t()
    st = lib.csa_index_topk(ctypes.byref(p), 4, ctypes.byref(q), 16, ctypes.byref(k), 1, 100, None, 16, 16, None, 16,
                            1 << 20, None)
    assert st == 1 and b"topk" in lib.csa_last_error()
    p.topk = 64
    st = lib.csa_index_topk(ctypes.byref(p), 4, ctypes.byref(q), 16, ctypes.byref(k), 1, 1000, None, 16, 16, None, 16,
                            64, None)
    assert st == 3 and b"workspace" in lib.csa_last_error()
    fp8k = _t(dtype=csa.CSA_FP8_E4M3, scale=None, group=128)
    st = lib.csa_index_topk(ctypes.byref(p), 4, ctypes.byref(q), 16, ctypes.byref(fp8k), 1, 1000, None, 16, 16, None, 16,
                            1 << 30, None)
    assert st == 1 and b"scales" in lib.csa_last_error()


def test_attention_rejects_bad_arguments(lib):
    p = csa.params(4, 512, 128, 64, 64, 64, 128, 64)  # swa_cap < window
    q, kv, out = _t(), _t(), _t()
    st = lib.csa_sparse_swa_attention(ctypes.byref(p), 2, ctypes.byref(q), ctypes.byref(kv), 1, 100, 16, 16, None, None,
                                      None, 16, None, None, ctypes.byref(out), None, 16, 1 << 30, None)
    assert st == 1 and b"swa_cap" in lib.csa_last_error()
    p.swa_cap = 128
    st = lib.csa_sparse_swa_attention(ctypes.byref(p), 2, ctypes.byref(q), ctypes.byref(kv), 1, 100, 16, 16, None, None,
                                      None, 16, None, None, ctypes.byref(out), None, 16, 1 << 30, None)
    assert st == 1 and b"swa_k" in lib.csa_last_error()


def test_workspace_size_grows_with_problem(lib):
    p = csa.params(4, 512, 128, 64, 64, 1024, 128, 128)
    a = csa.csa_workspace_size(p, 4, 262144)
    b = csa.csa_workspace_size(p, 8, 262144)
    # room for one fp32 score per visible entry and request (the many-query indexer path)
    assert a >= 4 * 262144 * 4 and b >= 8 * 262144 * 4
    p.topk = 0
    assert csa.csa_workspace_size(p, 4, 2048) > 0
    # many queries (chunked prefill: more queries than SMs)
    p.topk = 512
    assert csa.csa_workspace_size(p, 4096, 33792) >= 4096 * 33792 * 4


def test_pool_entry_points_reject_bad_arguments(lib):
    p = csa.params(4, 512, 128, 64, 64, 64, 128, 128)
    q, k = _t(), _t()
    ws = csa.csa_index_pool_workspace_size(p, 4, 262144, 8, 2048)
    # the Full layer keeps every score and every block maximum
    assert ws >= 4 * 262144 * 4 + 4 * (262144 // 8) * 4
    for block in (0, 3, 256):
        st = lib.csa_index_topk_pool(ctypes.byref(p), 4, ctypes.byref(q), 16, ctypes.byref(k), 1, 1000, None, 16,
                                     block, 64, 16, None, None, 16, 1 << 30, None)
        assert st == 1 and b"block" in lib.csa_last_error()
    st = lib.csa_index_topk_pool(ctypes.byref(p), 4, ctypes.byref(q), 16, ctypes.byref(k), 1, 1000, None, 16,
                                 8, 0, 16, None, None, 16, 1 << 30, None)
    assert st == 1 and b"pool_blocks" in lib.csa_last_error()
    st = lib.csa_index_topk_pool(ctypes.byref(p), 4, ctypes.byref(q), 16, ctypes.byref(k), 1, 1000, None, 16,
                                 8, 64, 16, None, None, 16, 64, None)
    assert st == 3 and b"workspace" in lib.csa_last_error()
    st = lib.csa_index_topk_reindex(ctypes.byref(p), 4, ctypes.byref(q), 16, ctypes.byref(k), 1, 1000, None, 16,
                                    None, 8, 64, 16, None, 16, 1 << 30, None)
    assert st == 1 and b"pool" in lib.csa_last_error()
    st = lib.csa_index_topk_reindex(ctypes.byref(p), 4, ctypes.byref(q), 16, ctypes.byref(k), 1, 1000, None, 16,
                                    16, 8, 64, 16, None, 16, 64, None)
    assert st == 3 and b"workspace" in lib.csa_last_error()
    p.topk = 0
    st = lib.csa_index_topk_reindex(ctypes.byref(p), 4, ctypes.byref(q), 16, ctypes.byref(k), 1, 1000, None, 16,
                                    16, 8, 64, 16, None, 16, 1 << 30, None)
    assert st == 1 and b"topk" in lib.csa_last_error()


def _decode_args(kv_dtype=csa.CSA_FP8_E4M3, kv_scale=32, kv_group=64):
    """A decode step's arguments that pass host validation (fake aligned
    device addresses: every case below changes one field so that the call
    returns before any launch)."""
    p = csa.params(4, 512, 128, 64, 64, 64, 128, 128)
    bf = lambda: _t()  # noqa: E731
    caches = csa.DecodeCaches(_t(dtype=kv_dtype, scale=kv_scale, group=kv_group),
                              _t(dtype=csa.CSA_FP8_E4M3, scale=32, group=128), bf(), bf(), bf(), bf(), 1024)
    tok = csa.DecodeToken(bf(), bf(), bf(), bf(), bf(), bf(), 16, None, bf())
    return p, caches, tok


def _decode(lib, p, caches, tok, batch=4, pos=16, out=None, ws=16, ws_bytes=64):
    out = out if out is not None else _t()
    return lib.csa_decode_step(ctypes.byref(p), batch, ctypes.byref(caches), ctypes.byref(tok), pos,
                               ctypes.byref(out), None, None, ws, ws_bytes, None)


def test_decode_step_rejects_bad_arguments(lib):
    p, caches, tok = _decode_args()
    # the valid arguments reach the workspace check, which a 64-byte workspace fails
    assert _decode(lib, p, caches, tok) == 3 and b"workspace" in lib.csa_last_error()
    assert _decode(lib, p, caches, tok, batch=0) == 0  # nothing to do, nothing launched
    assert _decode(lib, p, caches, tok, pos=None) == 1 and b"null" in lib.csa_last_error()
    p.window = 0
    assert _decode(lib, p, caches, tok) == 1 and b"window" in lib.csa_last_error()
    p, caches, tok = _decode_args()
    tok.w_ik = csa.Tensor(None, None, 0, 0)
    assert _decode(lib, p, caches, tok) == 1 and b"w_ik" in lib.csa_last_error()
    p, caches, tok = _decode_args()
    p.d_idx = 48  # the projection needs a multiple of 32
    st = _decode(lib, p, caches, tok)
    assert st in (1, 2) and b"d_idx" in lib.csa_last_error()
    p, caches, tok = _decode_args()
    tok.z = _t(dtype=csa.CSA_F32)
    assert _decode(lib, p, caches, tok) == 1 and b"one dtype" in lib.csa_last_error()
    p, caches, tok = _decode_args()
    caches.open_c = _t(dtype=csa.CSA_F32)
    assert _decode(lib, p, caches, tok) == 1 and b"open-block" in lib.csa_last_error()
    p, caches, tok = _decode_args()
    caches.kv = _t(dtype=csa.CSA_FP8_E4M3, scale=32, group=128)  # main-KV FP8 groups are 64 channels
    assert _decode(lib, p, caches, tok) == 1 and b"scale_group" in lib.csa_last_error()


def test_decode_step_mxfp4_layout_rules(lib):
    # MXFP4 main KV: one E4M3 scale byte per 16 elements, 16-byte aligned scales
    p, caches, tok = _decode_args(kv_dtype=csa.CSA_MXFP4_E2M1, kv_scale=32, kv_group=16)
    assert _decode(lib, p, caches, tok) == 3 and b"workspace" in lib.csa_last_error()
    p, caches, tok = _decode_args(kv_dtype=csa.CSA_MXFP4_E2M1, kv_scale=32, kv_group=32)
    assert _decode(lib, p, caches, tok) == 1 and b"scale_group must be 16" in lib.csa_last_error()
    p, caches, tok = _decode_args(kv_dtype=csa.CSA_MXFP4_E2M1, kv_scale=None, kv_group=16)
    assert _decode(lib, p, caches, tok) == 1 and b"scales" in lib.csa_last_error()
    p, caches, tok = _decode_args(kv_dtype=csa.CSA_MXFP4_E2M1, kv_scale=40, kv_group=16)
    assert _decode(lib, p, caches, tok) == 1 and b"aligned" in lib.csa_last_error()
    # rows must hold whole 32-element pairs of scale groups (16 bytes of codes)
    p, caches, tok = _decode_args(kv_dtype=csa.CSA_MXFP4_E2M1, kv_scale=32, kv_group=16)
    p.d = 48
    assert _decode(lib, p, caches, tok) == 1 and b"multiple of 16 bytes" in lib.csa_last_error()


def test_compress_mxfp4_output_rules(lib):
    C, Z = _t(), _t()
    bad_group = _t(dtype=csa.CSA_MXFP4_E2M1, scale=32, group=32)
    st = lib.csa_compress(ctypes.byref(C), ctypes.byref(Z), 1, 64, 128, 4, ctypes.byref(bad_group), 16, None, 0,
                          None, None)
    assert st == 1 and b"scale_group must be 16" in lib.csa_last_error()
    no_scale = _t(dtype=csa.CSA_MXFP4_E2M1, scale=None, group=16)
    st = lib.csa_compress(ctypes.byref(C), ctypes.byref(Z), 1, 64, 128, 4, ctypes.byref(no_scale), 16, None, 0,
                          None, None)
    assert st == 1 and b"scales" in lib.csa_last_error()


def test_topk_rejects_bad_arguments(lib):
    assert lib.csa_topk(16, 2, 64, 16, 0, 16, None, None, 0, None) == 1 and b"bad shape" in lib.csa_last_error()
    assert lib.csa_topk(16, -1, 64, 16, 4, 16, None, None, 0, None) == 1
    assert lib.csa_topk(16, 0, 64, 16, 4, 16, None, None, 0, None) == 0  # no rows: nothing launched
    assert lib.csa_topk(None, 2, 64, 16, 4, 16, None, None, 0, None) == 1 and b"null" in lib.csa_last_error()
    assert lib.csa_topk(16, 2, 64, None, 4, 16, None, None, 0, None) == 1
    # the multi-CTA control words grow with the rows
    assert csa.csa_topk_workspace_size(8) >= csa.csa_topk_workspace_size(1) > 0


def test_key_counts_beyond_int32_are_rejected(lib):
    """The keys of one query (selection or, dense, the cache's rows, plus the
    window) are counted in 64 bits: a count past 2^31 - 1 is refused, never
    wrapped into a small positive number that would pass the workspace or
    scratch checks."""
    p = csa.params(4, 512, 128, 64, 64, 0, 128, 128)  # dense (HCA)
    huge = (1 << 31) - 64
    assert csa.csa_workspace_size(p, 2, huge) == 0
    q, kv, out = _t(), _t(), _t()
    sk, sv = _t(), _t()
    st = lib.csa_sparse_swa_attention(ctypes.byref(p), 2, ctypes.byref(q), ctypes.byref(kv), 1, huge, None, 16, None,
                                      ctypes.byref(sk), ctypes.byref(sv), 16, None, None, ctypes.byref(out), None, 16,
                                      1 << 40, None)
    assert st == 1 and b"2^31" in lib.csa_last_error()
    st = lib.csa_sparse_swa_attention_noalloc(ctypes.byref(p), 2, ctypes.byref(q), ctypes.byref(kv), 1, huge, None, 16,
                                              None, ctypes.byref(sk), ctypes.byref(sv), 16, None, None,
                                              ctypes.byref(out), None, None)
    assert st == 1 and b"2^31" in lib.csa_last_error()
    p2, caches, tok = _decode_args()
    p2.topk = 0
    caches.cap = huge
    assert _decode(lib, p2, caches, tok) == 1 and b"2^31" in lib.csa_last_error()


def test_noalloc_validates_params_before_sizing_its_scratch(lib):
    """Bad parameters give the status csa_sparse_swa_attention gives
    (CSA_ERR_INVALID_ARG), not a capacity error from a scratch size computed
    out of them; the previous call's message does not linger."""
    q, kv, out = _t(), _t(), _t()
    for field, value in (("h_q", -64), ("d", -512), ("window", -1)):
        p = csa.params(4, 512, 128, 64, 64, 64, 128, 128)
        setattr(p, field, value)
        st = lib.csa_sparse_swa_attention_noalloc(ctypes.byref(p), 2, ctypes.byref(q), ctypes.byref(kv), 1, 100, 16,
                                                  16, None, None, None, 16, None, None, ctypes.byref(out), None, None)
        assert st == 1 and b"params" in lib.csa_last_error(), (field, lib.csa_last_error())
