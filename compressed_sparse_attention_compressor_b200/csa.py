"""Python binding of the C ABI in include/csa.h (ctypes; argument marshalling
only -- every step of the path runs in the CUDA kernels of libcsa.so).

Device memory comes from torch tensors; the library never allocates.  Each
function keeps the C name and argument order, takes :class:`DevTensor`
objects for ``csa_tensor_t`` arguments, and raises :class:`CsaError` on a
non-zero status.  The library is the in-tree ``libcsa.so``; importing this
module fails loudly if it has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa.so")

CSA_F32, CSA_BF16, CSA_FP8_E4M3, CSA_MXFP4_E2M1 = 0, 1, 2, 3
_DTYPES = {"f32": CSA_F32, "bf16": CSA_BF16, "fp8": CSA_FP8_E4M3, "mxfp4": CSA_MXFP4_E2M1}
STATUS = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED", 3: "CSA_ERR_CAPACITY",
          4: "CSA_ERR_TIMEOUT", 5: "CSA_ERR_CUDA"}

EXPORTS = ["csa_workspace_size", "csa_compress", "csa_index_topk", "csa_index_score", "csa_topk",
           "csa_sparse_swa_attention", "csa_decode_step", "csa_last_error", "csa_sync_status", "csa_profile_start",
           "csa_profile_stop", "csa_profile_count", "csa_profile_get", "csa_sparse_swa_attention_noalloc",
           "csa_index_topk_pool", "csa_index_topk_reindex", "csa_index_pool_workspace_size",
           "csa_topk_workspace_size", "csa_test_expire_next_barrier"]


class CsaError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")
        self.status = status


class Tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("scale_group", ctypes.c_int32)]


class Params(ctypes.Structure):
    _fields_ = [("m", ctypes.c_int32), ("d", ctypes.c_int32), ("d_idx", ctypes.c_int32), ("h_q", ctypes.c_int32),
                ("h_idx", ctypes.c_int32), ("topk", ctypes.c_int32), ("window", ctypes.c_int32),
                ("swa_cap", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


class DecodeCaches(ctypes.Structure):
    _fields_ = [("kv", Tensor), ("kidx", Tensor), ("swa_k", Tensor), ("swa_v", Tensor), ("open_c", Tensor),
                ("open_z", Tensor), ("cap", ctypes.c_int64)]


class DecodeToken(ctypes.Structure):
    _fields_ = [("c", Tensor), ("z", Tensor), ("k_swa", Tensor), ("v_swa", Tensor), ("q", Tensor),
                ("q_idx", Tensor), ("w", ctypes.c_void_p), ("sink", ctypes.c_void_p), ("w_ik", Tensor)]


_lib = None


def load() -> ctypes.CDLL:
    """The in-tree libcsa.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m compressed_sparse_attention_compressor_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, V, I32, I64, SZ = ctypes.POINTER, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    T = P(Tensor)
    sig = {
        "csa_workspace_size": (SZ, [P(Params), I32, I64]),
        "csa_compress": (I32, [T, T, I32, I64, I32, I32, T, I64, T, I32, T, V]),
        "csa_index_topk": (I32, [P(Params), I32, T, V, T, I32, I64, V, V, V, V, V, SZ, V]),
        "csa_index_score": (I32, [P(Params), I32, T, V, T, I32, I64, V, V, V, I64, V]),
        "csa_topk": (I32, [V, I32, I64, V, I32, V, V, V, SZ, V]),
        "csa_index_topk_pool": (I32, [P(Params), I32, T, V, T, I32, I64, V, V, I32, I32, V, V, V, V, SZ, V]),
        "csa_index_topk_reindex": (I32, [P(Params), I32, T, V, T, I32, I64, V, V, V, I32, I32, V, V, V, SZ, V]),
        "csa_index_pool_workspace_size": (SZ, [P(Params), I32, I64, I32, I32]),
        "csa_topk_workspace_size": (SZ, [I32]),
        "csa_sparse_swa_attention": (I32, [P(Params), I32, T, T, I32, I64, V, V, V, T, T, V, V, V, T, V, V, SZ, V]),
        "csa_sparse_swa_attention_noalloc": (I32, [P(Params), I32, T, T, I32, I64, V, V, V, T, T, V, V, V, T, V, V]),
        "csa_decode_step": (I32, [P(Params), I32, P(DecodeCaches), P(DecodeToken), V, T, V, V, V, SZ, V]),
        "csa_last_error": (ctypes.c_char_p, []),
        "csa_sync_status": (I32, [V]),
        "csa_test_expire_next_barrier": (I32, [I32, ctypes.c_uint32]),
        "csa_profile_start": (I32, [I32]),
        "csa_profile_stop": (I32, []),
        "csa_profile_count": (I32, []),
        "csa_profile_get": (I32, [I32, P(ctypes.c_char_p), P(ctypes.c_float)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


# ---------------------------------------------------------------------------
# device tensors in storage format
# ---------------------------------------------------------------------------
@dataclass
class DevTensor:
    """A device tensor in storage format: ``data`` (float32 / int16 bf16 bits /
    uint8 E4M3 codes / uint8 pairs of E2M1 codes) plus, for 'fp8', fp32
    ``scale`` with one value per ``group`` consecutive elements of a row, for
    'mxfp4', uint8 E4M3 scale codes, one per 16 elements."""

    data: torch.Tensor
    dtype: str
    scale: torch.Tensor | None = None
    group: int = 0

    def c(self) -> Tensor:
        return Tensor(self.data.data_ptr(), self.scale.data_ptr() if self.scale is not None else None,
                      _DTYPES[self.dtype], self.group if self.dtype in ("fp8", "mxfp4") else 0)

    @staticmethod
    def empty(shape, dtype: str, device="cuda", group: int = 0) -> "DevTensor":
        if dtype == "mxfp4":
            lead = tuple(shape[:-1])
            return DevTensor(torch.zeros(lead + (shape[-1] // 2,), dtype=torch.uint8, device=device), "mxfp4",
                             torch.zeros(lead + (shape[-1] // 16,), dtype=torch.uint8, device=device), 16)
        tdt = {"f32": torch.float32, "bf16": torch.int16, "fp8": torch.uint8}[dtype]
        data = torch.zeros(tuple(shape), dtype=tdt, device=device)
        scale = None
        if dtype == "fp8":
            scale = torch.ones(tuple(shape[:-1]) + (shape[-1] // group,), dtype=torch.float32, device=device)
        return DevTensor(data, dtype, scale, group)

    @staticmethod
    def from_stored(st, device="cuda") -> "DevTensor":
        """From a host tensor with numpy ``data``/``scale`` (e.g. workloads.Stored)."""
        import numpy as np

        arr = st.data
        if st.dtype == "bf16":
            arr = arr.view(np.int16)
        data = torch.from_numpy(np.ascontiguousarray(arr)).to(device)
        scale = torch.from_numpy(np.ascontiguousarray(st.scale)).to(device) if st.scale is not None else None
        return DevTensor(data, st.dtype, scale, st.group)

    def host(self):
        """(data, scale) as numpy arrays in storage format (bf16 as uint16)."""
        import numpy as np

        d = self.data.cpu().numpy()
        if self.dtype == "bf16":
            d = d.view(np.uint16)
        return d, (self.scale.cpu().numpy() if self.scale is not None else None)

    def offset_rows(self, row0: int) -> "DevTensor":
        """A view starting at row ``row0`` of a [rows][d] layout (flattened over
        leading axes), for appending into a cache."""
        flat = self.data.reshape(-1, self.data.shape[-1])
        sc = self.scale.reshape(-1, self.scale.shape[-1])[row0:] if self.scale is not None else None
        return DevTensor(flat[row0:], self.dtype, sc, self.group)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(status: int, where: str):
    if status != 0:
        raise CsaError(status, where, load().csa_last_error().decode())


def params(m, d, d_idx, h_q, h_idx, topk, window, swa_cap, softmax_scale=1.0) -> Params:
    return Params(m, d, d_idx, h_q, h_idx, topk, window, swa_cap, softmax_scale)


# ---------------------------------------------------------------------------
# the entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def csa_workspace_size(p: Params, n_queries: int, max_entries: int) -> int:
    return load().csa_workspace_size(ctypes.byref(p), n_queries, max_entries)


def csa_compress(C: DevTensor, Z: DevTensor, batch: int, n_tokens: int, d: int, m: int, out: DevTensor,
                 out_rows: int, w_ik: DevTensor | None = None, d_idx: int = 0, kidx_out: DevTensor | None = None,
                 stream=None):
    cw = ctypes.byref(w_ik.c()) if w_ik is not None else None
    ck = ctypes.byref(kidx_out.c()) if kidx_out is not None else None
    _check(load().csa_compress(ctypes.byref(C.c()), ctypes.byref(Z.c()), batch, n_tokens, d, m,
                               ctypes.byref(out.c()), out_rows, cw, d_idx, ck, _stream(stream)), "csa_compress")


def csa_index_topk(p: Params, n_queries: int, q_idx: DevTensor, w: torch.Tensor, k_idx: DevTensor, batch: int,
                   cap: int, q_req: torch.Tensor | None, n_visible: torch.Tensor, out_idx: torch.Tensor,
                   out_score: torch.Tensor | None, workspace: torch.Tensor, stream=None):
    _check(load().csa_index_topk(ctypes.byref(p), n_queries, ctypes.byref(q_idx.c()), _ptr(w), ctypes.byref(k_idx.c()),
                                 batch, cap, _ptr(q_req), _ptr(n_visible), _ptr(out_idx), _ptr(out_score), _ptr(workspace),
                                 workspace.numel() * workspace.element_size() if workspace is not None else 0,
                                 _stream(stream)), "csa_index_topk")


def csa_index_score(p: Params, n_queries: int, q_idx: DevTensor, w: torch.Tensor, k_idx: DevTensor, batch: int,
                    cap: int, q_req: torch.Tensor | None, n_visible: torch.Tensor, scores: torch.Tensor, ld: int,
                    stream=None):
    _check(load().csa_index_score(ctypes.byref(p), n_queries, ctypes.byref(q_idx.c()), _ptr(w),
                                  ctypes.byref(k_idx.c()), batch, cap, _ptr(q_req), _ptr(n_visible), _ptr(scores), ld,
                                  _stream(stream)), "csa_index_score")


def csa_topk_workspace_size(n_rows: int) -> int:
    return load().csa_topk_workspace_size(n_rows)


def csa_topk(scores: torch.Tensor, n_rows: int, ld: int, n_valid: torch.Tensor, k: int, out_idx: torch.Tensor,
             out_score: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    _check(load().csa_topk(_ptr(scores), n_rows, ld, _ptr(n_valid), k, _ptr(out_idx), _ptr(out_score),
                           _ptr(workspace), workspace.numel() * workspace.element_size() if workspace is not None else 0,
                           _stream(stream)), "csa_topk")


def _nbytes(t):
    return t.numel() * t.element_size() if t is not None else 0


def csa_index_pool_workspace_size(p: Params, n_queries: int, max_entries: int, block: int, pool_blocks: int) -> int:
    return load().csa_index_pool_workspace_size(ctypes.byref(p), n_queries, max_entries, block, pool_blocks)


def csa_index_topk_pool(p: Params, n_queries: int, q_idx: DevTensor, w: torch.Tensor, k_idx: DevTensor, batch: int,
                        cap: int, q_req: torch.Tensor | None, n_visible: torch.Tensor, block: int, pool_blocks: int,
                        out_pool: torch.Tensor, out_idx: torch.Tensor | None, out_score: torch.Tensor | None,
                        workspace: torch.Tensor, stream=None):
    _check(load().csa_index_topk_pool(ctypes.byref(p), n_queries, ctypes.byref(q_idx.c()), _ptr(w),
                                      ctypes.byref(k_idx.c()), batch, cap, _ptr(q_req), _ptr(n_visible), block,
                                      pool_blocks, _ptr(out_pool), _ptr(out_idx), _ptr(out_score), _ptr(workspace),
                                      _nbytes(workspace), _stream(stream)), "csa_index_topk_pool")


def csa_index_topk_reindex(p: Params, n_queries: int, q_idx: DevTensor, w: torch.Tensor, k_idx: DevTensor,
                           batch: int, cap: int, q_req: torch.Tensor | None, n_visible: torch.Tensor,
                           pool: torch.Tensor, block: int, pool_blocks: int, out_idx: torch.Tensor,
                           out_score: torch.Tensor | None, workspace: torch.Tensor, stream=None):
    _check(load().csa_index_topk_reindex(ctypes.byref(p), n_queries, ctypes.byref(q_idx.c()), _ptr(w),
                                         ctypes.byref(k_idx.c()), batch, cap, _ptr(q_req), _ptr(n_visible),
                                         _ptr(pool), block, pool_blocks, _ptr(out_idx), _ptr(out_score),
                                         _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "csa_index_topk_reindex")


def csa_sparse_swa_attention(p: Params, n_queries: int, q: DevTensor, kv: DevTensor, batch: int, cap: int,
                             idx: torch.Tensor | None, n_visible: torch.Tensor, q_req: torch.Tensor | None,
                             swa_k: DevTensor | None, swa_v: DevTensor | None, q_pos: torch.Tensor,
                             swa_lo: torch.Tensor | None, sink: torch.Tensor | None, out: DevTensor,
                             lse: torch.Tensor | None, workspace: torch.Tensor | None, stream=None):
    sk = ctypes.byref(swa_k.c()) if swa_k is not None else None
    sv = ctypes.byref(swa_v.c()) if swa_v is not None else None
    _check(load().csa_sparse_swa_attention(
        ctypes.byref(p), n_queries, ctypes.byref(q.c()), ctypes.byref(kv.c()), batch, cap, _ptr(idx), _ptr(n_visible),
        _ptr(q_req), sk, sv, _ptr(q_pos), _ptr(swa_lo), _ptr(sink), ctypes.byref(out.c()), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size() if workspace is not None else 0,
        _stream(stream)), "csa_sparse_swa_attention")


def csa_sparse_swa_attention_noalloc(p: Params, n_queries: int, q: DevTensor, kv: DevTensor, batch: int, cap: int,
                                     idx: torch.Tensor | None, n_visible: torch.Tensor, q_req: torch.Tensor | None,
                                     swa_k: DevTensor | None, swa_v: DevTensor | None, q_pos: torch.Tensor,
                                     swa_lo: torch.Tensor | None, sink: torch.Tensor | None, out: DevTensor,
                                     lse: torch.Tensor | None, stream=None):
    """csa_sparse_swa_attention without a workspace: for callers that cannot
    allocate device memory; its scratch is a fixed array inside the library
    (see include/csa.h)."""
    sk = ctypes.byref(swa_k.c()) if swa_k is not None else None
    sv = ctypes.byref(swa_v.c()) if swa_v is not None else None
    _check(load().csa_sparse_swa_attention_noalloc(
        ctypes.byref(p), n_queries, ctypes.byref(q.c()), ctypes.byref(kv.c()), batch, cap, _ptr(idx),
        _ptr(n_visible), _ptr(q_req), sk, sv, _ptr(q_pos), _ptr(swa_lo), _ptr(sink), ctypes.byref(out.c()),
        _ptr(lse), _stream(stream)), "csa_sparse_swa_attention_noalloc")


def decode_caches(kv, kidx, swa_k, swa_v, open_c, open_z, cap) -> DecodeCaches:
    none = Tensor(None, None, 0, 0)
    return DecodeCaches(kv.c(), kidx.c() if kidx is not None else none, swa_k.c(), swa_v.c(), open_c.c(),
                        open_z.c(), cap)


def decode_token(c, z, k_swa, v_swa, q, q_idx, w, sink, w_ik) -> DecodeToken:
    none = Tensor(None, None, 0, 0)
    return DecodeToken(c.c(), z.c(), k_swa.c(), v_swa.c(), q.c(), q_idx.c() if q_idx is not None else none,
                       _ptr(w), _ptr(sink), w_ik.c() if w_ik is not None else none)


def csa_decode_step(p: Params, batch: int, caches: DecodeCaches, tok: DecodeToken, pos: torch.Tensor,
                    out: DevTensor, lse: torch.Tensor | None, out_idx: torch.Tensor | None, workspace: torch.Tensor,
                    stream=None):
    _check(load().csa_decode_step(ctypes.byref(p), batch, ctypes.byref(caches), ctypes.byref(tok), _ptr(pos),
                                  ctypes.byref(out.c()), _ptr(lse), _ptr(out_idx), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)), "csa_decode_step")


def csa_last_error() -> str:
    return load().csa_last_error().decode()


def csa_sync_status(stream=None):
    _check(load().csa_sync_status(_stream(stream)), "csa_sync_status")


def csa_test_expire_next_barrier(cta: int, polls: int):
    """Test support: the next fused-indexer launch's CTA ``cta`` skips its
    first grid-barrier arrival and its waits give up after ``polls`` polls
    (see include/csa.h)."""
    _check(load().csa_test_expire_next_barrier(cta, polls), "csa_test_expire_next_barrier")


def csa_profile_start(max_launches: int):
    _check(load().csa_profile_start(max_launches), "csa_profile_start")


def csa_profile_stop():
    _check(load().csa_profile_stop(), "csa_profile_stop")


def csa_profile_records() -> list[tuple[str, float]]:
    """(kernel name, milliseconds) of every recorded launch, in launch order."""
    lib = load()
    out = []
    for i in range(lib.csa_profile_count()):
        name, ms = ctypes.c_char_p(), ctypes.c_float()
        _check(lib.csa_profile_get(i, ctypes.byref(name), ctypes.byref(ms)), "csa_profile_get")
        out.append((name.value.decode(), ms.value))
    return out


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A caller-owned workspace buffer of at least ``nbytes`` bytes."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
