"""Shared helpers of the GPU parity tests: upload seeded inputs, run the CUDA
path through the C ABI, and compare with the oracle under the stated
tolerances.

Tolerances (the acceptance bar of the path):
* attention outputs and lse, max-abs error against the fp64 oracle:
  1e-4 for fp32 workloads, 2e-2 for bf16 / FP8 / MXFP4 workloads; and, so
  that the bar scales with outputs far below it (bf16 workloads whose
  values are N(0,1)/sqrt(d) give outputs of about 0.005-0.1), the output's
  max-abs error must also stay within the same number times max |oracle
  output|: an all-zero or garbage-but-small output fails;
* selected index sets: fp32 workloads bit-exact, except for swaps at a
  near-tie -- an entry in only one of the two sets must score within the
  fp32 error bound 1e-5 (1 + max|s|) of the oracle's k-th score (reported
  with a warning); bf16 / FP8 workloads may differ only by boundary swaps
  whose oracle scores lie within 1e-3 of the oracle's k-th score;
* scores the kernel reports: |gpu - oracle| <= 1e-4 * (1 + |oracle|);
* compressor outputs: fp32 1e-5 * (1 + |x|); bf16 half an ulp (2^-8 |x| at
  worst, just above a power of two) plus 1e-7; FP8 scales to 1e-5 relative
  and codes within one step of the
  oracle's round-to-nearest-even code (a step only where the oracle value sits
  within 1e-5 relative of a rounding midpoint); MXFP4 scale bytes equal the
  oracle's E4M3 rounding of max|x| / 6 and codes the oracle's E2M1 rounding
  of x / scale, a neighbour only at a rounding midpoint.
"""
from __future__ import annotations

import warnings

import numpy as np
import torch

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200 import workloads as Wk
from compressed_sparse_attention_compressor_b200.csa import DevTensor
from oracle import csa_oracle as O

ATT_TOL = {"f32": 1e-4, "bf16": 2e-2, "fp8": 2e-2, "mxfp4": 2e-2}
BOUNDARY_GAP = 1e-3
FP32_TIE = 1e-5  # relative fp32 error bound of an indexer score (times 1 + max|s|)


def dev(st) -> DevTensor:
    return DevTensor.from_stored(st)


def i32(a):
    return torch.as_tensor(np.asarray(a, np.int32)).cuda()


def i64(a):
    return torch.as_tensor(np.asarray(a, np.int64)).cuda()


def f32(a):
    return torch.as_tensor(np.asarray(a, np.float32)).cuda()


def to_f64(t: DevTensor) -> np.ndarray:
    """GPU tensor in storage format -> fp64 numpy (torch casts)."""
    if t.dtype == "f32":
        return t.data.double().cpu().numpy()
    if t.dtype == "bf16":
        return t.data.view(torch.bfloat16).double().cpu().numpy()
    if t.dtype == "mxfp4":  # no torch cast for E2M1: the pinned oracle decoder
        return O.decode(t.data.cpu().numpy(), "mxfp4", t.scale.cpu().numpy(), 16)
    v = t.data.view(torch.float8_e4m3fn).double()
    sc = t.scale.double().repeat_interleave(t.group, dim=-1)
    return (v * sc).cpu().numpy()


def out_dtype(wl) -> str:
    return "f32" if wl.act_dtype == "f32" else "bf16"


def params_of(wl, swa_cap: int, tau: float = 1.0):
    return csa.params(wl.m, wl.d, wl.d_idx, wl.h_q, wl.h_idx, wl.topk, wl.window, swa_cap, tau)


# ---------------------------------------------------------------------------
# running the CUDA path
# ---------------------------------------------------------------------------
class GpuDecode:
    """Device copies of a DecodeInputs plus the step's outputs."""

    def __init__(self, inp: Wk.DecodeInputs, tau: float = 1.0):
        wl = inp.wl
        self.inp, self.wl = inp, wl
        self.p = params_of(wl, inp.swa_cap, tau)
        self.kv, self.kidx = dev(inp.kv), dev(inp.kidx)
        self.swa_k, self.swa_v = dev(inp.swa_k), dev(inp.swa_v)
        self.open_c, self.open_z = dev(inp.open_c), dev(inp.open_z)
        self.c_t, self.z_t, self.k_t, self.v_t = dev(inp.c_t), dev(inp.z_t), dev(inp.k_t), dev(inp.v_t)
        self.q, self.q_idx, self.w_ik = dev(inp.q), dev(inp.q_idx), dev(inp.w_ik)
        self.w, self.sink = f32(inp.w), f32(inp.sink)
        self.pos = i64(inp.pos)
        self.out = DevTensor.empty((wl.batch, wl.h_q, wl.d), out_dtype(wl))
        self.lse = torch.empty((wl.batch, wl.h_q), dtype=torch.float32, device="cuda")
        # the step's selection (sparse workloads), -7 so that unwritten slots show
        self.idx = None if wl.dense else torch.full((wl.batch, wl.topk), -7, dtype=torch.int32, device="cuda")
        self.ws = csa.workspace(csa.csa_workspace_size(self.p, wl.batch, inp.cap))
        self.caches = csa.decode_caches(self.kv, self.kidx, self.swa_k, self.swa_v, self.open_c, self.open_z, inp.cap)
        self.tok = csa.decode_token(self.c_t, self.z_t, self.k_t, self.v_t, self.q, self.q_idx, self.w, self.sink,
                                    self.w_ik)

    def step(self, stream=None):
        csa.csa_decode_step(self.p, self.wl.batch, self.caches, self.tok, self.pos, self.out, self.lse, self.idx,
                            self.ws, stream)

    def check_selections(self, ref, requests=None) -> int:
        """The step's selection of every request (or of ``requests``, in the
        order of ``ref``) against the oracle decode step's scores; returns
        the boundary swaps accepted."""
        if self.idx is None:
            return 0
        reqs = list(range(self.wl.batch)) if requests is None else list(requests)
        gi = self.idx.cpu().numpy()
        exact = self.wl.act_dtype == "f32" and self.wl.idx_dtype == "f32"
        return sum(check_selection(gi[b], ref["scores"][n], self.wl.topk, exact) for n, b in enumerate(reqs))


def gpu_index_topk(wl, q_idx_st, w, kidx_st, batch, cap, q_req, n_vis, k=None):
    p = params_of(wl, max(wl.window, 1))
    if k is not None:
        p.topk = k
    nq = q_idx_st.data.shape[0]
    q_idx, kidx = dev(q_idx_st), dev(kidx_st)
    out_idx = torch.full((nq, p.topk), -7, dtype=torch.int32, device="cuda")
    out_score = torch.empty((nq, p.topk), dtype=torch.float32, device="cuda")
    ws = csa.workspace(csa.csa_workspace_size(p, nq, cap))
    csa.csa_index_topk(p, nq, q_idx, f32(w), kidx, batch, cap, i32(q_req) if q_req is not None else None, i32(n_vis),
                       out_idx, out_score, ws)
    torch.cuda.synchronize()
    return out_idx.cpu().numpy(), out_score.cpu().numpy()


# ---------------------------------------------------------------------------
# comparisons
# ---------------------------------------------------------------------------
def check_selection(gpu_row: np.ndarray, scores: np.ndarray, k: int, exact: bool, gpu_scores=None) -> int:
    """Checks one query's selected set against the oracle; returns the number
    of boundary swaps accepted."""
    n = scores.shape[0]
    kk = min(k, n)
    valid = gpu_row[gpu_row >= 0]
    assert np.all(gpu_row[gpu_row < 0] == -1), "padding must be -1"
    assert valid.shape[0] == kk, f"selected {valid.shape[0]} entries, expected {kk}"
    assert np.unique(valid).shape[0] == kk, "duplicate indices"
    assert np.all(valid < n), "index beyond the visible entries"
    if gpu_scores is not None:
        gs = gpu_scores[gpu_row >= 0]
        ref = scores[valid]
        assert np.all(np.abs(gs - ref) <= 1e-4 * (1 + np.abs(ref))), "reported scores differ from the oracle"
    o = O.topk(scores, k)
    oset = set(o[o >= 0].tolist())
    diff = oset.symmetric_difference(valid.tolist())
    if not diff:
        return 0
    kth = np.sort(scores)[::-1][kk - 1]
    # fp32: only a near-tie at fp32 resolution may swap; bf16 / FP8: 1e-3
    tol = FP32_TIE * (1.0 + np.abs(scores).max()) if exact else BOUNDARY_GAP
    for j in diff:
        assert abs(scores[j] - kth) <= tol, \
            f"entry {j} is in one set only and scores {abs(scores[j] - kth):g} from the k-th (allowed {tol:g})"
    if exact:
        warnings.warn(f"fp32 near-tie at the top-k boundary (oracle gap {O.boundary_gap(scores, k):g}); "
                      f"sets differ by {len(diff)} entries within {tol:g} of the k-th score")
    return len(diff) // 2


def check_attention(gpu_out, gpu_lse, ref_out, ref_lse, dtype: str):
    tol = ATT_TOL[dtype]
    err = np.abs(gpu_out - ref_out).max() if ref_out.size else 0.0
    assert err <= tol, f"attention max-abs error {err:g} > {tol:g}"
    scale = np.abs(ref_out).max() if ref_out.size else 0.0
    assert err <= tol * scale, \
        f"attention max-abs error {err:g} > {tol:g} x max|oracle output| {scale:g} (the output-scaled bar)"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(gpu_lse)), "lse finiteness differs"
    if fin.any():
        lerr = np.abs(gpu_lse[fin] - ref_lse[fin]).max()
        assert lerr <= tol, f"lse max-abs error {lerr:g} > {tol:g}"
    return float(err)


def check_rows(gpu_vals: np.ndarray, ref: np.ndarray, dtype: str, group: int = 0, gpu_scale=None, gpu_codes=None):
    """Compressor / projection outputs.  gpu_vals: GPU rows decoded to fp64;
    for FP8 also the raw codes and the fp32 scales."""
    ref = np.asarray(ref, np.float64)
    if dtype == "f32":
        assert np.all(np.abs(gpu_vals - ref) <= 1e-5 * (1 + np.abs(ref))), \
            f"fp32 rows differ by {np.abs(gpu_vals - ref).max():g}"
    elif dtype == "bf16":
        # round to nearest: at most half an ulp, 2^-8 |x| (x just above a power of 2)
        assert np.all(np.abs(gpu_vals - ref) <= 2.0 ** -8 * np.abs(ref) * (1 + 1e-5) + 1e-7), \
            f"bf16 rows differ by {np.abs(gpu_vals - ref).max():g}"
    elif dtype == "mxfp4":
        check_mxfp4_rows(ref, gpu_codes, gpu_scale)
    else:
        codes, scale = O.quantize_groups(ref, group)
        # the kernel's group maximum is an fp32 pooled value: a few fp32 ulps
        # of the block's inputs away from the fp64 one
        rel = np.abs(gpu_scale - scale) / scale
        assert np.all(rel <= 1e-5), f"FP8 scales differ by {rel.max():.3g} relative"
        gv = O.e4m3_to_f64(gpu_codes)
        ov = O.e4m3_to_f64(codes)
        off = gv != ov
        if off.any():
            x = (ref / np.repeat(scale, group, axis=-1))[off]
            a, b = gv[off], ov[off]
            # the two codes must be neighbours around x, with x at their midpoint
            # (up to the fp32 error of the kernel's x / scale)
            assert np.all(np.minimum(a, b) <= x + 1e-9) and np.all(x <= np.maximum(a, b) + 1e-9), \
                "FP8 code is not a neighbour of the value"
            mid = (a + b) / 2
            assert np.all(np.abs(x - mid) <= 1e-5 * np.abs(x) + 1e-9), "FP8 code differs away from a rounding midpoint"


def _neighbours_at_midpoint(x, a, b, what):
    """Codes a != b (as values) are acceptable only as the two neighbours of
    x with x at their midpoint, up to the fp32 error of the kernel's input."""
    assert np.all(np.minimum(a, b) <= x + 1e-9) and np.all(x <= np.maximum(a, b) + 1e-9), \
        f"{what} code is not a neighbour of the value"
    assert np.all(np.abs(x - (a + b) / 2) <= 1e-5 * np.abs(x) + 1e-9), f"{what} code differs away from a midpoint"


def check_mxfp4_rows(ref, gpu_codes, gpu_scale):
    """MXFP4 rows: the GPU's E4M3 group scales equal the oracle's rounding of
    max|x| / 6 (a neighbour only at an E4M3 midpoint), and every element the
    oracle's E2M1 rounding of x / (the GPU's scale) (a neighbour only at an
    E2M1 midpoint).  ref: the oracle's fp64 rows [n][d]; gpu_codes [n][d/2],
    gpu_scale [n][d/16] (uint8)."""
    ref = np.asarray(ref, np.float64)
    g = ref.reshape(ref.shape[:-1] + (-1, 16))
    want = O.e4m3_to_f64(O.e4m3_round(np.abs(g).max(axis=-1) / O.E2M1_MAX))
    got = O.e4m3_to_f64(gpu_scale)
    off = got != want
    if off.any():
        _neighbours_at_midpoint((np.abs(g).max(axis=-1) / O.E2M1_MAX)[off], got[off], want[off], "MXFP4 scale")
    b = np.asarray(gpu_codes, np.uint8)
    codes = np.stack([b & 0xF, b >> 4], axis=-1).reshape(ref.shape)
    gv = O.E2M1_VALUES[codes]
    sc = np.repeat(got, 16, axis=-1)
    zero = sc == 0
    assert np.all(gv[zero] == 0), "a zero scale must store zero codes"
    x = np.where(zero, 0.0, ref / np.where(zero, 1.0, sc))
    ov = O.E2M1_VALUES[O.e2m1_round(x)]
    off = (gv != ov) & ~zero
    if off.any():
        _neighbours_at_midpoint(np.clip(x[off], -O.E2M1_MAX, O.E2M1_MAX), gv[off], ov[off], "E2M1")
