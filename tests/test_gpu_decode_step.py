"""a6 decode step (append + compress + index + top-k + attention) through
csa_decode_step, vs the oracle's decode step, on scaled-down versions of
every decode workload; plus the pipeline from the compressor (tiny and
chunked-prefill workloads) through csa_compress -> csa_index_topk ->
csa_sparse_swa_attention."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200 import workloads as Wk
from compressed_sparse_attention_compressor_b200.csa import DevTensor
from oracle import csa_oracle as O
from tests._harness import (GpuDecode, check_attention, check_rows, check_selection, dev, f32, i32, i64, params_of,
                            to_f64)

pytestmark = pytest.mark.gpu

DECODE = {
    "tiny": Wk.WORKLOADS["tiny"].scaled(context=1024),
    "tiny_open": Wk.WORKLOADS["tiny"].scaled(context=1022),           # block not closed by this token
    "decode64k": Wk.WORKLOADS["decode64k"].scaled(batch=3, context=4096 + 4 * 37),
    "decode1m": Wk.WORKLOADS["decode1m"].scaled(batch=2, context=8192),
    "decode1m_open": Wk.WORKLOADS["decode1m"].scaled(batch=2, context=8190),  # appended in the indexer, block open
    "hybrid_csa": Wk.WORKLOADS["hybrid_csa"].scaled(batch=2, context=3000),
    "hybrid_hca": Wk.WORKLOADS["hybrid_hca"].scaled(batch=2, context=128 * 40),
    "hybrid_ratio1": Wk.WORKLOADS["hybrid_ratio1"].scaled(batch=2, context=2500, topk=300),
    "short_context": Wk.WORKLOADS["decode64k"].scaled(batch=2, context=60),  # fewer entries than top-k, window > T
    "decode1m_fp4": Wk.WORKLOADS["decode1m_fp4"].scaled(batch=2, context=8192),
    "decode1m_fp4_open": Wk.WORKLOADS["decode1m_fp4"].scaled(batch=2, context=8190),
    "decode1m_fp4_simt_index": Wk.WORKLOADS["decode1m_fp4"].scaled(batch=3, context=4096, idx_dtype="bf16",
                                                                   h_idx=32),
    "tiny_fp4": Wk.WORKLOADS["tiny"].scaled(context=1024, kv_dtype="mxfp4", kv_group=16),
}


def _dtype_tol(wl):
    # MXFP4 rows: an element of a freshly pooled row at an E2M1 rounding
    # midpoint may take either neighbour (a full step), so even fp32
    # workloads get the quantised tolerance
    return "f32" if wl.act_dtype == "f32" and wl.kv_dtype != "mxfp4" else wl.kv_dtype


@pytest.mark.parametrize("name", list(DECODE))
def test_decode_step_matches_oracle(name, cuda_lib):
    wl = DECODE[name]
    inp = Wk.make_decode_inputs(wl)
    g = GpuDecode(inp)
    g.step()
    torch.cuda.synchronize()
    ref = O.decode_step(inp)
    check_attention(to_f64(g.out), g.lse.double().cpu().numpy(), ref["out"], ref["lse"], _dtype_tol(wl))
    g.check_selections(ref)
    t = int(inp.pos[0])
    if (t + 1) % wl.m == 0:
        j = (t + 1) // wl.m - 1
        kv = to_f64(g.kv)
        for b in range(wl.batch):
            quant = wl.kv_dtype in ("fp8", "mxfp4")
            sc = g.kv.scale[b, j:j + 1].cpu().numpy() if quant else None
            codes = g.kv.data[b, j:j + 1].cpu().numpy() if quant else None
            check_rows(kv[b, j:j + 1], ref["new_rows"][b][None], wl.kv_dtype, 64, sc, codes)
            if not wl.dense:
                ki = to_f64(g.kidx)
                kf = wl.idx_dtype == "fp8"
                ksc = g.kidx.scale[b, j:j + 1].cpu().numpy() if kf else None
                kc = g.kidx.data[b, j:j + 1].cpu().numpy() if kf else None
                check_rows(ki[b, j:j + 1], ref["new_keys"][b][None], wl.idx_dtype, wl.d_idx, ksc, kc)
    # the token's SWA row landed in its ring slot, the open block holds c_t
    sk = to_f64(g.swa_k)
    assert np.array_equal(sk[:, t % inp.swa_cap], O.decode_stored(inp.k_t))
    oc = to_f64(g.open_c)
    assert np.array_equal(oc[:, t % wl.m], O.decode_stored(inp.c_t))


# Requests of one batch at different positions: the first token (no entry
# visible, the window holds the token alone), the token that closes the first
# block (one entry), an open block, and a closing block past top-k.  Rows of
# the caches beyond a request's visible entries hold stale values that must
# not be read.
RAGGED = {
    "decode1m": (Wk.WORKLOADS["decode1m"].scaled(batch=4, context=8192), [0, 3, 4097, 8191]),
    "decode1m_fp4": (Wk.WORKLOADS["decode1m_fp4"].scaled(batch=4, context=8192), [8191, 1, 3, 5002]),
    "decode64k": (Wk.WORKLOADS["decode64k"].scaled(batch=3, context=4096), [4095, 0, 2050]),
    "hybrid_hca": (Wk.WORKLOADS["hybrid_hca"].scaled(batch=3, context=128 * 40), [127, 5, 128 * 40 - 1]),
    "tiny": (Wk.WORKLOADS["tiny"].scaled(batch=2, context=1024), [3, 1023]),
}


@pytest.mark.parametrize("name", list(RAGGED))
def test_decode_step_ragged_positions(name, cuda_lib):
    wl, positions = RAGGED[name]
    inp = Wk.make_decode_inputs(wl)
    inp.pos = np.array(positions, np.int64)
    g = GpuDecode(inp)
    g.step()
    torch.cuda.synchronize()
    ref = O.decode_step(inp)
    check_attention(to_f64(g.out), g.lse.double().cpu().numpy(), ref["out"], ref["lse"], _dtype_tol(wl))
    g.check_selections(ref)
    kv = to_f64(g.kv)
    quant = wl.kv_dtype in ("fp8", "mxfp4")
    closed = 0
    for b, t in enumerate(positions):
        if (t + 1) % wl.m == 0:
            j = (t + 1) // wl.m - 1
            sc = g.kv.scale[b, j:j + 1].cpu().numpy() if quant else None
            codes = g.kv.data[b, j:j + 1].cpu().numpy() if quant else None
            check_rows(kv[b, j:j + 1], ref["new_rows"][closed][None], wl.kv_dtype, 64, sc, codes)
            closed += 1
        assert np.array_equal(to_f64(g.swa_k)[b, t % inp.swa_cap], O.decode_stored(inp.k_t)[b])
        assert np.array_equal(to_f64(g.open_c)[b, t % wl.m], O.decode_stored(inp.c_t)[b])
    assert closed == len(ref["new_rows"])


def test_decode_step_is_repeatable(cuda_lib):
    """Same position twice: identical outputs (the step only overwrites the
    slots it owns)."""
    inp = Wk.make_decode_inputs(DECODE["decode64k"])
    g = GpuDecode(inp)
    g.step()
    a = g.out.data.clone()
    g.step()
    torch.cuda.synchronize()
    assert torch.equal(a, g.out.data)


def test_tiny_pipeline_end_to_end(cuda_lib):
    """The tiny workload at its published size: C, Z [4096][128] fp32 ->
    compressor (+ indexer-key projection) -> indexer + top-k 64 ->
    attention with the 128-token window and sink 0."""
    wl = Wk.WORKLOADS["tiny"]
    inp = Wk.make_tiny_pipeline_inputs(wl)
    _run_pipeline(inp, exact=True)


def test_prefill_pipeline_scaled(cuda_lib):
    """Chunked prefill: 256 new queries after 2,048 cached tokens, bf16,
    causal visibility of blocks closed inside the chunk."""
    wl = Wk.WORKLOADS["prefill"].scaled(context=2048, chunk=256)
    inp = Wk.make_prefill_inputs(wl)
    _run_pipeline(inp, exact=False)


@pytest.mark.parametrize("name", ["tiny", "prefill"])
def test_pipeline_with_mxfp4_main_kv(name, cuda_lib):
    """The main KV stored as MXFP4 (E2M1 codes, an E4M3 scale per 16
    channels): the compressor quantises its pooled rows, the attention
    dequantises the cached and the new rows."""
    if name == "tiny":
        inp = Wk.make_tiny_pipeline_inputs(Wk.WORKLOADS["tiny"].scaled(kv_dtype="mxfp4", kv_group=16))
        _run_pipeline(inp, exact=True)
    else:
        wl = Wk.WORKLOADS["prefill"].scaled(context=2048, chunk=256, kv_dtype="mxfp4", kv_group=16)
        _run_pipeline(Wk.make_prefill_inputs(wl), exact=False)


def _run_pipeline(inp, exact, queries=None):
    wl = inp.wl
    m, d = wl.m, wl.d
    B = 1
    nq = inp.q_pos.shape[0]
    n_new = inp.C.data.shape[1] // m
    cap = inp.cap
    if inp.kv_cached is not None:
        kv, kidx = dev(inp.kv_cached), dev(inp.kidx_cached)
    else:
        kv = DevTensor.empty((B, cap, d), wl.kv_dtype, group=64)
        kidx = DevTensor.empty((B, cap, wl.d_idx), wl.idx_dtype, group=wl.d_idx)
    n0 = inp.n_cached
    csa.csa_compress(dev(inp.C), dev(inp.Z), B, inp.C.data.shape[1], d, m, kv.offset_rows(n0), cap, dev(inp.w_ik),
                     wl.d_idx, kidx.offset_rows(n0))
    p = params_of(wl, inp.swa_cap)
    n_vis = ((inp.q_pos + 1) // m).astype(np.int32)
    out_idx = torch.empty((nq, wl.topk), dtype=torch.int32, device="cuda")
    out_score = torch.empty((nq, wl.topk), dtype=torch.float32, device="cuda")
    ws = csa.workspace(csa.csa_workspace_size(p, nq, cap))
    csa.csa_index_topk(p, nq, dev(inp.q_idx), f32(inp.w), kidx, B, cap, i32(inp.q_req), i32(n_vis), out_idx, out_score,
                       ws)
    out = DevTensor.empty((nq, wl.h_q, d), "f32" if wl.act_dtype == "f32" else "bf16")
    lse = torch.empty((nq, wl.h_q), dtype=torch.float32, device="cuda")
    csa.csa_sparse_swa_attention(p, nq, dev(inp.q), kv, B, cap, out_idx, i32(n_vis), i32(inp.q_req), dev(inp.swa_k),
                                 dev(inp.swa_v), i64(inp.q_pos), None, f32(inp.sink), out, lse, ws)
    torch.cuda.synchronize()
    qs = list(range(nq)) if queries is None else queries
    ref = O.pipeline(inp, qs)
    # compressor output rows and keys
    kvh, kih = to_f64(kv), to_f64(kidx)
    f8, k8 = wl.kv_dtype in ("fp8", "mxfp4"), wl.idx_dtype == "fp8"
    check_rows(kvh[0, n0:n0 + n_new], ref["rows"], wl.kv_dtype, 64,
               kv.scale[0, n0:n0 + n_new].cpu().numpy() if f8 else None,
               kv.data[0, n0:n0 + n_new].cpu().numpy() if f8 else None)
    check_rows(kih[0, n0:n0 + n_new], ref["keys"], wl.idx_dtype, wl.d_idx,
               kidx.scale[0, n0:n0 + n_new].cpu().numpy() if k8 else None,
               kidx.data[0, n0:n0 + n_new].cpu().numpy() if k8 else None)
    gi, gs = out_idx.cpu().numpy(), out_score.cpu().numpy()
    got, got_lse = to_f64(out), lse.double().cpu().numpy()
    swaps = 0
    for n, i in enumerate(qs):
        swaps += check_selection(gi[i], ref["scores"][n], wl.topk, exact, gs[i])
    check_attention(got[qs], got_lse[qs], ref["out"], ref["lse"], _dtype_tol(wl))
    return swaps
