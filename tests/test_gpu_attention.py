"""a4 + a5: sparse / dense attention + sliding window + sink, CUDA path vs
the fp64 oracle, on explicit seeded selections (isolating the attention)."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200 import workloads as Wk
from compressed_sparse_attention_compressor_b200.csa import DevTensor
from oracle import csa_oracle as O
from tests._harness import ATT_TOL, check_attention, dev, f32, i32, i64, params_of, to_f64

pytestmark = pytest.mark.gpu

# name: (workload, n_queries, batch, cap, swa_cap, dense, use_sink, use_lo, tau)
CASES = {
    "tiny_f32": (Wk.WORKLOADS["tiny"], 3, 2, 1024, 128, False, True, False, 1.0),
    "bf16_csa": (Wk.WORKLOADS["decode64k"], 5, 3, 3000, 128, False, True, False, 1.0),
    "fp8_csa": (Wk.WORKLOADS["decode1m"], 3, 3, 4000, 128, False, True, False, 1.0),
    "bf16_hca": (Wk.WORKLOADS["hybrid_hca"], 3, 2, 700, 128, True, True, False, 1.0),
    "bf16_nosink_replay": (Wk.WORKLOADS["decode64k"], 4, 2, 2000, 256, False, False, True, 1.0),
    "bf16_sharp": (Wk.WORKLOADS["decode64k"], 2, 2, 1500, 128, False, True, False, float(np.sqrt(512))),
    "f32_prefill_like": (Wk.WORKLOADS["tiny"].scaled(h_q=16), 40, 1, 300, 512, False, True, True, 1.0),
    "bf16_no_window": (Wk.WORKLOADS["decode64k"].scaled(window=0), 3, 3, 800, 128, False, True, False, 1.0),
    # enough queries that the per-query clusters shrink to the smallest size
    # that fits (window values then re-gathered instead of held in registers)
    "bf16_many_queries": (Wk.WORKLOADS["decode64k"], 40, 4, 1200, 128, False, True, False, 1.0),
    # MXFP4 main KV (E2M1 + an E4M3 scale per 16 channels), dequantised to bf16 / fp32
    "mxfp4_csa": (Wk.WORKLOADS["decode1m_fp4"], 3, 3, 4000, 128, False, True, False, 1.0),
    "mxfp4_hca": (Wk.WORKLOADS["hybrid_hca"].scaled(kv_dtype="mxfp4", kv_group=16), 3, 2, 700, 128, True, True,
                  False, 1.0),
    "mxfp4_many_queries": (Wk.WORKLOADS["decode1m_fp4"], 40, 4, 1200, 128, False, True, False, 1.0),
    "tiny_mxfp4": (Wk.WORKLOADS["tiny"].scaled(kv_dtype="mxfp4", kv_group=16), 3, 2, 1024, 128, False, True, False,
                   1.0),
    # more than 64 queries: one CTA per query looping over 128-key tiles
    # (the chunked-prefill path), every main-KV format, dense and sparse
    "many_bf16_csa": (Wk.WORKLOADS["decode64k"], 96, 3, 3000, 128, False, True, False, 1.0),
    "many_fp8_csa": (Wk.WORKLOADS["decode1m"], 80, 2, 4000, 128, False, True, False, 1.0),
    "many_mxfp4_csa": (Wk.WORKLOADS["decode1m_fp4"], 72, 2, 4000, 128, False, True, False, 1.0),
    "many_bf16_hca": (Wk.WORKLOADS["hybrid_hca"], 70, 2, 700, 128, True, True, False, 1.0),
    "many_nosink_replay": (Wk.WORKLOADS["decode64k"], 66, 2, 2000, 256, False, False, True, 1.0),
    "many_no_window": (Wk.WORKLOADS["decode64k"].scaled(window=0), 65, 3, 800, 128, False, True, False, 1.0),
    # logits spread over tens of nats: a head's running maximum moves by more
    # than the lazy threshold between tiles, so O is rescaled in TMEM
    "many_very_sharp": (Wk.WORKLOADS["decode64k"], 68, 2, 1500, 128, False, True, False, 512.0),
    "many_top300": (Wk.WORKLOADS["decode64k"].scaled(topk=300), 90, 2, 2000, 128, False, True, False, 1.0),
}


@pytest.mark.parametrize("name", list(CASES))
def test_attention_matches_oracle(name, cuda_lib):
    wl, nq, B, cap, swa_cap, dense, use_sink, use_lo, tau = CASES[name]
    seed = 4000 + len(name) * 7
    d = wl.d
    sd = 1 / np.sqrt(d)
    kv_std = 1.0 if wl.kv_dtype == "fp8" else sd
    if wl.kv_dtype == "mxfp4":
        kv = Wk.random_mxfp4(seed, "kv", (B, cap, d))
    else:
        kv = Wk.store(Wk.normal(seed, "kv", (B, cap, d), kv_std), wl.kv_dtype, 64)
    act = wl.act_dtype
    swa_k = Wk.store(Wk.normal(seed, "sk", (B, swa_cap, d), sd), act)
    swa_v = Wk.store(Wk.normal(seed, "sv", (B, swa_cap, d), sd), act)
    q = Wk.store(Wk.normal(seed, "q", (nq, wl.h_q, d), sd), act)
    q_req = (np.arange(nq) % B).astype(np.int32)
    g = Wk.rng(seed, "shape")
    n_vis = g.integers(1, cap + 1, size=nq).astype(np.int32)
    n_vis[0] = cap
    n_vis[-1] = min(5, cap)
    if wl.window > 0:
        q_pos = g.integers(0, 10 * cap, size=nq).astype(np.int64)
        q_pos[-1] = 3  # a window shorter than W (start of the sequence)
    else:
        q_pos = np.full(nq, 100, np.int64)
    lo = (q_pos - g.integers(0, wl.window + 1, size=nq)).astype(np.int64) if use_lo else None
    sink = Wk.normal(seed, "sink", (wl.h_q,)) if use_sink else None
    k = wl.topk
    idx = None if dense else Wk.make_indices(seed, n_vis, k, pad_frac=0.3)

    p = params_of(wl, swa_cap, tau)
    out = DevTensor.empty((nq, wl.h_q, d), "f32" if act == "f32" else "bf16")
    lse = torch.empty((nq, wl.h_q), dtype=torch.float32, device="cuda")
    max_keys = (cap if dense else k) + wl.window
    ws = csa.workspace(csa.csa_workspace_size(p, nq, cap))
    csa.csa_sparse_swa_attention(p, nq, dev(q), dev(kv), B, cap, None if dense else i32(idx), i32(n_vis), i32(q_req),
                                 dev(swa_k), dev(swa_v), i64(q_pos), i64(lo) if lo is not None else None,
                                 f32(sink) if sink is not None else None, out, lse, ws)
    torch.cuda.synchronize()
    got, got_lse = to_f64(out), lse.double().cpu().numpy()

    qd = O.decode_stored(q)
    sk, sv = O.decode_stored(swa_k), O.decode_stored(swa_v)
    worst = 0.0
    for i in range(nq):
        b = q_req[i]
        rows = O.decode(kv.data[b], kv.dtype, None if kv.scale is None else kv.scale[b], 64)
        o, l = O.sparse_swa_attention(qd[i], rows, None if dense else idx[i], int(n_vis[i]), sk[b], sv[b], swa_cap,
                                      int(q_pos[i]), wl.window, sink, tau, 0 if lo is None else int(lo[i]))
        worst = max(worst, check_attention(got[i], got_lse[i], o, l, act if act == "f32" else wl.kv_dtype))
    print(f"{name}: max-abs error {worst:.3g} (tolerance {ATT_TOL[act if act == 'f32' else wl.kv_dtype]:g})")


def test_attention_empty_and_sink_only(cuda_lib):
    """No visible entry, no window: out = 0; lse = sink, or -inf without one."""
    wl = Wk.WORKLOADS["decode64k"].scaled(window=0)
    d, hq = wl.d, wl.h_q
    kv = Wk.store(np.zeros((1, 16, d)), "bf16")
    q = Wk.store(Wk.normal(1, "q", (2, hq, d)), "bf16")
    sink = Wk.normal(1, "sink", (hq,))
    p = params_of(wl, 128)
    for s in (sink, None):
        out = DevTensor.empty((2, hq, d), "bf16")
        lse = torch.empty((2, hq), dtype=torch.float32, device="cuda")
        ws = csa.workspace(csa.csa_workspace_size(p, 2, 16))
        csa.csa_sparse_swa_attention(p, 2, dev(q), dev(kv), 1, 16, i32(np.full((2, wl.topk), -1)), i32([0, 0]),
                                     i32([0, 0]), None, None, i64([0, 0]), None, f32(s) if s is not None else None,
                                     out, lse, ws)
        torch.cuda.synchronize()
        assert np.all(to_f64(out) == 0)
        l = lse.cpu().numpy()
        if s is None:
            assert np.all(np.isneginf(l))
        else:
            assert np.allclose(l, np.stack([s, s]), atol=1e-6)
