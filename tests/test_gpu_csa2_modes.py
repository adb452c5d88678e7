"""A CSA2 decoder layer group, Full / Reindex / Reuse, through the C ABI:
every layer's selection and attention output against the oracle."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200 import workloads as Wk
from compressed_sparse_attention_compressor_b200.csa import DevTensor
from oracle import csa_oracle as O
from tests._harness import check_attention, dev, f32, i32, i64, params_of, to_f64

pytestmark = pytest.mark.gpu

# the decoder's pattern: a group opened by a Full layer, then one opened by Reindex
MODES = ["full", "reuse", "reuse", "reuse", "reindex", "reuse", "reuse", "reuse"]


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "mxfp4"])
@pytest.mark.parametrize("per_request", [True, False])
def test_decoder_group_matches_oracle(kv_dtype, per_request, cuda_lib):
    """Indexer inputs are small integers (every fp32 score exact), so the
    selections and the pool must equal the oracle's; the attention outputs
    then differ only by the attention's own rounding.  per_request: one query
    per request without q_req (the fused tensor-core indexer)."""
    wl = Wk.WORKLOADS["decode64k"].scaled(topk=128, kv_dtype=kv_dtype, kv_group=16 if kv_dtype == "mxfp4" else 64)
    B, cap, block, pool_blocks, L = 2, 6000, 8, 64, len(MODES)
    seed = 4700 + len(kv_dtype)
    g = np.random.default_rng(seed)
    d, sd = wl.d, 1 / np.sqrt(wl.d)
    kidx = Wk.store(g.integers(-2, 3, size=(B, cap, wl.d_idx)).astype(np.float32), "bf16")
    q_idx = [Wk.store(g.integers(-2, 3, size=(B, wl.h_idx, wl.d_idx)).astype(np.float32), "bf16") for _ in range(L)]
    w = [g.choice(np.array([0.5, 1.0, 2.0], np.float32), size=(B, wl.h_idx)) for _ in range(L)]
    if kv_dtype == "mxfp4":
        kv = Wk.random_mxfp4(seed, "kv", (B, cap, d))
    else:
        kv = Wk.store(Wk.normal(seed, "kv", (B, cap, d), 1.0 if kv_dtype == "fp8" else sd), kv_dtype, 64)
    swa_cap = 128
    q = [Wk.store(Wk.normal(seed + l, "q", (B, wl.h_q, d), sd), "bf16") for l in range(L)]
    swa_k = [Wk.store(Wk.normal(seed + l, "sk", (B, swa_cap, d), sd), "bf16") for l in range(L)]
    swa_v = [Wk.store(Wk.normal(seed + l, "sv", (B, swa_cap, d), sd), "bf16") for l in range(L)]
    sink = [Wk.normal(seed + l, "sink", (wl.h_q,)) for l in range(L)]
    n_vis = np.array([cap, cap - 13], np.int32)
    q_pos = (n_vis.astype(np.int64) * wl.m + 2).astype(np.int64)
    q_req = None if per_request else np.arange(B, dtype=np.int32)

    p = params_of(wl, swa_cap)
    ws = csa.workspace(max(csa.csa_index_pool_workspace_size(p, B, cap, block, pool_blocks),
                           csa.csa_workspace_size(p, B, cap)))
    kidx_d, kv_d = dev(kidx), dev(kv)
    pool = torch.full((B, pool_blocks), -7, dtype=torch.int32, device="cuda")
    idx = torch.full((B, wl.topk), -7, dtype=torch.int32, device="cuda")
    sels, outs = [], []
    for l, mode in enumerate(MODES):
        if mode == "full":
            csa.csa_index_topk_pool(p, B, dev(q_idx[l]), f32(w[l]), kidx_d, B, cap,
                                    i32(q_req) if q_req is not None else None, i32(n_vis), block, pool_blocks,
                                    pool, idx, None, ws)
        elif mode == "reindex":
            fresh = torch.empty_like(idx)
            csa.csa_index_topk_reindex(p, B, dev(q_idx[l]), f32(w[l]), kidx_d, B, cap,
                                       i32(q_req) if q_req is not None else None, i32(n_vis), pool, block,
                                       pool_blocks, fresh, None, ws)
            idx = fresh
        out = DevTensor.empty((B, wl.h_q, d), "bf16")
        lse = torch.empty((B, wl.h_q), dtype=torch.float32, device="cuda")
        csa.csa_sparse_swa_attention(p, B, dev(q[l]), kv_d, B, cap, idx, i32(n_vis),
                                     i32(q_req) if q_req is not None else None, dev(swa_k[l]), dev(swa_v[l]),
                                     i64(q_pos), None, f32(sink[l]), out, lse, ws)
        torch.cuda.synchronize()
        sels.append(idx.cpu().numpy().copy())
        outs.append((to_f64(out), lse.double().cpu().numpy()))
    gpu_pool = pool.cpu().numpy()

    for b in range(B):
        n = int(n_vis[b])
        keys = O.decode(kidx.data[b, :n], "bf16")
        ref_sel, ref_pool = O.csa2_group_selections(MODES, [O.decode_stored(x)[b] for x in q_idx],
                                                    [x[b] for x in w], keys, block, pool_blocks, wl.topk)
        assert np.array_equal(gpu_pool[b], ref_pool), f"request {b}: candidate pool"
        rows = O.decode(kv.data[b], kv.dtype, None if kv.scale is None else kv.scale[b], kv.group)
        for l in range(L):
            assert np.array_equal(np.sort(sels[l][b]), np.sort(ref_sel[l])), f"request {b} layer {l}: selection"
            o, lse_ref = O.sparse_swa_attention(O.decode_stored(q[l])[b], rows, ref_sel[l], n,
                                                O.decode_stored(swa_k[l])[b], O.decode_stored(swa_v[l])[b], swa_cap,
                                                int(q_pos[b]), wl.window, sink[l], 1.0)
            check_attention(outs[l][0][b], outs[l][1][b], o, lse_ref, kv_dtype)
