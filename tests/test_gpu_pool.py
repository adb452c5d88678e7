"""Hierarchical sparse indexer (candidate pool of the Full layer, re-indexing
inside it): CUDA path vs the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200 import workloads as Wk
from oracle import csa_oracle as O
from tests._harness import check_selection, dev, f32, i32, params_of

pytestmark = pytest.mark.gpu


def gpu_pool(wl, q_idx_st, w, kidx_st, batch, cap, q_req, n_vis, block, pool_blocks, with_idx=True):
    p = params_of(wl, max(wl.window, 1))
    nq = q_idx_st.data.shape[0]
    out_pool = torch.full((nq, pool_blocks), -7, dtype=torch.int32, device="cuda")
    out_idx = torch.full((nq, p.topk), -7, dtype=torch.int32, device="cuda") if with_idx else None
    ws = csa.workspace(csa.csa_index_pool_workspace_size(p, nq, cap, block, pool_blocks))
    csa.csa_index_topk_pool(p, nq, dev(q_idx_st), f32(w), dev(kidx_st), batch, cap,
                            i32(q_req) if q_req is not None else None, i32(n_vis), block, pool_blocks, out_pool,
                            out_idx, None, ws)
    torch.cuda.synchronize()
    return out_pool.cpu().numpy(), (out_idx.cpu().numpy() if with_idx else None)


def gpu_reindex(wl, q_idx_st, w, kidx_st, batch, cap, q_req, n_vis, pool, block, k=None):
    p = params_of(wl, max(wl.window, 1))
    if k is not None:
        p.topk = k
    nq, pool_blocks = pool.shape
    out_idx = torch.full((nq, p.topk), -7, dtype=torch.int32, device="cuda")
    out_score = torch.empty((nq, p.topk), dtype=torch.float32, device="cuda")
    ws = csa.workspace(csa.csa_index_pool_workspace_size(p, nq, cap, block, pool_blocks))
    csa.csa_index_topk_reindex(p, nq, dev(q_idx_st), f32(w), dev(kidx_st), batch, cap,
                               i32(q_req) if q_req is not None else None, i32(n_vis), i32(pool), block, pool_blocks,
                               out_idx, out_score, ws)
    torch.cuda.synchronize()
    return out_idx.cpu().numpy(), out_score.cpu().numpy()


def keys_of(kidx, r, n):
    return O.decode(kidx.data[r, :n], kidx.dtype, None if kidx.scale is None else kidx.scale[r, :n], kidx.group)


def check_pool_row(gpu_pool_row, scores, block, pool_blocks, exact):
    """The pool as a set of blocks (boundary swaps allowed unless exact),
    written in ascending block order, -1 padded at the end."""
    valid = gpu_pool_row[gpu_pool_row >= 0]
    assert np.all(gpu_pool_row[valid.shape[0]:] == -1), "padding must follow the block ids"
    assert np.all(np.diff(valid) > 0), "pool block ids must ascend"
    bs = O.block_scores(scores, block)
    if exact:
        assert np.array_equal(gpu_pool_row, O.candidate_pool(scores, block, pool_blocks))
        return 0
    return check_selection(gpu_pool_row, bs, pool_blocks, False)


def check_reindex_row(gpu_ids, gpu_sc, pool_row, block, keys, q, w, k, exact):
    """A Reindex selection: entry ids drawn from the pool, compared with the
    oracle's top k of the pool's scores (as pool positions)."""
    ent = O.pool_entries(pool_row, block, keys.shape[0])
    ref_ids, s_pool = O.reindex_topk(q, w, keys, pool_row, block, k)
    if exact:
        assert np.array_equal(np.sort(gpu_ids), np.sort(ref_ids))
        sel = gpu_ids >= 0
        assert np.array_equal(gpu_sc[sel].astype(np.float64), O.index_scores(q, w, keys[gpu_ids[sel]]))
        return 0
    where = {int(e): i for i, e in enumerate(ent)}
    assert all(int(e) in where for e in gpu_ids[gpu_ids >= 0]), "selected entry outside the pool"
    pos = np.array([where[int(e)] if e >= 0 else -1 for e in gpu_ids], np.int64)
    gsc = np.where(gpu_ids >= 0, gpu_sc, -np.inf)
    return check_selection(pos, s_pool, k, False, gsc)


# ---------------------------------------------------------------------------
# exact: small-integer keys, queries and weights make every fp32 score exact,
# so the GPU must reproduce the oracle's pool and selections bit for bit,
# including the tie rules (many equal scores, duplicated blocks)
# ---------------------------------------------------------------------------
def integer_inputs(seed, wl, nq, B, cap, dup_blocks, block):
    g = np.random.default_rng(seed)
    k = g.integers(-2, 3, size=(B, cap, wl.d_idx)).astype(np.float32)
    for b in range(B):  # exact block ties: copies of block 3 further on
        for c in dup_blocks:
            if (c + 1) * block <= cap and 4 * block <= cap:
                k[b, c * block:(c + 1) * block] = k[b, 3 * block:4 * block]
    q = g.integers(-2, 3, size=(nq, wl.h_idx, wl.d_idx)).astype(np.float32)
    w = g.choice(np.array([0.5, 1.0, 2.0], np.float32), size=(nq, wl.h_idx))
    return Wk.store(k, wl.idx_dtype, wl.d_idx), Wk.store(q, wl.act_dtype), w


EXACT = {
    # name: (workload, n_queries, batch, cap, block, pool_blocks)
    "f32_b8": (Wk.WORKLOADS["tiny"].scaled(topk=40), 3, 2, 1000 + 5, 8, 24),
    "f32_b1": (Wk.WORKLOADS["tiny"].scaled(topk=40), 2, 2, 700, 1, 64),
    "bf16_b8": (Wk.WORKLOADS["decode64k"].scaled(topk=128), 3, 3, 6000 + 3, 8, 96),
    "bf16_b128": (Wk.WORKLOADS["decode64k"].scaled(topk=128), 2, 2, 9000, 128, 7),
    "bf16_b32_many_chunks": (Wk.WORKLOADS["decode64k"].scaled(topk=256), 2, 2, 150000, 32, 300),
    # 70,000 single-entry blocks per query: the pool is selected by several CTAs per query (> 65,536)
    "bf16_b1_long_rows": (Wk.WORKLOADS["decode64k"].scaled(topk=128), 2, 2, 70000, 1, 3000),
}


@pytest.mark.parametrize("per_request", [False, True])
@pytest.mark.parametrize("name", list(EXACT))
def test_pool_and_reindex_exact(name, per_request, cuda_lib):
    """per_request: one query per request without q_req, the form that the
    fused tensor-core indexer takes for bf16 / FP8 keys of 64 x 128."""
    wl, nq, B, cap, block, pool_blocks = EXACT[name]
    if per_request and nq != B:
        pytest.skip("needs one query per request")
    seed = 4200 + len(name)
    kidx, q_idx, w = integer_inputs(seed, wl, nq, B, cap, dup_blocks=(7, 11, 40), block=block)
    q_req = (np.arange(nq) % B).astype(np.int32)
    # full cache, a partial last block, fewer blocks than the pool holds
    n_vis = np.array([cap, cap - block // 2 - 1, min(cap, block * pool_blocks // 2 + 3)][:nq], np.int32)
    gp, gi = gpu_pool(wl, q_idx, w, kidx, B, cap, None if per_request else q_req, n_vis, block, pool_blocks)
    qd = O.decode_stored(q_idx)
    pools = []
    for i in range(nq):
        keys = keys_of(kidx, q_req[i], n_vis[i])
        s = O.index_scores(qd[i], w[i], keys)
        check_pool_row(gp[i], s, block, pool_blocks, exact=True)
        assert np.array_equal(np.sort(gi[i]), np.sort(O.topk(s, wl.topk))), "Full layer top-k"
        pools.append(O.candidate_pool(s, block, pool_blocks))
    # a Reindex layer: its own query and weights over the oracle's pool
    _, q2, w2 = integer_inputs(seed + 1, wl, nq, B, cap, (), block)
    pool = np.stack(pools).astype(np.int32)
    ri, rs = gpu_reindex(wl, q2, w2, kidx, B, cap, None if per_request else q_req, n_vis, pool, block)
    q2d = O.decode_stored(q2)
    for i in range(nq):
        check_reindex_row(ri[i], rs[i], pool[i], block, keys_of(kidx, q_req[i], n_vis[i]), q2d[i], w2[i], wl.topk,
                          exact=True)


# ---------------------------------------------------------------------------
# seeded normal inputs in the workloads' precisions
# ---------------------------------------------------------------------------
CASES = {
    "fp8": (Wk.WORKLOADS["decode1m"], 3, 3, 40000 + 8, 8, 512),
    "fp8_ragged_cap": (Wk.WORKLOADS["decode1m"], 3, 3, 40000 + 4, 8, 512),
    "fp8_b16": (Wk.WORKLOADS["decode1m"], 2, 2, 60000, 16, 300),
    "bf16": (Wk.WORKLOADS["decode64k"], 2, 2, 20000, 8, 256),
    "f32": (Wk.WORKLOADS["tiny"], 2, 1, 3000, 16, 40),
}


@pytest.mark.parametrize("per_request", [False, True])
@pytest.mark.parametrize("name", list(CASES))
def test_pool_and_reindex_match_oracle(name, per_request, cuda_lib):
    wl, nq, B, cap, block, pool_blocks = CASES[name]
    if per_request and nq != B:
        pytest.skip("needs one query per request")
    seed = 4300 + len(name)
    sI = 1 / np.sqrt(wl.d_idx)
    kidx = Wk.store(Wk.normal(seed, "kidx", (B, cap, wl.d_idx), sI), wl.idx_dtype, wl.d_idx)
    q_idx = Wk.store(Wk.normal(seed, "q_idx", (nq, wl.h_idx, wl.d_idx), sI), wl.act_dtype)
    w = Wk.uniform(seed, "w", (nq, wl.h_idx))
    q_req = (np.arange(nq) % B).astype(np.int32)
    n_vis = np.array([cap, cap - 3, block * pool_blocks // 3 + 1][:nq], np.int32)
    gp, gi = gpu_pool(wl, q_idx, w, kidx, B, cap, None if per_request else q_req, n_vis, block, pool_blocks)
    exact = wl.idx_dtype == "f32"
    qd = O.decode_stored(q_idx)
    swaps = 0
    for i in range(nq):
        keys = keys_of(kidx, q_req[i], n_vis[i])
        s = O.index_scores(qd[i], w[i], keys)
        swaps += check_pool_row(gp[i], s, block, pool_blocks, exact=False)
        swaps += check_selection(gi[i], s, wl.topk, exact)
    # Reindex over a seeded pool: ascending random blocks, -1 padded, one
    # block running past the visible entries
    q2 = Wk.store(Wk.normal(seed + 1, "q_idx", (nq, wl.h_idx, wl.d_idx), sI), wl.act_dtype)
    w2 = Wk.uniform(seed + 1, "w", (nq, wl.h_idx))
    g = np.random.default_rng(seed)
    pool = np.full((nq, pool_blocks), -1, np.int32)
    for i in range(nq):
        nb = (int(n_vis[i]) + block - 1) // block
        take = min(nb, pool_blocks - 5)
        # the last (possibly partial) block is always in the pool
        ch = np.sort(g.choice(nb - 1, size=take - 1, replace=False)) if take > 1 else np.zeros(0, np.int64)
        pool[i, :take] = np.append(ch, nb - 1)
    ri, rs = gpu_reindex(wl, q2, w2, kidx, B, cap, None if per_request else q_req, n_vis, pool, block)
    q2d = O.decode_stored(q2)
    for i in range(nq):
        swaps += check_reindex_row(ri[i], rs[i], pool[i], block, keys_of(kidx, q_req[i], n_vis[i]), q2d[i], w2[i],
                                   wl.topk, exact=False)
    print(f"{name}: boundary swaps {swaps}")


def test_reindex_pool_smaller_than_k_and_empty_slots(cuda_lib):
    """Fewer candidates than k: every candidate is kept, the rest is -1 /
    -inf; empty pool slots and blocks past n_visible contribute nothing."""
    wl = Wk.WORKLOADS["decode64k"].scaled(topk=64)
    B, cap, block = 1, 4096, 8
    seed = 4400
    sI = 1 / np.sqrt(wl.d_idx)
    kidx = Wk.store(Wk.normal(seed, "kidx", (B, cap, wl.d_idx), sI), wl.idx_dtype, wl.d_idx)
    q_idx = Wk.store(Wk.normal(seed, "q_idx", (1, wl.h_idx, wl.d_idx), sI), wl.act_dtype)
    w = Wk.uniform(seed, "w", (1, wl.h_idx))
    n_vis = np.array([1003], np.int32)  # block 125 holds 3 visible entries
    pool = np.array([[2, 9, 125, 126, 400, -1, -1, -1]], np.int32)
    ri, rs = gpu_reindex(wl, q_idx, w, kidx, B, cap, None, n_vis, pool, block)
    expect = set(O.pool_entries(pool[0], block, 1003).tolist())
    assert len(expect) == 8 + 8 + 3
    got = ri[0][ri[0] >= 0]
    assert set(got.tolist()) == expect and got.shape[0] == len(expect)
    assert np.all(ri[0][ri[0] < 0] == -1) and np.all(np.isneginf(rs[0][ri[0] < 0]))


@pytest.mark.slow
def test_pool_full_size_decode1m(cuda_lib):
    """The page's pool at 1M context: 262,144 entries (m = 4), blocks of 8,
    a 2,048-block (16,384-candidate) pool, top 1,024; FP8 keys, 4 requests."""
    wl = Wk.WORKLOADS["decode1m"]
    B, cap, block, pool_blocks = wl.batch, wl.context // wl.m, 8, 2048
    seed = 4500
    sI = 1 / np.sqrt(wl.d_idx)
    kidx = Wk.store(Wk.normal(seed, "kidx", (B, cap, wl.d_idx), sI), wl.idx_dtype, wl.d_idx)
    q_idx = Wk.store(Wk.normal(seed, "q_idx", (B, wl.h_idx, wl.d_idx), sI), wl.act_dtype)
    w = Wk.uniform(seed, "w", (B, wl.h_idx))
    n_vis = np.array([cap, cap - 1, cap - 5, cap // 2 + 3], np.int32)
    gp, gi = gpu_pool(wl, q_idx, w, kidx, B, cap, None, n_vis, block, pool_blocks)
    qd = O.decode_stored(q_idx)
    pools = []
    for i in range(B):
        keys = keys_of(kidx, i, n_vis[i])
        s = O.index_scores(qd[i], w[i], keys)
        check_pool_row(gp[i], s, block, pool_blocks, exact=False)
        check_selection(gi[i], s, wl.topk, False)
        pools.append(O.candidate_pool(s, block, pool_blocks))
    # the Reindex layer runs over the oracle's pool
    pool = np.stack(pools).astype(np.int32)
    q2 = Wk.store(Wk.normal(seed + 1, "q_idx", (B, wl.h_idx, wl.d_idx), sI), wl.act_dtype)
    w2 = Wk.uniform(seed + 1, "w", (B, wl.h_idx))
    ri, rs = gpu_reindex(wl, q2, w2, kidx, B, cap, None, n_vis, pool, block)
    q2d = O.decode_stored(q2)
    for i in range(B):
        check_reindex_row(ri[i], rs[i], pool[i], block, keys_of(kidx, i, n_vis[i]), q2d[i], w2[i], wl.topk,
                          exact=False)


@pytest.mark.parametrize("per_request", [False, True])
def test_pool_and_reindex_edge_cases(per_request, cuda_lib):
    """Requests with no visible entry, fewer entries than one block, exactly
    one block, and exactly pool_blocks blocks; k larger than the candidates."""
    wl = Wk.WORKLOADS["decode64k"].scaled(topk=64)
    B, cap, block, pool_blocks = 4, 2048, 8, 16
    seed = 4900
    kidx, q_idx, w = integer_inputs(seed, wl, B, B, cap, (), block)
    n_vis = np.array([0, 5, 8, block * pool_blocks], np.int32)
    q_req = None if per_request else np.arange(B, dtype=np.int32)
    gp, gi = gpu_pool(wl, q_idx, w, kidx, B, cap, q_req, n_vis, block, pool_blocks)
    qd = O.decode_stored(q_idx)
    pools = []
    for i in range(B):
        keys = keys_of(kidx, i, n_vis[i])
        s = O.index_scores(qd[i], w[i], keys) if n_vis[i] else np.zeros(0)
        ref_pool = O.candidate_pool(s, block, pool_blocks) if n_vis[i] else np.full(pool_blocks, -1)
        assert np.array_equal(gp[i], ref_pool), f"request {i}: pool"
        assert np.array_equal(np.sort(gi[i]), np.sort(O.topk(s, wl.topk))), f"request {i}: top-k"
        pools.append(ref_pool)
    pool = np.stack(pools).astype(np.int32)
    _, q2, w2 = integer_inputs(seed + 1, wl, B, B, cap, (), block)
    ri, rs = gpu_reindex(wl, q2, w2, kidx, B, cap, q_req, n_vis, pool, block)
    q2d = O.decode_stored(q2)
    for i in range(B):
        keys = keys_of(kidx, i, n_vis[i])
        ent = O.pool_entries(pool[i], block, int(n_vis[i]))
        if ent.shape[0] == 0:
            assert np.all(ri[i] == -1) and np.all(np.isneginf(rs[i])), f"request {i}: empty pool"
            continue
        check_reindex_row(ri[i], rs[i], pool[i], block, keys, q2d[i], w2[i], wl.topk, exact=True)
