"""a2 indexer + a3 top-k: CUDA path vs the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200 import workloads as Wk
from oracle import csa_oracle as O
from tests._harness import check_selection, gpu_index_topk, i32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("multi", [False, True])
@pytest.mark.parametrize("k,n_cols,pad", [(1, 10, 5), (64, 1000, 5), (512, 20000, 5), (1024, 100000, 5), (7, 5, 5),
                                         (1024, 100000, 4), (2048, 131072, 0), (33, 5003, 1)])
def test_topk_alone_is_bit_exact_with_ties(k, n_cols, pad, multi, cuda_lib):
    """Same fp32 scores on both sides: selection must match exactly,
    including planted exact ties, -0 vs +0, and rows with n_valid <= k.
    pad: row stride - n_cols (a multiple of 4 gives 16-byte aligned rows)."""
    rows = 6
    s = Wk.make_scores(3000 + k, rows, n_cols)
    n_valid = np.array([n_cols, n_cols - 1, min(n_cols, k), min(n_cols, k + 1), 0, max(n_cols // 3, 1)], np.int32)
    ld = n_cols + pad
    buf = np.zeros((rows, ld), np.float32)
    buf[:, :n_cols] = s
    scores = torch.from_numpy(buf).cuda()
    out_idx = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
    out_score = torch.empty((rows, k), dtype=torch.float32, device="cuda")
    # with a workspace, rows of more than 65,536 columns are split over several CTAs
    ws = csa.workspace(csa.csa_topk_workspace_size(rows)) if multi else None
    csa.csa_topk(scores, rows, ld, i32(n_valid), k, out_idx, out_score, ws)
    torch.cuda.synchronize()
    gi, gs = out_idx.cpu().numpy(), out_score.cpu().numpy()
    for r in range(rows):
        n = int(n_valid[r])
        ref = O.topk(buf[r, :n].astype(np.float64), k)
        assert np.array_equal(np.sort(gi[r]), np.sort(ref)), f"row {r}"
        sel = gi[r] >= 0
        assert np.array_equal(gs[r][sel], buf[r, gi[r][sel]])
        assert np.all(np.isneginf(gs[r][~sel]))


@pytest.mark.parametrize("n", [5000, 70000])
def test_topk_all_equal_scores_takes_lowest_indices(n, cuda_lib):
    """70,000 columns with a workspace: the rows are split over CTAs."""
    k = 300
    scores = torch.zeros((2, n), dtype=torch.float32, device="cuda")
    scores[1, ::2] = -0.0
    out_idx = torch.empty((2, k), dtype=torch.int32, device="cuda")
    csa.csa_topk(scores, 2, n, i32([n, n]), k, out_idx, None, csa.workspace(csa.csa_topk_workspace_size(2)))
    torch.cuda.synchronize()
    for r in range(2):
        assert np.array_equal(np.sort(out_idx[r].cpu().numpy()), np.arange(k))



def _shaped_rows(n):
    """Score rows whose shape decides which form of the row top-k runs:
    typical rows are selected among sampled candidates, while sorted rows
    (all winners in one warp's segment), rows whose sampled positions hold
    the largest scores (too few candidates), rows of few distinct values
    (many ties at the k-th score) and mostly -inf rows stress the sample's
    threshold and the fallback over the whole row."""
    g = Wk.rng(4100 + n, "shaped")
    rows = {
        "normal": g.standard_normal(n, dtype=np.float32),
        "ascending": np.arange(n, dtype=np.float32) / n,
        "descending": (n - np.arange(n, dtype=np.float32)) / n,
        "few_values": np.round(g.standard_normal(n)).astype(np.float32),
        "mostly_neg_inf": np.where(g.random(n) < 0.9, -np.inf, g.standard_normal(n)).astype(np.float32),
    }
    planted = (g.standard_normal(n) * 0.01).astype(np.float32)
    planted[np.arange(2048) * n // 2048] = 5 + g.random(2048, dtype=np.float32)
    rows["sample_positions_largest"] = planted
    return rows


@pytest.mark.parametrize("k", [512, 2048])
@pytest.mark.parametrize("n", [8192, 8193, 33000, 131072])
def test_topk_row_shapes_are_bit_exact(n, k, cuda_lib):
    """One CTA per row (no workspace): every row shape gives the oracle's
    selection, whichever form of the selection it takes."""
    shapes = _shaped_rows(n)
    names = list(shapes)
    buf = np.stack([shapes[x] for x in names])
    rows = buf.shape[0]
    scores = torch.from_numpy(buf).cuda()
    out_idx = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
    out_score = torch.empty((rows, k), dtype=torch.float32, device="cuda")
    csa.csa_topk(scores, rows, n, i32([n] * rows), k, out_idx, out_score, None)
    torch.cuda.synchronize()
    gi, gs = out_idx.cpu().numpy(), out_score.cpu().numpy()
    for r, name in enumerate(names):
        ref = O.topk(buf[r].astype(np.float64), k)
        assert np.array_equal(np.sort(gi[r]), np.sort(ref)), name
        assert np.array_equal(gs[r], buf[r, gi[r]]), name
        # the order inside a row is unspecified; the kernel writes at most two
        # runs of ascending indices (entries above the k-th score, then the
        # ones equal to it, or one run when the search ended on a whole bin)
        assert int(np.sum(np.diff(gi[r]) < 0)) <= 1, name

IDX_CASES = {
    # name: (workload, n_queries, batch, cap)
    "tiny_f32": (Wk.WORKLOADS["tiny"], 3, 3, 1024 + 37),
    "bf16": (Wk.WORKLOADS["decode64k"], 4, 2, 3000),
    "fp8": (Wk.WORKLOADS["decode1m"], 3, 3, 5000),
    "bf16_ratio1": (Wk.WORKLOADS["hybrid_ratio1"].scaled(topk=256), 2, 2, 2500),
}


@pytest.mark.parametrize("name", list(IDX_CASES))
def test_index_topk_matches_oracle(name, cuda_lib):
    wl, nq, B, cap = IDX_CASES[name]
    seed = 3100 + len(name)
    sI = 1 / np.sqrt(wl.d_idx)
    kidx = Wk.store(Wk.normal(seed, "kidx", (B, cap, wl.d_idx), sI), wl.idx_dtype, wl.d_idx)
    q_idx = Wk.store(Wk.normal(seed, "q_idx", (nq, wl.h_idx, wl.d_idx), sI), wl.act_dtype)
    w = Wk.uniform(seed, "w", (nq, wl.h_idx))
    q_req = np.arange(nq, dtype=np.int32) % B
    n_vis = np.array([cap, cap - 17, max(wl.topk // 2, 1), cap - 1][:nq], np.int32)
    gi, gs = gpu_index_topk(wl, q_idx, w, kidx, B, cap, q_req, n_vis)
    exact = wl.idx_dtype == "f32"
    qd = O.decode_stored(q_idx)
    swaps = 0
    for i in range(nq):
        keys = O.decode(kidx.data[q_req[i], : n_vis[i]], kidx.dtype,
                        None if kidx.scale is None else kidx.scale[q_req[i], : n_vis[i]], kidx.group)
        s = O.index_scores(qd[i], w[i], keys)
        swaps += check_selection(gi[i], s, wl.topk, exact, gs[i])
    print(f"{name}: boundary swaps {swaps}")


def test_index_topk_all_negative_dots_select_first_indices(cuda_lib):
    """Every score is exactly 0 (ReLU of negative dots): the tie rule picks
    indices 0..k-1."""
    wl = Wk.WORKLOADS["decode64k"]
    cap, k = 2000, 512
    keys = np.abs(Wk.normal(7, "k", (1, cap, wl.d_idx))) / 10
    q = -np.abs(Wk.normal(7, "q", (1, wl.h_idx, wl.d_idx))) / 10
    gi, gs = gpu_index_topk(wl, Wk.store(q, "bf16"), Wk.uniform(7, "w", (1, wl.h_idx)), Wk.store(keys, "bf16"), 1, cap,
                            None, np.array([cap], np.int32), k=k)
    assert np.array_equal(np.sort(gi[0]), np.arange(k))
    assert np.all(gs[0] == 0)


# one query per request, q_req = NULL: the fused tensor-core kernel
TC_CASES = {
    "fp8_ragged": (Wk.WORKLOADS["decode1m"], 3, 5000, [5000, 4983, 700]),
    "bf16": (Wk.WORKLOADS["decode64k"], 2, 3000, [3000, 2999]),
    "fp8_one_request_many_ctas": (Wk.WORKLOADS["decode1m"], 1, 20000, [19999]),
    "bf16_k2048": (Wk.WORKLOADS["hybrid_ratio1"], 2, 9000, [9000, 8000]),
    "bf16_fewer_than_k": (Wk.WORKLOADS["decode64k"], 2, 700, [300, 512]),
}


@pytest.mark.parametrize("name", list(TC_CASES))
def test_index_topk_tensor_core_path(name, cuda_lib):
    wl, B, cap, n_vis = TC_CASES[name]
    seed = 3300 + len(name)
    sI = 1 / np.sqrt(wl.d_idx)
    kidx = Wk.store(Wk.normal(seed, "kidx", (B, cap, wl.d_idx), sI), wl.idx_dtype, wl.d_idx)
    q_idx = Wk.store(Wk.normal(seed, "q_idx", (B, wl.h_idx, wl.d_idx), sI), wl.act_dtype)
    w = Wk.uniform(seed, "w", (B, wl.h_idx))
    n_vis = np.array(n_vis, np.int32)
    gi, gs = gpu_index_topk(wl, q_idx, w, kidx, B, cap, None, n_vis)
    qd = O.decode_stored(q_idx)
    swaps = 0
    for i in range(B):
        keys = O.decode(kidx.data[i, : n_vis[i]], kidx.dtype,
                        None if kidx.scale is None else kidx.scale[i, : n_vis[i]], kidx.group)
        s = O.index_scores(qd[i], w[i], keys)
        swaps += check_selection(gi[i], s, wl.topk, False, gs[i])
    print(f"{name}: boundary swaps {swaps}")


@pytest.mark.parametrize("dt", ["fp8", "bf16"])
def test_index_topk_tensor_core_all_ties(dt, cuda_lib):
    """Every score is exactly 0 across many CTAs: the selection is the k
    lowest indices, assembled by the last CTA of each request."""
    wl = Wk.WORKLOADS["decode1m" if dt == "fp8" else "decode64k"]
    B, cap = 2, 30000
    keys = np.abs(Wk.normal(8, "k", (B, cap, wl.d_idx))) / 10
    q = -np.abs(Wk.normal(8, "q", (B, wl.h_idx, wl.d_idx))) / 10
    gi, gs = gpu_index_topk(wl, Wk.store(q, "bf16"), Wk.uniform(8, "w", (B, wl.h_idx)),
                            Wk.store(keys, dt, wl.d_idx), B, cap, None, np.array([cap, cap - 5], np.int32))
    for i in range(B):
        assert np.array_equal(gi[i], np.arange(wl.topk)), "ties must keep the lowest indices, in index order"
        assert np.all(gs[i] == 0)


def test_index_topk_tensor_core_is_deterministic(cuda_lib):
    wl = Wk.WORKLOADS["decode1m"]
    B, cap = 2, 40000
    kidx = Wk.store(Wk.normal(9, "kidx", (B, cap, wl.d_idx)), "fp8", wl.d_idx)
    q_idx = Wk.store(Wk.normal(9, "q", (B, wl.h_idx, wl.d_idx)), "bf16")
    w = Wk.uniform(9, "w", (B, wl.h_idx))
    n_vis = np.array([cap, cap], np.int32)
    a, sa = gpu_index_topk(wl, q_idx, w, kidx, B, cap, None, n_vis)
    b, sb = gpu_index_topk(wl, q_idx, w, kidx, B, cap, None, n_vis)
    assert np.array_equal(a, b) and np.array_equal(sa, sb)


@pytest.mark.parametrize("dt", ["fp8", "bf16"])
def test_index_topk_tensor_core_zero_ties_resolved_in_shared_memory(dt, cuda_lib):
    """A few hundred keys score above zero, every other key scores exactly 0
    and the zeros fit the shared-memory boundary list: the selection is every
    positive key plus the lowest-index zeros, bit-exact."""
    wl = Wk.WORKLOADS["decode1m" if dt == "fp8" else "decode64k"]
    cap, k, n_pos = 8000, 512, 300
    rng = np.random.default_rng(11)
    pos_rows = np.sort(rng.choice(cap, n_pos, replace=False))
    keys = np.abs(Wk.normal(11, "k", (1, cap, wl.d_idx))) / 10
    keys[0, pos_rows] *= -1.0  # q < 0 everywhere: these rows have positive dots
    q = -np.abs(Wk.normal(11, "q", (1, wl.h_idx, wl.d_idx))) / 10
    gi, gs = gpu_index_topk(wl, Wk.store(q, "bf16"), Wk.uniform(11, "w", (1, wl.h_idx)),
                            Wk.store(keys, dt, wl.d_idx), 1, cap, None, np.array([cap], np.int32), k=k)
    zeros = np.setdiff1d(np.arange(cap), pos_rows)[: k - n_pos]
    assert np.array_equal(np.sort(gi[0]), np.sort(np.concatenate([pos_rows, zeros])))
    sel_zero = np.isin(gi[0], zeros)
    assert np.all(gs[0][sel_zero] == 0) and np.all(gs[0][~sel_zero] > 0)


def test_index_topk_tensor_core_crowded_bin_takes_second_level(cuda_lib):
    """All scores within a few per cent of each other: the top 12 key bits
    put more than the shared-memory list holds into the boundary bin, so the
    kernel narrows the boundary with a second distributed histogram level."""
    wl = Wk.WORKLOADS["decode64k"]
    cap = 30000
    sI = 1 / np.sqrt(wl.d_idx)
    base = Wk.normal(12, "base", (1, 1, wl.d_idx), sI)
    keys = base + 0.03 * Wk.normal(12, "noise", (1, cap, wl.d_idx), sI)
    kidx = Wk.store(keys, "bf16")
    q_idx = Wk.store(Wk.normal(12, "q", (1, wl.h_idx, wl.d_idx), sI), "bf16")
    w = Wk.uniform(12, "w", (1, wl.h_idx))
    gi, gs = gpu_index_topk(wl, q_idx, w, kidx, 1, cap, None, np.array([cap], np.int32))
    s = O.index_scores(O.decode_stored(q_idx)[0], w[0], O.decode(kidx.data[0], "bf16", None, 0))
    top = np.sort(s)[::-1]
    assert top[0] / top[-1] < 1.1, "the scores are meant to crowd one 12-bit key bin"
    check_selection(gi[0], s, wl.topk, False, gs[0])
