"""csa_sparse_swa_attention_noalloc: the attention entry point for callers
that cannot allocate device memory (a plugin whose host application owns all
device memory, or a loop that cannot pay cudaMalloc's device-wide
synchronisation).  It must give the same results as the workspace entry
point, call after call, and refuse problems larger than its fixed scratch.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200 import workloads as Wk
from compressed_sparse_attention_compressor_b200.csa import CsaError, DevTensor
from oracle import csa_oracle as O
from tests._harness import check_attention, dev, f32, i32, i64, params_of, to_f64

pytestmark = pytest.mark.gpu


def _problem(nq=4, cap=20000):
    wl = Wk.WORKLOADS["decode1m"]
    d = wl.d
    kv = Wk.store(Wk.normal(51, "kv", (nq, cap, d)), "fp8", 64)
    sk = Wk.store(Wk.normal(51, "sk", (nq, 128, d), 1 / np.sqrt(d)), "bf16")
    sv = Wk.store(Wk.normal(51, "sv", (nq, 128, d), 1 / np.sqrt(d)), "bf16")
    q = Wk.store(Wk.normal(51, "q", (nq, wl.h_q, d), 1 / np.sqrt(d)), "bf16")
    n_vis = np.full(nq, cap, np.int32)
    idx = Wk.make_indices(51, n_vis, wl.topk)
    args = dict(q=dev(q), kv=dev(kv), idx=i32(idx), n_vis=i32(n_vis), swa_k=dev(sk), swa_v=dev(sv),
                q_pos=i64(np.full(nq, 4 * cap - 1)), sink=f32(Wk.normal(51, "sink", (wl.h_q,))))
    return wl, params_of(wl, 128), nq, cap, args


def _run(fn, wl, p, nq, cap, a, with_ws):
    out = DevTensor.empty((nq, wl.h_q, wl.d), "bf16")
    lse = torch.empty((nq, wl.h_q), dtype=torch.float32, device="cuda")
    extra = [csa.workspace(csa.csa_workspace_size(p, nq, cap))] if with_ws else []
    fn(p, nq, a["q"], a["kv"], nq, cap, a["idx"], a["n_vis"], None, a["swa_k"], a["swa_v"], a["q_pos"], None,
       a["sink"], out, lse, *extra)
    torch.cuda.synchronize()
    return to_f64(out), lse.double().cpu().numpy()


def test_noalloc_matches_workspace_entry_point_twice(cuda_lib):
    """Top-1,024 + window per query: one cluster per query, merged in
    distributed shared memory (no scratch written).  The same kernels run on
    the same inputs, so the bytes must be equal."""
    wl, p, nq, cap, a = _problem()
    ref_out, ref_lse = _run(csa.csa_sparse_swa_attention, wl, p, nq, cap, a, True)
    for _ in range(2):
        out, lse = _run(csa.csa_sparse_swa_attention_noalloc, wl, p, nq, cap, a, False)
        assert np.array_equal(out, ref_out) and np.array_equal(lse, ref_lse)


def _dense_problem(seed, nq=2, cap=3000):
    """Dense (HCA) attention over up to 3,000 bf16 entries + the window:
    25 key tiles per query, more than one cluster of 16 CTAs holds, so the
    kernel takes its split path -- per-tile partial softmax states in the
    scratch, then a merge kernel.  (The scratch the call reserves, about
    13 MB, stays under the library's fixed 16 MiB.)"""
    wl = Wk.WORKLOADS["hybrid_hca"]
    d = wl.d
    sd = 1 / np.sqrt(d)
    kv = Wk.store(Wk.normal(seed, "kv", (nq, cap, d), sd), "bf16")
    sk = Wk.store(Wk.normal(seed, "sk", (nq, 128, d), sd), "bf16")
    sv = Wk.store(Wk.normal(seed, "sv", (nq, 128, d), sd), "bf16")
    q = Wk.store(Wk.normal(seed, "q", (nq, wl.h_q, d), sd), "bf16")
    sink = Wk.normal(seed, "sink", (wl.h_q,))
    n_vis = np.array([cap, cap - 1000][:nq], np.int32)
    q_pos = (4 * n_vis.astype(np.int64) + 3)
    args = dict(q=dev(q), kv=dev(kv), idx=None, n_vis=i32(n_vis), swa_k=dev(sk), swa_v=dev(sv), q_pos=i64(q_pos),
                sink=f32(sink))
    host = dict(q=q, kv=kv, sk=sk, sv=sv, sink=sink, n_vis=n_vis, q_pos=q_pos)
    return wl, params_of(wl, 128), nq, cap, args, host


def test_noalloc_split_path_uses_its_scratch_and_matches(cuda_lib):
    """The split path writes every query's per-tile (max, sum, O) states into
    the library's scratch array and merges them.  Two calls in a row, with a
    different problem in between that leaves other values in the scratch:
    each result equals the workspace entry point's bit for bit, and the
    oracle within the tolerance."""
    wl, p, nq, cap, a, h = _dense_problem(61)
    need = csa.csa_workspace_size(p, nq, cap)
    assert need > 4 * nq * 64 * 514 * 4, "the problem must need split states (scratch)"
    ref_out, ref_lse = _run(csa.csa_sparse_swa_attention, wl, p, nq, cap, a, True)
    wl2, p2, nq2, cap2, a2, _ = _dense_problem(62)
    for _ in range(2):
        out, lse = _run(csa.csa_sparse_swa_attention_noalloc, wl, p, nq, cap, a, False)
        assert np.array_equal(out, ref_out) and np.array_equal(lse, ref_lse)
        _run(csa.csa_sparse_swa_attention_noalloc, wl2, p2, nq2, cap2, a2, False)  # other scratch contents
    qd = O.decode_stored(h["q"])
    sk, sv = O.decode_stored(h["sk"]), O.decode_stored(h["sv"])
    for i in range(nq):
        rows = O.decode(h["kv"].data[i], "bf16")
        o, l = O.sparse_swa_attention(qd[i], rows, None, int(h["n_vis"][i]), sk[i], sv[i], 128, int(h["q_pos"][i]),
                                      wl.window, h["sink"], 1.0)
        check_attention(out[i], lse[i], o, l, "bf16")


def test_noalloc_refuses_problems_beyond_its_scratch(cuda_lib):
    """Two queries, dense over a very long claimed context: many splits per
    query, whose partial states need more than the fixed scratch.  The call
    is refused before any launch (nothing visible is read either way)."""
    wl, p, nq, cap, a = _problem(nq=4, cap=4000)
    two = 2
    q = DevTensor.empty((two, wl.h_q, wl.d), "bf16")
    out = DevTensor.empty((two, wl.h_q, wl.d), "bf16")
    p.topk = 0
    with pytest.raises(CsaError) as e:
        csa.csa_sparse_swa_attention_noalloc(p, two, q, a["kv"], nq, 1 << 20, None, i32(np.zeros(two)), None,
                                             a["swa_k"], a["swa_v"], i64(np.zeros(two)), None, None, out, None)
    assert "scratch" in str(e.value) and e.value.status == 3
