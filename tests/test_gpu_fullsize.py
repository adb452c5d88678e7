"""Full-size parity: every published decode workload through csa_decode_step
(the launch configuration bench.py times), compared with the oracle on
sampled requests; the chunked-prefill workload at full size through the
pipeline entry points, compared on sampled queries."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import workloads as Wk
from oracle import csa_oracle as O
from tests._harness import GpuDecode, check_attention, check_selection, gpu_index_topk, to_f64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = {
    "decode1m": [0, 1, 2, 3],
    "decode64k": [0, 7, 15],
    "hybrid_csa": [0, 5],
    "hybrid_hca": [0, 7],
    "hybrid_ratio1": [3],
    "decode1m_fp4": [1, 2],
}


@pytest.mark.parametrize("name", list(FULL))
def test_decode_full_size(name, cuda_lib):
    wl = Wk.WORKLOADS[name]
    inp = Wk.make_decode_inputs(wl)
    g = GpuDecode(inp)
    g.step()
    torch.cuda.synchronize()
    reqs = FULL[name]
    ref = O.decode_step(inp, requests=reqs)
    got, got_lse = to_f64(g.out)[reqs], g.lse.double().cpu().numpy()[reqs]
    err = check_attention(got, got_lse, ref["out"], ref["lse"], wl.kv_dtype)
    # the selection of the fused indexer (with the token's append inside it)
    swaps = g.check_selections(ref, reqs)
    print(f"{name}: requests {reqs}, max-abs error {err:.3g}, boundary swaps {swaps}")


@pytest.mark.parametrize("name", ["decode1m", "hybrid_csa", "hybrid_ratio1"])
def test_index_topk_full_size(name, cuda_lib):
    """csa_index_topk alone over a full-size cache (the fused indexer without
    the append: decode1m's FP8 keys, 262,144 per request, top-1,024;
    hybrid_csa's 65,536 bf16 keys, top-512; hybrid_ratio1's 262,144 bf16
    keys, top-2,048): every request's set against the oracle's, with its
    reported scores."""
    wl = Wk.WORKLOADS[name]
    inp = Wk.make_decode_inputs(wl)
    B, cap = wl.batch, inp.cap
    n_vis = np.full(B, cap, np.int32)
    gi, gs = gpu_index_topk(wl, inp.q_idx, inp.w, inp.kidx, B, cap, None, n_vis)
    swaps = 0
    for b in FULL[name]:
        keys = O.decode(inp.kidx.data[b], inp.kidx.dtype, None if inp.kidx.scale is None else inp.kidx.scale[b],
                        inp.kidx.group)
        s = O.index_scores(O.decode(inp.q_idx.data[b], inp.q_idx.dtype), inp.w[b], keys)
        swaps += check_selection(gi[b], s, wl.topk, False, gs[b])
    print(f"{name}: index top-{wl.topk} of {cap} entries, requests {FULL[name]}, boundary swaps {swaps}")


def test_prefill_full_size_sampled(cuda_lib):
    from tests.test_gpu_decode_step import _run_pipeline

    inp = Wk.make_prefill_inputs(Wk.WORKLOADS["prefill"])
    swaps = _run_pipeline(inp, exact=False, queries=[0, 1, 1000, 2047, 3000, 4095])
    print(f"prefill: boundary swaps {swaps}")
