"""Full-size parity: every published decode workload through csa_decode_step
(the launch configuration bench.py times), compared with the oracle on
sampled requests; the chunked-prefill workload at full size through the
pipeline entry points, compared on sampled queries."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import workloads as Wk
from oracle import csa_oracle as O
from tests._harness import GpuDecode, check_attention, check_selection, to_f64

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
    print(f"{name}: requests {reqs}, max-abs error {err:.3g}")


def test_prefill_full_size_sampled(cuda_lib):
    from tests.test_gpu_decode_step import _run_pipeline

    inp = Wk.make_prefill_inputs(Wk.WORKLOADS["prefill"])
    swaps = _run_pipeline(inp, exact=False, queries=[0, 1, 1000, 2047, 3000, 4095])
    print(f"prefill: boundary swaps {swaps}")
