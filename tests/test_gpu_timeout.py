"""Failure detection of the bounded device-side waits, without a fault: a
test request makes one CTA of the fused indexer skip its arrival at the
first per-request grid barrier, with a short poll limit.  The request's
waits must give up, the host must see CSA_ERR_TIMEOUT from csa_sync_status,
and the next call on the same stream must run normally and match the
oracle.  Nothing traps, faults or waits without a limit."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200 import workloads as Wk
from compressed_sparse_attention_compressor_b200.csa import CsaError
from oracle import csa_oracle as O
from tests._harness import check_selection, dev, f32, i32, params_of

pytestmark = pytest.mark.gpu


def _index_problem():
    wl = Wk.WORKLOADS["decode1m"].scaled(batch=2, context=4 * 40000)
    inp = Wk.make_decode_inputs(wl)
    B, cap = wl.batch, inp.cap
    return wl, inp, B, cap


def _call(wl, inp, B, cap, out_idx, ws):
    p = params_of(wl, 128)
    csa.csa_index_topk(p, B, dev(inp.q_idx), f32(inp.w), dev(inp.kidx), B, cap, None, i32(np.full(B, cap)), out_idx,
                       None, ws)


def test_expired_grid_barrier_reports_timeout_then_recovers(cuda_lib):
    wl, inp, B, cap = _index_problem()
    p = params_of(wl, 128)
    ws = csa.workspace(csa.csa_workspace_size(p, B, cap))
    out_idx = torch.full((B, wl.topk), -7, dtype=torch.int32, device="cuda")
    csa.csa_sync_status()  # nothing latched before the test
    # CTA 1 (request 0, whose chunks need every CTA's arrival) never arrives;
    # every wait of the launch gives up after 2,000 polls (~0.1 ms)
    csa.csa_test_expire_next_barrier(1, 2000)
    _call(wl, inp, B, cap, out_idx, ws)
    with pytest.raises(CsaError) as e:
        csa.csa_sync_status()
    assert e.value.status == 4, str(e.value)  # CSA_ERR_TIMEOUT
    csa.csa_sync_status()  # the error was reported once and cleared
    # the same stream, the next call: a normal launch, the oracle's selection
    out_idx.fill_(-7)
    _call(wl, inp, B, cap, out_idx, ws)
    csa.csa_sync_status()
    gi = out_idx.cpu().numpy()
    for b in range(B):
        keys = O.decode(inp.kidx.data[b], inp.kidx.dtype, inp.kidx.scale[b], inp.kidx.group)
        s = O.index_scores(O.decode(inp.q_idx.data[b], inp.q_idx.dtype), inp.w[b], keys)
        check_selection(gi[b], s, wl.topk, exact=False)


def test_withdrawn_request_leaves_launches_normal(cuda_lib):
    wl, inp, B, cap = _index_problem()
    p = params_of(wl, 128)
    ws = csa.workspace(csa.csa_workspace_size(p, B, cap))
    out_idx = torch.full((B, wl.topk), -7, dtype=torch.int32, device="cuda")
    csa.csa_test_expire_next_barrier(0, 10)
    csa.csa_test_expire_next_barrier(-1, 0)  # withdrawn before any launch
    _call(wl, inp, B, cap, out_idx, ws)
    csa.csa_sync_status()
    assert (out_idx >= 0).all()
