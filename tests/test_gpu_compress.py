"""a1 compressor: CUDA path vs the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import csa
from compressed_sparse_attention_compressor_b200 import workloads as Wk
from compressed_sparse_attention_compressor_b200.csa import DevTensor
from oracle import csa_oracle as O
from tests._harness import check_rows, dev, to_f64

pytestmark = pytest.mark.gpu

# (in dtype, out dtype, key dtype, batch, n_tokens, d, m, d_idx)
CASES = [
    ("f32", "f32", "f32", 1, 4099, 128, 4, 32),      # tiny shapes, ragged tail
    ("bf16", "bf16", "bf16", 2, 1031, 512, 4, 128),  # decode/prefill shapes
    ("bf16", "fp8", "fp8", 3, 515, 512, 4, 128),     # FP8 caches, per-64 / per-row scales
    ("bf16", "bf16", "bf16", 2, 1030, 512, 128, 128),  # HCA ratio
    ("f32", "f32", "f32", 1, 300, 64, 1, 32),          # ratio 1
    ("bf16", "bf16", "bf16", 2, 97, 512, 1, 128),
    ("bf16", "fp8", "fp8", 1, 130, 512, 2, 64),
]


def _inputs(i, dt, B, T, d, d_idx):
    C = Wk.store(Wk.normal(2000 + i, "C", (B, T, d), 1 / np.sqrt(d)), dt)
    Z = Wk.store(Wk.normal(2000 + i, "Z", (B, T, d), 2.0), dt)
    W = Wk.store(Wk.normal(2000 + i, "W", (d, d_idx), 1 / np.sqrt(d)), dt)
    return C, Z, W


@pytest.mark.parametrize("case", range(len(CASES)))
def test_compress_matches_oracle(case, cuda_lib):
    dt, odt, kdt, B, T, d, m, d_idx = CASES[case]
    C, Z, W = _inputs(case, dt, B, T, d, d_idx)
    n = T // m
    rows_cap = n + 3  # request stride larger than the rows written
    out = DevTensor.empty((B, rows_cap, d), odt, group=64)
    kout = DevTensor.empty((B, rows_cap, d_idx), kdt, group=d_idx)
    csa.csa_compress(dev(C), dev(Z), B, T, d, m, out, rows_cap, dev(W), d_idx, kout)
    torch.cuda.synchronize()
    got = to_f64(out)
    gotk = to_f64(kout)
    Cd, Zd, Wd = O.decode_stored(C), O.decode_stored(Z), O.decode_stored(W)
    for b in range(B):
        ref = O.compress(Cd[b], Zd[b], m)
        keys = O.project_index_keys(ref, Wd)
        sc = out.scale[b, :n].cpu().numpy() if odt == "fp8" else None
        ksc = kout.scale[b, :n].cpu().numpy() if kdt == "fp8" else None
        codes = out.data[b, :n].cpu().numpy() if odt == "fp8" else None
        kcodes = kout.data[b, :n].cpu().numpy() if kdt == "fp8" else None
        check_rows(got[b, :n], ref, odt, 64, sc, codes)
        check_rows(gotk[b, :n], keys, kdt, d_idx, ksc, kcodes)
        assert np.all(got[b, n:] == 0), "rows past the last complete block were written"
        if m == 1 and odt == dt:
            assert np.array_equal(got[b, :n], Cd[b]), "ratio 1 must copy C exactly"


def test_compress_without_projection_and_offset(cuda_lib):
    """Appending after cached rows through an offset view; no projection."""
    C, Z, _ = _inputs(99, "bf16", 1, 64, 512, 128)
    out = DevTensor.empty((1, 40, 512), "bf16")
    csa.csa_compress(dev(C), dev(Z), 1, 64, 512, 4, out.offset_rows(24), 16)
    torch.cuda.synchronize()
    got = to_f64(out)[0]
    ref = O.compress(O.decode_stored(C)[0], O.decode_stored(Z)[0], 4)
    assert np.all(got[:24] == 0)
    check_rows(got[24:40], ref, "bf16")
