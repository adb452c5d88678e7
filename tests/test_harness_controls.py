"""Negative controls of the GPU parity checks (CPU only): the comparisons in
tests/_harness.py must reject outputs that are wrong, however small the
outputs are.  bf16 workloads draw values as N(0,1)/sqrt(d), so their
attention outputs are about 0.005-0.1: an absolute 2e-2 bar alone would pass
an all-zero output."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_compressor_b200 import workloads as Wk
from oracle import csa_oracle as O
from tests._harness import check_attention, check_selection


@pytest.fixture(scope="module")
def small_bf16_step():
    wl = Wk.WORKLOADS["decode64k"].scaled(batch=2, context=2048)
    ref = O.decode_step(Wk.make_decode_inputs(wl))
    assert np.abs(ref["out"]).max() < 2e-2  # the regime the scaled bar exists for
    return ref


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).double().numpy()


def test_correct_bf16_output_passes(small_bf16_step):
    ref = small_bf16_step
    check_attention(_bf16(ref["out"]), ref["lse"].astype(np.float32), ref["out"], ref["lse"], "bf16")


@pytest.mark.parametrize("wrong", ["zeros", "scaled_0.9", "noise", "permuted_heads"])
def test_wrong_small_output_fails(small_bf16_step, wrong):
    ref = small_bf16_step
    out = ref["out"]
    g = np.random.default_rng(3)
    bad = {"zeros": np.zeros_like(out), "scaled_0.9": 0.9 * out,
           "noise": g.standard_normal(out.shape) * np.abs(out).max() * 0.1,
           "permuted_heads": out[:, ::-1]}[wrong]
    with pytest.raises(AssertionError):
        check_attention(_bf16(bad), ref["lse"], out, ref["lse"], "bf16")


def test_wrong_lse_fails(small_bf16_step):
    ref = small_bf16_step
    with pytest.raises(AssertionError):
        check_attention(_bf16(ref["out"]), ref["lse"] + 0.05, ref["out"], ref["lse"], "bf16")


def test_selection_checks():
    g = np.random.default_rng(4)
    s = g.standard_normal(200)
    k = 20
    o = O.topk(s, k)
    check_selection(o.copy(), s, k, exact=True)
    # a swap far from the boundary fails, on both bars
    order = np.argsort(-s, kind="stable")
    far = o.copy()
    far[0] = order[150]
    for exact in (True, False):
        with pytest.raises(AssertionError):
            check_selection(far, s, k, exact=exact)
    # an exact tie at the boundary broken the other way: accepted (a warning for fp32)
    t = s.copy()
    a, b = order[k - 1], order[k]
    t[b] = t[a]
    lo, hi = min(a, b), max(a, b)
    ot = O.topk(t, k)
    assert lo in ot and hi not in ot
    swapped = np.where(ot == lo, hi, ot)
    with pytest.warns(UserWarning):
        check_selection(swapped, t, k, exact=True)
    # padding and duplicates
    with pytest.raises(AssertionError):
        check_selection(np.concatenate([o[:-1], [o[0]]]), s, k, exact=False)
    with pytest.raises(AssertionError):
        check_selection(np.concatenate([o[:-1], [-7]]), s, k, exact=False)
