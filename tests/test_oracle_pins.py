"""Pins of the CPU oracle to facts outside itself.

Each test checks the oracle against something it does not compute: a library
routine on a special case (torch's dtype casts, scaled_dot_product_attention,
topk), a closed form, an invariant the pages state, a worked case of a
printed formula (tests/golden/page_facts.json), or brute force on tiny
inputs.  A plausible slip in the oracle (dropped term, wrong sign or index,
transposed operand) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _facts():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------- formats
def test_e4m3_table_matches_torch_cast():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = O.e4m3_to_f64(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])
    assert O.e4m3_to_f64(np.array([0x7E]))[0] == 448.0
    assert O.e4m3_to_f64(np.array([0x38]))[0] == 1.0
    assert O.e4m3_to_f64(np.array([0x01]))[0] == 2.0 ** -9


def test_e4m3_round_matches_torch_cast():
    g = np.random.default_rng(5)
    x = np.concatenate([
        g.standard_normal(20000) * 30, g.standard_normal(5000) * 0.01,
        g.uniform(-460, 460, 5000),
    ]).astype(np.float32)
    ref = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = O.e4m3_round(x.astype(np.float64))
    # +0 / -0 codes may differ for values that round to zero; compare values
    assert np.array_equal(O.e4m3_to_f64(ref), O.e4m3_to_f64(mine))


def test_e4m3_round_ties_and_saturation():
    v = O.e4m3_to_f64
    r = lambda a: v(O.e4m3_round(np.array([a])))[0]
    assert r(0.5 * 2 ** -9) == 0.0                # tie 0 | 2^-9 -> even (0)
    assert r(1.5 * 2 ** -9) == 2 * 2 ** -9        # tie code1 | code2 -> code2
    assert r(500.0) == 448.0 and r(-1e9) == -448.0
    assert r(1.0 + 1 / 16) == 1.0                  # tie 1.0 | 1.125 -> 1.0 (even)
    assert r(1.0 + 3 / 16) == 1.25                 # tie 1.125 | 1.25 -> 1.25 (even)


def test_bf16_decode_and_round_match_torch():
    g = np.random.default_rng(6)
    x = (g.standard_normal(50000) * np.exp(g.uniform(-20, 20, 50000))).astype(np.float32)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_to_f64(bits), ref)
    assert np.array_equal(O.bf16_round(x.astype(np.float64)), ref)


def test_quantize_groups_scale_and_error_bound():
    g = np.random.default_rng(7)
    x = g.standard_normal((13, 128))
    codes, scale = O.quantize_groups(x, 64)
    assert scale.shape == (13, 2)
    amax = np.abs(x.reshape(13, 2, 64)).max(-1)
    assert np.allclose(scale, amax / 448.0, rtol=0, atol=0)
    deq = O.decode(codes, "fp8", scale, 64)
    # E4M3 keeps 4 significant bits: relative error <= 2^-4, plus the
    # subnormal step 2^-10 * scale near zero
    bound = np.maximum(np.abs(x) * 2.0 ** -4, np.repeat(scale, 64, -1) * 2.0 ** -10)
    assert np.all(np.abs(deq - x) <= bound + 1e-15)
    # the group maximum maps to exactly +-448
    assert np.allclose(np.abs(deq).reshape(13, 2, 64).max(-1), amax, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- compressor
def test_compress_ratio1_is_copy():
    g = np.random.default_rng(1)
    C, Z = g.standard_normal((37, 16)), g.standard_normal((37, 16)) * 5
    assert np.array_equal(O.compress(C, Z, 1), C)


def test_compress_constant_gate_is_block_mean():
    g = np.random.default_rng(2)
    C = g.standard_normal((24, 8))
    Z = np.repeat(g.standard_normal((6, 1, 8)), 4, axis=1).reshape(24, 8)
    ref = C.reshape(6, 4, 8).mean(axis=1)
    assert np.allclose(O.compress(C, Z, 4), ref, rtol=0, atol=1e-14)


def test_compress_m2_sigmoid_closed_form():
    g = np.random.default_rng(3)
    C, Z = g.standard_normal((20, 8)), g.standard_normal((20, 8)) * 3
    c1, c2, z1, z2 = C[0::2], C[1::2], Z[0::2], Z[1::2]
    sig = 1.0 / (1.0 + np.exp(-(z1 - z2)))
    ref = sig * c1 + (1.0 - sig) * c2
    assert np.allclose(O.compress(C, Z, 2), ref, rtol=0, atol=1e-14)


def test_compress_dominant_gate_selects_row_per_channel():
    g = np.random.default_rng(4)
    C = g.standard_normal((8, 6))
    Z = np.zeros((8, 6))
    pick = g.integers(0, 4, size=(2, 6))
    for j in range(2):
        for c in range(6):
            Z[j * 4 + pick[j, c], c] = 1000.0
    out = O.compress(C, Z, 4)
    for j in range(2):
        for c in range(6):
            assert out[j, c] == C[j * 4 + pick[j, c], c]


def test_compress_gate_shift_invariance_and_tail():
    g = np.random.default_rng(8)
    C, Z = g.standard_normal((10, 5)), g.standard_normal((10, 5))
    shift = np.repeat(g.standard_normal((2, 1, 5)) * 50, 4, axis=1).reshape(8, 5)
    Z2 = Z.copy()
    Z2[:8] += shift
    Z2[8:] += 1e6  # rows of the partial trailing block are ignored
    assert O.compress(C, Z, 4).shape == (2, 5)
    assert np.allclose(O.compress(C, Z, 4), O.compress(C, Z2, 4), rtol=0, atol=1e-13)


def test_compress_blocks_do_not_overlap():
    """Golden: non-overlapping groups of m consecutive tokens."""
    for case in _facts()["ratio_blocks"]["cases"]:
        m, T = case["m"], case["T"]
        g = np.random.default_rng(m * 100 + T)
        C, Z = g.standard_normal((T, 3)), g.standard_normal((T, 3))
        base = O.compress(C, Z, m)
        assert base.shape[0] == len(case["blocks"])
        for t in range(T):
            C2 = C.copy()
            C2[t] += 1.0
            changed = np.nonzero(np.any(O.compress(C2, Z, m) != base, axis=1))[0].tolist()
            expect = [j for j, blk in enumerate(case["blocks"]) if t in blk]
            assert changed == expect


def test_compress_brute_force_tiny():
    g = np.random.default_rng(9)
    m, n, d = 3, 4, 5
    C, Z = g.standard_normal((m * n, d)), g.standard_normal((m * n, d))
    out = O.compress(C, Z, m)
    for j in range(n):
        for c in range(d):
            den = sum(math.exp(Z[j * m + i, c]) for i in range(m))
            num = sum(math.exp(Z[j * m + i, c]) * C[j * m + i, c] for i in range(m))
            assert abs(out[j, c] - num / den) < 1e-13


def test_project_index_keys_identity_projection():
    g = np.random.default_rng(10)
    rows = g.standard_normal((7, 6))
    assert np.array_equal(O.project_index_keys(rows, np.eye(6)), rows)
    sel = np.zeros((6, 2))
    sel[4, 0] = 1.0
    sel[1, 1] = -2.0
    assert np.array_equal(O.project_index_keys(rows, sel), np.stack([rows[:, 4], -2 * rows[:, 1]], 1))


# ---------------------------------------------------------------- indexer
def test_index_scores_single_head_is_relu_dot():
    g = np.random.default_rng(11)
    K, q = g.standard_normal((50, 16)), g.standard_normal((1, 16))
    ref = torch.relu(torch.mv(torch.from_numpy(K), torch.from_numpy(q[0]))).numpy()
    assert np.allclose(O.index_scores(q, np.ones(1), K), ref, rtol=0, atol=1e-13)


def test_index_scores_brute_force_and_linearity():
    g = np.random.default_rng(12)
    K, q = g.standard_normal((9, 4)), g.standard_normal((3, 4))
    w1, w2 = g.random(3), g.random(3)
    s = O.index_scores(q, w1, K)
    for j in range(9):
        ref = 0.0
        for h in range(3):
            dot = sum(q[h, c] * K[j, c] for c in range(4))
            ref += w1[h] * (dot if dot > 0 else 0.0)
        assert abs(s[j] - ref) < 1e-13
    assert np.allclose(O.index_scores(q, w1 + w2, K), s + O.index_scores(q, w2, K), atol=1e-13)


def test_index_scores_all_negative_dots_are_exact_zero():
    g = np.random.default_rng(13)
    K = np.abs(g.standard_normal((20, 8)))
    q = -np.abs(g.standard_normal((4, 8)))
    assert np.all(O.index_scores(q, g.random(4), K) == 0.0)


# ---------------------------------------------------------------- top-k
def test_topk_matches_torch_on_distinct_scores():
    g = np.random.default_rng(14)
    s = g.standard_normal(1000)
    ref = torch.topk(torch.from_numpy(s), 37).indices.numpy()
    assert np.array_equal(O.topk(s, 37), ref)


def test_topk_ties_lower_index_wins():
    assert O.topk(np.zeros(10), 4).tolist() == [0, 1, 2, 3]
    assert O.topk(np.array([0.0, -0.0, 0.0, -1.0]), 2).tolist() == [0, 1]
    assert O.topk(np.array([1.0, 2.0, 2.0, 1.0, 2.0]), 2).tolist() == [1, 2]


def test_topk_pads_when_fewer_candidates():
    assert O.topk(np.array([3.0, 1.0, 2.0]), 5).tolist() == [0, 2, 1, -1, -1]
    assert O.topk(np.zeros(0), 2).tolist() == [-1, -1]


def test_topk_brute_force_definition():
    g = np.random.default_rng(15)
    s = np.round(g.standard_normal(60) * 2) / 2  # many exact ties
    k = 17
    chosen = set(O.topk(s, k).tolist())
    for i in range(60):
        rank = sum(1 for j in range(60) if s[j] > s[i] or (s[j] == s[i] and j < i))
        assert (i in chosen) == (rank < k)


def test_boundary_gap_on_hand_written_rows():
    """s_(k) - s_(k+1), the k-th largest score minus the (k+1)-th, by hand:
    sorted descending, [5, 3, 3, 1] has gaps 2 (k = 1), 0 (k = 2, a tie), 2
    (k = 3); nothing is cut off for k >= n or k <= 0.  The same row shuffled
    gives the same gaps (the scores are ranked, not read in input order);
    -0 and +0 are a tie."""
    row = np.array([5.0, 3.0, 3.0, 1.0])
    want = {1: 2.0, 2: 0.0, 3: 2.0}
    for perm in ([0, 1, 2, 3], [3, 2, 0, 1], [1, 3, 0, 2]):
        r = row[perm]
        for k, gap in want.items():
            assert O.boundary_gap(r, k) == gap, (perm, k)
        for k in (0, 4, 5):
            assert O.boundary_gap(r, k) == math.inf
    assert O.boundary_gap(np.array([-0.0, 0.0, -1.0]), 1) == 0.0
    assert O.boundary_gap(np.array([-0.0, 0.0, -1.0]), 2) == 1.0
    # distinct gaps at every k: an index off by one anywhere changes the answer
    r = np.array([10.0, 0.5, 7.0, 3.0, 6.0])  # sorted: 10, 7, 6, 3, 0.5
    assert [O.boundary_gap(r, k) for k in range(1, 5)] == [3.0, 1.0, 3.0, 2.5]


def test_boundary_gap_brute_force_definition():
    """Against its definition: the smallest selected score minus the largest
    score left out, with the selection the top-k."""
    g = np.random.default_rng(16)
    for n in (2, 7, 40):
        s = np.round(g.standard_normal(n) * 3) / 3
        for k in range(1, n):
            sel = O.topk(s, k)
            rest = np.setdiff1d(np.arange(n), sel)
            assert O.boundary_gap(s, k) == s[sel].min() - s[rest].max()


# ---------------------------------------------------------------- attention
def _sdpa(q, k, v, mask=None):
    qt = torch.from_numpy(q)[None]
    return torch.nn.functional.scaled_dot_product_attention(
        qt, torch.from_numpy(k)[None], torch.from_numpy(v)[None], attn_mask=mask, scale=1.0)[0].numpy()


def test_dense_no_window_no_sink_equals_sdpa():
    g = np.random.default_rng(16)
    q, E = g.standard_normal((8, 32)) * 0.3, g.standard_normal((50, 32))
    out, lse = O.attend(q, E, np.zeros((0, 32)), np.zeros((0, 32)), None, 1.0)
    assert np.allclose(out, _sdpa(q, E, E), rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(torch.from_numpy(q @ E.T), dim=1).numpy()
    assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_sink_is_an_extra_zero_value_key():
    g = np.random.default_rng(17)
    h, d = 4, 16
    q, E = g.standard_normal((h, d)), g.standard_normal((30, d))
    wk, wv = g.standard_normal((5, d)), g.standard_normal((5, d))
    sink = g.standard_normal(h) * 2
    out, _ = O.attend(q, E, wk, wv, sink, 0.7)
    for i in range(h):
        qa = np.concatenate([q[i] * 0.7, [1.0]])[None]
        K = np.concatenate([np.concatenate([E, wk]), np.zeros((35, 1))], 1)
        K = np.concatenate([K, np.concatenate([np.zeros(d), [sink[i]]])[None]])
        V = np.concatenate([E, wv, np.zeros((1, d))])
        assert np.allclose(out[i], _sdpa(qa, K, V)[0], rtol=0, atol=1e-12)


def test_full_window_without_entries_is_causal_attention():
    g = np.random.default_rng(18)
    T, d, h = 12, 8, 3
    q, K, V = g.standard_normal((T, h, d)), g.standard_normal((T, d)), g.standard_normal((T, d))
    cap = 16
    ring_k, ring_v = np.zeros((cap, d)), np.zeros((cap, d))
    ring_k[np.arange(T) % cap], ring_v[np.arange(T) % cap] = K, V
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.transpose(1, 0, 2)), torch.from_numpy(K)[None].expand(h, T, d),
        torch.from_numpy(V)[None].expand(h, T, d), is_causal=True, scale=1.0).numpy()
    for t in range(T):
        out, _ = O.sparse_swa_attention(q[t], np.zeros((1, d)), np.zeros(0, np.int64), 0, ring_k, ring_v,
                                        cap, t, W=T, sink=None, tau=1.0)
        assert np.allclose(out, ref[:, t], rtol=0, atol=1e-12)


def test_sliding_window_band_matches_masked_sdpa():
    g = np.random.default_rng(19)
    T, d, W = 20, 8, 5
    q, K, V = g.standard_normal((T, 1, d)), g.standard_normal((T, d)), g.standard_normal((T, d))
    cap = 8
    for t in range(T):
        ring_k, ring_v = np.zeros((cap, d)), np.zeros((cap, d))
        for p in range(max(0, t - cap + 1), t + 1):
            ring_k[p % cap], ring_v[p % cap] = K[p], V[p]
        mask = torch.zeros(1, T, dtype=torch.bool)
        mask[0, max(0, t - W + 1): t + 1] = True
        ref = _sdpa(q[t], K, V, mask)
        out, _ = O.sparse_swa_attention(q[t], np.zeros((1, d)), None, 0, ring_k, ring_v, cap, t, W, None, 1.0)
        assert np.allclose(out, ref, rtol=0, atol=1e-12)


def test_window_rule_golden():
    f = _facts()["window_rule"]
    for c in f["cases"]:
        pos = O.window_positions(c["i"], f["W"], c["s"])
        assert pos[0] == c["first"] and pos[-1] == c["last"] and len(pos) == c["last"] - c["first"] + 1


def test_split_merge_invariance():
    g = np.random.default_rng(20)
    q, E = g.standard_normal((6, 16)), g.standard_normal((40, 16))
    z = np.zeros((0, 16))
    o1, l1 = O.attend(q, E[:13], z, z, None, 1.0)
    o2, l2 = O.attend(q, E[13:], z, z, None, 1.0)
    o, l = O.attend(q, E, z, z, None, 1.0)
    M = np.maximum(l1, l2)
    a1, a2 = np.exp(l1 - M), np.exp(l2 - M)
    assert np.allclose(o, (o1 * a1[:, None] + o2 * a2[:, None]) / (a1 + a2)[:, None], atol=1e-12)
    assert np.allclose(l, M + np.log(a1 + a2), atol=1e-12)


def test_selection_order_does_not_matter():
    g = np.random.default_rng(21)
    q, rows = g.standard_normal((4, 8)), g.standard_normal((30, 8))
    idx = g.permutation(30)[:10]
    ring = np.zeros((4, 8))
    a = O.sparse_swa_attention(q, rows, idx, 30, ring, ring, 4, 0, 0, None, 1.0)[0]
    b = O.sparse_swa_attention(q, rows, idx[::-1].copy(), 30, ring, ring, 4, 0, 0, None, 1.0)[0]
    assert np.allclose(a, b, atol=1e-13)
    # padding entries (-1) are ignored
    c = O.sparse_swa_attention(q, rows, np.concatenate([idx, [-1, -1]]), 30, ring, ring, 4, 0, 0, None, 1.0)[0]
    assert np.allclose(a, c, atol=1e-13)


def test_degenerate_cases():
    g = np.random.default_rng(22)
    q, row = g.standard_normal((3, 8)), g.standard_normal((1, 8))
    z = np.zeros((0, 8))
    out, lse = O.attend(q, row, z, z, None, 1.0)
    assert np.allclose(out, np.repeat(row, 3, 0), atol=1e-14)
    sink = np.array([0.5, -1.0, 2.0])
    out, lse = O.attend(q, z, z, z, sink, 1.0)
    assert np.all(out == 0) and np.allclose(lse, sink)
    out, lse = O.attend(q, z, z, z, None, 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_visibility_rule():
    assert O.n_visible(2, 4) == 0 and O.n_visible(3, 4) == 1 and O.n_visible(7, 4) == 2
    assert O.n_visible(0, 1) == 1 and O.n_visible(126, 128) == 0 and O.n_visible(127, 128) == 1


# ---------------------------------------------------------------- decode step
def _small_decode(**kw):
    from compressed_sparse_attention_compressor_b200 import workloads as Wk

    wl = Wk.WORKLOADS["decode64k"].scaled(batch=2, context=64, d=16, h_q=3, h_idx=2, d_idx=8, **kw)
    return Wk.make_decode_inputs(wl)


def test_decode_step_dense_no_window_equals_sdpa():
    inp = _small_decode(topk=0, window=0, sink="zero", m=4, act_dtype="f32", kv_dtype="f32",
                        idx_dtype="f32")
    res = O.decode_step(inp)
    kv = O.decode_stored(inp.kv)
    for b in range(2):
        rows = kv[b].copy()
        rows[15] = res["new_rows"][b].astype(np.float32)  # stored as fp32
        q = O.decode_stored(inp.q)[b]
        # sink 0 is an extra key with logit 0 and value 0
        K = np.concatenate([np.concatenate([rows, np.zeros((16, 1))], 1), [[0.0] * 16 + [1.0]]])
        V = np.concatenate([rows, np.zeros((1, 16))])
        qa = np.concatenate([q, np.zeros((3, 1))], 1)
        assert np.allclose(res["out"][b], _sdpa(qa, K, V), atol=1e-10)


def test_decode_step_ratio1_appends_the_token_row():
    inp = _small_decode(m=1, topk=4, window=3, act_dtype="f32", kv_dtype="f32", idx_dtype="f32")
    res = O.decode_step(inp)
    c_t = O.decode_stored(inp.c_t)
    for b in range(2):
        assert np.array_equal(res["new_rows"][b], c_t[b])
        assert np.allclose(res["new_keys"][b], c_t[b] @ O.decode_stored(inp.w_ik), atol=1e-13)


def _small_prefill(**kw):
    from compressed_sparse_attention_compressor_b200 import workloads as Wk

    base = dict(batch=1, context=16, chunk=8, d=16, h_q=3, h_idx=2, d_idx=8, act_dtype="f32",
                kv_dtype="f32", idx_dtype="f32")
    base.update(kw)
    return Wk.make_prefill_inputs(Wk.WORKLOADS["prefill"].scaled(**base))


def test_pipeline_ratio1_dense_no_window_is_causal_attention_over_the_tokens():
    # ratio 1 keeps every token as an entry; with no top-k, no window and a
    # zero sink, query i (position 16 + i) attends causally over the 16 cached
    # rows and the chunk's first i + 1 rows, the sink an extra key of logit 0
    # and value 0
    inp = _small_prefill(m=1, topk=0, window=0, sink="zero")
    res = O.pipeline(inp)
    cached = O.decode_stored(inp.kv_cached)[0][:16]
    C = O.decode_stored(inp.C)[0]
    rows = np.concatenate([cached, C])
    q = O.decode_stored(inp.q)
    for i in range(8):
        ent = rows[:17 + i]
        K = np.concatenate([np.concatenate([ent, np.zeros((len(ent), 1))], 1), [[0.0] * 16 + [1.0]]])
        V = np.concatenate([ent, np.zeros((1, 16))])
        qa = np.concatenate([q[i], np.zeros((3, 1))], 1)
        assert np.allclose(res["out"][i], _sdpa(qa, K, V), rtol=0, atol=1e-12)


def test_pipeline_topk_covering_every_entry_equals_dense():
    # a top-k at least the visible entry count selects them all: the CSA path
    # equals the dense (HCA) path over the same compressed cache, window and sink
    sparse = O.pipeline(_small_prefill(m=2, topk=64, window=3, sink="normal"))
    dense = O.pipeline(_small_prefill(m=2, topk=0, window=3, sink="normal"))
    assert np.allclose(sparse["out"], dense["out"], rtol=0, atol=1e-12)
    assert np.allclose(sparse["lse"], dense["lse"], rtol=0, atol=1e-12)
    for i, t in enumerate(range(16, 24)):
        sel = sparse["idx"][i]
        assert sorted(sel[sel >= 0].tolist()) == list(range((t + 1) // 2))


def test_pipeline_window_reads_the_ring_slots_of_the_last_w_positions():
    # with m above every position no compressed entry is visible, so the
    # output is attention over the window alone: keys and values of ring slots
    # p % swa_cap for p in [t - W + 1, t]; positions 40..47 wrap the 16-slot ring
    inp = _small_prefill(context=40, m=128, topk=0, window=4, sink="zero")
    assert inp.swa_cap == 16
    res = O.pipeline(inp)
    K = O.decode_stored(inp.swa_k)[0]
    V = O.decode_stored(inp.swa_v)[0]
    q = O.decode_stored(inp.q)
    for i, t in enumerate(range(40, 48)):
        slots = [p % 16 for p in range(t - 3, t + 1)]
        Kw = np.concatenate([np.concatenate([K[slots], np.zeros((4, 1))], 1), [[0.0] * 16 + [1.0]]])
        Vw = np.concatenate([V[slots], np.zeros((1, 16))])
        qa = np.concatenate([q[i], np.zeros((3, 1))], 1)
        assert np.allclose(res["out"][i], _sdpa(qa, Kw, Vw), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# hierarchical sparse indexer: candidate pool and re-indexing
# ---------------------------------------------------------------------------
def _brute_pool(scores, block, pool_blocks):
    """Pool by the definition, in plain Python: every block's maximum, blocks
    ranked by (maximum descending, block id ascending), the first pool_blocks
    ids in ascending order."""
    s = [float(x) for x in scores]
    maxima = []
    for b in range(0, len(s), block):
        maxima.append(max(s[b:b + block]))
    ranked = sorted(range(len(maxima)), key=lambda i: (-maxima[i], i))
    chosen = sorted(ranked[:pool_blocks])
    return chosen + [-1] * (pool_blocks - len(chosen))


def test_pool_sizes_from_the_page():
    with open(GOLDEN) as f:
        g = json.load(f)["candidate_pool"]
    assert g["pool_blocks"] * g["block"] == g["pool_positions"] == 16384
    assert round(100.0 * g["pool_positions"] / g["context"], 1) == g["fraction_percent_about"]
    # a pool built with those sizes holds exactly pool_positions entries
    s = np.random.default_rng(0).standard_normal(200_000)
    pool = O.candidate_pool(s, g["block"], g["pool_blocks"])
    assert O.pool_entries(pool, g["block"], s.shape[0]).shape[0] == g["pool_positions"]


def test_block_scores_partial_tail_and_ties():
    s = np.array([1.0, 5.0, 2.0, 2.0, 7.0, 0.0, 0.0, 0.0, 5.0, 5.0, 1.0, 1.0, 3.0])
    assert np.array_equal(O.block_scores(s, 4), [5.0, 7.0, 5.0, 3.0])  # last block: entry 12 alone
    # blocks 0 and 2 tie at 5: the lower block wins the second place
    assert np.array_equal(O.candidate_pool(s, 4, 2), [0, 1])
    assert np.array_equal(O.candidate_pool(s, 4, 3), [0, 1, 2])
    assert np.array_equal(O.candidate_pool(s, 4, 6), [0, 1, 2, 3, -1, -1])
    assert np.array_equal(O.pool_entries(O.candidate_pool(s, 4, 6), 4, 13), np.arange(13))


def test_pool_matches_brute_force():
    rng = np.random.default_rng(1)
    for n, block, pb in [(37, 4, 3), (64, 8, 5), (100, 1, 10), (9, 8, 1), (50, 7, 50)]:
        s = np.round(rng.standard_normal(n), 1)  # coarse values: many exact ties
        assert list(O.candidate_pool(s, block, pb)) == _brute_pool(s, block, pb), (n, block, pb)


def test_pool_of_single_entry_blocks_is_the_top_entries():
    s = np.random.default_rng(2).standard_normal(500)
    assert np.array_equal(O.candidate_pool(s, 1, 40), np.sort(O.topk(s, 40)))


def test_reindex_over_every_block_is_the_plain_top_k():
    rng = np.random.default_rng(3)
    keys = rng.standard_normal((300, 8))
    q, w = rng.standard_normal((3, 8)), rng.random(3)
    pool = O.candidate_pool(rng.standard_normal(300), 8, 64)  # 38 blocks <= 64: all of them
    ids, _ = O.reindex_topk(q, w, keys, pool, 8, 20)
    assert np.array_equal(ids, O.topk(O.index_scores(q, w, keys), 20))


def test_reindex_selects_inside_the_pool_by_brute_force():
    rng = np.random.default_rng(4)
    keys = np.round(rng.standard_normal((120, 6)), 1)
    q, w = rng.standard_normal((2, 6)), np.ones(2)
    pool = O.candidate_pool(rng.standard_normal(120), 8, 4)
    ids, _ = O.reindex_topk(q, w, keys, pool, 8, 10)
    members = [b * 8 + i for b in pool if b >= 0 for i in range(8) if b * 8 + i < 120]
    sc = {j: sum(max(0.0, float(np.dot(q[h], keys[j]))) * w[h] for h in range(2)) for j in members}
    want = sorted(members, key=lambda j: (-sc[j], j))[:10]
    assert sorted(ids.tolist()) == sorted(want)
    # fewer pool entries than k: all of them, padded with -1
    ids2, _ = O.reindex_topk(q, w, keys, pool, 8, 40)
    assert sorted(ids2[ids2 >= 0].tolist()) == sorted(members) and np.all(ids2[len(members):] == -1)


# ---------------------------------------------------------------- MXFP4 main KV
def test_e2m1_values_embed_in_the_torch_pinned_e4m3_table():
    """E2M1 (1 sign, 2 exponent, 1 mantissa bit) is the set of E4M3 values in
    [0, 6] with at most two significant bits and a multiple of 0.5: a
    derivation from torch's E4M3 cast, independent of the oracle's formula."""
    e4 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()

    def two_significant_bits(n):  # n > 0: its odd part has at most two bits
        return (n // (n & -n)).bit_length() <= 2

    cand = sorted({float(v) for v in e4 if np.isfinite(v) and 0 <= v <= 6 and 2 * v == int(2 * v)
                   and (v == 0 or two_significant_bits(int(2 * v)))})
    assert np.array_equal(O.E2M1_VALUES[:8], np.array(cand))
    assert np.array_equal(O.E2M1_VALUES[8:], -O.E2M1_VALUES[:8])


def test_mxfp4_ceiling_from_the_page():
    f = _facts()["mxfp4"]
    assert O.E2M1_MAX == f["e2m1_max"] and O.E4M3_MAX == f["e4m3_max"] and O.MXFP4_GROUP == f["group"]
    top = np.abs(np.outer(O.E2M1_VALUES, O.e4m3_to_f64(np.arange(0x7F)))).max()
    assert top == f["ceiling"] == f["e4m3_max"] * f["e2m1_max"]
    # a group at the ceiling is stored exactly; beyond it, it saturates there
    x = np.zeros((1, 32))
    x[0, 3], x[0, 20] = 2688.0, -1e6
    c, s = O.quantize_mxfp4(x)
    y = O.decode(c, "mxfp4", s, 16)
    assert y[0, 3] == 2688.0 and y[0, 20] == -2688.0
    # the largest magnitude seen in training sits > 100x below the ceiling
    assert f["ceiling"] / f["largest_observed_about"] > 100


def test_e2m1_round_is_nearest_with_ties_to_even_by_brute_force():
    mags = O.E2M1_VALUES[:8]
    g = np.random.default_rng(11)
    mids = (mags[1:] + mags[:-1]) / 2
    x = np.concatenate([g.uniform(-8, 8, 4000), mids, -mids, mags, -mags, [0.0, 6.5, -100.0]])
    got = O.E2M1_VALUES[O.e2m1_round(x)]
    for xi, gi in zip(x, got):
        a = min(abs(xi), 6.0)
        d = np.abs(mags - a)
        best = np.flatnonzero(d == d.min())
        code = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert abs(gi) == mags[code] and (gi == 0 or np.sign(gi) == np.sign(xi))


def test_mxfp4_round_trip_error_bound_and_layout():
    g = np.random.default_rng(12)
    # values on the grid of a group whose largest code is 6: stored exactly
    s = O.e4m3_to_f64(g.integers(0x20, 0x60, size=(50, 4)))
    codes = g.integers(0, 16, size=(50, 4, 16))
    codes[:, :, 5] = 7
    x = (O.E2M1_VALUES[codes] * s[..., None]).reshape(50, 64)
    c, sc = O.quantize_mxfp4(x)
    assert np.array_equal(O.decode(c, "mxfp4", sc, 16), x)
    # Gaussian rows: the error of an element is at most its group's scale
    y = g.standard_normal((40, 512)) * np.exp(g.uniform(-3, 3, (40, 1)))
    c, sc = O.quantize_mxfp4(y)
    err = np.abs(O.decode(c, "mxfp4", sc, 16) - y)
    assert np.all(err <= np.repeat(O.e4m3_to_f64(sc), 16, axis=-1) * (1 + 1e-12))
    # element 2i in the low nibble of byte i; the sign in bit 3 of a nibble
    b = np.array([[0x72, 0x0F] + [0] * 14], np.uint8)
    v = O.decode(b, "mxfp4", np.array([[0x38, 0x38]], np.uint8), 16)
    assert v[0, :4].tolist() == [1.0, 6.0, -6.0, 0.0]
    # a 512-channel row: 256 code bytes + 32 scale bytes = 288, vs 544 for FP8
    # with an fp32 scale per 64 ("nearly halves")
    assert 512 // 2 + 512 // 16 == 288 and 288 / (512 + 4 * 8) < 0.55
    # an all-zero group keeps a zero scale and zero codes
    c, sc = O.quantize_mxfp4(np.zeros((1, 32)))
    assert np.all(c == 0) and np.all(sc == 0)


# ---------------------------------------------------------------- CSA2 layer modes
def _group_inputs(seed, n=300, H=3, D=8, layers=6):
    g = np.random.default_rng(seed)
    keys = g.standard_normal((n, D))
    qs = g.standard_normal((layers, H, D))
    ws = g.uniform(0, 1, (layers, H))
    return keys, qs, ws


def test_csa2_reuse_layers_repeat_the_latest_selection():
    keys, qs, ws = _group_inputs(31)
    modes = ["full", "reuse", "reuse", "reindex", "reuse", "reuse"]
    sel, pool = O.csa2_group_selections(modes, qs, ws, keys, 8, 10, 16)
    assert np.array_equal(sel[1], sel[0]) and np.array_equal(sel[2], sel[0])
    assert np.array_equal(sel[4], sel[3]) and np.array_equal(sel[5], sel[3])
    # the Full layer is the plain top-k of its own query; the pool is its blocks
    assert np.array_equal(sel[0], O.topk(O.index_scores(qs[0], ws[0], keys), 16))
    assert np.array_equal(pool, O.candidate_pool(O.index_scores(qs[0], ws[0], keys), 8, 10))
    # the Reindex layer's picks lie inside the pool
    inside = set(O.pool_entries(pool, 8, keys.shape[0]).tolist())
    assert set(sel[3][sel[3] >= 0].tolist()) <= inside


def test_csa2_reindex_over_a_pool_of_every_block_equals_a_full_layer():
    keys, qs, ws = _group_inputs(32, n=203)
    nb = (203 + 7) // 8
    sel, _ = O.csa2_group_selections(["full", "reindex"], qs, ws, keys, 8, nb, 20)
    full, _ = O.csa2_group_selections(["full", "full"], qs, ws, keys, 8, nb, 20)
    assert np.array_equal(np.sort(sel[1]), np.sort(full[1]))


def test_csa2_pool_comes_from_the_first_full_layer_only():
    keys, qs, ws = _group_inputs(33)
    sel, pool = O.csa2_group_selections(["full", "full", "reindex"], qs, ws, keys, 8, 6, 12)
    assert np.array_equal(pool, O.candidate_pool(O.index_scores(qs[0], ws[0], keys), 8, 6))
    assert not np.array_equal(pool, O.candidate_pool(O.index_scores(qs[1], ws[1], keys), 8, 6))
    with pytest.raises(ValueError):
        O.csa2_group_selections(["reindex"], qs, ws, keys, 8, 6, 12)
    with pytest.raises(ValueError):
        O.csa2_group_selections(["reuse"], qs, ws, keys, 8, 6, 12)
