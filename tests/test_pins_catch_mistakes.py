"""The oracle's pins must catch plausible mistakes: each case below plants one
wrong variant of an oracle function (on the CPU, for the duration of the
case) and checks that at least one of the pins aimed at it fails.  A pin set
that still passes with the mistake planted would not pin that function."""
import numpy as np
import pytest

from oracle import csa_oracle as O
from tests import test_oracle_pins as P

pytestmark = pytest.mark.filterwarnings("ignore")


def _compress_unnormalised(C, Z, m):
    C, Z = np.asarray(C, np.float64), np.asarray(Z, np.float64)
    n = C.shape[0] // m
    Cb, Zb = C[: n * m].reshape(n, m, -1), Z[: n * m].reshape(n, m, -1)
    return (np.exp(Zb - Zb.max(axis=1, keepdims=True)) * Cb).sum(axis=1)  # the softmax's division dropped


def _compress_softmax_over_channels(C, Z, m):
    C, Z = np.asarray(C, np.float64), np.asarray(Z, np.float64)
    n = C.shape[0] // m
    Cb, Zb = C[: n * m].reshape(n, m, -1), Z[: n * m].reshape(n, m, -1)
    e = np.exp(Zb - Zb.max(axis=2, keepdims=True))
    return (e / e.sum(axis=2, keepdims=True) * Cb).sum(axis=1)  # normalised over the wrong axis


def _compress_overlapping(C, Z, m):
    C, Z = np.asarray(C, np.float64), np.asarray(Z, np.float64)
    n = C.shape[0] // m
    out = np.empty((n, C.shape[1]))
    for j in range(n):
        lo = max(0, j * m - 1)  # the previous block's last row leaks in
        zb, cb = Z[lo:(j + 1) * m], C[lo:(j + 1) * m]
        e = np.exp(zb - zb.max(axis=0))
        out[j] = (e / e.sum(axis=0) * cb).sum(axis=0)
    return out


def _scores_without_relu(q_idx, w, keys):
    dots = np.asarray(keys, np.float64) @ np.asarray(q_idx, np.float64).T
    return (dots * np.asarray(w, np.float64)[None, :]).sum(axis=1)


def _scores_unweighted(q_idx, w, keys):
    dots = np.asarray(keys, np.float64) @ np.asarray(q_idx, np.float64).T
    return np.maximum(dots, 0.0).sum(axis=1)


def _topk_ties_to_higher_index(scores, k):
    s = np.asarray(scores, np.float64)
    order = np.lexsort((-np.arange(s.shape[0]), -s))
    out = np.full(k, -1, np.int64)
    take = order[: min(k, s.shape[0])]
    out[: take.shape[0]] = take
    return out


def _n_visible_one_early(t, m):
    return np.asarray(t) // m


def _window_one_too_long(t, W, lo=0):
    start = max(lo, t - W, 0)
    return np.arange(start, t + 1, dtype=np.int64) if W > 0 else np.zeros(0, np.int64)


def _attend_sink_dropped(q, entries, win_k, win_v, sink, tau):
    return _real["attend"](q, entries, win_k, win_v, None, tau)


def _attend_without_tau(q, entries, win_k, win_v, sink, tau):
    return _real["attend"](q, entries, win_k, win_v, sink, 1.0 if tau != 1.0 else 0.5)


def _e4m3_truncating(x):
    x = np.asarray(x, np.float64)
    finite = O.E4M3_VALUES[:127]
    mag = np.minimum(np.abs(x), O.E4M3_MAX)
    code = np.maximum(np.searchsorted(finite, mag, side="right") - 1, 0).astype(np.uint8)
    return (code | np.where((x < 0) & (code != 0), 0x80, 0)).astype(np.uint8)


def _bf16_truncating(x):
    f, e = np.frexp(np.asarray(x, np.float64))
    return np.ldexp(np.trunc(f * 256.0), e - 8)


def _e2m1_ties_away(y):
    y = np.asarray(y, np.float64)
    mags = O.E2M1_VALUES[:8]
    a = np.minimum(np.abs(y), O.E2M1_MAX)
    hi = np.minimum(np.searchsorted(mags, a, side="left"), 7)
    lo = np.maximum(hi - 1, 0)
    code = np.where(a - mags[lo] < mags[hi] - a, lo, hi)  # a tie goes to the larger magnitude
    return (code | np.where(np.signbit(y), 8, 0)).astype(np.uint8)


def _pool_unsorted(scores, block, pool_blocks):
    chosen = O.topk(O.block_scores(scores, block), pool_blocks)  # best first, not ascending
    return chosen


def _block_scores_mean(scores, block):
    s = np.asarray(scores, np.float64)
    nb = (s.shape[0] + block - 1) // block
    return np.array([s[b * block:(b + 1) * block].mean() for b in range(nb)])


def _gap_off_by_one(scores, k):
    s = np.sort(np.asarray(scores, np.float64))[::-1]
    if k <= 0 or k + 1 >= s.shape[0]:
        return float("inf")
    return float(s[k] - s[k + 1])  # the (k+1)-th minus the (k+2)-th


def _gap_unsorted(scores, k):
    s = np.asarray(scores, np.float64)  # the row's own order, not ranked
    if k <= 0 or k >= s.shape[0]:
        return float("inf")
    return float(s[k - 1] - s[k])


def _gap_ascending(scores, k):
    s = np.sort(np.asarray(scores, np.float64))  # ranked the wrong way round
    if k <= 0 or k >= s.shape[0]:
        return float("inf")
    return float(s[k - 1] - s[k])


_real = {"attend": O.attend}

# (name, oracle attribute, wrong variant, pins aimed at it)
MISTAKES = [
    ("compress: softmax not normalised", "compress", _compress_unnormalised,
     ["test_compress_constant_gate_is_block_mean", "test_compress_m2_sigmoid_closed_form",
      "test_compress_brute_force_tiny"]),
    ("compress: softmax over channels", "compress", _compress_softmax_over_channels,
     ["test_compress_constant_gate_is_block_mean", "test_compress_m2_sigmoid_closed_form",
      "test_compress_dominant_gate_selects_row_per_channel"]),
    ("compress: overlapping blocks", "compress", _compress_overlapping,
     ["test_compress_blocks_do_not_overlap", "test_compress_brute_force_tiny"]),
    ("indexer: ReLU dropped", "index_scores", _scores_without_relu,
     ["test_index_scores_single_head_is_relu_dot", "test_index_scores_all_negative_dots_are_exact_zero"]),
    ("indexer: head weights dropped", "index_scores", _scores_unweighted,
     ["test_index_scores_brute_force_and_linearity"]),
    ("top-k: ties to the higher index", "topk", _topk_ties_to_higher_index,
     ["test_topk_ties_lower_index_wins", "test_topk_brute_force_definition"]),
    ("visibility one block early", "n_visible", _n_visible_one_early,
     ["test_visibility_rule", "test_pipeline_ratio1_dense_no_window_is_causal_attention_over_the_tokens"]),
    ("window one position too long", "window_positions", _window_one_too_long,
     ["test_window_rule_golden", "test_pipeline_window_reads_the_ring_slots_of_the_last_w_positions"]),
    ("attention: sink dropped", "attend", _attend_sink_dropped,
     ["test_sink_is_an_extra_zero_value_key", "test_decode_step_dense_no_window_equals_sdpa"]),
    ("attention: softmax scale ignored", "attend", _attend_without_tau,
     ["test_dense_no_window_no_sink_equals_sdpa", "test_split_merge_invariance", "test_degenerate_cases",
      "test_full_window_without_entries_is_causal_attention", "test_sliding_window_band_matches_masked_sdpa"]),
    ("E4M3 rounding truncates", "e4m3_round", _e4m3_truncating,
     ["test_e4m3_round_matches_torch_cast", "test_e4m3_round_ties_and_saturation"]),
    ("bf16 rounding truncates", "bf16_round", _bf16_truncating,
     ["test_bf16_decode_and_round_match_torch"]),
    ("E2M1 ties away from zero", "e2m1_round", _e2m1_ties_away,
     ["test_e2m1_round_is_nearest_with_ties_to_even_by_brute_force"]),
    ("pool not in ascending order", "candidate_pool", _pool_unsorted,
     ["test_pool_matches_brute_force", "test_pool_of_single_entry_blocks_is_the_top_entries"]),
    ("block score = mean, not max", "block_scores", _block_scores_mean,
     ["test_block_scores_partial_tail_and_ties", "test_pool_matches_brute_force"]),
    ("boundary gap one rank too deep", "boundary_gap", _gap_off_by_one,
     ["test_boundary_gap_on_hand_written_rows", "test_boundary_gap_brute_force_definition"]),
    ("boundary gap in input order", "boundary_gap", _gap_unsorted,
     ["test_boundary_gap_on_hand_written_rows", "test_boundary_gap_brute_force_definition"]),
    ("boundary gap ranked ascending", "boundary_gap", _gap_ascending,
     ["test_boundary_gap_on_hand_written_rows", "test_boundary_gap_brute_force_definition"]),
]


@pytest.mark.parametrize("name,attr,wrong,pins", MISTAKES, ids=[m[0] for m in MISTAKES])
def test_a_planted_mistake_fails_a_pin(name, attr, wrong, pins, monkeypatch):
    for pin in pins:
        getattr(P, pin)()  # every pin passes on the real oracle
    monkeypatch.setattr(O, attr, wrong)
    failed = []
    for pin in pins:
        try:
            getattr(P, pin)()
        except AssertionError:  # a pin's check, not a crash of the planted variant
            failed.append(pin)
    assert failed, f"no pin caught the planted mistake '{name}'"
