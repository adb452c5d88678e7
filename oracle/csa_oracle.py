"""CPU oracle of the compressed-sparse-attention hot path (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library; it reads the same seeded storage-format inputs.

It is a plain, slow, obviously correct restatement of what the method
computes.  Every input is first decoded exactly to fp64 (bf16 bit patterns,
E4M3 codes times their fp32 scale); every step then runs in fp64 with numpy
reductions and ``@`` as the only library primitives.

Sources (web pages; cited by page title and section):

* "DeepSeek-V4.1-Flash, illustrated" (mxino.github.io/illustrations/
  deepseek-v41-flash), Equation (1) figure: the compressor turns the projected
  KV entries C_l and compression weights Z_l into pooled entries; ratio 1 is
  the unpooled main-KV projection; non-overlapping pairs at ratio 2.
* "Model architectures" atlas (llm-switchboard.icompaas.com/app/architectures),
  "compressed KV" entry: CSA squeezes every m KV tokens into one entry with
  learned compression weights, then runs top-k lightning-indexer selection
  over the compressed entries plus a sliding window; HCA compresses harder and
  runs dense attention over the short stream.  "Sliding-window attention"
  entry: token t attends to the previous W tokens, rolling buffer.  "MLA"
  entry: attention runs over the latent directly (K = V = latent).
* Tech-report tour (astryx-dracula tech-report.tsx), chapter "Compressed
  Sparse Attention 2": section "The indexer selects, SWA covers the rest"
  (indexer query x indexer key scores main KV entries, top 512 per query, the
  query attends to those entries together with the sliding-window KV; ratio 1
  is the uncompressed special case); section "A simpler compressor" (no
  overlap, no absolute position term, indexer K projected from main KV);
  chapter "SWA Bounded Replay", section "Replay only the window" (keys in
  [max(s, i-W+1), i]).

Readings taken where the pages are silent or garbled:

* Equation (1)'s body is not extracted.  Reading: within each block of m
  consecutive tokens the pooling weights are a softmax over the block's m
  gate logits Z, taken separately for every channel, and the entry is the
  weighted sum of the block's C rows.  A partial trailing block emits nothing.
* Indexer score: s_j = sum_h w_h * ReLU(q_h . k_j), no softmax, no scale.
* Top-k order: score descending, index ascending on exact ties (-0 == +0).
* One online softmax covers the selected (or all, for HCA) compressed entries,
  the window keys, and a per-head sink logit that only adds exp(sink) to the
  denominator.  Window and compressed entries are not de-duplicated.
* A compressed block j is visible to a query at absolute position t iff its
  last token (j+1)m-1 <= t, i.e. n_visible(t) = floor((t+1)/m).

Parity unpinned: the exact form of Equation (1) is not printed on the pages;
only the invariants the pages fix (ratio 1 = unpooled copy, non-overlapping
blocks, no positional term) and closed forms of the per-channel softmax
reading pin the compressor.
"""
from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0


# ===========================================================================
# storage formats
# ===========================================================================
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit pattern -> value: the upper 16 bits of an IEEE binary32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def _e4m3_table() -> np.ndarray:
    """Value of every E4M3 (OCP 'fn' variant) code, from the format definition.

    Layout s eeee mmm, exponent bias 7.  e == 0: subnormal m/8 * 2^-6.
    e == 15 and m == 7: NaN (no infinities).  Otherwise (1 + m/8) * 2^(e-7).
    """
    t = np.empty(256, np.float64)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            t[code] = np.nan
        elif e == 0:
            t[code] = s * (m / 8.0) * 2.0 ** -6
        else:
            t[code] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return t


E4M3_VALUES = _e4m3_table()


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    return E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


# ---------------------------------------------------------------------------
# MXFP4 main KV.  Tech-report tour, chapter "Engram, DSpark, FP4", section
# "FP4 main KV cache": elements are FP4 E2M1, one E4M3 scale per 16 channels,
# no second-level (global) scale, so the largest storable magnitude is
# 448 * 6 = 2688; values are dequantised before attention.
# ---------------------------------------------------------------------------
def _e2m1_table() -> np.ndarray:
    """Value of every E2M1 code (OCP FP4), from the format definition.

    Layout s ee m, exponent bias 1.  e == 0: subnormal m/2.  Otherwise
    (1 + m/2) * 2^(e-1).  No infinities or NaN.
    """
    t = np.empty(16, np.float64)
    for code in range(16):
        sgn = -1.0 if code & 0x8 else 1.0
        e, m = (code >> 1) & 0x3, code & 0x1
        t[code] = sgn * (m / 2.0 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1))
    return t


E2M1_VALUES = _e2m1_table()
E2M1_MAX = 6.0
MXFP4_GROUP = 16


def e2m1_round(y: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest E2M1 value, ties to the even code,
    saturating at +-6 (tech-report tour, "FP4 main KV cache": E2M1
    elements; the rounding rule is a reading, the page names none).  Returns codes 0..15 (sign in bit 3; a negative value
    that rounds to zero keeps its sign bit)."""
    y = np.asarray(y, np.float64)
    mags = E2M1_VALUES[:8]                       # codes 0..7, ascending
    a = np.minimum(np.abs(y), E2M1_MAX)
    hi = np.minimum(np.searchsorted(mags, a, side="left"), 7)
    lo = np.maximum(hi - 1, 0)
    d_hi, d_lo = mags[hi] - a, a - mags[lo]
    code = np.where((d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0)), lo, hi)
    code = np.where(a == mags[hi], hi, code)
    return (code | np.where(np.signbit(y), 8, 0)).astype(np.uint8)


def quantize_mxfp4(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """MXFP4 storage of fp64 values (last axis a multiple of 32).

    Reading of the section cited above: per 16 channels, the scale is the
    E4M3 value nearest max|x| / 6 (round to nearest even, saturating at 448),
    so that the largest magnitude lands on the largest E2M1 value; each
    element is the E2M1 value nearest x / scale (saturating at 6); a zero
    scale stores zero codes.  Returns (packed codes [.., d/2] uint8, element
    2i in the low nibble of byte i; E4M3 scale codes [.., d/16] uint8)."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    g = x.reshape(x.shape[:-1] + (d // MXFP4_GROUP, MXFP4_GROUP))
    sc_code = e4m3_round(np.abs(g).max(axis=-1) / E2M1_MAX)
    sc = e4m3_to_f64(sc_code)
    safe = np.where(sc > 0, sc, 1.0)
    codes = np.where(sc[..., None] > 0, e2m1_round(g / safe[..., None]), 0).astype(np.uint8).reshape(x.shape)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, sc_code


def decode(data: np.ndarray, dtype: str, scale: np.ndarray | None = None, group: int = 0) -> np.ndarray:
    """Exact fp64 value of a stored tensor (codes times group scale for FP8
    and MXFP4)."""
    if dtype == "f32":
        return np.asarray(data, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_to_f64(data)
    if dtype == "fp8":
        v = e4m3_to_f64(data)
        sc = np.repeat(np.asarray(scale, np.float64), group, axis=-1)
        return v * sc
    if dtype == "mxfp4":
        b = np.asarray(data, np.uint8)
        codes = np.stack([b & 0xF, b >> 4], axis=-1).reshape(b.shape[:-1] + (2 * b.shape[-1],))
        sc = np.repeat(e4m3_to_f64(scale), MXFP4_GROUP, axis=-1)
        return E2M1_VALUES[codes] * sc
    raise ValueError(dtype)


def decode_stored(t) -> np.ndarray:
    """Decode a ``workloads.Stored`` (duck-typed: data, dtype, scale, group)."""
    return decode(t.data, t.dtype, t.scale, t.group)


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest E4M3 value, ties to even code,
    saturating at +-448 (the largest finite value).  The FP8 storage of the
    1M-token decode configuration; the rounding rule is a reading (the pages
    name E4M3, not how values are rounded into it).  Returns codes (uint8)."""
    x = np.asarray(x, np.float64)
    finite = E4M3_VALUES[:127]                  # codes 0x00..0x7E, ascending
    mag = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(finite, mag, side="left")   # first value >= mag
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_hi = finite[hi] - mag
    d_lo = mag - finite[lo]
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(pick_lo, lo, hi).astype(np.uint8)
    code = np.where(mag == finite[hi], hi, code).astype(np.uint8)
    neg = (x < 0) & (code != 0)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (8 significant bits), ties
    to even (a reading: the configurations store bf16 and name no rounding).  Normal range only, which covers every value the path stores."""
    x = np.asarray(x, np.float64)
    f, e = np.frexp(x)                      # x = f * 2^e, 0.5 <= |f| < 1
    return np.ldexp(np.rint(f * 256.0), e - 8)


def round_to_storage(x: np.ndarray, dtype: str, group: int = 0) -> np.ndarray:
    """Value that remains after storing fp64 ``x`` in format ``dtype``:
    fp32 (IEEE round-to-nearest-even cast), bf16 (``bf16_round``) or E4M3
    with a per-group scale (``quantize_groups``, then decoded)."""
    if dtype == "f32":
        return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_round(x)
    if dtype == "fp8":
        codes, scale = quantize_groups(x, group)
        return decode(codes, "fp8", scale, group)
    if dtype == "mxfp4":
        codes, scale = quantize_mxfp4(x)
        return decode(codes, "mxfp4", scale, MXFP4_GROUP)
    raise ValueError(dtype)


def quantize_groups(x: np.ndarray, group: int) -> tuple[np.ndarray, np.ndarray]:
    """E4M3 storage of fp64 values: per ``group`` channels, scale = max|x|/448
    (1.0 for an all-zero group), codes = RNE-saturating E4M3 of x/scale."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    g = x.reshape(x.shape[:-1] + (d // group, group))
    amax = np.abs(g).max(axis=-1)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    codes = e4m3_round(g / scale[..., None]).reshape(x.shape)
    return codes, scale


# ===========================================================================
# a1: the compressor
# ===========================================================================
def compress(C: np.ndarray, Z: np.ndarray, m: int) -> np.ndarray:
    """Pool every m consecutive rows of C into one entry.

    "DeepSeek-V4.1-Flash, illustrated", Equation (1) (C_l, Z_l rule) and the
    atlas's "compressed KV" entry (every m KV tokens -> one entry with learned
    compression weights); tech-report tour, "A simpler compressor"
    (non-overlapping groups, no absolute positional term).

    For block j and channel c:
        a_i = exp(Z[i,c]) / sum_{i' in block j} exp(Z[i',c])
        out[j,c] = sum_{i in block j} a_i * C[i,c]
    computed with the block maximum subtracted before exp.  Rows after the
    last complete block are ignored.  C, Z: [T][d] -> [T // m][d].
    """
    C = np.asarray(C, np.float64)
    Z = np.asarray(Z, np.float64)
    T, d = C.shape
    n = T // m
    Cb = C[: n * m].reshape(n, m, d)
    Zb = Z[: n * m].reshape(n, m, d)
    M = Zb.max(axis=1, keepdims=True)
    e = np.exp(Zb - M)
    a = e / e.sum(axis=1, keepdims=True)
    return (a * Cb).sum(axis=1)


def project_index_keys(C_hat: np.ndarray, w_ik: np.ndarray) -> np.ndarray:
    """Indexer keys projected from main-KV entries: k_I = C_hat @ W_IK.

    Tech-report tour, "A simpler compressor": CSA2 derives indexer K by
    projecting main KV entries.  [n][d] @ [d][d_idx] -> [n][d_idx].
    """
    return np.asarray(C_hat, np.float64) @ np.asarray(w_ik, np.float64)


# ===========================================================================
# a2 / a3: lightning indexer and per-query top-k
# ===========================================================================
def n_visible(t: int | np.ndarray, m: int):
    """Compressed blocks whose last token is at or before position t.

    "DeepSeek-V4.1-Flash, illustrated", the CSA2 figure (each decoder query
    scores its causally visible context).  Reading: block j, made of tokens
    jm .. jm+m-1, is visible to position t once it is complete, (j+1)m-1 <= t.
    """
    return (np.asarray(t) + 1) // m


def index_scores(q_idx: np.ndarray, w: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Lightning-indexer scores of one query against ``keys``.

    s_j = sum_h w_h * max(0, q_h . k_j).  Atlas, "Trained sparse attention"
    entry (DSA: lightning indexer + top-k token selection) and "compressed
    KV" entry; tech-report tour, "The indexer selects, SWA covers the rest".
    q_idx [h][d_idx], w [h], keys [n][d_idx] -> [n].
    """
    dots = np.asarray(keys, np.float64) @ np.asarray(q_idx, np.float64).T   # [n][h]
    return (np.maximum(dots, 0.0) * np.asarray(w, np.float64)[None, :]).sum(axis=1)


def topk(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores: score descending, index ascending on
    exact ties (-0 equals +0).  Fewer than k candidates: pad with -1.
    Tech-report tour, "The indexer selects, SWA covers the rest"."""
    s = np.asarray(scores, np.float64)
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))
    take = order[: min(k, n)]
    out = np.full(k, -1, np.int64)
    out[: take.shape[0]] = take
    return out


def boundary_gap(scores: np.ndarray, k: int) -> float:
    """s_(k) - s_(k+1) of the sorted scores (inf when nothing is cut off)."""
    s = np.sort(np.asarray(scores, np.float64))[::-1]
    if k <= 0 or k >= s.shape[0]:
        return math.inf
    return float(s[k - 1] - s[k])


# ===========================================================================
# hierarchical sparse indexer: the candidate pool and re-indexing inside it
# ===========================================================================
def block_scores(scores: np.ndarray, block: int) -> np.ndarray:
    """Score of each block of ``block`` consecutive entries: the maximum of its
    entries' index scores; a partial last block takes the maximum over the
    entries it has.  Tech-report tour, chapter "Compressed Sparse Attention
    2", section "The Hierarchical Sparse Indexer" (block score = max of its
    positions)."""
    s = np.asarray(scores, np.float64)
    n = s.shape[0]
    nb = (n + block - 1) // block
    out = np.empty(nb, np.float64)
    for b in range(nb):
        out[b] = s[b * block: min(n, (b + 1) * block)].max()
    return out


def candidate_pool(scores: np.ndarray, block: int, pool_blocks: int) -> np.ndarray:
    """The candidate pool the first Full layer builds for one query: the
    ``pool_blocks`` best blocks of ``block`` entries (block score descending,
    lower block first on exact ties), as block ids in ascending order, padded
    with -1 when fewer blocks exist.  Same section as block_scores (2,048
    blocks of 8 positions, a pool of 16,384 candidates)."""
    bs = block_scores(scores, block)
    chosen = topk(bs, pool_blocks)
    chosen = np.sort(chosen[chosen >= 0])
    out = np.full(pool_blocks, -1, np.int64)
    out[: chosen.shape[0]] = chosen
    return out


def pool_entries(pool: np.ndarray, block: int, n_vis: int) -> np.ndarray:
    """Visible entry ids of a pool, ascending: the positions a Reindex layer
    scores.  Tech-report tour, "The Hierarchical Sparse Indexer" (later
    indexers search only the pool's candidate positions)."""
    ids = [b * block + i for b in np.asarray(pool) if b >= 0 for i in range(block) if b * block + i < n_vis]
    return np.asarray(ids, np.int64)


def reindex_topk(q_idx: np.ndarray, w: np.ndarray, keys: np.ndarray, pool: np.ndarray, block: int, k: int):
    """A Reindex layer's selection: the lightning-indexer scores of the pool's
    entries only (its own query, the shared keys), top k of them (score
    descending, lower entry first on exact ties), as entry ids padded with
    -1.  Tech-report tour, chapter "Compressed Sparse Attention 2", sections
    "Full, Reindex, and Reuse" (Reindex rescores the candidate pool) and "The
    Hierarchical Sparse Indexer" (later indexers search only the pool).
    keys [n_vis][d_idx] are the visible keys; returns (ids, scores of the pool)."""
    ent = pool_entries(pool, block, keys.shape[0])
    s = index_scores(q_idx, w, keys[ent]) if ent.shape[0] else np.zeros(0)
    sel = topk(s, k)
    ids = np.where(sel >= 0, ent[np.maximum(sel, 0)] if ent.shape[0] else -1, -1)
    return ids.astype(np.int64), s


def csa2_group_selections(modes, layer_q_idx, layer_w, keys, block: int, pool_blocks: int, k: int):
    """The index selection every layer of one CSA2 layer group attends over,
    for one query.  Tech-report tour, chapter "Compressed Sparse Attention
    2": section "Full, Reindex, and Reuse" (modes table: Full computes fresh
    Top-K indices; Reindex keeps the shared main KV and indexer K and
    rescores the candidate pool with its own indexer query; Reuse takes the
    latest selection and runs no indexer) and section "The Hierarchical Sparse
    Indexer" (the first Full layer of the group builds the candidate pool
    that later indexers search).

    modes: "full" / "reindex" / "reuse" per layer, the first "full" or
    "reindex"; layer_q_idx[l] [h_idx][d_idx] and layer_w[l] [h_idx] are that
    layer's indexer query and weights (unused for Reuse); keys [n_vis][d_idx]
    the group's shared visible indexer keys.  Returns (selections, pool):
    selections[l] the entry ids (-1 padded) layer l attends over; pool the
    block ids the first Full layer kept (None if the group has no Full
    layer, which then needs no Reindex layer either).

    Reading: a Reindex layer before the group's first Full layer has no pool
    to rescore, so the first indexing layer must be Full or the group must
    have no Reindex layer."""
    sel, pool, latest = [], None, None
    for l, mode in enumerate(modes):
        if mode == "full":
            s = index_scores(layer_q_idx[l], layer_w[l], keys)
            latest = topk(s, k)
            if pool is None:
                pool = candidate_pool(s, block, pool_blocks)
        elif mode == "reindex":
            if pool is None:
                raise ValueError("a Reindex layer needs a preceding Full layer's pool")
            latest, _ = reindex_topk(layer_q_idx[l], layer_w[l], keys, pool, block, k)
        elif mode == "reuse":
            if latest is None:
                raise ValueError("a Reuse layer needs a preceding Full or Reindex layer")
        else:
            raise ValueError(mode)
        sel.append(np.asarray(latest, np.int64).copy())
    return sel, pool


# ===========================================================================
# a4 / a5: sparse (or dense) attention + sliding window + sink, one softmax
# ===========================================================================
def window_positions(t: int, W: int, lo: int = 0) -> np.ndarray:
    """Absolute key positions of the sliding window of a query at t.

    Atlas, "Sliding-window attention" entry (token t sees the previous W
    tokens); tech-report tour, "Replay only the window": a replay starting at
    s restricts the keys to [max(s, i-W+1), i].
    """
    start = max(lo, t - W + 1, 0)
    return np.arange(start, t + 1, dtype=np.int64) if W > 0 else np.zeros(0, np.int64)


def attend(q: np.ndarray, entries: np.ndarray, win_k: np.ndarray, win_v: np.ndarray,
           sink: np.ndarray | None, tau: float) -> tuple[np.ndarray, np.ndarray]:
    """One softmax over compressed entries (K = V = entry), window keys and a
    sink logit per head.

    For head h:  l_j = tau q_h . e_j,  l_p = tau q_h . k_p,
      M = max(sink_h, all l),  L = exp(sink_h - M) + sum exp(l - M),
      out_h = (sum_j exp(l_j - M) e_j + sum_p exp(l_p - M) v_p) / L,
      lse_h = M + log L.
    q [h][d], entries [n][d], win_k / win_v [p][d], sink [h] or None.
    With nothing to attend to and no sink: out = 0, lse = -inf.

    Atlas, "compressed KV" entry (sparse attention over the selected
    compressed entries, or dense over all of them) and "MLA" entry (attention
    runs over the latent, so K = V = the entry); tech-report tour, "The
    indexer selects, SWA covers the rest" (the query attends to the selected
    entries together with the layer's sliding-window KV, one softmax).  The
    sink follows the atlas's entry on attention sinks and activation outliers
    (give the model the rescaling it improvises); its form, one logit per
    head in the denominator only, is a reading: the pages print no formula.
    """
    q = np.asarray(q, np.float64)
    keys = np.concatenate([np.asarray(entries, np.float64).reshape(-1, q.shape[1]),
                           np.asarray(win_k, np.float64).reshape(-1, q.shape[1])], axis=0)
    vals = np.concatenate([np.asarray(entries, np.float64).reshape(-1, q.shape[1]),
                           np.asarray(win_v, np.float64).reshape(-1, q.shape[1])], axis=0)
    h = q.shape[0]
    logits = tau * (q @ keys.T)                             # [h][n+p]
    s = np.full(h, -np.inf) if sink is None else np.asarray(sink, np.float64)
    M = np.maximum(s, logits.max(axis=1) if logits.shape[1] else np.full(h, -np.inf))
    out = np.zeros_like(q)
    lse = np.full(h, -np.inf)
    ok = np.isfinite(M)
    if ok.any():
        e = np.exp(logits[ok] - M[ok, None])
        L = e.sum(axis=1) + np.exp(s[ok] - M[ok])
        out[ok] = (e @ vals) / L[:, None]
        lse[ok] = M[ok] + np.log(L)
    return out, lse


def sparse_swa_attention(q, kv_rows, idx, n_vis, swa_k, swa_v, swa_cap, t, W, sink, tau,
                         swa_lo: int = 0):
    """Attention of one query token (all heads) at absolute position t.

    kv_rows: this request's compressed entries [cap][d] (fp64).
    idx: selected entry indices (-1 = padding); None selects all n_vis
         visible entries (the HCA branch, atlas "compressed KV" entry).
    swa_k / swa_v: [swa_cap][d] ring, position p in slot p % swa_cap.
    """
    if idx is None:
        sel = np.arange(n_vis, dtype=np.int64)
    else:
        sel = np.asarray(idx, np.int64)
        sel = sel[sel >= 0]
    ent = np.asarray(kv_rows, np.float64)[sel]
    pos = window_positions(t, W, swa_lo)
    slots = pos % swa_cap
    return attend(q, ent, np.asarray(swa_k, np.float64)[slots], np.asarray(swa_v, np.float64)[slots],
                  sink, tau)


# ===========================================================================
# a6: one decode step
# ===========================================================================
def _rows(t, b: int, rows) -> np.ndarray:
    """fp64 value of rows ``rows`` of request ``b`` of a [B][n][d] stored tensor."""
    data = t.data[b][rows]
    scale = None if t.scale is None else t.scale[b][rows]
    return decode(data, t.dtype, scale, t.group)


def decode_step(inp, tau: float = 1.0, requests=None):
    """One decode step for the requests of a ``workloads.DecodeInputs``.

    Tech-report tour, "Full, Reindex, and Reuse" (Full mode: compute main KV,
    project indexer K, select a fresh top-k) and "The indexer selects, SWA
    covers the rest".  Steps per request b with the new token at position t:
      1. the token's SWA key/value enter ring slot t % swa_cap;
      2. its C/Z row enters open-block slot t % m; if (t+1) % m == 0 the block
         is pooled (``compress``) into entry (t+1)/m - 1, and its indexer key
         is projected from it (``project_index_keys``);
      3. scores of the n_visible(t) entries, top-k (skipped when dense);
      4. one softmax over selected entries + window + sink.
    The new entry and its indexer key are stored in the caches' formats
    (``round_to_storage``) before they are scored and attended, as the
    caches hold them in storage format.  ``requests`` restricts the work to
    some requests (all by default); only the cache rows a request touches
    are decoded.
    Returns dict with out [R][h_q][d], lse [R][h_q], idx [R][k] (or None),
    scores (list), and the new cache rows / keys (fp64, before storage
    rounding) of the requests that closed a block.
    """
    wl = inp.wl
    m = wl.m
    reqs = list(range(wl.batch)) if requests is None else list(requests)
    outs, lses, idxs, scores, new_rows, new_keys = [], [], [], [], [], []
    w_ik = decode_stored(inp.w_ik)
    for b in reqs:
        t = int(inp.pos[b])
        swa_k = _rows(inp.swa_k, b, slice(None)).copy()
        swa_v = _rows(inp.swa_v, b, slice(None)).copy()
        swa_k[t % inp.swa_cap] = decode(inp.k_t.data[b], inp.k_t.dtype)
        swa_v[t % inp.swa_cap] = decode(inp.v_t.data[b], inp.v_t.dtype)
        nv = int(n_visible(t, m))
        new_row = new_key = None
        if (t + 1) % m == 0:
            open_c = _rows(inp.open_c, b, slice(None)).copy()
            open_z = _rows(inp.open_z, b, slice(None)).copy()
            open_c[t % m] = decode(inp.c_t.data[b], inp.c_t.dtype)
            open_z[t % m] = decode(inp.z_t.data[b], inp.z_t.dtype)
            row = compress(open_c, open_z, m)[0]
            key = project_index_keys(row[None], w_ik)[0]
            new_row = round_to_storage(row[None], inp.kv.dtype, inp.kv.group)[0]
            new_key = round_to_storage(key[None], inp.kidx.dtype, inp.kidx.group)[0]
            new_rows.append(row)
            new_keys.append(key)
        if wl.dense:
            sel, s = None, None
            ent = _rows(inp.kv, b, slice(0, nv)).copy()
            if new_row is not None:
                ent[nv - 1] = new_row
        else:
            keys = _rows(inp.kidx, b, slice(0, nv)).copy()
            if new_key is not None:
                keys[nv - 1] = new_key
            q_idx = decode(inp.q_idx.data[b], inp.q_idx.dtype)
            s = index_scores(q_idx, inp.w[b], keys)
            sel = topk(s, wl.topk)
            take = sel[sel >= 0]
            ent = _rows(inp.kv, b, take)
            if new_row is not None:
                ent[take == nv - 1] = new_row
        q = decode(inp.q.data[b], inp.q.dtype)
        pos = window_positions(t, wl.window)
        slots = pos % inp.swa_cap
        o, l = attend(q, ent, swa_k[slots], swa_v[slots], inp.sink, tau)
        outs.append(o)
        lses.append(l)
        idxs.append(sel)
        scores.append(s)
    return {
        "out": np.stack(outs), "lse": np.stack(lses),
        "idx": None if wl.dense else np.stack(idxs),
        "scores": scores, "new_rows": new_rows, "new_keys": new_keys,
    }


def pipeline(inp, queries=None, tau: float = 1.0):
    """The path from the compressor for a ``workloads.PipelineInputs``
    (single request): pool the new C/Z rows into entries appended after the
    ``n_cached`` cached ones (stored in the cache format), project their
    indexer keys, then for each query i (all, or ``queries``) at position
    q_pos[i]: scores over its n_visible entries, top-k, and attention over
    the selection + window + sink.  Causal visibility: block j is visible to
    position t iff (j+1)m - 1 <= t ("Compressed Sparse Attention 2": each
    query attends over causally visible entries)."""
    wl = inp.wl
    m = wl.m
    C = decode_stored(inp.C)[0]
    Z = decode_stored(inp.Z)[0]
    rows = compress(C, Z, m)
    keys = project_index_keys(rows, decode_stored(inp.w_ik))
    n_new = rows.shape[0]
    kv_dt = wl.kv_dtype
    idx_dt = wl.idx_dtype
    stored_rows = round_to_storage(rows, kv_dt, wl.kv_group)
    stored_keys = round_to_storage(keys, idx_dt, wl.d_idx)
    n0 = inp.n_cached
    if n0 > 0:
        cached_keys = _rows(inp.kidx_cached, 0, slice(0, n0))
        all_keys = np.concatenate([cached_keys, stored_keys])
    else:
        all_keys = stored_keys

    def kv_rows(sel):
        sel = np.asarray(sel, np.int64)
        out = np.empty((sel.shape[0], wl.d))
        old = sel < n0
        if old.any():
            out[old] = _rows(inp.kv_cached, 0, sel[old])
        out[~old] = stored_rows[sel[~old] - n0]
        return out

    swa_k = decode_stored(inp.swa_k)[0]
    swa_v = decode_stored(inp.swa_v)[0]
    q_all, qi_all = inp.q, inp.q_idx
    qs = range(inp.q_pos.shape[0]) if queries is None else queries
    outs, lses, idxs, scores = [], [], [], []
    for i in qs:
        t = int(inp.q_pos[i])
        nv = int(n_visible(t, m))
        if wl.dense:
            sel, s = None, None
            ent = kv_rows(np.arange(nv))
        else:
            s = index_scores(decode(qi_all.data[i], qi_all.dtype), inp.w[i], all_keys[:nv])
            sel = topk(s, wl.topk)
            ent = kv_rows(sel[sel >= 0])
        pos = window_positions(t, wl.window)
        slots = pos % inp.swa_cap
        o, l = attend(decode(q_all.data[i], q_all.dtype), ent, swa_k[slots], swa_v[slots], inp.sink, tau)
        outs.append(o)
        lses.append(l)
        idxs.append(sel)
        scores.append(s)
    return {"rows": rows, "keys": keys, "n_new": n_new, "out": np.stack(outs), "lse": np.stack(lses),
            "idx": None if wl.dense else np.stack(idxs), "scores": scores}
