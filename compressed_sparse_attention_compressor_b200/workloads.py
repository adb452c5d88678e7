"""Seeded synthetic inputs for the compressed-sparse-attention hot path.

This module only draws random numbers and stores them in the storage formats
the kernels read: fp32, bf16 bit patterns, and FP8 E4M3 codes with fp32
scales.  It holds none of the method's arithmetic (no pooling, no scoring, no
selection, no attention), so that the CPU oracle and the CUDA path can both be
fed from it without sharing any code with one another.  Rounding to bf16 and
to E4M3 is done by torch's own dtype casts (a library routine).

Workloads (shapes and distributions of the five published configurations):

* ``tiny``      -- batch 1, 4,096-token context, fp32, d=128, m=4, indexer
                   4 heads x 32, top-k 64, 8 query heads, W=128, sink 0.0.
                   C, Z, the SWA keys/values and the indexer query come from
                   seeded projections of N(0,1) hidden states of width 256.
* ``decode64k`` -- batch 16 at 65,536 tokens, bf16, d=512, 64 query heads,
                   indexer 64 x 128, top-k 512, W=128, per-head sinks N(0,1).
* ``prefill``   -- 4,096 new queries on a 131,072-token cached context, bf16.
* ``decode1m``  -- batch 4 at 1,048,576 tokens; FP8 E4M3 main KV with one fp32
                   scale per 64 channels, FP8 indexer keys with one fp32 scale
                   per row, top-k 1,024.
* ``hybrid_csa`` / ``hybrid_hca`` / ``hybrid_ratio1`` -- batch 8 at 262,144
                   tokens: m=4 with top-k 512; m=128 dense over all entries;
                   m=1 with top-k 2,048.

Every workload can be shrunk with :meth:`Workload.scaled` for parity tests.
"""
from __future__ import annotations

import dataclasses
import zlib
from dataclasses import dataclass

import numpy as np

FP8_MAX = 448.0  # largest finite E4M3 value; used to choose storage scales


# --------------------------------------------------------------------------
# storage containers
# --------------------------------------------------------------------------
@dataclass
class Stored:
    """A tensor in its storage format.

    ``data`` is float32 (dtype 'f32'), uint16 bf16 bit patterns ('bf16') or
    uint8 E4M3 codes ('fp8').  For 'fp8', ``scale`` holds one float32 per
    ``group`` consecutive elements of the last axis.
    """

    data: np.ndarray
    dtype: str
    scale: np.ndarray | None = None
    group: int = 0

    @property
    def shape(self):
        return self.data.shape


def _torch():
    import torch  # local import: torch is only a casting library here

    return torch


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even float -> bf16 bit patterns (torch cast)."""
    torch = _torch()
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def to_e4m3_codes(x: np.ndarray, group: int) -> tuple[np.ndarray, np.ndarray]:
    """Store ``x`` as E4M3 codes with one fp32 scale per ``group`` elements.

    The scale of a group is its largest magnitude divided by 448 (1.0 for an
    all-zero group); codes are torch's round-to-nearest-even cast of x/scale.
    """
    torch = _torch()
    x = np.ascontiguousarray(x, dtype=np.float32)
    d = x.shape[-1]
    assert d % group == 0
    g = x.reshape(x.shape[:-1] + (d // group, group))
    amax = np.abs(g).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(FP8_MAX), np.float32(1.0)).astype(np.float32)
    y = (g / scale[..., None]).astype(np.float32)
    y = np.clip(y, -FP8_MAX, FP8_MAX)
    codes = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes.reshape(x.shape), scale


def store(x: np.ndarray, dtype: str, group: int = 0) -> Stored:
    """Store float64/float32 values ``x`` in format ``dtype``."""
    if dtype == "f32":
        return Stored(np.ascontiguousarray(x, dtype=np.float32), "f32")
    if dtype == "bf16":
        return Stored(to_bf16_bits(x), "bf16")
    if dtype == "fp8":
        codes, scale = to_e4m3_codes(x, group)
        return Stored(codes, "fp8", scale, group)
    raise ValueError(dtype)


def empty_stored(shape, dtype: str, group: int = 0) -> Stored:
    """A zero-filled tensor in storage format ``dtype`` (scales of 1.0; MXFP4:
    zero codes and zero scale bytes)."""
    if dtype == "mxfp4":
        return Stored(np.zeros(tuple(shape[:-1]) + (shape[-1] // 2,), np.uint8), "mxfp4",
                      np.zeros(tuple(shape[:-1]) + (shape[-1] // 16,), np.uint8), 16)
    if dtype == "f32":
        return Stored(np.zeros(shape, np.float32), "f32")
    if dtype == "bf16":
        return Stored(np.zeros(shape, np.uint16), "bf16")
    if dtype == "fp8":
        sshape = tuple(shape[:-1]) + (shape[-1] // group,)
        return Stored(np.zeros(shape, np.uint8), "fp8", np.ones(sshape, np.float32), group)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# random streams
# --------------------------------------------------------------------------
def rng(seed: int, tag: str) -> np.random.Generator:
    """Independent PCG64 stream for (seed, tag)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, zlib.crc32(tag.encode())])))


def normal(seed: int, tag: str, shape, std: float = 1.0) -> np.ndarray:
    g = rng(seed, tag)
    return g.standard_normal(size=shape, dtype=np.float32) * np.float32(std)


def random_mxfp4(seed: int, tag: str, shape) -> Stored:
    """An MXFP4 tensor drawn directly in storage form (no rounding): every
    E2M1 code uniform over its 16 values, every E4M3 scale byte uniform over
    0x28 .. 0x2F (0.25 .. 0.46875), so that a group's largest magnitude (6 x
    scale, 1.5 .. 2.8) and the rms (about 1) are those of N(0, 1) entries.
    ``shape`` is the logical [.., d] shape."""
    g = rng(seed, tag)
    data = g.integers(0, 256, size=tuple(shape[:-1]) + (shape[-1] // 2,), dtype=np.uint8)
    scale = g.integers(0x28, 0x30, size=tuple(shape[:-1]) + (shape[-1] // 16,), dtype=np.uint8)
    return Stored(data, "mxfp4", scale, 16)


def uniform(seed: int, tag: str, shape) -> np.ndarray:
    return rng(seed, tag).random(size=shape, dtype=np.float32)


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    """Shape, precision and distribution recipe of one hot-path workload.

    context:  decode -- tokens in context including the current one (the
              current token sits at position context-1);
              prefill -- cached tokens before the new chunk.
    chunk:    0 for decode; number of new query tokens for chunked prefill.
    topk:     <= 0 selects dense attention over every visible entry (HCA).
    """

    name: str
    batch: int
    context: int
    m: int
    d: int
    h_q: int
    h_idx: int
    d_idx: int
    topk: int
    window: int
    kv_dtype: str
    idx_dtype: str
    act_dtype: str
    sink: str  # 'zero' | 'normal'
    chunk: int = 0
    kv_group: int = 64
    hidden: int = 0  # >0: C/Z/SWA/indexer query projected from hidden states
    seed: int = 1000

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def is_prefill(self) -> bool:
        return self.chunk > 0

    @property
    def idx_group(self) -> int:
        return self.d_idx  # one scale per indexer-key row

    @property
    def dense(self) -> bool:
        return self.topk <= 0


WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 4096, 4, 128, 8, 4, 32, 64, 128, "f32", "f32", "f32", "zero",
                     hidden=256, seed=1001),
    "decode64k": Workload("decode64k", 16, 65536, 4, 512, 64, 64, 128, 512, 128, "bf16", "bf16", "bf16",
                          "normal", seed=1002),
    "prefill": Workload("prefill", 1, 131072, 4, 512, 64, 64, 128, 512, 128, "bf16", "bf16", "bf16",
                        "normal", chunk=4096, seed=1003),
    "decode1m": Workload("decode1m", 4, 1048576, 4, 512, 64, 64, 128, 1024, 128, "fp8", "fp8", "bf16",
                         "normal", seed=1004),
    "hybrid_csa": Workload("hybrid_csa", 8, 262144, 4, 512, 64, 64, 128, 512, 128, "bf16", "bf16", "bf16",
                           "normal", seed=1005),
    "hybrid_hca": Workload("hybrid_hca", 8, 262144, 128, 512, 64, 64, 128, 0, 128, "bf16", "bf16", "bf16",
                           "normal", seed=1006),
    "hybrid_ratio1": Workload("hybrid_ratio1", 8, 262144, 1, 512, 64, 64, 128, 2048, 128, "bf16", "bf16",
                              "bf16", "normal", seed=1007),
    # a decoder group of the hierarchical indexer: ratio 1 at 1M tokens, top
    # 512, a pool of 2,048 blocks of 8 positions
    "hier1m": Workload("hier1m", 4, 1048576, 1, 512, 64, 64, 128, 512, 128, "fp8", "fp8", "bf16", "normal",
                       seed=1008),
    # decode1m with the main KV in MXFP4 (E2M1 + one E4M3 scale per 16)
    "decode1m_fp4": Workload("decode1m_fp4", 4, 1048576, 4, 512, 64, 64, 128, 1024, 128, "mxfp4", "fp8", "bf16",
                             "normal", kv_group=16, seed=1009),
}

# candidate pool of the hierarchical indexer: (block, pool_blocks)
HIER_POOL = (8, 2048)


# --------------------------------------------------------------------------
# decode-step inputs
# --------------------------------------------------------------------------
@dataclass
class DecodeInputs:
    """Everything one decode step of ``batch`` requests reads.

    Caches hold ``cap`` rows per request; rows [0, n_prev) are filled.  The
    current token of every request sits at absolute position ``pos``.
    The SWA ring has ``swa_cap`` slots; position p lives in slot p % swa_cap.
    The open-block buffer holds the C/Z rows of the not-yet-closed block in
    slots p % m.
    """

    wl: Workload
    pos: np.ndarray        # [B] int64
    n_prev: int            # compressed rows present before the step
    cap: int
    kv: Stored             # [B][cap][d]
    kidx: Stored           # [B][cap][d_idx]
    swa_k: Stored          # [B][swa_cap][d]
    swa_v: Stored
    swa_cap: int
    open_c: Stored         # [B][m][d]
    open_z: Stored
    c_t: Stored            # [B][d]
    z_t: Stored
    k_t: Stored            # [B][d]
    v_t: Stored
    q: Stored              # [B][h_q][d]
    q_idx: Stored          # [B][h_idx][d_idx]
    w: np.ndarray          # [B][h_idx] float32
    sink: np.ndarray       # [h_q] float32
    w_ik: Stored           # [d][d_idx]


def _sink(wl: Workload) -> np.ndarray:
    if wl.sink == "zero":
        return np.zeros(wl.h_q, np.float32)
    return normal(wl.seed, "sink", (wl.h_q,))


def _kv_cache(seed: int, wl: Workload, kv: np.ndarray, n_filled: int) -> Stored:
    """The main-KV cache in storage format: ``kv`` stored, or for MXFP4 rows
    [0, n_filled) drawn directly in storage form and the rest zero."""
    if wl.kv_dtype != "mxfp4":
        return store(kv, wl.kv_dtype, wl.kv_group)
    st = random_mxfp4(seed, "kv", kv.shape)
    st.data[:, n_filled:] = 0
    st.scale[:, n_filled:] = 0
    return st


def make_decode_inputs(wl: Workload) -> DecodeInputs:
    assert not wl.is_prefill
    B, T, m, d = wl.batch, wl.context, wl.m, wl.d
    pos = T - 1
    n_prev = pos // m
    cap = T // m
    sd, sI = 1.0 / np.sqrt(d), 1.0 / np.sqrt(wl.d_idx)
    s = wl.seed
    kv_std = 1.0 if wl.kv_dtype == "fp8" else sd
    kv = np.zeros((B, cap, d), np.float32)
    if wl.kv_dtype != "mxfp4":
        kv[:, :n_prev] = normal(s, "kv", (B, n_prev, d), kv_std)
    kv_st = _kv_cache(s, wl, kv, n_prev)
    kidx = np.zeros((B, cap, wl.d_idx), np.float32)
    kidx[:, :n_prev] = normal(s, "kidx", (B, n_prev, wl.d_idx), sI)
    W = wl.window
    swa_cap = max(W, 1)
    act = wl.act_dtype
    return DecodeInputs(
        wl=wl,
        pos=np.full(B, pos, np.int64),
        n_prev=n_prev,
        cap=cap,
        kv=kv_st,
        kidx=store(kidx, wl.idx_dtype, wl.idx_group),
        swa_k=store(normal(s, "swa_k", (B, swa_cap, d), sd), act),
        swa_v=store(normal(s, "swa_v", (B, swa_cap, d), sd), act),
        swa_cap=swa_cap,
        open_c=store(normal(s, "open_c", (B, m, d), sd), act),
        open_z=store(normal(s, "open_z", (B, m, d)), act),
        c_t=store(normal(s, "c_t", (B, d), sd), act),
        z_t=store(normal(s, "z_t", (B, d)), act),
        k_t=store(normal(s, "k_t", (B, d), sd), act),
        v_t=store(normal(s, "v_t", (B, d), sd), act),
        q=store(normal(s, "q", (B, wl.h_q, d), sd), act),
        q_idx=store(normal(s, "q_idx", (B, wl.h_idx, wl.d_idx), sI), act),
        w=uniform(s, "w", (B, wl.h_idx)),
        sink=_sink(wl),
        w_ik=store(normal(s, "w_ik", (d, wl.d_idx), sd), act),
    )


# --------------------------------------------------------------------------
# pipeline inputs: compressor input C/Z plus one query per request
# --------------------------------------------------------------------------
@dataclass
class PipelineInputs:
    """Inputs of the full path starting at the compressor.

    Request b has ``n_tokens`` raw rows C[b], Z[b]; the query sits at position
    n_tokens-1 (decode) or at positions ``q_pos`` (prefill).  For prefill the
    cache already holds ``n_cached`` compressed rows and C/Z are the new chunk.
    """

    wl: Workload
    C: Stored               # [B][n_new][d]
    Z: Stored
    n_cached: int
    kv_cached: Stored | None   # [B][cap][d] with rows [0, n_cached) filled
    kidx_cached: Stored | None
    cap: int
    swa_k: Stored           # [B][swa_cap][d]
    swa_v: Stored
    swa_cap: int
    q: Stored               # [nq][h_q][d]
    q_idx: Stored           # [nq][h_idx][d_idx]
    w: np.ndarray           # [nq][h_idx]
    q_pos: np.ndarray       # [nq] int64
    q_req: np.ndarray       # [nq] int32
    sink: np.ndarray
    w_ik: Stored            # [d][d_idx]


def make_tiny_pipeline_inputs(wl: Workload) -> PipelineInputs:
    """Hidden-state driven inputs (the tiny configuration).

    H ~ N(0,1) of width ``hidden``; W_KV, W_Z, W_K, W_V, W_IQ ~ N(0, 1/hidden);
    W_IK ~ N(0, 1/d).  C = H W_KV, Z = H W_Z, SWA K/V = H W_K / H W_V, the
    indexer query is H[t] W_IQ split into heads, the main query is
    N(0,1)/sqrt(d) per head, indexer head weights U(0,1).
    """
    assert wl.hidden > 0 and wl.batch == 1 and not wl.is_prefill
    s, T, d, hd = wl.seed, wl.context, wl.d, wl.hidden
    H = normal(s, "H", (T, hd)).astype(np.float64)

    def proj(tag, fan_in, n_out):
        return normal(s, tag, (fan_in, n_out), 1.0 / np.sqrt(fan_in)).astype(np.float64)

    C = H @ proj("W_KV", hd, d)
    Z = H @ proj("W_Z", hd, d)
    Kw = H @ proj("W_K", hd, d)
    Vw = H @ proj("W_V", hd, d)
    qI = (H[T - 1] @ proj("W_IQ", hd, wl.h_idx * wl.d_idx)).reshape(1, wl.h_idx, wl.d_idx)
    w_ik = proj("W_IK", d, wl.d_idx)
    W = wl.window
    swa_cap = W
    t0 = max(0, T - W)
    sk = np.zeros((1, swa_cap, d))
    sv = np.zeros((1, swa_cap, d))
    for p in range(t0, T):
        sk[0, p % swa_cap] = Kw[p]
        sv[0, p % swa_cap] = Vw[p]
    f = wl.act_dtype
    return PipelineInputs(
        wl=wl,
        C=store(C[None], f), Z=store(Z[None], f),
        n_cached=0, kv_cached=None, kidx_cached=None, cap=T // wl.m,
        swa_k=store(sk, f), swa_v=store(sv, f), swa_cap=swa_cap,
        q=store(normal(s, "q", (1, wl.h_q, d), 1.0 / np.sqrt(d)), f),
        q_idx=store(qI, f),
        w=uniform(s, "w", (1, wl.h_idx)),
        q_pos=np.array([T - 1], np.int64),
        q_req=np.zeros(1, np.int32),
        sink=_sink(wl),
        w_ik=store(w_ik, f),
    )


def make_prefill_inputs(wl: Workload) -> PipelineInputs:
    """Chunked prefill: ``chunk`` new tokens after ``context`` cached tokens.

    Cached compressed rows are N(0,1)/sqrt(d); cached indexer keys
    N(0,1)/sqrt(d_idx).  The chunk's C is N(0,1)/sqrt(d), Z is N(0,1).  SWA
    keys/values for the W-1 tokens before the chunk and for every chunk token
    are N(0,1)/sqrt(d), held in a ring of ``swa_cap`` >= chunk + W slots.
    """
    assert wl.is_prefill and wl.batch == 1
    s, d, m, L = wl.seed, wl.d, wl.m, wl.chunk
    T0 = wl.context
    n_cached = T0 // m
    cap = (T0 + L) // m
    sd, sI = 1.0 / np.sqrt(d), 1.0 / np.sqrt(wl.d_idx)
    kv = np.zeros((1, cap, d), np.float32)
    kv[:, :n_cached] = normal(s, "kv", (1, n_cached, d), sd)
    kidx = np.zeros((1, cap, wl.d_idx), np.float32)
    kidx[:, :n_cached] = normal(s, "kidx", (1, n_cached, wl.d_idx), sI)
    swa_cap = 1
    while swa_cap < L + wl.window:
        swa_cap *= 2
    f = wl.act_dtype
    return PipelineInputs(
        wl=wl,
        C=store(normal(s, "C", (1, L, d), sd), f),
        Z=store(normal(s, "Z", (1, L, d)), f),
        n_cached=n_cached,
        kv_cached=_kv_cache(s, wl, kv, n_cached),
        kidx_cached=store(kidx, wl.idx_dtype, wl.idx_group),
        cap=cap,
        swa_k=store(normal(s, "swa_k", (1, swa_cap, d), sd), f),
        swa_v=store(normal(s, "swa_v", (1, swa_cap, d), sd), f),
        swa_cap=swa_cap,
        q=store(normal(s, "q", (L, wl.h_q, d), sd), f),
        q_idx=store(normal(s, "q_idx", (L, wl.h_idx, wl.d_idx), sI), f),
        w=uniform(s, "w", (L, wl.h_idx)),
        q_pos=np.arange(T0, T0 + L, dtype=np.int64),
        q_req=np.zeros(L, np.int32),
        sink=_sink(wl),
        w_ik=store(normal(s, "w_ik", (d, wl.d_idx), sd), f),
    )


def make_scores(seed: int, n_rows: int, n_cols: int, tie_frac: float = 0.1) -> np.ndarray:
    """Random fp32 score rows with planted exact ties (zeros, repeated values
    and negative zero) for testing selection on its own."""
    g = rng(seed, "scores")
    s = g.standard_normal((n_rows, n_cols), dtype=np.float32)
    mask = g.random((n_rows, n_cols)) < tie_frac
    s[mask] = 0.0
    neg0 = g.random((n_rows, n_cols)) < tie_frac / 4
    s[neg0] = -0.0
    rep = g.random((n_rows, n_cols)) < tie_frac
    vals = np.round(g.standard_normal((n_rows, n_cols)).astype(np.float32) * 4) / 4
    s[rep] = vals[rep]
    return s


def make_indices(seed: int, n_vis: np.ndarray, k: int, pad_frac: float = 0.0) -> np.ndarray:
    """Random distinct entry indices per query (an explicit selection for
    testing attention on its own): row i holds min(k, n_vis[i]) distinct
    indices below n_vis[i] in random order, then -1 padding; with
    ``pad_frac`` > 0 some rows hold fewer entries."""
    g = rng(seed, "indices")
    out = np.full((n_vis.shape[0], k), -1, np.int32)
    for i, n in enumerate(n_vis):
        take = min(k, int(n))
        if pad_frac > 0 and g.random() < pad_frac:
            take = int(g.integers(0, take + 1))
        out[i, :take] = g.permutation(int(n))[:take]
    return out
