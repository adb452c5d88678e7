"""Decode-step throughput of the compressed-sparse-attention hot path on B200.

One step = csa_decode_step for every request of the workload: append the new
token (SWA ring + open block), pool the block it closes and project its
indexer key, score all visible compressed entries, select the top-k, and run
the single-softmax attention over the selection + window + sink.

Default workload: ``decode1m`` -- batch 4 at 1,048,576 tokens, m = 4
(262,144 compressed entries per request), FP8 E4M3 main KV (fp32 scale per
64 channels) and FP8 indexer keys (fp32 scale per row), 64 bf16 query heads
of dim 512, indexer 64 x 128, top-k 1,024, W = 128.  Inputs are seeded and
synthetic and resident in HBM.  The timed steps run back to back on
rotating copies of the caches: consecutive steps read different copies and
at least twice the L2's size is read between two steps on the same copy, so
every step's inputs come from HBM, while the kernels' code stays warm in L2
(as when one kernel serves every layer of a model).  ``e2e`` is the host's
wall clock over K back-to-back steps through the public API, each with its
host-to-device input copy and device-to-host output copy (on their own
streams, overlapping the neighbouring steps' kernels), one synchronize at the
end.  (``--path hier`` and ``--path prefill`` flush L2 between steps.)

Metric: decode tokens/s (requests finished per second, all ranks).
Multi-GPU: every rank runs its own batch (independent requests, no
collective on the data path): weak scaling, max-over-ranks device time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle as the reference arm
  python bench.py --path hier ...        # the hierarchical sparse indexer (hier1m)
  python bench.py --path prefill ...     # chunked prefill (query-tokens/s)

``--path hier`` times one Reindex layer of a decoder group at 1M tokens
(ratio 1, FP8 indexer keys, top 512): the lightning indexer over the
16,384-position candidate pool that the group's Full layer built (2,048
blocks of 8), its top-512, and the pool-position -> entry mapping.  The Full
layer (full scan + block maxima + pool) and a full scan with the Reindex
layer's query are timed beside it.

``--path prefill`` times one 4,096-token chunk after 131,072 cached tokens:
the chunk's compressor (1,024 new entries and their indexer keys), then the
indexer, top-512 and attention (selection + window + sink) of its 4,096
queries, each over the entries causally visible to it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from compressed_sparse_attention_compressor_b200 import workloads as Wk  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode1m", choices=[k for k, v in Wk.WORKLOADS.items() if not v.is_prefill])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", default="step", choices=["step", "hier", "prefill"])
    ap.add_argument("--copies", type=int, default=0,
                    help="cache copies the decode steps rotate over (0: enough that no step finds its inputs in "
                         "L2; a profiler run may ask for fewer to hold less memory)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# byte accounting (algorithmic bytes: what the path must read / write once)
# ---------------------------------------------------------------------------
def _eb(dt):
    return {"f32": 4, "bf16": 2, "fp8": 1}[dt]


def key_row_bytes(wl):
    return wl.d_idx * _eb(wl.idx_dtype) + (4 if wl.idx_dtype == "fp8" else 0)


def kv_row_bytes(wl):
    if wl.kv_dtype == "mxfp4":
        return wl.d // 2 + wl.d // 16  # two E2M1 codes per byte, one E4M3 scale byte per 16
    return wl.d * _eb(wl.kv_dtype) + (4 * wl.d // wl.kv_group if wl.kv_dtype == "fp8" else 0)


def step_bytes(wl, n_vis):
    """Headline bytes of one decode step: the visible indexer keys, the
    selected (or, dense, all visible) compressed rows, the window K/V rows."""
    B = wl.batch
    keys = 0 if wl.dense else B * n_vis * key_row_bytes(wl)
    rows = B * (n_vis if wl.dense else min(wl.topk, n_vis)) * kv_row_bytes(wl)
    window = B * 2 * wl.window * wl.d * _eb(wl.act_dtype)
    return keys + rows + window


def kernel_bytes(name, wl, n_vis):
    """Algorithmic bytes of one launch of a kernel of the decode step: what it
    must read or write once (the attention: the selected or, dense, all
    visible compressed rows, the window's K and V rows, the queries and the
    outputs; the merge: the split states it combines and the outputs)."""
    B, ea = wl.batch, _eb(wl.act_dtype)
    if name.startswith("index_"):
        return B * n_vis * key_row_bytes(wl) + B * wl.h_idx * (wl.d_idx * ea + 4)
    if name.startswith("attn_merge"):
        splits = -(-((n_vis if wl.dense else min(wl.topk, n_vis)) + wl.window) // 128)
        return B * splits * wl.h_q * (wl.d + 2) * 4 + B * wl.h_q * wl.d * ea
    if name.startswith("attn_"):
        rows = n_vis if wl.dense else min(wl.topk, n_vis)
        return (B * rows * kv_row_bytes(wl) + B * 2 * wl.window * wl.d * ea + 2 * B * wl.h_q * wl.d * ea)
    if name.startswith("topk"):
        return B * n_vis * 4 + B * wl.topk * 4
    if name.startswith("decode_append"):
        # the token's four rows, the open block's C / Z rows, the pooled row
        # and its indexer key, W_IK
        return B * wl.d * ea * (4 + 2 * wl.m) + B * (kv_row_bytes(wl) + key_row_bytes(wl)) + wl.d * wl.d_idx * ea
    return None


def rank_workload(name, rank):
    """Every rank runs its own requests: the workload's shapes, its own seed
    (replicas: the requests are independent, nothing is exchanged)."""
    base = Wk.WORKLOADS[name]
    return base.scaled(seed=base.seed + 100 * rank)


def max_over_ranks(x, dist, device):
    """The largest x over the ranks (x itself without a process group)."""
    if dist is None:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def tokens_per_s(batch_per_rank, world, ms_per_step):
    """Whole-job decode throughput: every rank's requests over the slowest
    rank's step time."""
    return batch_per_rank * world / (ms_per_step * 1e-3)


def step_stats(ms):
    """Median and 10th / 90th percentiles of per-step times (ms), this rank's."""
    v = np.asarray(list(ms), dtype=np.float64)
    if v.size == 0:
        return None
    p10, p50, p90 = np.percentile(v, [10, 50, 90])
    return {"p10_ms": float(p10), "median_ms": float(p50), "p90_ms": float(p90)}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def load_traffic(name, workload):
    """DRAM bytes per launch from the committed ncu summary of a kernel on a
    workload (profiles/<kernel>_<workload>.md), if the kernel's source is
    unchanged since the capture (else None)."""
    for path in [os.path.join(ROOT, "profiles", f"{name}_{workload}.md")]:
        import re
        try:
            text = open(path).read()
            nbytes = int(re.search(r"traffic_bytes_per_launch:\s*(\d+)", text).group(1))
            src = re.search(r"- source:\s*(\S+)", text).group(1)
            want = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", text).group(1)
            cur = os.path.join(ROOT, "compressed_sparse_attention_compressor_b200", "csrc", src)
            if hashlib.sha256(open(cur, "rb").read()).hexdigest()[:16] == want:
                return float(nbytes)
        except Exception:
            continue
    return None


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-i", str(self.index), "-lms", "200"], stdout=subprocess.PIPE,
                                      stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.p = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.p is not None:
            time.sleep(0.3)
            self.p.terminate()
            try:
                self.out, _ = self.p.communicate(timeout=5)
            except Exception:
                self.p.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def n_copies(step_bytes_, copy_bytes, budget=24 << 30):
    """Copies of the caches the timed steps rotate through: consecutive steps
    read different copies, and at least twice the L2's size is read between
    two steps on the same copy, so no step finds its inputs in L2 (the
    kernels' code and the small per-step buffers stay warm, as they do when
    one kernel serves every layer of a model)."""
    c = max(2, -(-2 * L2_BYTES // max(int(step_bytes_), 1)) + 1)
    return int(min(c, max(2, budget // max(int(copy_bytes), 1))))


def run_ours(args, rank, world, local_rank):
    import torch

    from compressed_sparse_attention_compressor_b200 import csa
    from compressed_sparse_attention_compressor_b200.csa import DevTensor

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist_
        dist = dist_

    wl = rank_workload(args.workload, rank)
    inp = Wk.make_decode_inputs(wl)
    B = wl.batch
    up = DevTensor.from_stored
    n_vis = int((inp.pos[0] + 1) // wl.m)
    sbytes = step_bytes(wl, n_vis)
    cache_st = (inp.kv, inp.kidx, inp.swa_k, inp.swa_v, inp.open_c, inp.open_z)
    copy_bytes = sum(t.data.nbytes + (t.scale.nbytes if t.scale is not None else 0) for t in cache_st)
    ncp = args.copies if args.copies > 0 else n_copies(sbytes, copy_bytes)
    caches, keep = [], []
    for _ in range(ncp):
        kv, kidx, swa_k, swa_v, open_c, open_z = (up(t) for t in cache_st)
        keep.append((kv, kidx, swa_k, swa_v, open_c, open_z))
        caches.append(csa.decode_caches(kv, kidx, swa_k, swa_v, open_c, open_z, inp.cap))
    c_t, z_t, k_t, v_t, q, q_idx, w_ik = (up(inp.c_t), up(inp.z_t), up(inp.k_t), up(inp.v_t), up(inp.q),
                                          up(inp.q_idx), up(inp.w_ik))
    w = torch.from_numpy(inp.w).cuda()
    sink = torch.from_numpy(inp.sink).cuda()
    pos = torch.from_numpy(inp.pos).cuda()
    p = csa.params(wl.m, wl.d, wl.d_idx, wl.h_q, wl.h_idx, wl.topk, wl.window, inp.swa_cap, 1.0)
    out = DevTensor.empty((B, wl.h_q, wl.d), "bf16" if wl.act_dtype != "f32" else "f32")
    lse = torch.empty((B, wl.h_q), dtype=torch.float32, device="cuda")
    ws = csa.workspace(csa.csa_workspace_size(p, B, inp.cap))
    # a dense (HCA) layer has no indexer: no indexer query, weights or key projection
    sparse = not wl.dense
    tok = csa.decode_token(c_t, z_t, k_t, v_t, q, q_idx if sparse else None, w if sparse else None, sink,
                           w_ik if sparse else None)
    stream = torch.cuda.current_stream()
    del inp

    def step(i, tk=tok, o=out):
        csa.csa_decode_step(p, B, caches[i % ncp], tk, pos, o, lse, None, ws, stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    def head_start():
        # the GPU idles ~1 ms while the host queues the first steps, so that
        # no step's events wait on the host's launch calls
        torch.cuda._sleep(2_000_000)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # ---- timed region: K back-to-back steps on rotating cache copies, one
    # event pair around all of them (the K steps' device time, gaps included) ----
    K = args.steps
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        head_start()
        t_start.record(stream)
        for i in range(K):
            step(i)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), dist, "cuda")
    ms_per_step = total_ms / K
    # the spread of single steps: the same K steps with an event pair around each
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    head_start()
    for i in range(K):
        e0[i].record(stream)
        step(i)
        e1[i].record(stream)
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in zip(e0, e1)]

    # ---- per-kernel times: the same K steps with events around every launch ----
    csa.csa_profile_start(64 * K)
    head_start()
    for i in range(K):
        step(i)
    torch.cuda.synchronize()
    csa.csa_profile_stop()
    recs = csa.csa_profile_records()
    per = {}
    for name, ms in recs:
        c = per.setdefault(name, [0, 0.0])
        c[0] += 1
        c[1] += ms
    launches_per_step = len(recs) / K
    dom = max(per, key=lambda n: per[n][1])
    dom_ms = per[dom][1] / per[dom][0]
    dom_bytes = kernel_bytes(dom, wl, n_vis)
    peak, peak_src = load_peaks()
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9 if dom_bytes else None

    # ---- end to end: host inputs -> device -> step -> host output ----
    # The token's inputs sit back to back in one pinned host buffer and one device
    # buffer (256-byte aligned slots), so each step moves them with one copy; the
    # step reads views of the device buffer.  Two device buffers and two outputs
    # alternate, so that step i + 1's input copy and step i - 1's output copy run
    # on their own streams while step i computes (a serving loop's pipeline).
    toks = (c_t, z_t, k_t, v_t, q, q_idx) if sparse else (c_t, z_t, k_t, v_t, q)
    srcs = [t.data for t in toks] + ([w] if sparse else []) + [t.scale for t in toks if t.scale is not None]
    offs, total = [], 0
    for t in srcs:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    nt = len(toks)

    def make_pack():
        dev = torch.empty(total, dtype=torch.uint8, device="cuda")
        views = []
        for t, o in zip(srcs, offs):
            v_ = dev[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
            v_.copy_(t)
            views.append(v_)
        sc_views = iter(views[nt + (1 if sparse else 0):])
        tv = [DevTensor(vw, t.dtype, next(sc_views) if t.scale is not None else None, t.group)
              for vw, t in zip(views[:nt], toks)]
        if sparse:
            return dev, csa.decode_token(*tv, views[nt], sink, w_ik)
        return dev, csa.decode_token(*tv, None, None, sink, None)

    packs, tok_ps = zip(*(make_pack() for _ in range(2)))
    host_pack = packs[0].cpu().pin_memory()
    outs = (out, DevTensor.empty(tuple(out.data.shape), "bf16" if wl.act_dtype != "f32" else "f32"))
    host_outs = [torch.empty_like(o.data, device="cpu").pin_memory() for o in outs]
    h2d = host_pack.numel()
    d2h = host_outs[0].numel() * host_outs[0].element_size()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]   # pack b holds its step's inputs
    in_free = [torch.cuda.Event() for _ in range(2)]    # the step that read pack b is done
    out_ready = [torch.cuda.Event() for _ in range(2)]  # output b holds its step's result
    out_free = [torch.cuda.Event() for _ in range(2)]   # output b has been read back

    def e2e_loop(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(in_free[b])
                packs[b].copy_(host_pack, non_blocking=True)
                in_ready[b].record(h2d_s)
            stream.wait_event(in_ready[b])
            if i >= 2:
                stream.wait_event(out_free[b])
            step(i, tok_ps[b], outs[b])
            in_free[b].record(stream)
            out_ready[b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(out_ready[b])
                host_outs[b].copy_(outs[b].data, non_blocking=True)
                out_free[b].record(d2h_s)
        stream.wait_stream(d2h_s)

    # host wall clock: K back-to-back steps through the public API, every
    # launch and copy issued by the host inside the region, one synchronize
    # at its end (no head start: the host's own cost is part of the number)
    e2e_loop(2)
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e2e_loop(K)
    torch.cuda.synchronize()
    wall_ms = (time.perf_counter() - t0) * 1e3
    barrier()
    e2e_ms = max_over_ranks(wall_ms, dist, "cuda") / K
    # the same loop timed on the device: from before the first input copy to
    # after the last output copy (events on the launch stream)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    head_start()
    f0.record(stream)
    h2d_s.wait_stream(stream)
    e2e_loop(K)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_dev_ms = max_over_ranks(f0.elapsed_time(f1), dist, "cuda") / K

    value = tokens_per_s(B, world, ms_per_step)
    res = {
        "metric": "decode tokens/s (CSA+SWA attention step)",
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "step_ms": step_stats(step_ms),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.kv_dtype if wl.kv_dtype in ("fp8", "mxfp4") else wl.act_dtype,
        "data": "synthetic (seeded Gaussian caches and queries)",
        "config": {
            "workload": wl.name, "batch_per_gpu": B, "context": wl.context, "m": wl.m,
            "compressed_entries": n_vis, "topk": wl.topk, "window": wl.window, "d": wl.d, "h_q": wl.h_q,
            "indexer": f"{wl.h_idx}x{wl.d_idx}", "kv_dtype": wl.kv_dtype, "idx_dtype": wl.idx_dtype,
            "parallelism": f"replicas x{world}",
            "l2": (f"inputs larger than L2: steps rotate over {ncp} copies of the caches, "
                   f"{ncp * sbytes / 1e6:.0f} MB of step reads between two reads of one copy (L2 126 MB)"),
        },
        "step_hbm": {"bytes": sbytes, "gbs": sbytes / (ms_per_step * 1e-3) / 1e9,
                     "frac_of_peak": sbytes / (ms_per_step * 1e-3) / 1e9 / peak,
                     "frac_of_8tbs": sbytes / (ms_per_step * 1e-3) / 1e9 / 8000.0},
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak if achieved else None, "traffic": load_traffic(dom, wl.name),
                     "algorithmic_bytes": dom_bytes, "avg_ms": dom_ms, "peak_source": f"{peak_src} hbm_gbs"},
        "kernels": {n: {"launches": c, "total_ms": t, "avg_us": 1e3 * t / c,
                        "share": t / sum(v[1] for v in per.values()),
                        "algorithmic_bytes": kernel_bytes(n, wl, n_vis)}
                    for n, (c, t) in per.items()},
        "gpu_launches": int(round(launches_per_step * K)),
        "e2e": {"value": tokens_per_s(B, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "timing": ("host wall clock over K back-to-back steps, one sync at the end; every step copies its "
                           "inputs in and its output back, on their own streams, overlapping the neighbouring "
                           "steps' compute (two input buffers, two outputs)"),
                "device_timed": {"value": tokens_per_s(B, world, e2e_dev_ms), "ms_per_step": e2e_dev_ms}},
        "clocks": clk.summary(),
    }
    return res


def run_hier(args, rank, world, local_rank):
    """The hierarchical sparse indexer: one Reindex layer over the Full
    layer's candidate pool, on hier1m."""
    import torch

    from compressed_sparse_attention_compressor_b200 import csa
    from compressed_sparse_attention_compressor_b200.csa import DevTensor

    torch.cuda.set_device(local_rank)
    wl = rank_workload("hier1m", rank)
    block, pool_blocks = Wk.HIER_POOL
    B, cap, s = wl.batch, wl.context // wl.m, wl.seed
    sI = 1.0 / np.sqrt(wl.d_idx)
    up = DevTensor.from_stored
    kidx_st = Wk.store(Wk.normal(s, "kidx", (B, cap, wl.d_idx), sI), wl.idx_dtype, wl.idx_group)
    qf_st = Wk.store(Wk.normal(s, "q_idx", (B, wl.h_idx, wl.d_idx), sI), wl.act_dtype)
    qr_st = Wk.store(Wk.normal(s, "q_idx_reindex", (B, wl.h_idx, wl.d_idx), sI), wl.act_dtype)
    wf_np, wr_np = Wk.uniform(s, "w", (B, wl.h_idx)), Wk.uniform(s, "w_reindex", (B, wl.h_idx))
    kidx, q_full, q_re = up(kidx_st), up(qf_st), up(qr_st)
    w_full, w_re = torch.from_numpy(wf_np).cuda(), torch.from_numpy(wr_np).cuda()
    n_vis = torch.full((B,), cap, dtype=torch.int32, device="cuda")
    p = csa.params(wl.m, wl.d, wl.d_idx, wl.h_q, wl.h_idx, wl.topk, wl.window, max(wl.window, 1), 1.0)
    ws = csa.workspace(max(csa.csa_index_pool_workspace_size(p, B, cap, block, pool_blocks),
                           csa.csa_workspace_size(p, B, cap)))
    pool = torch.empty((B, pool_blocks), dtype=torch.int32, device="cuda")
    idx_full = torch.empty((B, wl.topk), dtype=torch.int32, device="cuda")
    idx_re = torch.empty((B, wl.topk), dtype=torch.int32, device="cuda")
    idx_scan = torch.empty((B, wl.topk), dtype=torch.int32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    evict = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def flush_l2():
        flush.zero_()
        evict.sum()
        torch.cuda._sleep(200_000)

    def full():
        csa.csa_index_topk_pool(p, B, q_full, w_full, kidx, B, cap, None, n_vis, block, pool_blocks, pool, idx_full,
                                None, ws, stream)

    def reindex():
        csa.csa_index_topk_reindex(p, B, q_re, w_re, kidx, B, cap, None, n_vis, pool, block, pool_blocks, idx_re,
                                   None, ws, stream)

    def scan():
        csa.csa_index_topk(p, B, q_re, w_re, kidx, B, cap, None, n_vis, idx_scan, None, ws, stream)

    def timed(fn, K):
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        for i in range(K):
            flush_l2()
            e0[i].record(stream)
            fn()
            e1[i].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in zip(e0, e1)]

    full()
    for _ in range(args.warmup):
        for fn in (full, reindex, scan):
            flush_l2()
            fn()
    torch.cuda.synchronize()
    K = args.steps
    with ClockSampler(local_rank) as clk:
        re_ms = timed(reindex, K)
    full_ms = timed(full, K)
    scan_ms = timed(scan, K)
    ms = float(sum(re_ms)) / K

    csa.csa_profile_start(64 * K)
    for _ in range(K):
        flush_l2()
        reindex()
    torch.cuda.synchronize()
    csa.csa_profile_stop()
    per = {}
    for name, t in csa.csa_profile_records():
        c = per.setdefault(name, [0, 0.0])
        c[0] += 1
        c[1] += t
    dom = max(per, key=lambda n: per[n][1])
    dom_ms = per[dom][1] / per[dom][0]
    P = block * pool_blocks
    # the dominant launch reads the pool's keys (code bytes + row scale), the
    # pool itself, the queries and the weights
    peak, peak_src = load_peaks()
    dom_bytes = B * (P * key_row_bytes(wl) + pool_blocks * 4 + wl.h_idx * (wl.d_idx * _eb(wl.act_dtype) + 4))
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    res = {
        "metric": "Reindex-layer selections/s (top-512 over a 16,384-candidate pool, 1M tokens)",
        "value": B / (ms * 1e-3),
        "unit": "queries/s",
        "n_gpus": 1,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "step_ms": step_stats(re_ms),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8",
        "data": "synthetic (seeded Gaussian indexer keys and queries)",
        "config": {"workload": wl.name, "batch": B, "context": wl.context, "m": wl.m, "entries": cap,
                   "block": block, "pool_blocks": pool_blocks, "candidates": P, "topk": wl.topk,
                   "indexer": f"{wl.h_idx}x{wl.d_idx}", "idx_dtype": wl.idx_dtype,
                   "l2": "flushed between timed steps (256 MB write, then 256 MB read)"},
        "full_layer_ms": float(sum(full_ms)) / K,
        "full_scan_ms": float(sum(scan_ms)) / K,
        "reindex_vs_full_scan": (float(sum(scan_ms)) / K) / ms,
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": load_traffic(dom, "hier1m_reindex"),
                     "algorithmic_bytes": dom_bytes, "avg_ms": dom_ms, "peak_source": f"{peak_src} hbm_gbs"},
        "kernels": {n: {"launches": c, "total_ms": t, "share": t / sum(v[1] for v in per.values())}
                    for n, (c, t) in per.items()},
        "gpu_launches": sum(c for c, _ in per.values()),
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        # the oracle on request 0: its Full layer builds the pool (not timed),
        # its Reindex layer is the sample
        from oracle import csa_oracle as O

        keys = O.decode(kidx_st.data[0], kidx_st.dtype, kidx_st.scale[0], kidx_st.group)
        qf, qr = O.decode_stored(qf_st)[0], O.decode_stored(qr_st)[0]
        opool = O.candidate_pool(O.index_scores(qf, wf_np[0], keys), block, pool_blocks)
        n_s, t_s = 0, 0.0
        while n_s < 3 or t_s < 5.0:
            t0 = time.perf_counter()
            O.reindex_topk(qr, wr_np[0], keys, opool, block, wl.topk)
            t_s += time.perf_counter() - t0
            n_s += 1
        res["cpu_baseline"] = {"value": n_s / t_s, "unit": "queries/s", "cores": _threads(), "kind": "oracle",
                               "sample": f"{n_s} Reindex-layer selections of request 0 ({t_s:.1f} s)"}
    return res


def prefill_kernel_work(name, wl, sum_vis, sum_keys):
    """Algorithmic work of one launch of a chunked-prefill kernel: (amount,
    kind) with kind 'alu' (fp32 flops on CUDA cores), 'tensor' (bf16 flops)
    or 'hbm' (bytes).  sum_vis: visible entries summed over the queries;
    sum_keys: attended keys (selected entries + window) summed over them."""
    if name.startswith("index_many"):
        return 2.0 * wl.h_idx * wl.d_idx * sum_vis, "tensor"
    if name.startswith("index_score"):
        return 2.0 * wl.h_idx * wl.d_idx * sum_vis, "alu"
    if name.startswith("attn_tc") or name.startswith("attn_many"):
        return 4.0 * wl.h_q * wl.d * sum_keys, "tensor"
    if name.startswith("attn"):
        return 4.0 * wl.h_q * wl.d * sum_keys, "alu"
    if name.startswith("topk"):
        return 4.0 * sum_vis, "hbm"
    if name.startswith("compress"):
        n_tok = wl.chunk
        return (2.0 * n_tok * wl.d * _eb(wl.act_dtype) + n_tok // wl.m * (kv_row_bytes(wl) + key_row_bytes(wl))), "hbm"
    return None, None


def bf16_peak():
    """Measured dense bf16 tensor peak (TFLOP/s, burst), else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def alu_peak_tflops(sms):
    """fp32 FMA peak of the CUDA cores: SMs x 128 lanes x 2 flops x the
    measured maximum SM clock."""
    mhz = 1965.0
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mhz = float(json.load(f).get("sm_max_mhz", mhz))
    except Exception:
        pass
    return sms * 128 * 2 * mhz * 1e6 / 1e12


def run_prefill(args, rank, world, local_rank):
    """Chunked prefill: the chunk's compressor (4,096 tokens into 1,024
    entries appended to the cache), then the indexer, top-k and attention for
    its 4,096 queries, each over its causally visible entries."""
    import torch

    from compressed_sparse_attention_compressor_b200 import csa
    from compressed_sparse_attention_compressor_b200.csa import DevTensor

    torch.cuda.set_device(local_rank)
    wl = rank_workload("prefill", rank)
    inp = Wk.make_prefill_inputs(wl)
    up = DevTensor.from_stored
    m, d, cap, n0 = wl.m, wl.d, inp.cap, inp.n_cached
    nq, n_tok = inp.q_pos.shape[0], inp.C.data.shape[1]
    kv, kidx = up(inp.kv_cached), up(inp.kidx_cached)
    C, Z, q, q_idx, w_ik = up(inp.C), up(inp.Z), up(inp.q), up(inp.q_idx), up(inp.w_ik)
    swa_k, swa_v = up(inp.swa_k), up(inp.swa_v)
    w = torch.from_numpy(inp.w).cuda()
    sink = torch.from_numpy(inp.sink).cuda()
    q_pos = torch.from_numpy(inp.q_pos).cuda()
    q_req = torch.from_numpy(inp.q_req).cuda()
    n_vis_np = ((inp.q_pos + 1) // m).astype(np.int32)
    n_vis = torch.from_numpy(n_vis_np).cuda()
    p = csa.params(m, d, wl.d_idx, wl.h_q, wl.h_idx, wl.topk, wl.window, inp.swa_cap, 1.0)
    ws = csa.workspace(csa.csa_workspace_size(p, nq, cap))
    out_idx = torch.empty((nq, wl.topk), dtype=torch.int32, device="cuda")
    out = DevTensor.empty((nq, wl.h_q, d), "bf16")
    lse = torch.empty((nq, wl.h_q), dtype=torch.float32, device="cuda")
    kv_new, kidx_new = kv.offset_rows(n0), kidx.offset_rows(n0)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    evict = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def flush_l2():
        flush.zero_()
        evict.sum()
        torch.cuda._sleep(200_000)

    def step():
        csa.csa_compress(C, Z, 1, n_tok, d, m, kv_new, cap, w_ik, wl.d_idx, kidx_new, stream)
        csa.csa_index_topk(p, nq, q_idx, w, kidx, 1, cap, q_req, n_vis, out_idx, None, ws, stream)
        csa.csa_sparse_swa_attention(p, nq, q, kv, 1, cap, out_idx, n_vis, q_req, swa_k, swa_v, q_pos, None, sink,
                                     out, lse, ws, stream)

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    K = args.steps
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    with ClockSampler(local_rank) as clk:
        for i in range(K):
            flush_l2()
            e0[i].record(stream)
            step()
            e1[i].record(stream)
        torch.cuda.synchronize()
    pre_ms = [a.elapsed_time(b) for a, b in zip(e0, e1)]
    ms = max_over_ranks(sum(pre_ms), None, "cuda") / K

    csa.csa_profile_start(64 * K)
    for _ in range(K):
        flush_l2()
        step()
    torch.cuda.synchronize()
    csa.csa_profile_stop()
    per = {}
    for name, t in csa.csa_profile_records():
        c = per.setdefault(name, [0, 0.0])
        c[0] += 1
        c[1] += t
    dom = max(per, key=lambda n: per[n][1])
    dom_ms = per[dom][1] / per[dom][0]
    sum_vis = float(n_vis_np.sum())
    win = np.minimum(inp.q_pos + 1, wl.window)
    sum_keys = float(np.minimum(n_vis_np, wl.topk).sum() + win.sum())
    work, kind = prefill_kernel_work(dom, wl, sum_vis, sum_keys)
    sms = torch.cuda.get_device_properties(local_rank).multi_processor_count
    if kind == "hbm":
        peak, src = load_peaks()
        roof = {"bound": "hbm", "unit": "GB/s", "achieved": work / (dom_ms * 1e-3) / 1e9, "peak": peak,
                "peak_source": f"{src} hbm_gbs"}
    elif kind == "alu":
        roof = {"bound": "alu", "unit": "TFLOP/s", "achieved": work / (dom_ms * 1e-3) / 1e12,
                "peak": alu_peak_tflops(sms), "peak_source": f"{sms} SMs x 128 fp32 lanes x 2 x sm_max_mhz"}
    elif kind == "tensor":
        roof = {"bound": "tensor", "unit": "TFLOP/s", "achieved": work / (dom_ms * 1e-3) / 1e12,
                "peak": 1682.4, "peak_source": "measured bf16_tflops"}
        try:
            with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                roof["peak"] = float(json.load(f)["bf16_tflops"])
        except Exception:
            roof["peak_source"] = "fallback bf16"
    else:
        roof = {"bound": None, "unit": None, "achieved": None, "peak": None, "peak_source": None}
    roof.update({"kernel": dom, "frac": roof["achieved"] / roof["peak"] if roof["achieved"] else None,
                 "traffic": load_traffic(dom, "prefill"), "algorithmic_work": work, "avg_ms": dom_ms})

    def kernel_roof(name, c, t):
        """Each kernel's own work against its own roof (tensor: measured bf16
        peak; hbm: measured copy bandwidth; alu: the CUDA cores' fp32 peak)."""
        wk, kd = prefill_kernel_work(name, wl, sum_vis, sum_keys)
        if wk is None:
            return {}
        sec = t / c * 1e-3
        if kd == "hbm":
            ach, pk = wk / sec / 1e9, load_peaks()[0]
        elif kd == "tensor":
            ach, pk = wk / sec / 1e12, roof["peak"] if roof["bound"] == "tensor" else bf16_peak()
        else:
            ach, pk = wk / sec / 1e12, alu_peak_tflops(sms)
        return {"bound": kd, "achieved": ach, "peak": pk, "frac": ach / pk}
    res = {
        "metric": "prefill query-tokens/s (a 4,096-token chunk after 131,072 cached tokens)",
        "value": nq / (ms * 1e-3),
        "unit": "query-tokens/s",
        "n_gpus": 1,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "step_ms": step_stats(pre_ms),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded Gaussian cache, chunk and queries)",
        "config": {"workload": wl.name, "context": wl.context, "chunk": n_tok, "m": m, "cached_entries": n0,
                   "new_entries": n_tok // m, "topk": wl.topk, "window": wl.window, "h_q": wl.h_q, "d": d,
                   "indexer": f"{wl.h_idx}x{wl.d_idx}",
                   "l2": "flushed between timed steps (256 MB write, then 256 MB read)"},
        "roofline": roof,
        "kernels": {n: {"launches": c, "total_ms": t, "avg_ms": t / c, "share": t / sum(v[1] for v in per.values()),
                        **kernel_roof(n, c, t)}
                    for n, (c, t) in per.items()},
        "gpu_launches": sum(c for c, _ in per.values()),  # over the K steps, as timed
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        # the oracle on 256 of the chunk's queries (every 16th); the chunk's
        # compressor is timed once and charged to the sample pro rata
        from oracle import csa_oracle as O

        qs = list(range(0, nq, max(nq // 256, 1)))[:256]
        t0 = time.perf_counter()
        rows = O.compress(O.decode_stored(inp.C)[0], O.decode_stored(inp.Z)[0], m)
        O.project_index_keys(rows, O.decode_stored(inp.w_ik))
        t_c = time.perf_counter() - t0
        t0 = time.perf_counter()
        O.pipeline(inp, qs)
        t_p = time.perf_counter() - t0
        t_q = max(t_p - t_c, 1e-9) + t_c * len(qs) / nq
        res["cpu_baseline"] = {"value": len(qs) / t_q, "unit": "query-tokens/s", "cores": _threads(),
                               "kind": "oracle",
                               "sample": f"{len(qs)} of the chunk's {nq} queries ({t_p:.1f} s with the chunk's "
                                         f"compressor, {t_c:.1f} s, charged {len(qs)}/{nq} of it)"}
    return res


# ---------------------------------------------------------------------------
# the CPU oracle (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
def _threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(wl_name, budget_s=12.0, min_reqs=1):
    """Times the oracle's decode step one request at a time until the budget
    is spent; returns (requests/s, requests timed, seconds)."""
    from oracle import csa_oracle as O

    wl = Wk.WORKLOADS[wl_name]
    inp = Wk.make_decode_inputs(wl)
    n, t = 0, 0.0
    while n < min_reqs or (t < budget_s and n < wl.batch * 4):
        b = n % wl.batch
        t0 = time.perf_counter()
        O.decode_step(inp, requests=[b])
        t += time.perf_counter() - t0
        n += 1
    return n / t, n, t


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle, one request per step (a bounded
    sample of the workload), on this host's cores."""
    from oracle import csa_oracle as O

    wl = Wk.WORKLOADS[args.workload]
    inp = Wk.make_decode_inputs(wl)
    for i in range(args.warmup):
        O.decode_step(inp, requests=[i % wl.batch])
    times = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        O.decode_step(inp, requests=[i % wl.batch])
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = 1.0 / (ms * 1e-3)
    sample = f"one request ({wl.context} tokens, {(wl.context) // wl.m} entries) per step, requests cycled"
    return {
        "metric": "decode tokens/s (CSA+SWA attention step)", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded Gaussian caches and queries)",
        "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "context": wl.context, "m": wl.m,
                   "topk": wl.topk, "window": wl.window},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if args.path == "hier":
        # one GPU's study of the hierarchical indexer: every rank runs it on
        # its own inputs, rank 0 prints its own line
        res = run_hier(args, rank, world, local_rank)
    elif args.path == "prefill":
        res = run_prefill(args, rank, world, local_rank)
    else:
        res = run_ours(args, rank, world, local_rank)
    if args.path == "step" and rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, t = oracle_sample(args.workload)
        res["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
                               "sample": f"{n} single-request decode steps of {args.workload} ({t:.1f} s)"}
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
