#!/usr/bin/env python
"""Benchmark of the fused attention forward (and split-KV decode) on B200.

One JSON line on stdout (rank 0).  A "step" is one attn_fwd call over the
causal prefill workload B=2, H=16, L=4096, d=64 (bf16, seed 1): the
configuration the headline metric is quoted on.  `value` is its mask-adjusted
throughput, 4*d*(visible query/key pairs) / kernel time, in TFLOP/s, summed
over ranks (weak scaling: every rank runs its own batch; no collective is on
the data path).  The other workloads (32K GQA prefill, draft+window+doc, and
the split-KV decodes) are timed in the same run and reported under
"workloads".

Timing: inputs already resident in HBM, L2 flushed (a 512 MiB write) before
every timed launch, CUDA events on the launching stream around each launch,
max over ranks.  `e2e` is the same metric through the same C-ABI call with
host buffers: pinned host -> device copies of Q, K, V, the call, and device ->
host copies of O and LSE, all inside the timed region.

`--impl reference` times the CPU oracle (double precision, OpenMP, the host's
cores) on a bounded sample of the same workload and prints the same metric.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import (CAUSAL_4K, CAUSAL_32K_GQA, DECODE_LQ1, DECODE_LQ16,  # noqa: E402
                       DRAFT_WINDOW_DOC, DRAFT_WINDOW_DOC_FULL, CONFIGS, make_inputs)

METRIC = "attn fwd mask-adjusted TFLOP/s & % BF16 TC peak; decode KV GB/s % of HBM"
HEADLINE = CAUSAL_4K
FLUSH_BYTES = 512 << 20  # > 4x the 126 MB L2


# ----------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def _row_intervals(cfg, b, doc_ids=None, kv_lens=None):
    """Visible key interval [lo, hi] of every query row of sequence b.

    Every mask here gives each query row one contiguous key interval; the
    document mask then keeps the keys of the row's document, which is again
    an interval because documents are contiguous runs of positions.
    """
    Lq, Lk = cfg.Lq, cfg.Lk
    lkb = Lk if kv_lens is None else int(kv_lens[b])
    p = np.arange(Lq, dtype=np.int64) + (lkb - Lq)
    lo = np.zeros(Lq, dtype=np.int64)
    hi = np.full(Lq, lkb - 1, dtype=np.int64)
    if cfg.mask == "causal":
        hi = np.minimum(hi, p)
    elif cfg.mask == "draft":
        bd = cfg.draft_block
        hi = np.minimum(hi, (np.floor_divide(p, bd) + 1) * bd - 1)
    wl, wr = cfg.window
    if wl >= 0:
        lo = np.maximum(lo, p - wl)
    if wr >= 0:
        hi = np.minimum(hi, p + wr)
    if doc_ids is not None:
        d = np.asarray(doc_ids[b], dtype=np.int64)
        starts = np.concatenate([[0], np.nonzero(np.diff(d))[0] + 1])
        ends = np.concatenate([starts[1:], [Lk]]) - 1
        run = np.searchsorted(starts, p, side="right") - 1
        lo = np.maximum(lo, starts[run])
        hi = np.minimum(hi, ends[run])
    return lo, hi


def visible_pairs(cfg, doc_ids=None, kv_lens=None) -> int:
    """Visible (query, key) pairs of one head summed over the batch."""
    total = 0
    for b in range(cfg.B):
        lo, hi = _row_intervals(cfg, b, doc_ids, kv_lens)
        total += int(np.maximum(hi - lo + 1, 0).sum())
    return total


def visible_keys(cfg, doc_ids=None) -> int:
    """Keys that at least one query row sees, summed over the batch (one head)."""
    total = 0
    for b in range(cfg.B):
        lo, hi = _row_intervals(cfg, b, doc_ids)
        seen = np.zeros(cfg.Lk + 1, dtype=np.int64)
        ok = hi >= lo
        np.add.at(seen, lo[ok], 1)
        np.add.at(seen, hi[ok] + 1, -1)
        total += int((np.cumsum(seen)[: cfg.Lk] > 0).sum())
    return total


def prefill_bytes(cfg, doc_ids=None) -> float:
    """Algorithmic HBM bytes of one prefill call: Q read, the K and V rows some
    query row sees (every KV head), O written, LSE written (and the document
    ids of the batch when given)."""
    q = cfg.B * cfg.Hq * cfg.Lq * cfg.d * 2
    kv = visible_keys(cfg, doc_ids) * cfg.Hkv * cfg.d * 2 * 2
    lse = cfg.B * cfg.Hq * cfg.Lq * 4
    doc = 0 if doc_ids is None else cfg.B * cfg.Lk * 4
    return float(2 * q + kv + lse + doc)


def algorithmic_flops(cfg, pairs_per_head):
    return 4.0 * cfg.d * pairs_per_head * cfg.Hq


def decode_bytes(cfg, kv_lens):
    """K and V rows read (kv_len per sequence, every KV head) + Q + O + LSE."""
    kv = float(np.asarray(kv_lens, dtype=np.int64).sum()) * cfg.Hkv * cfg.d * 2 * 2
    q = cfg.B * cfg.Hq * cfg.Lq * cfg.d * 2
    return kv + 2 * q + cfg.B * cfg.Hq * cfg.Lq * 4


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def profiled_traffic():
    """DRAM bytes per launch of the headline kernel from the committed ncu
    summary, or None when the kernel sources changed since that capture."""
    try:
        from sm_attn_fwd_b200 import build as _build
        fields = {}
        with open(os.path.join(ROOT, "profiles", "attn_prefill_causal4k_d64.md")) as f:
            for line in f:
                if ":" in line and line.split(":", 1)[0] in ("kernel_digest",
                                                             "traffic_bytes_per_launch"):
                    k, v = line.split(":", 1)
                    fields[k] = v.strip()
        if fields.get("kernel_digest") == _build.source_digest():
            return float(fields["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        pass
    return None


# ----------------------------------------------------------- GPU timing
def device_inputs(cfg):
    """The workload's inputs drawn with the CPU generator (the same draws the
    parity tests check against the oracle), then copied to the GPU."""
    inp = make_inputs(cfg, device="cpu")
    for name in ("q", "k", "v", "doc_ids", "kv_lens"):
        t = getattr(inp, name)
        if t is not None:
            setattr(inp, name, t.to("cuda").contiguous())
    torch.cuda.synchronize()
    return inp


class Timer:
    """CUDA-event timing of single launches on one stream, L2 flushed before each."""

    def __init__(self, stream):
        self.stream = stream
        self.flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def flush(self):
        with torch.cuda.stream(self.stream):
            self.flush_buf.fill_(1)

    def time(self, fn, steps, warmup):
        for _ in range(warmup):
            self.flush()
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for s, e in evs:
            self.flush()
            s.record(self.stream)
            fn()
            e.record(self.stream)
        self.stream.synchronize()
        return [s.elapsed_time(e) for s, e in evs]  # ms


def run_prefill(cfg, timer, steps, warmup, stream, batch_mult=1):
    import sm_attn_fwd_b200 as ab
    c = cfg.with_(B=cfg.B * batch_mult) if batch_mult != 1 else cfg
    inp = device_inputs(c)
    o = torch.empty_like(inp.q)
    lse = torch.empty(c.B, c.Hq, c.Lq, dtype=torch.float32, device="cuda")
    kw = dict(scale=c.softmax_scale, mask=c.mask, window=c.window, draft_block=c.draft_block,
              doc_ids=inp.doc_ids, o=o, lse=lse, stream=stream)
    fn = lambda: ab.attn_fwd(inp.q, inp.k, inp.v, **kw)  # noqa: E731
    ms = timer.time(fn, steps, warmup)
    st, bits = ab.attn_get_device_error(stream)
    if st != ab.ATTN_OK:
        raise RuntimeError(f"device error after {c.name}: {st} {bits}")
    doc = None if inp.doc_ids is None else inp.doc_ids.cpu().numpy()
    pairs = visible_pairs(c, doc_ids=doc)
    return c, inp, ms, algorithmic_flops(c, pairs), prefill_bytes(c, doc_ids=doc)


def run_alibi(cfg, timer, steps, warmup, stream):
    """The headline workload with the ALiBi score_mod (slopes 2^(-8 (h+1) / H))."""
    import sm_attn_fwd_b200 as ab
    inp = device_inputs(cfg)
    slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / cfg.Hq) for h in range(cfg.Hq)],
                          dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    o = torch.empty_like(inp.q)
    lse = torch.empty(cfg.B, cfg.Hq, cfg.Lq, dtype=torch.float32, device="cuda")
    fn = lambda: ab.attn_fwd_score_mod(inp.q, inp.k, inp.v, alibi_slopes=slopes,  # noqa: E731
                                       scale=cfg.softmax_scale, mask=cfg.mask, o=o, lse=lse,
                                       stream=stream)
    ms = timer.time(fn, steps, warmup)
    st, bits = ab.attn_get_device_error(stream)
    if st != ab.ATTN_OK:
        raise RuntimeError(f"device error after {cfg.name} with ALiBi: {st} {bits}")
    return ms, algorithmic_flops(cfg, visible_pairs(cfg))


def run_backward(cfg, timer, steps, warmup, stream, with_forward=False):
    """attn_bwd on a prefill workload.  Work: the two score GEMMs and three
    gradient GEMMs of 2*d flop per visible pair each, 10*d*pairs in all; with
    the forward in the same step (a training step's attention), 14*d*pairs."""
    import sm_attn_fwd_b200 as ab
    inp = device_inputs(cfg)
    g = torch.Generator()
    g.manual_seed(cfg.seed + 1000)
    dout = torch.randn(inp.q.shape, generator=g).to(torch.bfloat16).cuda()
    torch.cuda.synchronize()
    o = torch.empty_like(inp.q)
    lse = torch.empty(cfg.B, cfg.Hq, cfg.Lq, dtype=torch.float32, device="cuda")
    ab.attn_fwd(inp.q, inp.k, inp.v, scale=cfg.softmax_scale, mask=cfg.mask, o=o, lse=lse,
                stream=stream)
    ws = torch.empty(ab.load_library().attn_bwd_workspace_size(cfg.B, cfg.Hq, cfg.Lq, cfg.d),
                     dtype=torch.uint8, device="cuda")
    dq, dk, dv = torch.empty_like(inp.q), torch.empty_like(inp.k), torch.empty_like(inp.v)

    def fn():
        if with_forward:
            ab.attn_fwd(inp.q, inp.k, inp.v, scale=cfg.softmax_scale, mask=cfg.mask, o=o, lse=lse,
                        stream=stream)
        ab.attn_bwd(inp.q, inp.k, inp.v, o, lse, dout, scale=cfg.softmax_scale, mask=cfg.mask,
                    workspace=ws, dq=dq, dk=dk, dv=dv, stream=stream)

    ms = timer.time(fn, steps, warmup)
    st, bits = ab.attn_get_device_error(stream)
    if st != ab.ATTN_OK:
        raise RuntimeError(f"device error after attn_bwd on {cfg.name}: {st} {bits}")
    pairs = visible_pairs(cfg) * cfg.Hq
    return ms, (14.0 if with_forward else 10.0) * cfg.d * pairs


# Packed sequences: 16 documents with lengths drawn uniformly from [128, 4096]
# (seed 5), self-attention, causal, H = 16, d = 64.
VARLEN_NAME = "varlen_causal_16seqs_l128to4096_h16_d64"


def run_varlen(timer, steps, warmup, stream, *, n=16, lo=128, hi=4096, H=16, d=64, seed=5):
    import sm_attn_fwd_b200 as ab
    from workloads import packed_case, packed_lengths
    lens = packed_lengths(seed, n, lo, hi)
    q, k, v, cu_q, cu_k = (t.cuda() for t in packed_case(seed, lens, lens, H, H, d))
    torch.cuda.synchronize()
    o = torch.empty_like(q)
    lse = torch.empty(H, q.shape[0], dtype=torch.float32, device="cuda")
    fn = lambda: ab.attn_fwd_varlen(q, k, v, cu_q, cu_k, max(lens), mask="causal", o=o,  # noqa: E731
                                    lse=lse, stream=stream)
    ms = timer.time(fn, steps, warmup)
    st, bits = ab.attn_get_device_error(stream)
    if st != ab.ATTN_OK:
        raise RuntimeError(f"device error after {VARLEN_NAME}: {st} {bits}")
    pairs = sum(L * (L + 1) // 2 for L in lens)
    return ms, 4.0 * d * pairs * H, lens


def run_decode(cfg, timer, steps, warmup, stream):
    import sm_attn_fwd_b200 as ab
    inp = make_inputs(cfg, device="cuda")
    torch.cuda.synchronize()  # inputs are drawn on the default stream; launches use `stream`
    ws = torch.empty(ab.attn_decode_workspace_size(cfg.B, cfg.Hq, cfg.Hkv, cfg.Lq, cfg.Lk, cfg.d),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty_like(inp.q)
    lse = torch.empty(cfg.B, cfg.Hq, cfg.Lq, dtype=torch.float32, device="cuda")
    fn = lambda: ab.attn_decode_splitkv(inp.q, inp.k, inp.v, inp.kv_lens, scale=cfg.softmax_scale,  # noqa: E731
                                        workspace=ws, o=o, lse=lse, stream=stream)
    ms = timer.time(fn, steps, warmup)
    st, bits = ab.attn_get_device_error(stream)
    if st != ab.ATTN_OK:
        raise RuntimeError(f"device error after {cfg.name}: {st} {bits}")
    kv = inp.kv_lens.cpu().numpy()
    nsplit, chunk = ab.attn_decode_num_splits(cfg.B, cfg.Hq, cfg.Hkv, cfg.Lq, cfg.Lk, cfg.d)
    return inp, ms, decode_bytes(cfg, kv), (nsplit, chunk)


def run_decode_alibi(cfg, timer, steps, warmup, stream):
    """The decode workload with the ALiBi score_mod (slopes 2^(-8 (h+1) / Hq)), query row
    i of sequence b at position kv_lens[b] - Lq + i."""
    import sm_attn_fwd_b200 as ab
    inp = make_inputs(cfg, device="cuda")
    slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / cfg.Hq) for h in range(cfg.Hq)],
                          dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    ws = torch.empty(ab.attn_decode_workspace_size(cfg.B, cfg.Hq, cfg.Hkv, cfg.Lq, cfg.Lk, cfg.d),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty_like(inp.q)
    lse = torch.empty(cfg.B, cfg.Hq, cfg.Lq, dtype=torch.float32, device="cuda")
    fn = lambda: ab.attn_decode_splitkv_score_mod(  # noqa: E731
        inp.q, inp.k, inp.v, inp.kv_lens, alibi_slopes=slopes, scale=cfg.softmax_scale,
        workspace=ws, o=o, lse=lse, stream=stream)
    ms = timer.time(fn, steps, warmup)
    st, bits = ab.attn_get_device_error(stream)
    if st != ab.ATTN_OK:
        raise RuntimeError(f"device error after {cfg.name} with ALiBi: {st} {bits}")
    return ms, decode_bytes(cfg, inp.kv_lens.cpu().numpy())


def run_decode_paged(cfg, page_size, timer, steps, warmup, stream):
    """The decode workload with its cache moved into a shuffled page pool
    [num_pages, Hkv, page_size, d] addressed through a block table."""
    import sm_attn_fwd_b200 as ab
    inp = make_inputs(cfg, device="cuda")
    B, Hkv, L, d = inp.k.shape
    pps = L // page_size
    g = torch.Generator(device="cuda")
    g.manual_seed(cfg.seed + 1000)
    perm = torch.randperm(B * pps, generator=g, device="cuda")
    # logical page (b, i) goes to physical page perm[b * pps + i]
    def to_pool(x):
        pages = x.view(B, Hkv, pps, page_size, d).permute(0, 2, 1, 3, 4).reshape(B * pps, Hkv,
                                                                                   page_size, d)
        pool = torch.empty_like(pages)
        pool[perm] = pages
        return pool
    kp, vp = to_pool(inp.k), to_pool(inp.v)
    table = perm.view(B, pps).to(torch.int32).contiguous()
    del inp.k, inp.v
    torch.cuda.synchronize()
    ws = torch.empty(ab.attn_decode_workspace_size(cfg.B, cfg.Hq, cfg.Hkv, cfg.Lq, cfg.Lk, cfg.d),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty_like(inp.q)
    lse = torch.empty(cfg.B, cfg.Hq, cfg.Lq, dtype=torch.float32, device="cuda")
    fn = lambda: ab.attn_decode_paged(inp.q, kp, vp, table, inp.kv_lens, scale=cfg.softmax_scale,  # noqa: E731
                                      workspace=ws, o=o, lse=lse, stream=stream)
    ms = timer.time(fn, steps, warmup)
    st, bits = ab.attn_get_device_error(stream)
    if st != ab.ATTN_OK:
        raise RuntimeError(f"device error after paged {cfg.name}: {st} {bits}")
    return ms, decode_bytes(cfg, inp.kv_lens.cpu().numpy())


def e2e_prefill(cfg, steps, warmup, stream):
    """The public host-buffer call attn_fwd_host: per step the upload of Q, K, V
    from pinned host memory, the forward and the download of O and the LSE
    (pipelined by the library over chunks of heads), timed with events on the
    call's stream."""
    import sm_attn_fwd_b200 as ab
    inp = make_inputs(cfg, device="cpu")
    qh, kh, vh = (t.pin_memory() for t in (inp.q, inp.k, inp.v))
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    lh = torch.empty(cfg.B, cfg.Hq, cfg.Lq, dtype=torch.float32).pin_memory()
    ws = torch.empty(ab.attn_fwd_host_workspace_size(cfg.B, cfg.Hq, cfg.Hkv, cfg.Lq, cfg.Lk,
                                                     cfg.d), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()

    def step():
        ab.attn_fwd_host(qh, kh, vh, scale=cfg.softmax_scale, mask=cfg.mask, o=oh, lse=lh,
                         workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for s, e in evs:
        s.record(stream)
        step()
        e.record(stream)
    stream.synchronize()
    ms = [s.elapsed_time(e) for s, e in evs]
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
    return ms, h2d, d2h


# --------------------------------------------------------- CPU baseline
def cpu_oracle_sample(cfg, target_s=10.0, inp=None):
    """Time the oracle (as it stands) on an evenly strided subset of query rows
    of every head, sized for about target_s seconds; returns TFLOP/s."""
    import oracle
    if inp is None:
        inp = make_inputs(cfg, device="cpu")
    n_rows = cfg.B * cfg.Hq * cfg.Lq
    L = cfg.Lq

    def pairs_of(rows):
        i = rows % L
        if cfg.mask == "causal":
            return int((i + 1 + (cfg.Lk - cfg.Lq)).sum())
        return int(len(rows) * cfg.Lk)

    def run(stride):
        rows = np.arange(0, n_rows, stride, dtype=np.int64)
        t0 = time.perf_counter()
        oracle.attn_fwd(inp.q, inp.k, inp.v, scale=cfg.softmax_scale, mask=cfg.mask, rows=rows)
        return rows, time.perf_counter() - t0

    stride = 512
    rows, dt = run(stride)
    while dt < 0.5 and stride > 1:
        stride //= 4
        stride = max(stride, 1)
        rows, dt = run(stride)
    # scale the sample to ~target_s
    want = max(1, int(stride * dt / target_s)) if dt > 0 else stride
    if want != stride:
        stride = want
        rows, dt = run(stride)
    flops = 4.0 * cfg.d * pairs_of(rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"{len(rows)} of {n_rows} query rows (every {stride}th row across all "
                      f"heads) of {cfg.name}; {dt:.1f} s in double precision"}


# ---------------------------------------------------------------- main
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            backend="nccl" if torch.cuda.is_available() else "gloo",
            timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def reduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def main_reference(args, world, rank):
    if rank != 0:
        return
    cfg = HEADLINE
    inp = make_inputs(cfg, device="cpu")
    vals = []
    info = None
    for i in range(args.warmup + args.steps):
        info = cpu_oracle_sample(
            cfg, target_s=max(0.5, args.ref_seconds / max(1, args.steps + args.warmup)), inp=inp)
        if i >= args.warmup:
            vals.append(info["value"])
    v = statistics.median(vals)
    info["value"] = v
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": cfg.name},
           "cpu_baseline": info,
           "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--only", default=None, help="time a single workload by name (profiling)")
    ap.add_argument("--batch-mult", type=int, default=1,
                    help="with --only: multiply the batch (larger-than-L2 profiling case)")
    ap.add_argument("--batch", type=int, default=None,
                    help="with --only: set the batch size B (smaller profiling case)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="with --only on a prefill workload: Lq = Lk = this length (profiling)")
    ap.add_argument("--head-dim", type=int, default=None,
                    help="with --only on a prefill workload: this head dimension (profiling)")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="--impl reference: total CPU seconds across all steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="also time attn_bwd on the headline workload (reported under workloads);"
                         " with --only, time attn_bwd on that workload instead of the forward")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" and args.only is None else args.warmup

    world, rank, local = dist_setup()
    if args.impl == "reference":
        main_reference(args, world, rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    import sm_attn_fwd_b200 as ab
    ab.load_library()
    torch.cuda.set_device(local)
    stream = torch.cuda.Stream()
    timer = Timer(stream)
    peaks = load_peaks()

    if args.only is not None:
        cfg = CONFIGS[args.only]
        if args.batch is not None:
            cfg = cfg.with_(B=args.batch, name=f"{cfg.name}_B{args.batch}")
        if args.seq_len is not None and not cfg.decode:
            cfg = cfg.with_(Lq=args.seq_len, Lk=args.seq_len, name=f"{cfg.name}_L{args.seq_len}")
        if args.head_dim is not None and not cfg.decode:
            cfg = cfg.with_(d=args.head_dim, name=f"{cfg.name}_d{args.head_dim}")
        if args.backward and not cfg.decode:
            ms, flops = run_backward(cfg, timer, args.steps, args.warmup, stream)
            print(json.dumps({"workload": cfg.name + "_backward", "ms": ms,
                              "TFLOP/s": flops / (statistics.median(ms) * 1e9)}))
        elif cfg.decode:
            _, ms, nbytes, plan = run_decode(cfg, timer, args.steps, args.warmup, stream)
            print(json.dumps({"workload": cfg.name, "ms": ms, "GB/s": nbytes / (statistics.median(ms) * 1e6)}))
        else:
            c, _, ms, flops, _ = run_prefill(cfg, timer, args.steps, args.warmup, stream,
                                             batch_mult=args.batch_mult)
            print(json.dumps({"workload": c.name, "ms": ms,
                              "TFLOP/s": flops / (statistics.median(ms) * 1e9)}))
        return

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        cfg, _, ms, flops, _ = run_prefill(HEADLINE, timer, args.steps, args.warmup, stream)
        workloads = {}
        if not args.no_secondary:
            for sc in (CAUSAL_32K_GQA, DRAFT_WINDOW_DOC, DRAFT_WINDOW_DOC_FULL):
                c2, _, ms2, fl2, by2 = run_prefill(sc, timer, max(10, args.steps // 10), 3, stream)
                med = statistics.median(ms2)
                tf = fl2 / (med * 1e9)
                gbs = by2 / (med * 1e6)
                workloads[c2.name] = {"ms_median": med, "ms_min": min(ms2), "TFLOP/s": tf,
                                      "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
                                      "frac_of_bf16_sustained": tf / peaks["bf16_tflops_sustained"],
                                      "algorithmic_flop": fl2, "GB/s": gbs,
                                      "frac_of_hbm": gbs / peaks["hbm_gbs"],
                                      "algorithmic_bytes": by2}
            ms6, fl6 = run_alibi(HEADLINE, timer, max(5, args.steps // 10), 3, stream)
            med = statistics.median(ms6)
            tf = fl6 / (med * 1e9)
            workloads[HEADLINE.name + "_alibi"] = {"ms_median": med, "ms_min": min(ms6),
                                                   "TFLOP/s": tf,
                                                   "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
                                                   "frac_of_bf16_sustained":
                                                       tf / peaks["bf16_tflops_sustained"],
                                                   "algorithmic_flop": fl6}
            if args.backward:
                bwd_legs = [(HEADLINE.name + "_backward", HEADLINE, False),
                            (HEADLINE.name + "_train_fwd_bwd", HEADLINE, True),
                            (HEADLINE.name.replace("d64", "d128") + "_backward",
                             HEADLINE.with_(d=128, name=HEADLINE.name.replace("d64", "d128")),
                             False)]
                for leg, bcfg, with_fwd in bwd_legs:
                    ms7, fl7 = run_backward(bcfg, timer, max(5, args.steps // 10), 3, stream,
                                            with_forward=with_fwd)
                    med = statistics.median(ms7)
                    tf = fl7 / (med * 1e9)
                    workloads[leg] = {
                        "ms_median": med, "ms_min": min(ms7), "TFLOP/s": tf,
                        "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
                        "frac_of_bf16_sustained": tf / peaks["bf16_tflops_sustained"],
                        "algorithmic_flop": fl7}
            ms5, fl5, lens5 = run_varlen(timer, max(5, args.steps // 10), 3, stream)
            med = statistics.median(ms5)
            tf = fl5 / (med * 1e9)
            workloads[VARLEN_NAME] = {"ms_median": med, "ms_min": min(ms5), "TFLOP/s": tf,
                                      "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
                                      "frac_of_bf16_sustained": tf / peaks["bf16_tflops_sustained"],
                                      "algorithmic_flop": fl5, "tokens": sum(lens5)}
            for dc in (DECODE_LQ1, DECODE_LQ16):
                _, ms3, nb, plan = run_decode(dc, timer, max(5, args.steps // 10), 3, stream)
                med = statistics.median(ms3)
                gbs = nb / (med * 1e6)
                workloads[dc.name] = {"ms_median": med, "ms_min": min(ms3), "GB/s": gbs,
                                      "frac_of_hbm": gbs / peaks["hbm_gbs"],
                                      "frac_of_8TBs_nominal": gbs / 8000.0,
                                      "algorithmic_bytes": nb, "splits": plan[0],
                                      "chunk_keys": plan[1]}
            ms8, nb8 = run_decode_alibi(DECODE_LQ1, timer, max(5, args.steps // 10), 3, stream)
            med = statistics.median(ms8)
            gbs = nb8 / (med * 1e6)
            workloads[DECODE_LQ1.name + "_alibi"] = {
                "ms_median": med, "ms_min": min(ms8), "GB/s": gbs,
                "frac_of_hbm": gbs / peaks["hbm_gbs"], "algorithmic_bytes": nb8}
            for psz in (128, 16):
                ms4, nb4 = run_decode_paged(DECODE_LQ1, psz, timer, max(5, args.steps // 10), 3,
                                            stream)
                med = statistics.median(ms4)
                gbs = nb4 / (med * 1e6)
                workloads[f"{DECODE_LQ1.name}_paged{psz}"] = {
                    "ms_median": med, "ms_min": min(ms4), "GB/s": gbs,
                    "frac_of_hbm": gbs / peaks["hbm_gbs"], "algorithmic_bytes": nb4,
                    "page_size": psz}
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.summary()

    total_ms = sum(ms)
    total_ms_max = reduce_max(total_ms, world)
    ms_per_step = total_ms_max / len(ms)
    value = flops * world / (ms_per_step * 1e9)        # TFLOP/s, all ranks
    per_launch_tflops = flops / (statistics.mean(ms) * 1e9)

    e2e_ms, h2d, d2h = e2e_prefill(HEADLINE, max(10, args.steps // 10), 3, stream)
    e2e_ms_max = reduce_max(sum(e2e_ms) / len(e2e_ms), world)
    e2e_val = flops * world / (e2e_ms_max * 1e9)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(HEADLINE, target_s=10.0)

    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": HEADLINE.name, "B": HEADLINE.B, "H": HEADLINE.Hq,
                       "L": HEADLINE.Lq, "d": HEADLINE.d, "mask": "causal",
                       "parallelism": f"replicas x{world}" if world > 1 else "single gpu",
                       "l2": "flushed (512 MiB write) before every timed launch"},
            "roofline": {"bound": "tensor", "achieved": per_launch_tflops,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": per_launch_tflops / peaks["bf16_tflops"],
                         "frac_sustained": per_launch_tflops / peaks["bf16_tflops_sustained"],
                         "traffic": profiled_traffic(), "kernel": "attn_prefill_kernel<64>",
                         "algorithmic_flop_per_launch": flops,
                         "peak_source": f"{peaks['source']} bf16_tflops (burst)"},
            "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms_max,
                    "call": "attn_fwd_host (pinned host buffers in and out)"},
            "gpu_launches": len(ms),
            "clocks": clk,
            "cpu_baseline": cpu,
            "workloads": workloads,
            "peaks": peaks,
        }
        print(json.dumps(out))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
