"""Benchmark of the PIVOT indexer on B200 (libpivot, through its C ABI).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--seed S]

One step is one pass of the whole hot path over one synthetic sequence:
the dense indexer (every query scans its full causal prefix, keeps top-k),
then PIVOT -- proxy reduce, one proxy scan per group (top-C candidates),
PIVOT-Reuse and PIVOT-Refine -- so each step produces the dense, Reuse and
Refine index sets of all L queries.  ``value`` = L / step time (queries/s,
whole job).  With N > 1 ranks the one sequence's query rows are split
across the ranks by zig-zag group blocks (every rank holds all keys and
indexes its own rows; no exchange), so the total work is fixed (strong
scaling).  Per-mode times, Reuse/Refine recall against dense and the
neighbour overlap of dense are reported beside it, and (rank 0, N = 1) the
other prefill workloads -- dsa_prefill_16k and the dsa_prefill_64k sweep
over g in {8, 16} and C in {4096, 8192} -- each timed on its own.

Timing: W untimed warm-up steps, then K steps between CUDA events on the
launching stream, bracketed by a barrier and a device synchronize; the max
over ranks is reported.  The inputs (q alone is 1 GiB at L=128K) and the
score buffers are far larger than L2, so no flush is needed.

``--impl reference`` times the CPU oracle (``oracle/``, plain C, fp64) on a
bounded sample of the same workload and extrapolates to the full step; it
is the reference arm (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from top_token_selection_b200 import inputs as gen  # noqa: E402

METRIC = "indexer queries/s at L=128K (dense vs PIVOT-Reuse/Refine), % roofline; recall"
DEFAULT_WORKLOAD = "long_prefill_128k_fp8"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0   # nominal dense ratio (4.5 / 2.25 PFLOP/s)

# DRAM bytes per causal pair of the dense scan kernel, from one ncu capture
# of the fp8_prefill_16k dense scan (dram__bytes_read.sum +
# dram__bytes_write.sum over its causal pairs; the summary is under
# profiles/).  Valid only for the kernel sources and launch code it was
# taken on (api.cu sets the work items, whose query-block loads are part of
# the traffic): the bench reports it while these files hash (sha1, first 12
# hex digits) as listed, and null otherwise.
SCAN_TRAFFIC = {"bytes_per_pair": 5.121,
                "sources": {"scan_umma.cu": "3e8b3e987d59", "common.cuh": "e15e822467cd",
                            "segments.h": "fbc71176c053", "kernels.h": "cd53f91c3deb",
                            "api.cu": "2223bc936ec0"}}


# ---------------------------------------------------------------------------
# distributed plumbing (host logic, testable on CPU with gloo)
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def rank_rows(L: int, g: int, world: int, rank: int):
    """This rank's query row ranges of the one sequence: the whole sequence on
    one GPU, else its zig-zag group blocks (balanced causal work)."""
    from top_token_selection_b200.sharding import zigzag_ranges
    return [(0, L)] if world == 1 else zigzag_ranges(L, g, world, rank)


def max_over_ranks(x: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(total_queries: int, ms_max: float, steps: int) -> float:
    """Whole-job queries/s: the sequence's queries per step over the slowest
    rank's time (every rank holds a share of the same rows)."""
    return total_queries * steps / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v for v in vis.split(",") if v.strip()]
        self.dev = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.dev, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def make_inputs(wl, seed):
    return gen.make_prefill(wl["L"], wl["H"], wl["D"], wl["dtype"], kind=wl["kind"], seed=seed)


class Runner:
    """Device buffers and one step of the hot path through the C ABI over
    this rank's query row ranges (the whole sequence on one GPU)."""

    def __init__(self, p, wl, device, ranges=None):
        from top_token_selection_b200 import pivot as pv
        self.pv = pv
        pv.load()
        self.wl = wl
        self.L, self.H, self.D = p.L, p.H, p.D
        self.g, self.C, self.k = wl["g"], wl["C"], wl["topk"]
        self.G = -(-self.L // self.g)
        self.ranges = list(ranges) if ranges else [(0, self.L)]
        self.rows = sum(b - a for a, b in self.ranges)
        d = device
        self.host = {"q": p.q, "q_scale": p.q_scale, "w": p.w, "k": p.k, "k_scale": p.k_scale}
        self.dev = {n: (None if t is None else torch.empty_like(t, device=d))
                    for n, t in self.host.items()}
        for n, t in self.host.items():
            if t is not None:
                self.dev[n].copy_(t)
        self.seq = pv.make_seq(self.dev["q"], self.dev["q_scale"], self.dev["w"], self.dev["k"],
                               self.dev["k_scale"])
        store = {gen.F32: torch.float32, gen.BF16: torch.bfloat16,
                 gen.E4M3: torch.float8_e4m3fn}[wl["dtype"]]
        self.dense = torch.empty(self.L, self.k, dtype=torch.int32, device=d)
        self.reu = torch.empty(self.L, self.k, dtype=torch.int32, device=d)
        self.ref = torch.empty(self.L, self.k, dtype=torch.int32, device=d)
        self.cand = torch.empty(self.G, self.C, dtype=torch.int32, device=d)
        self.pq = torch.empty(self.G, self.H, self.D, dtype=store, device=d)
        self.pqs = (torch.empty(self.G, dtype=torch.float32, device=d)
                    if wl["dtype"] == gen.E4M3 else None)
        self.pw = torch.empty(self.G, self.H, dtype=torch.float32, device=d)
        wsb = 0
        for a, b in self.ranges:
            sq = self.range_seq(self.seq, a, b)
            wsb = max(wsb, pv.pivot_dense_index_workspace_size(sq, self.k),
                      pv.pivot_proxy_scan_workspace_size(sq, self.g, self.C),
                      pv.pivot_refine_workspace_size(sq, self.g, self.C, self.k))
        self.ws = torch.empty(wsb, dtype=torch.uint8, device=d)
        self.stream = torch.cuda.current_stream()

    def range_seq(self, seq, a, b):
        sq = self.pv.PivotSeq.from_buffer_copy(seq)
        sq.t_begin, sq.t_end = a, b
        return sq

    def _ptr(self, t):
        return None if t is None else t.data_ptr()

    def step(self, events=None, seq=None, outs=None):
        """One step on `seq` (default: this runner's sequence) into `outs` =
        (dense, reuse, refine) index buffers (default: this runner's), for
        every row range of this rank."""
        pv, s = self.pv, self.stream
        sp = pv._stream(s)
        ws, wsn = self.ws.data_ptr(), self.ws.numel()
        seq = self.seq if seq is None else seq
        dense, reu, ref = (self.dense, self.reu, self.ref) if outs is None else outs
        seqs = [(a, b, self.range_seq(seq, a, b)) for a, b in self.ranges]
        g, k, C = self.g, self.k, self.C

        def mark(i):
            if events is not None:
                events[i].record(s)

        def grp(a):   # this range's first group row in pq / pw / cand
            return a // g
        mark(0)
        for a, b, sq in seqs:
            pv._check(pv.pivot_dense_index(sq, k, dense[a].data_ptr(), None, ws, wsn, sp),
                      "dense")
        mark(1)
        for a, b, sq in seqs:
            pv._check(pv.pivot_proxy_reduce(sq, g, self.pq[grp(a)].data_ptr(),
                                            None if self.pqs is None else
                                            self.pqs[grp(a):].data_ptr(),
                                            self.pw[grp(a)].data_ptr(), sp), "reduce")
        mark(2)
        for a, b, sq in seqs:
            pv._check(pv.pivot_proxy_scan(sq, g, self.pq[grp(a)].data_ptr(),
                                          None if self.pqs is None else
                                          self.pqs[grp(a):].data_ptr(),
                                          self.pw[grp(a)].data_ptr(), C, k,
                                          self.cand[grp(a)].data_ptr(), None, ws, wsn, sp),
                      "scan")
        mark(3)
        for a, b, sq in seqs:
            pv._check(pv.pivot_reuse(a, b, g, self.cand[grp(a)].data_ptr(), C, k,
                                     reu[a].data_ptr(), sp), "reuse")
        mark(4)
        for a, b, sq in seqs:
            pv._check(pv.pivot_refine(sq, g, self.cand[grp(a)].data_ptr(), C, k,
                                      ref[a].data_ptr(), None, ws, wsn, sp), "refine")
        mark(5)

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.host.values() if t is not None)

    def d2h_bytes(self):
        return 3 * self.rows * self.k * 4


def recall_stats(dense, other, rows_per_chunk=4096):
    """Mean over rows of |other ∩ dense| / |dense| (both -1 padded)."""
    tot, n = 0.0, 0
    for r0 in range(0, dense.shape[0], rows_per_chunk):
        a = dense[r0:r0 + rows_per_chunk].long()
        b = other[r0:r0 + rows_per_chunk].long()
        big = torch.iinfo(torch.int64).max
        a_s, _ = torch.sort(torch.where(a >= 0, a, big), dim=1)
        pos = torch.searchsorted(a_s, b.contiguous())
        hit = (pos < a.shape[1]) & (torch.gather(a_s, 1, pos.clamp(max=a.shape[1] - 1)) == b)
        hit &= b >= 0
        cnt = (a >= 0).sum(1).clamp(min=1)
        tot += (hit.sum(1).double() / cnt.double()).sum().item()
        n += a.shape[0]
    return tot / max(n, 1)


def neighbour_overlap(dense, rows_per_chunk=4096):
    k = dense.shape[1]
    tot, n = 0.0, 0
    for r0 in range(0, dense.shape[0] - 1, rows_per_chunk):
        r1 = min(dense.shape[0] - 1, r0 + rows_per_chunk)
        a = dense[r0:r1]
        b = dense[r0 + 1:r1 + 1]
        full = (a >= 0).all(1) & (b >= 0).all(1)
        if full.any():
            tot += recall_stats(a[full], b[full]) * int(full.sum())
            n += int(full.sum())
    return tot / max(n, 1) if k else 0.0


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

def oracle_sample_time(p, wl, sample_rows=None, seed=0):
    """Time the oracle on a stratified sample of the step and extrapolate.

    Dense rows, proxy-scan groups and Refine rows are sampled evenly over
    positions; each part's time is scaled by (work of all rows) / (work of
    the sampled rows), work being the causal pairs the oracle scores.  The
    proxy reduce and Reuse run on sampled groups/rows and scale by count.
    Returns (seconds for one full step, description, threads)."""
    import oracle
    L, H, D, g, C, k = p.L, p.H, p.D, wl["g"], wl["C"], wl["topk"]
    G = -(-L // g)
    q, qs, w, kk, ks = p.codes()
    nd, ns, nr = sample_rows or (48, 24, 192)
    rng = np.random.default_rng(seed)
    dense_rows = np.unique(np.linspace(0, L - 1, nd).astype(np.int64) +
                           rng.integers(0, max(1, L // nd), nd)).clip(0, L - 1).astype(np.int32)
    groups = np.unique(np.linspace(0, G - 1, ns).astype(np.int64)).astype(np.int32)
    ref_rows = np.unique(np.linspace(0, L - 1, nr).astype(np.int64)).astype(np.int32)
    threads = oracle.max_threads()

    t0 = time.perf_counter()
    oracle.dense_index(p.dtype, q, qs, w, kk, ks, k, rows=dense_rows)
    t_dense = time.perf_counter() - t0
    all_pairs = L * (L + 1) / 2
    dense_full = t_dense * all_pairs / float(np.sum(dense_rows.astype(np.float64) + 1))

    t0 = time.perf_counter()
    pq, pqs, pw = oracle.proxy_reduce(p.dtype, q, qs, w, g, groups=groups)
    t_red = time.perf_counter() - t0
    red_full = t_red * G / len(groups)

    # proxy scan on the sampled groups: the oracle scan indexes pq by group id,
    # so place the sampled proxies in a full-size table
    store = pq.dtype
    pq_full = np.zeros((G, H, D), dtype=store)
    pw_full = np.zeros((G, H), dtype=np.float32)
    pqs_full = np.ones(G, dtype=np.float32) if pqs is not None else None
    pq_full[groups], pw_full[groups] = pq, pw
    if pqs is not None:
        pqs_full[groups] = pqs
    t0 = time.perf_counter()
    cand, _ = oracle.proxy_scan(p.dtype, pq_full, pqs_full, pw_full, kk, ks, L, g, C, k,
                                groups=groups)
    t_scan = time.perf_counter() - t0
    e = np.minimum(L, (groups.astype(np.float64) + 1) * g)
    scan_all = sum(min(L, (j + 1) * g) for j in range(G))
    scan_full = t_scan * scan_all / float(np.sum(e))

    # Refine and Reuse for the sampled rows, against candidates of their groups
    cand_full = np.full((G, C), -1, dtype=np.int32)
    cand_full[groups] = cand
    need = np.unique(ref_rows // g)
    missing = np.setdiff1d(need, groups).astype(np.int32)
    if len(missing):
        pq2, pqs2, pw2 = oracle.proxy_reduce(p.dtype, q, qs, w, g, groups=missing)
        pq_full[missing], pw_full[missing] = pq2, pw2
        if pqs2 is not None:
            pqs_full[missing] = pqs2
        c2, _ = oracle.proxy_scan(p.dtype, pq_full, pqs_full, pw_full, kk, ks, L, g, C, k,
                                  groups=missing)
        cand_full[missing] = c2
    t0 = time.perf_counter()
    oracle.refine(p.dtype, q, qs, w, kk, ks, g, cand_full, k, rows=ref_rows)
    t_ref = time.perf_counter() - t0
    m = min(C, L)
    ref_all = m * (m + 1) / 2 + (L - m) * C          # sum over t of min(C, t + 1)
    ref_full = t_ref * ref_all / float(np.sum(np.minimum(C, ref_rows.astype(np.float64) + 1)))
    t0 = time.perf_counter()
    oracle.reuse(L, g, cand_full, k, rows=ref_rows)
    t_reu = time.perf_counter() - t0
    reu_full = t_reu * L / len(ref_rows)

    total = dense_full + red_full + scan_full + ref_full + reu_full
    desc = (f"{len(dense_rows)} dense rows, {len(groups)} proxy-scan groups, {len(ref_rows)} "
            f"Refine/Reuse rows, {len(groups)} proxy groups, sampled evenly over positions; "
            f"each part scaled to the full step by causal pairs (dense, scan, Refine) or by "
            f"count (reduce, Reuse); sample CPU time {t_dense + t_red + t_scan + t_ref + t_reu:.1f}s")
    parts = {"dense_s": dense_full, "reduce_s": red_full, "scan_s": scan_full,
             "refine_s": ref_full, "reuse_s": reu_full}
    return total, desc, threads, parts


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_reference(args, wl):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    p = make_inputs(wl, args.seed)
    times = []
    desc, threads = "", 0
    for i in range(args.warmup + args.steps):
        total, desc, threads, _ = oracle_sample_time(p, wl, seed=i)
        if i >= args.warmup:
            times.append(total)
    t = float(np.mean(times))
    value = p.L / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": gen.DTYPE_NAMES[wl["dtype"]], "data": "synthetic",
            "config": config_of(wl, args),
            "cpu_baseline": {"value": value, "unit": "queries/s", "cores": threads,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl, args):
    return {"workload": args.workload, "L": wl["L"], "H": wl["H"], "D": wl["D"],
            "g": wl["g"], "C": wl["C"], "topk": wl["topk"],
            "q_k_format": gen.DTYPE_NAMES[wl["dtype"]] + (" + fp32 per-token scale"
                                                         if wl["dtype"] == gen.E4M3 else ""),
            "step": "dense index + proxy reduce + proxy scan + Reuse + Refine, all L queries",
            "parallelism": (f"zigzag{dist_env()[2]}: one sequence's query rows in 2N group "
                            "blocks, rank r takes blocks r and 2N-1-r; keys replicated"
                            if dist_env()[2] > 1 else "1 GPU, whole sequence"),
            "l2": "no flush: inputs and score buffers larger than L2 (q alone 1 GiB)",
            "selection": getattr(args, "selection", "library")}


def scan_traffic_per_pair():
    """DRAM bytes per causal pair of the scan kernel (SCAN_TRAFFIC), or None
    once the kernel sources differ from the ones it was measured on."""
    import hashlib
    bpp = SCAN_TRAFFIC.get("bytes_per_pair")
    if bpp is None or not SCAN_TRAFFIC.get("sources"):
        return None
    for name, digest in SCAN_TRAFFIC["sources"].items():
        src = os.path.join(ROOT, "top_token_selection_b200", "csrc", name)
        try:
            data = open(src, "rb").read()
        except OSError:
            return None
        if hashlib.sha1(data).hexdigest()[:len(digest)] != digest:
            return None
    return float(bpp)


def measure_fp8_peak(device, n=8192, sustain_s=3.0):
    """Dense FP8 (e4m3 x e4m3, fp32 accumulate, bf16 out) tensor throughput
    of the library GEMM, torch._scaled_mm at n^3: best of 10 (burst) and
    back to back for `sustain_s` seconds (sustained, the figure for kernels
    timed inside a long step).  TFLOP/s."""
    g = torch.Generator(device=device).manual_seed(0)
    a = (torch.randn(n, n, device=device, generator=g) * 0.5).to(torch.float8_e4m3fn)
    b = (torch.randn(n, n, device=device, generator=g) * 0.5).to(torch.float8_e4m3fn).t()
    one = torch.tensor(1.0, device=device)

    def mm():
        return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    for _ in range(3):
        mm()
    torch.cuda.synchronize()
    flop = 2.0 * n ** 3
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    iters = max(10, int(sustain_s / (best * 1e-3)))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        mm()
    e1.record()
    torch.cuda.synchronize()
    return {"burst": flop / (best * 1e-3) / 1e12,
            "sustained": flop * iters / (e0.elapsed_time(e1) * 1e-3) / 1e12,
            "how": f"torch._scaled_mm e4m3 {n}^3 (2 n^3 flop): best of 10, and {iters} back to "
                   f"back (~{sustain_s:.0f} s), CUDA events"}


def _event_ms(fn, stream, reps):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fn()
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def measure_extra(run, wl, device, peaks, seed, reps=3):
    """Steps outside the headline step, each timed on its own (CUDA events,
    warm): the MTP decode step on its workload in the three modes, Reuse with
    backfill and the window union on this prefill, and this prefill's tokens
    as ragged batches of 2048- and 256-token sequences (one call, and Refine
    sequence by sequence).  Not part of `value`."""
    pv, s = run.pv, run.stream
    sp = pv._stream(s)
    hbm = peaks["hbm_gbs"]
    out = {}
    # Reuse with backfill needs the proxy scores of the candidates
    cs = torch.empty(run.G, run.C, dtype=torch.float32, device=device)
    pv._check(pv.pivot_proxy_scan(run.seq, run.g, run.pq.data_ptr(), run._ptr(run.pqs),
                                  run.pw.data_ptr(), run.C, run.k, run.cand.data_ptr(),
                                  cs.data_ptr(), run.ws.data_ptr(), run.ws.numel(), sp), "scan")
    bf = torch.empty(run.L, run.k, dtype=torch.int32, device=device)
    ms = _event_ms(lambda: pv._check(pv.pivot_reuse_backfill(
        0, run.L, run.g, run.cand.data_ptr(), cs.data_ptr(), run.C, run.k, bf.data_ptr(), sp),
        "backfill"), s, reps)
    nbytes = run.G * run.C * 8 + run.L * run.k * 4     # candidates + scores read, rows written
    out["reuse_backfill"] = {"ms": ms, "queries_per_s": run.L / (ms / 1e3),
                             "gbs": nbytes / (ms / 1e3) / 1e9,
                             "frac_hbm": nbytes / (ms / 1e3) / 1e9 / hbm,
                             "bytes": nbytes}
    window = 128
    un = torch.empty(run.L, run.k + window, dtype=torch.int32, device=device)
    ms = _event_ms(lambda: pv._check(pv.pivot_window_union(
        run.dense.data_ptr(), run.L, run.k, 0, None, window, un.data_ptr(), sp), "union"), s, reps)
    nbytes = run.L * (2 * run.k + window) * 4
    out["window_union"] = {"window": window, "ms": ms, "gbs": nbytes / (ms / 1e3) / 1e9,
                           "frac_hbm": nbytes / (ms / 1e3) / 1e9 / hbm, "bytes": nbytes}
    # ragged batches: the prefill's tokens cut into equal sequences (each with
    # its own keys), every step as one launch over all of them, against the
    # same sequences through the single-sequence calls one after another
    def ragged(seg, C, topk):
        nseq = run.L // seg
        T = nseq * seg
        cu = [i * seg for i in range(nseq + 1)]
        dv = run.dev
        cut = lambda t: None if t is None else t[:T]
        batch = pv.make_varlen(cu, cut(dv["q"]), cut(dv["q_scale"]), cut(dv["w"]), cut(dv["k"]),
                               cut(dv["k_scale"]))
        rag = {"sequences": nseq, "tokens_each": seg, "g": run.g, "C": C, "topk": topk}
        idx = torch.empty(T, topk, dtype=torch.int32, device=device)
        for name, mode in (("dense", pv.DENSE), ("reuse", pv.REUSE), ("refine", pv.REFINE)):
            wsv = torch.empty(pv.pivot_index_varlen_workspace_size(batch, mode, run.g, C, topk),
                              dtype=torch.uint8, device=device)
            ms = _event_ms(lambda: pv._check(pv.pivot_index_varlen(
                batch, mode, run.g, C, topk, idx.data_ptr(), wsv.data_ptr(), wsv.numel(), sp),
                "varlen"), s, reps)
            rag[name] = {"ms": ms, "queries_per_s": T / (ms / 1e3)}
        seqs = [pv.make_seq(*(None if t is None else t[a:a + seg] for t in
                              (dv["q"], dv["q_scale"], dv["w"], dv["k"], dv["k_scale"])))
                for a in cu[:-1]]
        assert -(-seg // run.g) <= run.G and C <= run.C

        def per_sequence():   # Refine, sequence by sequence
            for i, sq in enumerate(seqs):
                pv._check(pv.pivot_proxy_reduce(sq, run.g, run.pq.data_ptr(), run._ptr(run.pqs),
                                                run.pw.data_ptr(), sp), "reduce")
                pv._check(pv.pivot_proxy_scan(sq, run.g, run.pq.data_ptr(), run._ptr(run.pqs),
                                              run.pw.data_ptr(), C, topk, run.cand.data_ptr(),
                                              None, run.ws.data_ptr(), run.ws.numel(), sp), "scan")
                pv._check(pv.pivot_refine(sq, run.g, run.cand.data_ptr(), C, topk,
                                          idx[i * seg:].data_ptr(), None, run.ws.data_ptr(),
                                          run.ws.numel(), sp), "refine")
        ms = _event_ms(per_sequence, s, reps)
        rag["refine_sequence_by_sequence"] = {"ms": ms, "queries_per_s": T / (ms / 1e3)}
        rag["refine"]["speedup_vs_sequence_by_sequence"] = ms / rag["refine"]["ms"]
        return rag

    if run.L >= 2 * 2048:
        out["ragged_batch"] = ragged(2048, run.C, run.k)
    if run.L >= 2 * 256 and run.C >= 256 and run.k >= 64:
        out["ragged_batch_short"] = ragged(256, 256, 64)
    # the MTP decode step (its own workload)
    dw = gen.WORKLOADS["mtp_decode_b32"]
    d = gen.make_decode(B=dw["B"], Gm=dw["Gm"], H=dw["H"], D=dw["D"], dtype=dw["dtype"],
                        len_lo=dw["len_lo"], len_hi=dw["len_hi"], seed=seed + 17)
    dev = [None if t is None else t.to(device) for t in
           (d.q, d.q_scale, d.w, d.kc, d.kc_scale, d.cache_len)]
    batch = pv.make_decode(*dev)
    rows = dw["B"] * dw["Gm"]
    keys = int(d.cache_len.sum())
    dec = {"workload": "mtp_decode_b32", "B": dw["B"], "Gm": dw["Gm"], "C": dw["C"],
           "topk": dw["topk"], "cached_keys": keys}
    for name, mode in (("dense", pv.DENSE), ("reuse", pv.REUSE), ("refine", pv.REFINE)):
        wsd = torch.empty(max(1, pv.pivot_decode_workspace_size(batch, mode, dw["C"], dw["topk"])),
                          dtype=torch.uint8, device=device)
        idx = torch.empty(dw["B"], dw["Gm"], dw["topk"], dtype=torch.int32, device=device)
        ms = _event_ms(lambda: pv._check(pv.pivot_decode(
            batch, mode, dw["C"], dw["topk"], idx.data_ptr(), None, wsd.data_ptr(), wsd.numel(),
            sp), "decode"), s, reps)
        dec[name] = {"ms": ms, "tokens_per_s": rows / (ms / 1e3)}
    dec["reuse"]["speedup_vs_dense"] = dec["dense"]["ms"] / dec["reuse"]["ms"]
    dec["refine"]["speedup_vs_dense"] = dec["dense"]["ms"] / dec["refine"]["ms"]
    out["decode"] = dec
    assert pv.device_error() == 0, "a kernel reported an error in the extra measurements"
    return out


def measure_layers(device, seed, nlayers=4, L=16384, rho=0.9, period=2, reps=3):
    """Cross-layer reuse of index rows (not in `value`): `nlayers` correlated
    layers of the 16K FP8 prefill; every layer runs the dense indexer
    (period 1) against every `period`-th layer running it and the others
    reusing its rows; the recall of each layer's rows against its own dense
    rows."""
    from top_token_selection_b200 import pivot as pv
    lay = gen.make_layers(nlayers, L, 64, 128, gen.E4M3, rho=rho, seed=seed + 29)
    seqs = []
    for p in lay:
        dev = [None if t is None else t.to(device) for t in (p.q, p.q_scale, p.w, p.k, p.k_scale)]
        seqs.append(pv.make_seq(*dev))
    own = pv.index_layers(seqs, pv.DENSE, 8, 4096, 2048, period=1)
    out = {"layers": nlayers, "L": L, "rho": rho, "period": period, "mode": "dense"}
    for per in (1, period):
        ms = _event_ms(lambda: pv.index_layers(seqs, pv.DENSE, 8, 4096, 2048, period=per),
                       torch.cuda.current_stream(), reps)
        out[f"period{per}_ms"] = ms
    got = pv.index_layers(seqs, pv.DENSE, 8, 4096, 2048, period=period)
    out["recall_per_layer"] = [recall_stats(o, r) for o, r in zip(own, got)]
    out["speedup"] = out["period1_ms"] / out[f"period{period}_ms"]
    assert pv.device_error() == 0
    return out


def time_modes(run, steps=3):
    """Per-stage CUDA-event times of `steps` warm steps of `run`: dense,
    Reuse (reduce + scan + Reuse) and Refine (reduce + scan + Refine)."""
    run.step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    for e in ev:
        run.step(e)
    torch.cuda.synchronize()
    st = np.zeros(5)
    for e in ev:
        for j in range(5):
            st[j] += e[j].elapsed_time(e[j + 1])
    dense, red, scan, reu, ref = st / steps
    L = run.rows
    out = {"dense": {"ms": dense, "queries_per_s": L / (dense / 1e3)},
           "reuse": {"ms": red + scan + reu, "queries_per_s": L / ((red + scan + reu) / 1e3),
                     "speedup_vs_dense": dense / (red + scan + reu)},
           "refine": {"ms": red + scan + ref, "queries_per_s": L / ((red + scan + ref) / 1e3),
                      "speedup_vs_dense": dense / (red + scan + ref)},
           "stages_ms": {"dense": dense, "proxy_reduce": red, "proxy_scan": scan,
                         "reuse": reu, "refine": ref}}
    return out


def measure_workloads(args, device, peaks, fp8_peak):
    """The other prefill workloads, each timed on its own (not in `value`):
    dsa_prefill_16k (bf16, g = 8, C = 4096) and dsa_prefill_64k (bf16) at
    g in {8, 16} x C in {4096, 8192}; per mode queries/s and speedup over
    dense, the scan's tensor throughput, and Reuse / Refine recall."""
    from top_token_selection_b200 import pivot as pv
    out = {}
    points = [("dsa_prefill_16k", 8, 4096)] + [("dsa_prefill_64k", g, C)
                                              for g in (8, 16) for C in (4096, 8192)]
    made = {}
    for name, g, C in points:
        wl = dict(gen.WORKLOADS[name], g=g, C=C)
        if name not in made:
            made.clear()
            made[name] = make_inputs(wl, args.seed)
        run = Runner(made[name], wl, device)
        pv.pivot_profile_enable(1)
        res = time_modes(run)
        pv.pivot_profile_enable(0)
        n, kms, work = pv.profile_read(0)     # scan: dense + proxy rows of the timed steps
        res["scan_tflops"] = work * 2.0 * run.H * run.D / (kms / 1e3) / 1e12 if kms else None
        res["recall"] = {"reuse_vs_dense": recall_stats(run.dense, run.reu),
                         "refine_vs_dense": recall_stats(run.dense, run.ref),
                         "dense_neighbour_overlap": neighbour_overlap(run.dense)}
        res.update({"L": wl["L"], "dtype": gen.DTYPE_NAMES[wl["dtype"]], "g": g, "C": C,
                    "topk": wl["topk"]})
        out[f"{name}_g{g}_C{C}"] = res
        del run
        torch.cuda.empty_cache()
    assert pv.device_error() == 0, "a kernel reported an error in the workload sweep"
    return out


def run_ours(args, wl):
    import torch.distributed as dist
    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1 and not dist.is_initialized():
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    # one sequence for the whole job: every rank builds the same inputs (the
    # keys are needed whole) and indexes its own zig-zag row ranges
    p = make_inputs(wl, args.seed)
    run = Runner(p, wl, device, rank_rows(wl["L"], wl["g"], world, rank))
    pv = run.pv
    if args.selection != "library":
        pv._check(pv.pivot_set_fused_selection(1 if args.selection == "fused" else 0, 4.5),
                  "selection mode")
    fp8 = wl["dtype"] == gen.E4M3
    fp8_peak = measure_fp8_peak(device) if fp8 else None

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        run.step()
    barrier()
    assert pv.device_error() == 0, "a kernel reported an error during warm-up"

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    pv.pivot_profile_enable(1)
    n0 = pv.pivot_launch_count()
    barrier()
    start.record(run.stream)
    for i in range(args.steps):
        run.step(ev[i])
    stop.record(run.stream)
    barrier()
    n1 = pv.pivot_launch_count()
    pv.pivot_profile_enable(0)
    clk = clocks.stop()
    ms = start.elapsed_time(stop)
    ms_max = max_over_ranks(ms, device)
    assert pv.device_error() == 0, "a kernel reported an error in the timed region"

    stage = np.zeros(5)
    for e in ev:
        for j in range(5):
            stage[j] += e[j].elapsed_time(e[j + 1])
    stage /= args.steps
    dense_ms, red_ms, scan_ms, reu_ms, ref_ms = stage
    L = run.L
    modes = {
        "dense": {"ms": dense_ms, "queries_per_s": L / (dense_ms / 1e3)},
        "reuse": {"ms": red_ms + scan_ms + reu_ms,
                  "queries_per_s": L / ((red_ms + scan_ms + reu_ms) / 1e3)},
        "refine": {"ms": red_ms + scan_ms + ref_ms,
                   "queries_per_s": L / ((red_ms + scan_ms + ref_ms) / 1e3)},
        "stages_ms": {"dense": dense_ms, "proxy_reduce": red_ms, "proxy_scan": scan_ms,
                      "reuse": reu_ms, "refine": ref_ms},
    }
    modes["reuse"]["speedup_vs_dense"] = dense_ms / modes["reuse"]["ms"]
    modes["refine"]["speedup_vs_dense"] = dense_ms / modes["refine"]["ms"]

    # kernels, roofline of the dominant one
    peaks, peak_src = load_peaks()
    kern = {}
    for kid, name in pv.KERNELS.items():
        n, kms, work = pv.profile_read(kid)
        kern[name] = {"launches": n, "ms": kms, "work": work}
    total_k = sum(v["ms"] for v in kern.values()) or 1.0
    for v in kern.values():
        v["share"] = v["ms"] / total_k
    flop_pair = 2.0 * run.H * run.D
    if fp8:   # the measured FP8 GEMM figures of this GPU
        tc_peak_burst, tc_peak = fp8_peak["burst"], fp8_peak["sustained"]
        tc_src = "measured fp8 sustained (" + fp8_peak["how"] + ")"
    else:
        tc_peak_burst, tc_peak = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
        tc_src = f"{peak_src} bf16 sustained"
    for name in ("scan", "refine"):
        v = kern[name]
        if v["ms"] > 0:
            v["tflops"] = v["work"] * flop_pair / (v["ms"] / 1e3) / 1e12
    for name in ("reduce", "reuse"):
        v = kern[name]
        if v["ms"] > 0:
            v["gbs"] = v["work"] / (v["ms"] / 1e3) / 1e9
    dom = max(kern, key=lambda n: kern[n]["ms"])
    dv = kern[dom]
    if dv["ms"] <= 0:
        roof = None
    elif dom in ("scan", "refine"):
        ach = dv["tflops"]
        bpp = scan_traffic_per_pair() if dom == "scan" else None
        pairs_per_launch = dv["work"] / max(dv["launches"], 1)
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": tc_peak,
                "unit": "TFLOP/s", "frac": ach / tc_peak,
                "traffic": None if bpp is None else bpp * pairs_per_launch,
                "traffic_source": None if bpp is None else
                    "ncu dram bytes of the dense scan at L=16384 (profiles/), per causal pair, "
                    "times this run's pairs per launch",
                "peak_source": tc_src,
                "frac_of_burst": ach / tc_peak_burst,
                "frac_of_nominal_x2_bf16": ach / (peaks["bf16_tflops_sustained"] *
                                                  (FP8_OVER_BF16 if fp8 else 1.0)),
                "per_launch": {"work_pairs": dv["work"] / max(dv["launches"], 1),
                               "ms": dv["ms"] / max(dv["launches"], 1)}}
    elif dom in ("reduce", "reuse"):
        ach = dv["gbs"]
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": ach / peaks["hbm_gbs"], "traffic": None,
                "peak_source": f"{peak_src} hbm"}
    else:   # the selection: its work is per row, not per byte
        roof = None

    # Refine + its top-k against HBM (algorithmic bytes: every group's C
    # candidate keys and scales gathered once, the members' queries and
    # weights read, the candidate rows read, the index rows written) and
    # against the tensor peak (member-candidate pairs x 2 H D)
    esz = {gen.F32: 4, gen.BF16: 2, gen.E4M3: 1}[wl["dtype"]]
    key_b = run.D * esz + (4 if fp8 else 0)
    groups = sum(-(-b // run.g) - a // run.g for a, b in run.ranges)
    gather = sum(min(run.C, min(run.L, (j + 1) * run.g)) for a, b in run.ranges
                 for j in range(a // run.g, -(-b // run.g)))
    ref_bytes = (gather * key_b + run.rows * (run.H * run.D * esz + run.H * 4 + 4)
                 + groups * run.C * 4 + run.rows * run.k * 4)
    ref_pairs = kern["refine"]["work"] / max(args.steps, 1)
    modes["refine_stage"] = {
        "ms": ref_ms, "algorithmic_bytes": ref_bytes,
        "gbs": ref_bytes / (ref_ms / 1e3) / 1e9,
        "frac_hbm": ref_bytes / (ref_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
        "tflops": ref_pairs * flop_pair / (ref_ms / 1e3) / 1e12,
        "frac_tensor": ref_pairs * flop_pair / (ref_ms / 1e3) / 1e12 / tc_peak}

    # quality (this rank's rows)
    rows_of = lambda t: torch.cat([t[a:b] for a, b in run.ranges])  # noqa: E731
    rec = {"reuse_vs_dense": recall_stats(rows_of(run.dense), rows_of(run.reu)),
           "refine_vs_dense": recall_stats(rows_of(run.dense), rows_of(run.ref)),
           "dense_neighbour_overlap": neighbour_overlap(rows_of(run.dense))}

    # end to end through host buffers (pinned), every step's copies inside the
    # timed region: step i's inputs go up while step i - 1 computes (two
    # device input sets), and each stage's indices come back while the later
    # stages compute (two device output sets), on their own copy streams
    e2e = None
    if not args.no_e2e:
        pinned = {n: (None if t is None else t.pin_memory()) for n, t in run.host.items()}
        outs = [torch.empty(run.L, run.k, dtype=torch.int32).pin_memory() for _ in range(3)]
        dev_in = [run.dev, {n: (None if t is None else torch.empty_like(t))
                            for n, t in run.dev.items()}]
        seqs = [run.seq, pv.make_seq(dev_in[1]["q"], dev_in[1]["q_scale"], dev_in[1]["w"],
                                     dev_in[1]["k"], dev_in[1]["k_scale"])]
        dev_out = [(run.dense, run.reu, run.ref),
                   tuple(torch.empty_like(run.dense) for _ in range(3))]
        comp, h2d, d2h = run.stream, torch.cuda.Stream(device), torch.cuda.Stream(device)
        mk = lambda: torch.cuda.Event(enable_timing=False)

        def pipelined(K):
            up = [mk(), mk()]            # inputs of set b landed
            used = [None, None]          # last step that read input set b finished
            back = [None, None]          # indices of output set b copied back
            h2d.wait_stream(comp)
            d2h.wait_stream(comp)

            def upload(b):
                if used[b] is not None:
                    h2d.wait_event(used[b])
                with torch.cuda.stream(h2d):
                    for n, t in pinned.items():
                        if t is not None:
                            dev_in[b][n].copy_(t, non_blocking=True)
                up[b].record(h2d)
            upload(0)
            for i in range(K):
                b = i % 2
                if i + 1 < K:
                    upload(1 - b)
                comp.wait_event(up[b])
                if back[b] is not None:
                    comp.wait_event(back[b])
                ev = [mk() for _ in range(6)]
                run.step(events=ev, seq=seqs[b], outs=dev_out[b])
                used[b] = ev[5]
                with torch.cuda.stream(d2h):
                    for o, dsrc, e in zip(outs, dev_out[b], (ev[1], ev[4], ev[5])):
                        d2h.wait_event(e)
                        for ra, rb in run.ranges:        # this rank's rows
                            o[ra:rb].copy_(dsrc[ra:rb], non_blocking=True)
                back[b] = mk()
                back[b].record(d2h)
            comp.wait_stream(h2d)
            comp.wait_stream(d2h)
        pipelined(2)
        barrier()
        k_e2e = args.steps
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(run.stream)
        pipelined(k_e2e)
        b.record(run.stream)
        barrier()
        e_ms = max_over_ranks(a.elapsed_time(b), device)
        # the host copies are the device results of the last step
        last = dev_out[(k_e2e - 1) % 2]
        ra, rb = run.ranges[0]
        for o, dsrc in zip(outs, last):
            assert torch.equal(o[ra:ra + 1024], dsrc[ra:ra + 1024].cpu()), \
                "host indices differ from the device's"
        e2e = {"value": job_value(L, e_ms, k_e2e), "unit": "queries/s",
               "h2d_bytes_per_step": run.h2d_bytes(), "d2h_bytes_per_step": run.d2h_bytes(),
               "ms_per_step": e_ms / k_e2e, "steps": k_e2e,
               "overlap": "inputs of step i+1 uploaded during step i; each stage's indices "
                          "copied back during the later stages"}

    extra = None
    if not args.no_extra and world == 1:
        extra = measure_extra(run, wl, device, peaks, args.seed)
        extra["workloads"] = measure_workloads(args, device, peaks, fp8_peak)
        extra["cross_layer_reuse"] = measure_layers(device, args.seed)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        total, desc, threads, parts = oracle_sample_time(p, wl)
        cpu = {"value": L / total, "unit": "queries/s", "cores": threads, "kind": "oracle",
               "sample": desc, "extrapolated_step_s": total, "parts_s": parts}

    value = job_value(L, ms_max, args.steps)      # the whole sequence's queries
    line = {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": gen.DTYPE_NAMES[wl["dtype"]], "data": "synthetic",
            "config": config_of(wl, args), "modes": modes, "recall": rec,
            "roofline": roof, "kernels": kern, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(n1 - n0), "clocks": clk, "fp8_peak_tflops": fp8_peak,
            "extra": extra}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=[k for k in gen.WORKLOADS if "decode" not in k])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the decode / backfill / window-union measurements")
    ap.add_argument("--selection", choices=["library", "fused", "scores"], default="library",
                    help="top-k of prefix rows: the library's default, fused into the scan, "
                         "or from every score written to the workspace")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = dict(gen.WORKLOADS[args.workload])
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
