"""Benchmark of the sparse-attention decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_32k] [--no-cpu-baseline] [--no-prefill] [--no-verify]
                    [--no-column] [--no-overlap] [--no-configs]

Workload (default): batched decode, batch 32, 32 query / 8 KV heads, d = 128,
context T = 32768, bf16 KV cache with fp32 accumulation, block 64, top-k 32 +
1 sink block + 4-block window (2369 keys per query), synthetic N(0,1) inputs
with 16 planted needle blocks per (sequence, KV head).  One step = one
``sa_sparse_attn_decode`` call over the whole batch, compressed keys
maintained: on this workload one cooperative launch that scores the
compressed keys, selects each pair's top-k and runs the split-KV sparse
attention (else a scoring + top-k kernel, then the attention kernel).

Timing: W untimed warm-up steps, then K steps; before every step the 126 MB
L2 is flushed (a 256 MB buffer written, then another 256 MB read so that the
dirty lines are written back before the step), and each step is bracketed by
CUDA events on the launching stream (the flush is outside the events).  Multi-GPU
(torchrun): every rank runs its own batch (weak scaling, no collective on the
data path); the per-rank device times are max-reduced.

Printed: one JSON line (rank 0).  ``value`` = sequences decoded per second
(whole job).  Also: the roofline of the step's one kernel (algorithmic bytes
over the timed launch, against the measured copy bandwidth), the attention
kernel alone on the same table, the causal prefill, the dense verify of a
draft chunk, column-sparse attention, the decode step with overlapping
compressed keys and the other decode workloads (tiny fp32, the 6-token draft
chunk, the 1M-token LSA decode), each with its kernels' rooflines,
the end-to-end number
through the C ABI with host buffers, clocks sampled during the timed region,
and the float64 CPU oracle timed on a bounded sample (rank 0, N = 1).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from top_block_sparse_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------- helpers --

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0) or 0), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region.

    nvidia-smi is started first and the timed work begins only once it has
    printed its first samples: its start-up (driver queries on the GPU) would
    otherwise fall inside a short timed region and slow the first steps."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 20

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.marks = []

    def _reader(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.lines.append((time.perf_counter(), ln))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", str(self.PERIOD_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        if self.proc is not None:
            self.thread = threading.Thread(target=self._reader, daemon=True)
            self.thread.start()
            t0 = time.perf_counter()
            while len(self.lines) < 3 and time.perf_counter() - t0 < 10.0 and self.proc.poll() is None:
                time.sleep(0.01)
        return self

    def mark(self):
        """Host time stamp taken right after a synchronize: the timed region
        lies between the first and the last mark."""
        self.marks.append(time.perf_counter())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(2.5 * self.PERIOD_MS / 1000)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=5)
        return False

    def summary(self):
        """Median SM clock and active throttle reasons of the samples taken
        inside the timed region (between the marks, widened by one sampling
        period), or of all samples if none falls inside."""
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = list(self.lines)
        if len(self.marks) >= 2:
            lo, hi = self.marks[0], self.marks[-1] + self.PERIOD_MS / 1000
            inside = [r for r in rows if lo <= r[0] <= hi]
            if inside:
                rows = inside
        sm, mx, reasons = [], None, set()
        for _, ln in rows:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "sample_period_ms": self.PERIOD_MS}


class nvtx_range:
    """An NVTX range around one benchmark leg (ncu --nvtx-include selects a
    leg's kernels by it)."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        torch.cuda.nvtx.range_pop()
        return False


def spread(ms_list):
    """Spread of per-step device times (ms): min, median, 90th percentile,
    max and mean."""
    s = sorted(ms_list)
    p90 = s[min(len(s) - 1, int(math.ceil(0.9 * len(s))) - 1)]
    return {"min": s[0], "median": statistics.median(s), "p90": p90, "max": s[-1],
            "mean": statistics.mean(s), "n": len(s)}


def decode_bytes(w) -> dict:
    """Algorithmic HBM bytes of one decode step (per the whole batch)."""
    el = 2 if w.dtype == "bf16" else 4
    b = w.block_size
    C = w.ctx_len
    s_end = min(w.sink_keys, C)
    w_begin = max(C - w.window_keys, s_end)
    nb = C // b
    cand = sum(1 for j in range(nb) if j * b < w_begin and (j + 1) * b > s_end)
    k = min(w.top_k, cand)
    keys = s_end + k * b + (C + w.n_q - w_begin)       # block keys inside sink/window are disjoint here
    pairs = w.batch * w.num_kv_heads
    kv = pairs * keys * w.head_dim * el * 2
    kc = pairs * nb * w.head_dim * 4
    q = w.batch * w.n_q * w.num_q_heads * w.head_dim * el
    o = w.batch * w.n_q * w.num_q_heads * w.head_dim * el
    return dict(kv=kv, kc=kc, q=q, o=o, keys_per_query=keys, attn=kv + q + o, step=kv + kc + 2 * q + o)


# the sources a kernel's traffic record depends on
TRAFFIC_SOURCES = {"decode_tc.cu": ("decode_tc.cu", "decode_units.cuh", "tc.cuh", "common.cuh", "internal.h")}


def src_hash(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "top_block_sparse_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(section: str, pairs: int):
    """DRAM bytes per launch of one instantiation of the decode kernel (the
    fused step `decode_tc_kernel<1, 4, 1>` or the attention alone
    `decode_tc_kernel<1, 4, 0>`) from the committed ncu summary: read + write
    of one launch at the captured batch, scaled by the number of (sequence,
    KV head) pairs (the traffic is per pair), if the summary was taken on the
    current source of the kernel; else None."""
    path = os.path.join(ROOT, "profiles", "decode_tc_kernel__decode_32k_b16.md")
    try:
        text = open(path).read()
        sha = re.search(r"source hash: `([0-9a-f]+)`", text).group(1)
        cap_pairs = int(re.search(r"captured pairs: (\d+)", text).group(1))
        if sha != src_hash(*TRAFFIC_SOURCES["decode_tc.cu"]):
            return None
        sec = text[text.index(f"## `{section}`"):]
        rd = float(re.search(r"dram__bytes_read\.sum`\) \| ([0-9.]+) Mbyte", sec).group(1))
        wr = float(re.search(r"dram__bytes_write\.sum`\) \| ([0-9.]+) Mbyte", sec).group(1))
        return (rd + wr) * 1e6 * pairs / cap_pairs
    except Exception:
        return None


class L2Flush:
    """Writes a 256 MB buffer (twice the 126 MB L2), then reads another 256 MB
    buffer: the read evicts the write's dirty lines, so their write-back to
    HBM happens here, outside the timed step, and the step starts with an L2
    holding nothing it will read."""

    def __init__(self, device):
        self.w = torch.empty(L2_FLUSH_BYTES // 4, device=device, dtype=torch.float32)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, device=device, dtype=torch.float32)
        self.sink = torch.empty((), device=device, dtype=torch.float32)

    def __call__(self):
        self.w.fill_(1.0)
        torch.sum(self.r, dim=0, out=self.sink)


def queue_ahead(steps):
    """Holds the stream for a few ms (a GPU spin, outside every timed
    region) so that the host enqueues the first steps before the GPU reaches
    them: without it the first step's start event fires while the host is
    still issuing that step's launch, and the host's launch latency would be
    timed as device time."""
    ms = min(50.0, 1.0 + 0.3 * steps)
    torch.cuda._sleep(int(ms * 1e-3 * 2.0e9))


def timed_steps(fn, steps, warmup, stream, flush, clk=None):
    """W warm-ups, then K steps each preceded by an L2 flush; returns the
    per-step device times (ms) from CUDA events on `stream`.  `clk` (a
    ClockSampler) gets host marks at both ends of the timed region."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush()
            fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if clk is not None:
        clk.mark()
    with torch.cuda.stream(stream):
        queue_ahead(steps)
        for s, e in evs:
            flush()
            s.record(stream)
            fn()
            e.record(stream)
    torch.cuda.synchronize()
    if clk is not None:
        clk.mark()
    return [s.elapsed_time(e) for s, e in evs]


def timed_interleaved(fns, steps, warmup, stream, flush, clk=None):
    """Like timed_steps for several functions at once: every round runs each
    function once (each after its own L2 flush), so they all see the same
    clocks and temperature.  Returns one list of per-step times (ms) per
    function."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            for fn in fns:
                flush()
                fn()
    torch.cuda.synchronize()
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in fns]
           for _ in range(steps)]
    if clk is not None:
        clk.mark()
    with torch.cuda.stream(stream):
        queue_ahead(steps * len(fns))
        for row in evs:
            for fn, (s, e) in zip(fns, row):
                flush()
                s.record(stream)
                fn()
                e.record(stream)
    torch.cuda.synchronize()
    if clk is not None:
        clk.mark()
    return [[row[i][0].elapsed_time(row[i][1]) for row in evs] for i in range(len(fns))]


# ------------------------------------------------------------- CPU oracle --

def oracle_sample(w, inp_cpu_pairs, n_pairs_total, min_seconds=10.0):
    """Times the float64 oracle (one thread) on the sampled pairs; returns
    (seconds per full step extrapolated, seconds measured, pairs)."""
    from threadpoolctl import threadpool_limits
    from oracle import sparse_attn_oracle as orc
    p = orc.OracleParams(block_size=w.block_size, top_k=w.top_k, sink_keys=w.sink_keys,
                         window_keys=w.window_keys, pool=w.pool)
    with threadpool_limits(limits=1):
        # compressed keys are maintained state of a decode step, as on the GPU
        Kcs = [orc.compress(K[:w.ctx_len], p) for (_, K, _) in inp_cpu_pairs]
        t0 = time.perf_counter()
        done = 0
        while True:     # repeat the sample until about min_seconds of CPU work
            for (q, K, V), Kc in zip(inp_cpu_pairs, Kcs):
                orc.decode_pair(q, K, V, w.ctx_len, p, Kc=Kc)
            done += len(inp_cpu_pairs)
            dt = time.perf_counter() - t0
            if dt >= min_seconds:
                break
    per_pair = dt / done
    return per_pair * n_pairs_total, dt, done


class ParityTally:
    """Per-config parity of the timed GPU results against the float64 oracle
    (one host core): selected sets identical / near-ties / mismatches, and
    the output errors of the pairs whose sets match (max abs, relative L2;
    for bf16 outputs also the max abs beyond half a bf16 step of the exact
    value, which the output format cannot come closer than)."""

    def __init__(self):
        self.n = self.match = self.near = self.mismatch = 0
        self.max_abs = self.max_abs_fmt = 0.0
        self.se = self.sr = 0.0
        self.oracle_s = 0.0

    def sets(self, got, sel):
        self.n += 1
        if got == sel.selected:
            self.match += 1
            return True
        if sel.near_tie:
            self.near += 1
        else:
            self.mismatch += 1
        return False

    def out(self, got, ref):
        import numpy as np
        g = got.double().cpu().numpy().reshape(ref.shape)
        d = np.abs(g - ref)
        self.max_abs = max(self.max_abs, float(d.max()) if d.size else 0.0)
        if got.dtype == torch.bfloat16:
            ax = np.abs(ref)
            half = np.where(ax > 0, np.exp2(np.floor(np.log2(np.where(ax > 0, ax, 1.0))) - 8), 0.0)
            d = np.maximum(d - half, 0.0)
        self.max_abs_fmt = max(self.max_abs_fmt, float(d.max()) if d.size else 0.0)
        self.se += float(((g - ref) ** 2).sum())
        self.sr += float((ref ** 2).sum())

    def report(self, sample, extrapolate=1.0):
        rel = math.sqrt(self.se / self.sr) if self.sr > 0 else 0.0
        return {"checked": self.n, "sets_match": self.match, "near_ties": self.near, "mismatches": self.mismatch,
                "max_abs": self.max_abs, "max_abs_beyond_bf16_rounding": self.max_abs_fmt, "rel_l2": rel,
                "oracle_s": self.oracle_s, "oracle_s_full_config": self.oracle_s * extrapolate,
                "oracle_cores": 1, "sample": sample}


def decode_parity(w, inp, O, idx, pairs, n_pairs_total, min_pairs_note=""):
    """Oracle decode of the sampled pairs on one core, compared with the
    GPU's index table and output of the same inputs."""
    from threadpoolctl import threadpool_limits
    from oracle import sparse_attn_oracle as orc
    op = orc.OracleParams(block_size=w.block_size, top_k=w.top_k, sink_keys=w.sink_keys,
                          window_keys=w.window_keys, pool=w.pool, pool_stride=w.pool_stride,
                          pool_kernel=w.pool_kernel)
    G = w.group
    t = ParityTally()
    with threadpool_limits(limits=1):
        for (b, h) in pairs:
            q = inp["Q"][b, :, h * G:(h + 1) * G].cpu().double().numpy()
            K = inp["K"][b, h, :w.kv_len].cpu().double().numpy()
            V = inp["V"][b, h, :w.kv_len].cpu().double().numpy()
            t0 = time.perf_counter()
            r = orc.decode_pair(q, K, V, w.ctx_len, op)
            t.oracle_s += time.perf_counter() - t0
            got = [int(x) for x in idx[b, h].tolist() if x >= 0]
            if t.sets(got, r["sel"]):
                t.out(O[b, :, h * G:(h + 1) * G], r["O"])
    sample = (f"every (sequence, KV head) pair ({len(pairs)})" if len(pairs) == n_pairs_total else
              f"{len(pairs)} of {n_pairs_total} (sequence, KV head) pairs, evenly spaced{min_pairs_note}")
    return t.report(sample, n_pairs_total / max(1, len(pairs)))


def prefill_parity(w, Q, K, V, O, idx, heads, tiles):
    """Oracle of sampled prefill tiles (selection and attention, one core)
    against the GPU's per-tile tables and output rows."""
    from threadpoolctl import threadpool_limits
    from oracle import sparse_attn_oracle as orc
    op = orc.OracleParams(block_size=w.block_size, top_k=w.top_k, sink_keys=w.sink_keys,
                          window_keys=w.window_keys)
    G, b = w.group, w.block_size
    t = ParityTally()
    with threadpool_limits(limits=1):
        for h in heads:
            Kh = K[0, h, :w.n_q].cpu().double().numpy()
            Vh = V[0, h, :w.n_q].cpu().double().numpy()
            t0 = time.perf_counter()
            Kc = orc.compress(Kh, op)
            t.oracle_s += time.perf_counter() - t0
            for i in tiles:
                q = Q[0, i * b:(i + 1) * b, h * G:(h + 1) * G].cpu().double().numpy()
                t0 = time.perf_counter()
                r = orc.prefill_tile(q, Kh, Vh, i, op, Kc)
                t.oracle_s += time.perf_counter() - t0
                got = [int(x) for x in idx[0, h, i].tolist() if x >= 0]
                if t.sets(got, r["sel"]):
                    t.out(O[0, i * b:(i + 1) * b, h * G:(h + 1) * G], r["O"])
    n_tiles = (w.n_q + b - 1) // b
    return t.report(f"{len(tiles)} of {n_tiles} query tiles (evenly spaced, the last included) x KV heads "
                    f"{list(heads)} of {w.num_kv_heads}; oracle_s_full_config extrapolates per tile, and later "
                    f"tiles cost more",
                    w.num_kv_heads * n_tiles / (len(heads) * len(tiles)))


def even_pairs(w, n):
    allp = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    if n >= len(allp):
        return allp
    step = len(allp) / n
    return [allp[int(i * step)] for i in range(n)]


def cpu_pairs(w, inp, n):
    G = w.group
    out = []
    pairs = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    step = max(1, len(pairs) // n)
    for (b, h) in pairs[::step][:n]:
        q = inp["Q"][b, :, h * G:(h + 1) * G].double().cpu().numpy()
        K = inp["K"][b, h, :w.kv_len].double().cpu().numpy()
        V = inp["V"][b, h, :w.kv_len].double().cpu().numpy()
        out.append((q, K, V))
    return out


def cpu_info():
    model = ""
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except Exception:
        pass
    return model, os.cpu_count()


# ---------------------------------------------------------------- ranks ---

def rank_seed(rank: int) -> int:
    """Input seed of a rank: every rank decodes its own batch (weak scaling)."""
    return 1000 + 1 + rank


def reduce_max(value: float, world: int, device) -> float:
    """Max over the ranks of a per-rank device time: the job takes as long as
    its slowest rank."""
    if world <= 1:
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------- arms ---

def run_reference(args, w, rank, world):
    """The float64 oracle on the host cores: each step is a bounded sample of
    the workload's (sequence, KV head) pairs; value extrapolated per step."""
    if rank != 0:
        return None
    inp = make_inputs(w.scaled(batch=1), seed=1000 + 1, device="cpu")
    n = min(args.ref_pairs, w.num_kv_heads)
    pairs = cpu_pairs(w.scaled(batch=1), inp, n)
    pairs_total = w.batch * w.num_kv_heads
    for _ in range(args.warmup):
        oracle_sample(w, pairs[:1], pairs_total, min_seconds=0.0)
    times = []
    for _ in range(args.steps):
        full, _, _ = oracle_sample(w, pairs, pairs_total, min_seconds=0.0)
        times.append(full)
    sec = statistics.mean(times)
    q_per_s = w.batch * w.n_q / sec
    model, ncpu = cpu_info()
    line = {
        "impl": "reference", "metric": METRIC, "value": q_per_s, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w),
        "cpu_baseline": {"value": q_per_s, "unit": "queries/s", "cores": 1, "kind": "oracle",
                         "sample": f"{len(pairs)} of {pairs_total} (sequence, KV head) pairs per step, "
                                   f"extrapolated to the full batch; {model}, {ncpu} host cores, 1 used"},
        "e2e": {"value": q_per_s, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


METRIC = "sparse-attn decode queries/s + achieved HBM GB/s at T=32k; prefill TFLOP/s"


def config_of(w):
    return {"workload": f"{w.name}: batched decode B={w.batch}, Hq={w.num_q_heads}, Hkv={w.num_kv_heads}, "
                        f"d={w.head_dim}, T={w.ctx_len}, {w.dtype} KV, block {w.block_size}, top-k {w.top_k} "
                        f"+ sink {w.sink_keys} keys + window {w.window_keys} keys",
            "batch": w.batch, "seq_len": w.ctx_len, "n_q": w.n_q, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
            "top_k": w.top_k, "sink_keys": w.sink_keys, "window_keys": w.window_keys,
            "l2": "flushed before every timed step, outside the step's events: 256 MB written, then "
                  "another 256 MB read so the written lines are evicted before the step",
            "parallelism": "replicas (weak scaling)"}


def run_ours(args, w, rank, world, local_rank):
    from top_block_sparse_b200 import sa
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    inp = make_inputs(w, seed=rank_seed(rank), device=dev)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    p = sa.params_for(w)
    nb = w.ctx_len // w.block_size
    Kc = torch.empty((w.batch, w.num_kv_heads, nb, w.head_dim), device=dev, dtype=torch.float32)
    O = torch.empty((w.batch, w.n_q, w.num_q_heads, w.head_dim), device=dev, dtype=Q.dtype)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device=dev, dtype=torch.float32)
    idx = torch.empty((w.batch, w.num_kv_heads, w.top_k), device=dev, dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_DECODE, device=dev)
    ws_g = sa.alloc_workspace(p, sa.SA_OP_GIVEN_IDX, device=dev)
    flush = L2Flush(dev)
    p_trusted = sa.params_for(w)
    p_trusted.flags = sa.SA_FLAG_TRUSTED_IDX
    torch.cuda.nvtx.range_push(w.name)
    with torch.cuda.stream(stream):
        sa.pool_keys(p, K, Kc, stream=stream)
    torch.cuda.synchronize()

    def step():
        sa.sparse_attn_decode(p, Q, K, V, Kc, O, lse, idx, ws, stream=stream)

    def attn_only():
        # the decode step's own (valid) table: only the attention kernel runs
        sa.sparse_attn_given_idx(p_trusted, Q, K, V, idx, O, lse, ws_g, stream=stream)

    def pool_only():
        sa.pool_keys(p, K, Kc, stream=stream)

    # --- the timed decode steps -------------------------------------------
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ClockSampler.PERIOD_MS = args.clock_period_ms
    with ClockSampler(local_rank) as clk:
        step_ms = timed_steps(step, args.steps, args.warmup, stream, flush, clk)
    if sa.read_status(ws, stream) != sa.SA_OK:
        raise RuntimeError("device status word set during the timed steps")
    ms = reduce_max(sum(step_ms) / len(step_ms), world, dev)
    parity = None
    if rank == 0 and not args.no_parity:
        torch.cuda.synchronize()
        parity = decode_parity(w, inp, O, idx, even_pairs(w, w.batch * w.num_kv_heads),
                               w.batch * w.num_kv_heads)
    # --- the attention kernel alone, rank-local ----------------------------
    attn_ms = statistics.mean(timed_steps(attn_only, max(50, args.steps // 4), 3, stream, flush))
    pool_ms = statistics.mean(timed_steps(pool_only, 10, 2, stream, flush))
    torch.cuda.nvtx.range_pop()
    # --- causal prefill (tensor cores), rank-local --------------------------
    prefill = None
    if not args.no_prefill:
        with nvtx_range("prefill"):
            prefill = run_prefill_bench(args, dev, stream, flush)
    # --- dense verify of a draft chunk, rank-local ----------------------------
    verify = None
    if not args.no_verify:
        with nvtx_range("verify"):
            verify = run_verify_bench(args, dev, stream, flush)
    # --- column-sparse attention, rank-local ----------------------------------
    column = None
    if not args.no_column:
        with nvtx_range("column"):
            column = run_column_bench(args, dev, stream, flush)
    # --- decode with overlapping compressed keys, rank-local ------------------
    overlap = None
    if not args.no_overlap:
        with nvtx_range("overlap"):
            overlap = run_overlap_bench(args, dev, stream, flush)
    # --- the other decode workloads, rank-local ---------------------------------
    configs = None
    if not args.no_configs:
        configs = run_decode_configs(args, dev, stream, flush)
    # --- LSA flat bucket retrieval, rank-local -----------------------------------
    buckets = None
    if not args.no_buckets:
        with nvtx_range("buckets"):
            buckets = run_bucket_bench(args, dev, stream, flush)
        torch.cuda.empty_cache()
    # --- end to end through the C ABI with host buffers -------------------
    with nvtx_range("e2e"):
        e2e = e2e_decode(args, w, p, Q, K, V, Kc, O, lse, idx, ws, stream, flush)
    e2e["ms"] = reduce_max(e2e["ms"], world, dev)
    e2e["serial_ms"] = reduce_max(e2e["serial_ms"], world, dev)
    if rank != 0:
        return None

    hbm, tfl, tfl_s, src = peaks()
    by = decode_bytes(w)
    q_per_s = world * w.batch * w.n_q / (ms * 1e-3)
    attn_gbs = by["attn"] / (attn_ms * 1e-3) / 1e9
    step_gbs = by["step"] / (ms * 1e-3) / 1e9
    pool_bytes = w.batch * w.num_kv_heads * (nb * w.block_size * w.head_dim * 2 + nb * w.head_dim * 4)
    line = {
        "metric": METRIC, "value": q_per_s, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) + needle blocks)",
        "config": config_of(w),
        "decode_hbm_gbs": step_gbs, "decode_hbm_frac": step_gbs / hbm,
        "decode_bytes_per_step": by["step"], "keys_per_query": by["keys_per_query"],
        # the timed step is one launch of the fused kernel: its roofline is the
        # step's (compressed keys + retained K/V bytes over the step time)
        "roofline": {"bound": "hbm",
                     "kernel": "decode_tc_kernel<fused> (scores, top-k and tcgen05 split-KV attention in one "
                               "cooperative launch)",
                     "achieved": step_gbs, "peak": hbm, "unit": "GB/s", "frac": step_gbs / hbm,
                     "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs, burst copy)" if src == "measured" else src,
                     "algorithmic_bytes_per_launch": by["step"], "launch_ms": ms,
                     "traffic": profiled_traffic("decode_tc_kernel<1, 4, 1>", w.batch * w.num_kv_heads),
                     "frac_of_spec_8tbs": step_gbs / 8000.0},
        # the attention kernel alone on the step's own table (the two-kernel
        # path's second launch), timed in its own loop after the timed steps
        "attention_alone": {"kernel": "decode_tc_kernel (tcgen05 split-KV attention, given index table)",
                            "achieved": attn_gbs, "peak": hbm, "unit": "GB/s", "frac": attn_gbs / hbm,
                            "algorithmic_bytes_per_launch": by["attn"], "launch_ms": attn_ms,
                            "traffic": profiled_traffic("decode_tc_kernel<1, 4, 0>", w.batch * w.num_kv_heads)},
        "pool": {"kernel": "pool_kernel", "ms": pool_ms, "gbs": pool_bytes / (pool_ms * 1e-3) / 1e9,
                 "note": "compression runs once after prefill / when a block fills; not part of a decode step"},
        "e2e": {"value": world * w.batch * w.n_q / (e2e["ms"] * 1e-3), "unit": "queries/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": e2e["ms"],
                "serial": {"value": world * w.batch * w.n_q / (e2e["serial_ms"] * 1e-3),
                           "ms_per_step": e2e["serial_ms"], "breakdown_us": e2e["breakdown_us"],
                           "note": "one step at a time on one stream, L2 flushed before each step"},
                "note": "per step: one pinned host -> device copy of the new tokens' Q, K, V rows (packed), "
                        "sa_append_kv into the cache and the decode call through the C ABI, device -> pinned "
                        "host copy of O; the KV cache and the compressed keys stay resident in HBM; steps "
                        "pipelined (copy-in, compute and copy-out streams, two staging slots), so a step's "
                        "copies overlap the decodes next to it"},
        "prefill": prefill,
        "verify": verify,
        "column": column,
        "overlap": overlap,
        "decode_configs": configs,
        "buckets": buckets,
        "parity": parity,
        "gpu_launches": sa.decode_launches(p) * args.steps,
        "clocks": clk.summary(),
    }
    # per-step spread of the timed steps, and the mean step in SM clock
    # cycles at the sampled median clock (a slower clock shows as fewer
    # cycles per step, not as a slower kernel)
    sp = spread(step_ms)
    line["step_ms_min"], line["step_ms_median"], line["step_ms_p90"] = sp["min"], sp["median"], sp["p90"]
    line["step_ms_max"] = sp["max"]
    line["step_us"] = [round(x * 1000, 1) for x in step_ms]
    mhz = line["clocks"].get("sm_mhz")
    line["step_kcycles_at_median_sm_mhz"] = ms * mhz if mhz else None
    return line


def prefill_counts(w):
    """Algorithmic and executed tensor-core FLOPs of one causal prefill of
    workload w (sink / window multiples of 64, tile = block = 64)."""
    T, b, k = w.n_q, w.block_size, w.top_k
    Hq, Hkv, G, d = w.num_q_heads, w.num_kv_heads, w.group, w.head_dim
    nt, nb = (T + b - 1) // b, T // b
    attn_alg = 0
    blocks = 0
    score_alg = 0
    for t in range(nt):
        C = t * b
        s_end = min(w.sink_keys, C)
        w_begin = max(C - w.window_keys, s_end)
        cand = sum(1 for j in range(min(nb, t)) if j * b < w_begin and (j + 1) * b > s_end)
        ke = min(k, cand)
        rows = min(b, T - C)
        ctx_keys = s_end + ke * b + (C - w_begin)
        attn_alg += Hq * 4 * d * (rows * ctx_keys + rows * (rows + 1) // 2)
        blocks += s_end // b + ke + (C - w_begin) // b + 1
        score_alg += Hkv * cand * rows * 2 * d
    attn_exec = Hkv * blocks * (G * b) * 4 * b * d            # S and PV, 256 rows x 64 keys x 128
    npairs = (nt + 1) // 2
    score_exec = 0
    for n in range(npairs):
        t = min(2 * n + 1, nt - 1)
        C = t * b
        s_end = min(w.sink_keys, C)
        w_begin = max(C - w.window_keys, s_end)
        j_lim = min(nb, -(-w_begin // b))
        if j_lim * b > s_end:
            score_exec += Hkv * (-(-j_lim // 128)) * 128 * 128 * 384 * 2
    return dict(attn_alg=attn_alg, attn_exec=attn_exec, score_alg=score_alg, score_exec=score_exec)


def prefill_report(w, full_l, score_l, attn_l, pk):
    """The prefill object of the benchmark line from the per-step times (ms)
    of the full call, the scoring call and the attention call, and the peaks
    (hbm GB/s, bf16 TFLOP/s, sustained TFLOP/s, source)."""
    T = w.n_q
    nb = T // 64
    full_ms, score_ms, attn_ms = (statistics.mean(x) for x in (full_l, score_l, attn_l))
    c = prefill_counts(w)
    hbm, tfl, tfl_s, src = pk
    q_bytes = T * w.num_q_heads * 128 * 2
    kc_bytes = w.num_kv_heads * nb * 128 * 4
    tf = lambda flop, ms: flop / (ms * 1e-3) / 1e12
    return {
        "workload": f"prefill_64k: causal prefill T={w.n_q}, Hq=32, Hkv=8, d=128, bf16, tile = block 64, "
                    "top-k 64 + sink 64 keys + window 256 keys",
        "ms": full_ms,
        "ms_spread": spread(full_l),
        "tflops": tf(c["attn_alg"] + c["score_alg"], full_ms),
        "tflops_note": "algorithmic attention + scoring FLOPs / whole prefill time (pool, score, top-k, attention)",
        "timing": "the full call, the scoring call and the attention call interleaved step by step (each after "
                  "its own L2 flush), so all three see the same clocks",
        "attention": {"kernel": "prefill_attn_kernel (tcgen05)", "ms": attn_ms, "ms_spread": spread(attn_l),
                      "alg_tflops": tf(c["attn_alg"], attn_ms),
                      "exec_tflops": tf(c["attn_exec"], attn_ms),
                      "frac_of_bf16_peak": tf(c["attn_alg"], attn_ms) / tfl,
                      "exec_frac_of_bf16_peak": tf(c["attn_exec"], attn_ms) / tfl,
                      "exec_flop": c["attn_exec"], "alg_flop": c["attn_alg"],
                      "note": "frac_of_bf16_peak counts the algorithmic FLOPs (attended keys only); the executed "
                              "count adds the masked half of each diagonal block"},
        "scoring": {"kernel": "kc_split + prefill_score_kernel (tcgen05, split bf16 x3) + prefill_topk_kernel",
                    "ms": score_ms, "ms_spread": spread(score_l),
                    "alg_tflops": tf(c["score_alg"], score_ms),
                    "exec_tflops": tf(c["score_exec"], score_ms),
                    "frac_of_bf16_peak": tf(c["score_alg"], score_ms) / tfl,
                    "exec_frac_of_bf16_peak": tf(c["score_exec"], score_ms) / tfl,
                    "hbm_bytes": q_bytes + kc_bytes,
                    "hbm_gbs": (q_bytes + kc_bytes) / (score_ms * 1e-3) / 1e9,
                    "hbm_frac": (q_bytes + kc_bytes) / (score_ms * 1e-3) / 1e9 / hbm,
                    "alg_gflop": c["score_alg"] / 1e9, "exec_gflop": c["score_exec"] / 1e9,
                    "note": "three readings: frac_of_bf16_peak = algorithmic FLOPs (GQA-summed query rows x the "
                            "causally visible compressed keys); exec_frac_of_bf16_peak = the MMA FLOPs executed "
                            "(three bf16 products per fp32 product for the split-precision scores, whole 128-block "
                            "chunks); hbm_frac = Q and Kc read once over the call"},
        "attention_plus_scoring_ms": attn_ms + score_ms,
        "peak_bf16_tflops": tfl, "peak_hbm_gbs": hbm, "peak_source": src,
    }


def run_prefill_bench(args, dev, stream, flush):
    """Times the full causal prefill and its two tensor-core kernels alone."""
    from top_block_sparse_b200 import sa
    w = WORKLOADS["prefill_64k"]
    if args.prefill_tokens:
        w = w.scaled(n_q=args.prefill_tokens)
    inp = make_inputs(w, seed=2001, device=dev)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    del inp
    p = sa.params_for(w)
    T = w.n_q
    nb, nt = T // 64, (T + 63) // 64
    Kc = torch.empty((1, w.num_kv_heads, nb, 128), device=dev)
    O = torch.empty((1, T, w.num_q_heads, 128), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((1, T, w.num_q_heads), device=dev)
    idx = torch.empty((1, w.num_kv_heads, nt, w.top_k), device=dev, dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_PREFILL, device=dev)
    ws_s = sa.alloc_workspace(p, sa.SA_OP_SCORE_TOPK, device=dev)
    pt = sa.params_for(w)
    pt.flags = sa.SA_FLAG_TRUSTED_IDX
    ws_g = sa.alloc_workspace(pt, sa.SA_OP_GIVEN_IDX, device=dev)

    def full():
        sa.sparse_attn_prefill(p, Q, K, V, Kc, O, lse, idx, ws, stream=stream)

    def score():
        sa.score_topk(p, Q, Kc, idx, None, ws_s, stream=stream)

    def attn():
        sa.sparse_attn_given_idx(pt, Q, K, V, idx, O, lse, ws_g, stream=stream)

    n = args.prefill_steps
    # the three calls interleaved step by step: a long run of tensor-core work
    # lowers the clock under the power cap, so timing them one after another
    # would give the later ones a lower clock
    with ClockSampler(torch.cuda.current_device()) as clk:
        full_l, score_l, attn_l = timed_interleaved([full, score, attn], n, 3, stream, flush, clk)
    if sa.read_status(ws, stream) != sa.SA_OK:
        raise RuntimeError("device status word set during the prefill runs")
    rep = prefill_report(w, full_l, score_l, attn_l, peaks())
    rep["clocks"] = clk.summary()
    if not args.no_parity:
        full()                     # the table and output of the full call
        torch.cuda.synchronize()
        nt = (T + 63) // 64
        tiles = sorted(set([int(i * (nt - 1) / 15) for i in range(16)] + [nt - 1]))
        rep["parity"] = prefill_parity(w, Q, K, V, O, idx, [0, w.num_kv_heads - 1], tiles)
    return rep


def run_verify_bench(args, dev, stream, flush):
    """Times the dense verify of a draft chunk (sa_verify_refresh) on the
    draft-chunk workload with the chunk's 6 tokens plus one (n_q = 7), and
    the dense attention alone (the same kernel through
    sa_sparse_attn_given_idx with the whole context as window)."""
    from top_block_sparse_b200 import sa
    w = WORKLOADS["draft_chunk_16k"].scaled(n_q=7)
    if args.batch:
        w = w.scaled(batch=args.batch)
    inp = make_inputs(w, seed=3001, device=dev)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    del inp
    p = sa.params_for(w, out_dtype="bf16")
    nb = w.ctx_len // w.block_size
    O = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device=dev)
    mass = torch.empty((w.batch, w.num_kv_heads, nb), device=dev)
    idx = torch.empty((w.batch, w.num_kv_heads, w.top_k), device=dev, dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_VERIFY, device=dev)
    pd = sa.params_for(w, out_dtype="bf16")
    pd.sink_keys, pd.window_keys, pd.top_k, pd.flags = 0, w.ctx_len, 0, sa.SA_FLAG_TRUSTED_IDX
    ws_d = sa.alloc_workspace(pd, sa.SA_OP_GIVEN_IDX, device=dev)

    def full():
        sa.verify_refresh(p, Q, K, V, O, mass, lse, idx, ws, stream=stream)

    def dense():
        sa.sparse_attn_given_idx(pd, Q, K, V, None, O, lse, ws_d, stream=stream)

    n = args.verify_steps
    full_ms = statistics.mean(timed_steps(full, n, 3, stream, flush))
    dense_ms = statistics.mean(timed_steps(dense, n, 3, stream, flush))
    if sa.read_status(ws, stream) != sa.SA_OK:
        raise RuntimeError("device status word set during the verify runs")
    hbm, _, _, src = peaks()
    pairs = w.batch * w.num_kv_heads
    kv = w.ctx_len + w.n_q
    qo = 2 * w.batch * w.n_q * w.num_q_heads * 128 * 2
    alg = pairs * kv * 128 * 2 * 2 + qo + pairs * nb * 4 + pairs * w.top_k * 4
    return {
        "workload": f"draft_chunk_16k dense verify: B={w.batch}, n_q={w.n_q} (6 draft tokens + 1), Hq={w.num_q_heads}, "
                    f"Hkv={w.num_kv_heads}, C={w.ctx_len}, d=128, bf16, block 64, refreshed top-k {w.top_k}",
        "ms": full_ms,
        "algorithmic_bytes": alg,
        "achieved_gbs": alg / (full_ms * 1e-3) / 1e9,
        "frac": alg / (full_ms * 1e-3) / 1e9 / hbm,
        "note": "algorithmic bytes = every K and V row once + Q, O, mass, table; K and V are read once (the "
                "attention pass also keeps per-32-key row sums that a small kernel turns into block masses)",
        "dense_attention": {"kernel": "decode_tc_kernel (the whole context as window)", "ms": dense_ms,
                            "gbs": (pairs * kv * 128 * 2 * 2 + qo) / (dense_ms * 1e-3) / 1e9,
                            "frac": (pairs * kv * 128 * 2 * 2 + qo) / (dense_ms * 1e-3) / 1e9 / hbm},
        "mass_overhead": {"what": "the row sums inside the attention pass + mass_finalize_kernel + "
                                  "mass_topk_kernel: the whole call minus the plain dense attention",
                          "ms": full_ms - dense_ms},
        "peak_gbs": hbm, "peak_source": src,
    }


def run_column_bench(args, dev, stream, flush):
    """Times column-sparse attention (sa_column_attn) on the 64k-token
    workload: every 64-token group attends to its 13120 listed columns."""
    from top_block_sparse_b200 import sa
    from top_block_sparse_b200.inputs import make_columns
    w = WORKLOADS["column_64k"]
    if args.column_tokens:
        # a smaller sequence (ncu captures) keeps the 20% of columns per group
        T = args.column_tokens
        w = w.scaled(n_q=T, top_k=max(64, (T // 5 + 63) // 64 * 64))
    inp = make_inputs(w, seed=4001, device=dev)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    del inp
    cols = make_columns(w, seed=4002, device=dev)
    n_valid = int((cols >= 0).sum().item())
    p = sa.params_for(w, out_dtype="bf16")
    p.flags = sa.SA_FLAG_TRUSTED_IDX
    O = torch.empty((1, w.n_q, w.num_q_heads, 128), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((1, w.n_q, w.num_q_heads), device=dev)
    ws = sa.alloc_workspace(p, sa.SA_OP_COLUMN, device=dev)

    def run():
        sa.column_attn(p, Q, K, V, cols, O, lse, ws, stream=stream)

    ms = statistics.mean(timed_steps(run, args.column_steps, 3, stream, flush))
    if sa.read_status(ws, stream) != sa.SA_OK:
        raise RuntimeError("device status word set during the column-sparse runs")
    _, tfl, _, src = peaks()
    rows = 64 * w.group                                   # query rows of one group
    alg = 2 * 2 * rows * 128 * n_valid                    # QK^T and PV over the listed columns
    chunks = int(((cols >= 0).sum(-1) + 63).div(64, rounding_mode="floor").clamp(min=1).sum().item())
    exe = 2 * 2 * rows * 128 * 64 * chunks                # 64-column chunks as executed
    return {
        "workload": f"column_64k: bidirectional column-sparse attention, T={w.n_q}, Hq={w.num_q_heads}, "
                    f"Hkv={w.num_kv_heads}, d=128, bf16, {w.top_k} columns per 64-token group (20% of T: a shared "
                    "random set per (sequence, KV head) plus the group's own tokens)",
        "ms": ms,
        "alg_tflops": alg / (ms * 1e-3) / 1e12,
        "exec_tflops": exe / (ms * 1e-3) / 1e12,
        "frac_of_bf16_peak": exe / (ms * 1e-3) / 1e12 / tfl,
        "kernel": "prefill_attn_kernel<column mode> (tcgen05; K and V rows gathered by cp.async)",
        "gathered_gb": n_valid * 512 / 1e9,
        "peak_bf16_tflops": tfl, "peak_source": src,
    }


def run_decode_configs(args, dev, stream, flush):
    """Times one sa_sparse_attn_decode call (compressed keys maintained) on
    each of the other decode workloads: the tiny fp32 decode, the 6-token
    draft chunk and the 1M-token decode with LSA centroids (whose one-time
    pooling of the whole context is timed too).  Median of
    --config-steps L2-flushed steps after 5 warm-ups."""
    from top_block_sparse_b200 import sa
    hbm, _, _, src = peaks()
    out = {"peak_gbs": hbm, "peak_source": src}
    for name, seed in (("tiny_decode", 6001), ("draft_chunk_16k", 6002), ("decode_1m", 6003)):
        torch.cuda.nvtx.range_push(name)
        w = WORKLOADS[name]
        if args.small and name != "tiny_decode":
            w = w.scaled(batch=max(1, w.batch // 8), ctx_len=min(w.ctx_len, 524288))
        inp = make_inputs(w, seed=seed, device=dev)
        Q, K, V = inp["Q"], inp["K"], inp["V"]
        del inp
        p = sa.params_for(w)
        nb = w.ctx_len // w.block_size
        Kc = torch.empty((w.batch, w.num_kv_heads, nb, 128), device=dev)
        odt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        O = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device=dev, dtype=odt)
        lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device=dev)
        idx = torch.empty((w.batch, w.num_kv_heads, w.top_k), device=dev, dtype=torch.int32)
        ws = sa.alloc_workspace(p, sa.SA_OP_DECODE, device=dev)

        def pool():
            sa.pool_keys(p, K, Kc, stream=stream)

        def step():
            sa.sparse_attn_decode(p, Q, K, V, Kc, O, lse, idx, ws, stream=stream)

        pool_ms = statistics.median(timed_steps(pool, 3, 3, stream, flush))
        ms = statistics.median(timed_steps(step, args.config_steps, 5, stream, flush))
        if sa.read_status(ws, stream) != sa.SA_OK:
            raise RuntimeError(f"device status word set during the {name} runs")
        parity = None
        if not args.no_parity:
            torch.cuda.synchronize()
            n_all = w.batch * w.num_kv_heads
            n_chk = n_all if name != "decode_1m" else 4
            parity = decode_parity(w, {"Q": Q, "K": K, "V": V}, O, idx, even_pairs(w, n_chk), n_all)
        by = decode_bytes(w)
        el = 2 if w.dtype == "bf16" else 4
        pool_b = w.batch * w.num_kv_heads * (nb * w.block_size * w.head_dim * el + nb * w.head_dim * 4)
        out[name] = {
            "workload": f"B={w.batch}, n_q={w.n_q}, Hq={w.num_q_heads}, Hkv={w.num_kv_heads}, C={w.ctx_len}, "
                        f"{w.dtype}, block {w.block_size}, {w.pool} pooling, top-k {w.top_k}, sink {w.sink_keys}, "
                        f"window {w.window_keys}",
            "ms": ms, "launches": sa.decode_launches(p),
            "token_queries_per_s": w.batch * w.n_q / (ms * 1e-3),
            "keys_per_query": by["keys_per_query"], "algorithmic_bytes": by["step"],
            "gbs": by["step"] / (ms * 1e-3) / 1e9, "frac": by["step"] / (ms * 1e-3) / 1e9 / hbm,
            "pool": {"ms": pool_ms, "gbs": pool_b / (pool_ms * 1e-3) / 1e9,
                     "note": "one-time compression of the whole context (each key read once)"},
            "parity": parity,
        }
        del Q, K, V, Kc, O, lse, idx, ws
        torch.cuda.empty_cache()
        torch.cuda.nvtx.range_pop()
    return out


def run_overlap_bench(args, dev, stream, flush):
    """Times the decode step with overlapping compressed keys on the 32k
    decode workload (windows of 32 keys every 16 keys, block = max over the
    windows touching it): one sa_sparse_attn_decode call = the scoring +
    top-k kernel over the windows, then the attention kernel.  Also the
    scoring kernel alone (sa_score_topk) and the window pooling."""
    from top_block_sparse_b200 import sa
    w = WORKLOADS["decode_32k_overlap"]
    if args.batch:
        w = w.scaled(batch=args.batch)
    inp = make_inputs(w, seed=5001, device=dev)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    del inp
    p = sa.params_for(w, out_dtype="bf16")
    pairs = w.batch * w.num_kv_heads
    nb = w.ctx_len // w.block_size
    n_c = (w.ctx_len - w.pool_kernel) // w.pool_stride + 1
    n_rows = min(n_c, nb * (w.block_size // w.pool_stride))     # windows touching a complete block
    Kc = torch.empty((w.batch, w.num_kv_heads, n_c, 128), device=dev)
    O = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device=dev)
    idx = torch.empty((w.batch, w.num_kv_heads, w.top_k), device=dev, dtype=torch.int32)
    idx2 = torch.empty_like(idx)
    ws = sa.alloc_workspace(p, sa.SA_OP_DECODE, device=dev)
    ws_s = sa.alloc_workspace(p, sa.SA_OP_SCORE_TOPK, device=dev)

    def pool():
        sa.pool_keys(p, K, Kc, stream=stream)

    def step():
        sa.sparse_attn_decode(p, Q, K, V, Kc, O, lse, idx, ws, stream=stream)

    def score():
        sa.score_topk(p, Q, Kc, idx2, None, ws_s, stream=stream)

    n = args.overlap_steps
    pool_ms = statistics.mean(timed_steps(pool, 5, 3, stream, flush))
    step_ms = statistics.mean(timed_steps(step, n, 3, stream, flush))
    score_ms = statistics.mean(timed_steps(score, n, 3, stream, flush))
    if sa.read_status(ws, stream) != sa.SA_OK or sa.read_status(ws_s, stream) != sa.SA_OK:
        raise RuntimeError("device status word set during the overlapping-window runs")
    if not torch.equal(idx, idx2):
        raise RuntimeError("the decode step and sa_score_topk selected different blocks")
    hbm, _, _, src = peaks()
    by = decode_bytes(w)
    win = pairs * n_rows * w.head_dim * 4
    step_b = by["kv"] + win + 2 * by["q"] + by["o"]
    score_b = win + by["q"] + pairs * w.top_k * 4
    pool_b = pairs * (n_c * w.pool_stride * w.head_dim * 2 + n_c * w.head_dim * 4)
    gbs = lambda b, ms: b / (ms * 1e-3) / 1e9
    return {
        "workload": f"decode_32k_overlap: B={w.batch}, Hq={w.num_q_heads}, Hkv={w.num_kv_heads}, C={w.ctx_len}, "
                    f"d=128, bf16, block {w.block_size}, windows of {w.pool_kernel} keys every {w.pool_stride} "
                    f"({n_rows} scored per pair, fp32), top-k {w.top_k}, sink {w.sink_keys}, window {w.window_keys}",
        "ms": step_ms,
        "queries_per_s": w.batch * w.n_q / (step_ms * 1e-3),
        "launches": sa.decode_launches(p),
        "algorithmic_bytes": step_b,
        "achieved_gbs": gbs(step_b, step_ms), "frac": gbs(step_b, step_ms) / hbm,
        "note": "algorithmic bytes = the scored windows (fp32) + the retained K and V rows + Q, O",
        "scoring": {"kernel": "score_topk_query0_kernel (window scores, block max, radix top-k)", "ms": score_ms,
                    "algorithmic_bytes": score_b, "gbs": gbs(score_b, score_ms),
                    "frac": gbs(score_b, score_ms) / hbm},
        "pool": {"kernel": "pool_kernel (overlapping windows)", "ms": pool_ms, "gbs": gbs(pool_b, pool_ms),
                 "note": "bytes = each key once + the windows written; runs when blocks fill, not per step"},
        "peak_gbs": hbm, "peak_source": src,
    }


def run_bucket_bench(args, dev, stream, flush):
    """Times LSA flat bucket retrieval on the 1M-token workload: the bucket
    cache build of all 2048 cluster blocks of every (sequence, KV head) pair
    (one-time, then per new cluster block), and one decode step
    (sa_bucket_decode: centroid scores, top-256 buckets, expansion to the
    2048 long-range keys of best own cosine, attention)."""
    from top_block_sparse_b200 import sa
    w = WORKLOADS["decode_1m_buckets"]
    if args.small:
        w = w.scaled(batch=1, ctx_len=262144)
    bucket_keys = 2048
    inp = make_inputs(w, seed=8001, device=dev)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    del inp
    p = sa.params_for(w, out_dtype="bf16")
    R = sa.bucket_rows(p)
    mcap = 16 // w.pool_stride
    cents = torch.empty((w.batch, w.num_kv_heads, R, 128), device=dev)
    members = torch.empty((w.batch, w.num_kv_heads, R, mcap), device=dev, dtype=torch.int32)
    kcap = bucket_keys // w.pool_stride
    O = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), device=dev)
    sel = torch.empty((w.batch, w.num_kv_heads, w.top_k), device=dev, dtype=torch.int32)
    kept = torch.empty((w.batch, w.num_kv_heads, kcap), device=dev, dtype=torch.int32)
    ws = sa.alloc_workspace(p, sa.SA_OP_BUCKET_DECODE, device=dev)

    def build():
        sa.bucket_build(p, K, cents, members, stream=stream)

    def step():
        sa.bucket_decode(p, Q, K, V, cents, members, O, lse, sel, kept, bucket_keys, ws, stream=stream)

    build_ms = statistics.median(timed_steps(build, 3, 1, stream, flush))
    ms_l = timed_steps(step, args.bucket_steps, 3, stream, flush)
    ms = statistics.mean(ms_l)
    if sa.read_status(ws, stream) != sa.SA_OK:
        raise RuntimeError("device status word set during the bucket runs")
    hbm, _, _, src = peaks()
    pairs = w.batch * w.num_kv_heads
    nblk = w.ctx_len // w.block_size
    n_bkt = nblk * (w.block_size // 8)
    n_kept = int((kept >= 0).sum().item())
    s_end = min(w.sink_keys, w.ctx_len)
    w_keys = min(w.window_keys, w.ctx_len - s_end)
    attn_keys = pairs * (s_end + w_keys + w.n_q) + n_kept * w.pool_stride
    by = {"centroids": pairs * n_bkt * 128 * 4,
          "members_of_selected": pairs * w.top_k * mcap * 4,
          "own_cosine_keys": pairs * w.top_k * mcap * w.pool_stride * 128 * 2,
          "attention_kv": attn_keys * 128 * 2 * 2,
          "q_o": 2 * w.batch * w.n_q * w.num_q_heads * 128 * 2}
    step_b = sum(by.values())
    build_b = pairs * nblk * w.block_size * 128 * 2 + pairs * n_bkt * (128 * 4 + mcap * 4)
    gbs = lambda b, t: b / (t * 1e-3) / 1e9
    return {
        "workload": f"decode_1m_buckets: B={w.batch}, Hq={w.num_q_heads}, Hkv={w.num_kv_heads}, C={w.ctx_len}, "
                    f"d=128, bf16, LSA pool keys of {w.pool_stride} keys, {w.block_size // 8} Ward buckets per "
                    f"{w.block_size}-key cluster block ({n_bkt} per pair), top-{w.top_k} buckets by centroid "
                    f"cosine, {bucket_keys} long-range keys by own cosine, sink {w.sink_keys}, window "
                    f"{w.window_keys}",
        "ms": ms, "ms_spread": spread(ms_l),
        "queries_per_s": w.batch * w.n_q / (ms * 1e-3),
        "launches": 5,
        "algorithmic_bytes": step_b, "bytes": by,
        "achieved_gbs": gbs(step_b, ms), "frac": gbs(step_b, ms) / hbm,
        "kept_pool_keys_per_pair": n_kept / pairs,
        "build": {"kernel": "ward_kernel (pool keys, Ward rounds, centroids, one CTA per cluster block)",
                  "ms": build_ms, "blocks": pairs * nblk, "us_per_block_per_sm":
                      build_ms * 1e3 * torch.cuda.get_device_properties(dev).multi_processor_count / (pairs * nblk),
                  "hbm_bytes": build_b, "gbs": gbs(build_b, build_ms),
                  "note": "one-time per context (then per new cluster block): reads every key once, writes "
                          "the centroids and member lists"},
        "peak_gbs": hbm, "peak_source": src,
    }


def e2e_decode(args, w, p, Q, K, V, Kc, O, lse, idx, ws, stream, flush):
    """One decode step as a serving loop runs it: the new tokens' Q, K and V
    arrive packed in one pinned host buffer, one copy takes them to the
    device, sa_append_kv writes the K and V rows into the cache, the decode
    runs on the staged Q, and O is copied back to pinned host memory."""
    from top_block_sparse_b200 import sa
    C = w.ctx_len
    shape_new = (w.batch, w.num_kv_heads, w.n_q, w.head_dim)
    nq, nk = Q.numel(), w.batch * w.num_kv_heads * w.n_q * w.head_dim
    h_stage = torch.empty(nq + 2 * nk, dtype=Q.dtype, pin_memory=True)
    d_stage = torch.empty(nq + 2 * nk, dtype=Q.dtype, device=Q.device)
    h_stage[:nq].copy_(Q.flatten().cpu())
    h_stage[nq:nq + nk].copy_(K[:, :, C:C + w.n_q].flatten().cpu())
    h_stage[nq + nk:].copy_(V[:, :, C:C + w.n_q].flatten().cpu())
    Qs = d_stage[:nq].view(Q.shape)
    Kn = d_stage[nq:nq + nk].view(shape_new)
    Vn = d_stage[nq + nk:].view(shape_new)
    hO = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)

    def one():
        d_stage.copy_(h_stage, non_blocking=True)
        sa.append_kv(p, Kn, Vn, K, V, stream=stream)
        sa.sparse_attn_decode(p, Qs, K, V, Kc, O, lse, idx, ws, stream=stream)
        hO.copy_(O, non_blocking=True)

    n = max(50, args.steps // 4)
    with torch.cuda.stream(stream):
        ms = statistics.mean(timed_steps(one, n, args.warmup, stream, flush))
    # where the step's time goes: the same four operations with an event
    # between each, in a loop of their own (the events add a little)
    parts = ["h2d_copy", "append_kv", "decode", "d2h_copy"]
    ops = [lambda: d_stage.copy_(h_stage, non_blocking=True),
           lambda: sa.append_kv(p, Kn, Vn, K, V, stream=stream),
           lambda: sa.sparse_attn_decode(p, Qs, K, V, Kc, O, lse, idx, ws, stream=stream),
           lambda: hO.copy_(O, non_blocking=True)]
    rec = []
    with torch.cuda.stream(stream):
        for _ in range(3):
            for op in ops:
                op()
        torch.cuda.synchronize()
        queue_ahead(20)
        for _ in range(20):
            flush()
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(ops) + 1)]
            evs[0].record(stream)
            for op, ev in zip(ops, evs[1:]):
                op()
                ev.record(stream)
            rec.append(evs)
    torch.cuda.synchronize()
    breakdown = {name: statistics.median(r[i].elapsed_time(r[i + 1]) for r in rec) * 1e3
                 for i, name in enumerate(parts)}
    piped = e2e_pipelined(args, w, p, h_stage, nq, nk, shape_new, Q, K, V, Kc, O, lse, idx, ws, stream)
    return {"ms": piped, "serial_ms": ms, "h2d": h_stage.numel() * h_stage.element_size(),
            "d2h": hO.numel() * O.element_size(), "breakdown_us": breakdown}


def e2e_pipelined(args, w, p, h_stage, nq, nk, shape_new, Q, K, V, Kc, O, lse, idx, ws, stream):
    """The serving loop with each step's copies overlapped with the decodes
    next to it: two staging slots (device inputs, device and pinned host
    outputs), a copy-in stream, the compute stream and a copy-out stream.
    Step i copies its packed Q, K, V rows into slot i % 2 once the decode two
    steps back has read them, appends and decodes on the compute stream, and
    copies O out on the copy-out stream; the compute stream waits for the
    copy-out two steps back before it overwrites that slot's O.  Every step's
    host -> device and device -> host copies are inside the timed region;
    no L2 flush between steps (each step reads its ~310 MB of retained K/V,
    more than the 126 MB L2).  Returns ms per step over the timed steps."""
    from top_block_sparse_b200 import sa
    dev = Q.device
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    slots = []
    for _ in range(2):
        d = torch.empty(h_stage.shape, dtype=h_stage.dtype, device=dev)
        slots.append(dict(d=d, Q=d[:nq].view(Q.shape), Kn=d[nq:nq + nk].view(shape_new),
                          Vn=d[nq + nk:].view(shape_new), O=torch.empty_like(O),
                          hO=torch.empty(O.shape, dtype=O.dtype, pin_memory=True),
                          h2d=torch.cuda.Event(), comp=torch.cuda.Event(), d2h=torch.cuda.Event()))

    def run(n):
        for i in range(n):
            sl = slots[i % 2]
            h2d_s.wait_event(sl["comp"])
            with torch.cuda.stream(h2d_s):
                sl["d"].copy_(h_stage, non_blocking=True)
                sl["h2d"].record(h2d_s)
            stream.wait_event(sl["h2d"])
            stream.wait_event(sl["d2h"])
            sa.append_kv(p, sl["Kn"], sl["Vn"], K, V, stream=stream)
            sa.sparse_attn_decode(p, sl["Q"], K, V, Kc, sl["O"], lse, idx, ws, stream=stream)
            sl["comp"].record(stream)
            d2h_s.wait_event(sl["comp"])
            with torch.cuda.stream(d2h_s):
                sl["hO"].copy_(sl["O"], non_blocking=True)
                sl["d2h"].record(d2h_s)

    run(max(4, args.warmup))
    torch.cuda.synchronize()
    n = max(50, args.steps // 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        queue_ahead(n)
        e0.record(stream)
    h2d_s.wait_event(e0)
    run(n)
    stream.wait_event(slots[(n - 1) % 2]["d2h"])
    stream.wait_event(slots[n % 2]["d2h"])
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_32k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clock-period-ms", type=int, default=20, help="nvidia-smi sampling period")
    ap.add_argument("--cpu-pairs", type=int, default=16)
    ap.add_argument("--ref-pairs", type=int, default=4)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--prefill-steps", type=int, default=10)
    ap.add_argument("--verify-steps", type=int, default=10)
    ap.add_argument("--no-verify", action="store_true")
    ap.add_argument("--column-steps", type=int, default=5)
    ap.add_argument("--no-column", action="store_true")
    ap.add_argument("--overlap-steps", type=int, default=50)
    ap.add_argument("--config-steps", type=int, default=30)
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--no-overlap", action="store_true")
    ap.add_argument("--no-buckets", action="store_true")
    ap.add_argument("--no-parity", action="store_true",
                    help="skip the per-config comparison of the timed results with the float64 oracle")
    ap.add_argument("--bucket-steps", type=int, default=20)
    ap.add_argument("--column-tokens", type=int, default=None,
                    help="override the column workload's sequence length (smaller cases for ncu captures)")
    ap.add_argument("--prefill-tokens", type=int, default=None,
                    help="override the prefill length (smaller cases for ncu captures)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for ncu captures)")
    ap.add_argument("--small", action="store_true",
                    help="every leg at a reduced size (a few GB on the device, inputs still larger than L2), "
                         "for ncu captures of single kernels; its numbers are not the benchmark's")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.small:
        args.batch = args.batch or 16
        args.prefill_tokens = args.prefill_tokens or 16384
        args.column_tokens = args.column_tokens or 16384

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]
    if args.batch is not None:
        w = w.scaled(batch=args.batch)

    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, w, rank, world, local_rank)
        if line is not None and world == 1 and not args.no_cpu_baseline:
            inp = make_inputs(w.scaled(batch=2), seed=1000 + 1, device="cuda")
            pairs = cpu_pairs(w.scaled(batch=2), inp, args.cpu_pairs)
            full, dt, n = oracle_sample(w, pairs, w.batch * w.num_kv_heads)
            model, ncpu = cpu_info()
            line["cpu_baseline"] = {
                "value": w.batch * w.n_q / full, "unit": "queries/s", "cores": 1, "kind": "oracle",
                "sample": f"float64 oracle, {n} (sequence, KV head) pair evaluations over {len(pairs)} distinct "
                          f"pairs in {dt:.1f} s (one step has {w.batch * w.num_kv_heads} pairs), "
                          f"extrapolated to the full step; {model}, {ncpu} host cores, 1 used"}
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
