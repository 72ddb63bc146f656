"""Benchmark of the TurboQuant paged KV path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload target64x8k] [--fmt 4]

One step = append one new token per sequence (tq_quantize_append) + one
decode over the whole paged cache (tq_paged_decode), on the workload named in
``config.workload``.  Inputs are resident in HBM when the timed region
starts; the cache (570 MB for the default workload) is larger than L2, so no
flush is needed between steps.  ``value`` is the effective KV bandwidth of
the step (algorithmic cache bytes read per step / step time); the line also
carries seq/s, the per-step and bulk append bandwidth, a roofline object for
the decode kernel, an end-to-end number through the C ABI with host buffers,
the oracle as a CPU baseline, the SM clocks seen around the timed region,
and ``per_config``: the decode and bulk append of every other synthetic
workload and format, timed alone with the L2 flushed before every launch.

With --gpus N (launched by torch.distributed.run) every rank runs an
independent replica on its own GPU: the workload has no exchange step, so
there is no collective on the data path; only the timings are reduced (max
over ranks).  ``--impl reference`` times the CPU oracle instead (rank 0
only).
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_paged_kv_tq_b200 import workloads as W  # noqa: E402

METRIC = "paged TurboQuant decode: effective KV GB/s (% of HBM peak), seq/s; append GB/s"
DEFAULT_WORKLOAD = "target64x8k"
FALLBACK_HBM_GBS = 6650.0


def max_over_ranks(times, world: int, device=None):
    """Element-wise maximum of per-rank times (all ranks call it in the same
    order; a no-op for one rank)."""
    if world <= 1:
        return list(times)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(times), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(bytes_per_rank_step: int, world: int, ms_step: float) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's step time
    (replicas with the same per-rank workload: weak scaling)."""
    return world * bytes_per_rank_step / (ms_step * 1e-3) / 1e9


def describe(w: W.Workload, fmt: int) -> str:
    names = FORMAT_NAMES
    lens = (f"{int(w.seq_lens[0])} tokens" if np.all(w.seq_lens == w.seq_lens[0])
            else f"lengths {int(w.seq_lens.min())}-{int(w.seq_lens.max())}")
    return (f"{w.name}: batch {w.batch} x {lens}, {w.num_q_heads} q / {w.num_kv_heads} kv "
            f"heads, head_dim {w.head_dim}, page {w.page_size}, {names[fmt]}, q_len {w.q_len}; "
            f"each step appends 1 token per sequence then decodes")


def step_bytes(w: W.Workload, fmt: int):
    kv = w.tokens_read() * 2 * W.row_bytes(fmt)                 # K and V rows read
    new = w.batch * w.num_kv_heads * 2
    append = new * (2 * w.head_dim + W.row_bytes(fmt)) + w.batch * 8
    return kv, append


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


DECODE_SOURCES = ("decode.cu", "decode_tc.cu", "tq_device.cuh")


def _code_only(src: str) -> str:
    """C/CUDA source without comments, blank lines or trailing blanks, so a
    comment edit does not change the fingerprint of the code."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def decode_sources_sha256() -> str:
    """sha256 over the code (comments stripped) of the decode kernels'
    sources, in DECODE_SOURCES order."""
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "quantized_paged_kv_tq_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()


def profiled_traffic(kernel: str):
    """dram read+write bytes per launch recorded in profiles/<kernel>*.md
    (e.g. k_decode_i8_target64x8k_turbo4.md), valid only while the decode
    sources are unchanged (their sha256 is recorded as decode_src_sha256)."""
    sha = decode_sources_sha256()
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for name in sorted(os.listdir(pdir)):
        if not name.startswith(kernel):
            continue
        vals = {}
        with open(os.path.join(pdir, name)) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    vals[k.strip()] = v.strip()
        if vals.get("decode_src_sha256") == sha and "traffic_bytes_per_launch" in vals:
            return float(vals["traffic_bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: int):
        self.gpu = gpu
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                if len(r) >= 9:
                    rows.append([x.strip() for x in r])
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ CPU oracle
def oracle_sample_decode(w: W.Workload, fmt: int, ntok: int, kv_head: int = 0, seq: int = 0):
    """Time the CPU oracle decoding one (sequence, kv head): the first `ntok`
    tokens of sequence `seq`, its `group` query heads, from a cache the
    oracle builds itself (untimed).  Returns (seconds, algorithmic bytes)."""
    import oracle
    P = w.page_size
    npages = (ntok + P - 1) // P
    phys = w.page_table[seq, :npages].astype(np.int64)
    slots = (phys[:, None] * P + np.arange(P)[None, :]).ravel()
    k, v = w.kv_for_slots(slots)
    k = np.ascontiguousarray(k[:, kv_head:kv_head + 1])
    v = np.ascontiguousarray(v[:, kv_head:kv_head + 1])
    bb = oracle.block_bytes(fmt, w.head_dim, P)
    if fmt == 16:
        kp = np.zeros((npages, 1, P, w.head_dim), np.uint16)
        vp = np.zeros_like(kp)
        oracle.append_bf16(k, v, np.arange(npages * P), P, kp, vp)
    else:
        kp = np.zeros((npages, 1, bb), np.uint8)
        vp = np.zeros_like(kp)
        oracle.quantize_append(k, v, np.arange(npages * P), fmt, P, kp, vp)
    q = w.queries()[seq:seq + 1, :, kv_head * w.group:(kv_head + 1) * w.group]
    pt = np.arange(npages, dtype=np.int32)[None]
    t0 = time.perf_counter()
    oracle.paged_decode(np.ascontiguousarray(q), fmt, P, kp, vp, pt,
                        np.array([ntok], np.int32), 1)
    dt = time.perf_counter() - t0
    return dt, ntok * 2 * W.row_bytes(fmt)


def cpu_baseline(w, fmt, budget_s=12.0):
    """The oracle, single-threaded, on a bounded sample of the workload."""
    n, secs, nbytes = 0, 0.0, 0
    ntok = int(w.seq_lens[0])
    while secs < budget_s and n < w.batch * w.num_kv_heads:
        seq, kvh = divmod(n, w.num_kv_heads)
        dt, b = oracle_sample_decode(w, fmt, min(ntok, int(w.seq_lens[seq])), kvh, seq)
        secs += dt
        nbytes += b
        n += 1
    return {"value": nbytes / secs / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} (sequence, kv head) decodes of up to {ntok} tokens x {w.group} "
                      f"q heads each ({nbytes / 1e6:.1f} MB of cache), single-threaded C, "
                      f"{os.cpu_count()} host cores present",
            "seconds": secs}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = W.make(args.workload)
    fmt = args.fmt or w.formats[0]
    budget = 90.0
    # calibrate the per-step sample so the whole run stays within ~budget
    ncal = min(1024, int(w.seq_lens[0]))
    dt, b = oracle_sample_decode(w, fmt, ncal)
    per_tok = dt / ncal
    ntok = int(max(16, min(int(w.seq_lens[0]), budget / (args.steps + args.warmup) / per_tok)))
    ntok = max(16, (ntok // 16) * 16)
    for i in range(args.warmup):
        oracle_sample_decode(w, fmt, ntok, i % w.num_kv_heads)
    secs, nbytes = 0.0, 0
    for i in range(args.steps):
        dt, b = oracle_sample_decode(w, fmt, ntok, i % w.num_kv_heads)
        secs += dt
        nbytes += b
    value = nbytes / secs / 1e9
    line = {"metric": METRIC, "impl": "reference", "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(w, fmt), "global_batch": w.batch,
                       "seq_len": int(w.seq_lens.max()), "parallelism": "cpu-1thread"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"each step: one (sequence, kv head) decode over "
                                       f"{ntok} tokens x {w.group} q heads, single-threaded C"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- GPU arm
# The (workload, format) pairs timed in `per_config`: every format of every
# synthetic workload (the bench workload itself is the line's main part).
PER_CONFIG = (("tiny", 4), ("batch8", 4), ("cbatch64", 3), ("cbatch64", 8), ("cbatch64", 16),
              ("cbatch64", 17), ("long128k", 4), ("long128k", 2), ("specverify", 4))
FORMAT_NAMES = {2: "turbo2", 3: "turbo3", 4: "turbo4", 8: "turbo8", 16: "bf16", 17: "fp8"}
L2_FLUSH_BYTES = 256 << 20         # > the 126 MB L2


def decode_kernel_label(fmt: int, G: int) -> str:
    """Name of the decode kernel instantiation the library launches for a
    format and G = q_len x GQA rows per kv head (a label for the report)."""
    if fmt == 16:
        return "k_decode<16>"
    if fmt != 17 and G >= 128:
        return f"k_prefill_tc<{fmt}>"
    rows = 4 if G <= 4 else (8 if G <= 8 else 16)
    if fmt == 17:
        return f"k_decode_tc<8,{rows},fp8>"
    if fmt == 3 or rows > 4:
        return f"k_decode_tc<{fmt},{rows}>"
    return f"k_decode_i8<{fmt},{rows}>"


def append_bytes(tokens: int, num_kv_heads: int, fmt: int, head_dim: int = 128) -> int:
    """Algorithmic bytes of appending `tokens` tokens: bf16 K and V read,
    codes and scales (or bf16 rows) written, one int64 slot read."""
    return tokens * (num_kv_heads * 2 * (2 * head_dim + W.row_bytes(fmt)) + 8)


def median(xs):
    return statistics.median(xs) if xs else float("nan")


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (libtq.so has no CPU path)")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from quantized_paged_kv_tq_b200 import build as tqbuild
    tqbuild.build()
    from quantized_paged_kv_tq_b200 import tq

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))

    def d_bf16(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(
            torch.bfloat16).to(dev)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def resident_fill_inputs(w, upto=None):
        """Every fill slot of w (positions [0, upto[b]) of each sequence) with
        its K/V values, resident on the device: (slots, k, v)."""
        n = len(w.fill_slots(upto))
        k_d = torch.empty((n, w.num_kv_heads, w.head_dim), dtype=torch.bfloat16, device=dev)
        v_d = torch.empty_like(k_d)
        s_d = torch.empty(n, dtype=torch.int64, device=dev)
        i = 0
        for slots, k, v in w.iter_fill(1 << 16, upto=upto):
            m = len(slots)
            k_d[i:i + m] = d_bf16(k)
            v_d[i:i + m] = d_bf16(v)
            s_d[i:i + m] = torch.from_numpy(slots.astype(np.int64)).to(dev)
            i += m
        return s_d, k_d, v_d

    def appender(cache, fmt):
        if fmt == 16:
            return lambda k, v, s: tq.tq_append_bf16(k, v, s, cache)
        return lambda k, v, s: tq.tq_quantize_append(k, v, s, fmt, cache)

    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def timed(fn, reps, flush):
        """Median / min device time (ms) of fn over reps launches, each
        bracketed by CUDA events on the launching stream; the L2 is flushed
        (an untimed 256 MB write) before each one when `flush`."""
        starts, ends = [ev() for _ in range(reps)], [ev() for _ in range(reps)]
        for r in range(reps):
            if flush:
                flush_buf.zero_()
            starts[r].record(stream)
            fn()
            ends[r].record(stream)
        torch.cuda.synchronize()
        t = [a.elapsed_time(b) for a, b in zip(starts, ends)]
        return median(t), min(t)

    def bulk_append_report(w, fmt, fill, s_d, k_d, v_d, flush):
        """The fill of a whole context as one append call (idempotent, so it
        can be repeated): time and bandwidth."""
        ms, ms_min = timed(lambda: fill(k_d, v_d, s_d), 3, flush)
        nbytes = append_bytes(int(s_d.numel()), w.num_kv_heads, fmt)
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"tokens": int(s_d.numel()), "us": ms * 1e3, "bytes": nbytes, "gbs": gbs,
                "frac_of_hbm": gbs / peak}

    # ================================================================ main
    w = W.make(args.workload)
    fmt = args.fmt or w.formats[0]

    # ---- resident cache: every context token but the last of each sequence,
    # appended by one timed bulk call
    cache = tq.Cache(fmt, w.num_pages, w.num_kv_heads, w.page_size, device=dev)
    fill = appender(cache, fmt)
    s_d, k_d, v_d = resident_fill_inputs(w, upto=w.seq_lens - 1)
    fill(k_d, v_d, s_d)
    main_bulk = bulk_append_report(w, fmt, fill, s_d, k_d, v_d,
                                   flush=append_bytes(int(s_d.numel()), w.num_kv_heads, fmt)
                                   < 2 * L2_FLUSH_BYTES)
    del s_d, k_d, v_d
    torch.cuda.empty_cache()

    # per-step inputs: a few distinct new-token sets, appended at position
    # seq_len - 1 of every sequence
    n_variants = 4
    new_slots = torch.from_numpy(np.array([w.slots_of(b, [int(w.seq_lens[b]) - 1])[0]
                                           for b in range(w.batch)], np.int64)).to(dev)
    new_k, new_v = [], []
    for i in range(n_variants):
        k, v = w.new_tokens(i, w.batch)
        new_k.append(d_bf16(k))
        new_v.append(d_bf16(v))
    q = d_bf16(w.queries())
    pt = torch.from_numpy(w.page_table).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    out = torch.empty((w.batch, w.q_len, w.num_q_heads, w.head_dim), dtype=torch.float32,
                      device=dev)
    max_len = w.max_seq_len
    ws = cache.workspace(w.batch, w.q_len, w.num_q_heads, max_len)
    decode = tq.tq_paged_decode_bf16 if fmt == 16 else tq.tq_paged_decode

    def append(i):
        j = i % n_variants
        fill(new_k[j], new_v[j], new_slots)

    def dec():
        decode(q, cache, pt, sl, w.q_len, out, max_seq_len=max_len, workspace=ws)

    torch.cuda.synchronize()

    # ---- in-run HBM roofline probes (untimed region)
    nbytes = 1 << 30
    a = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    bbuf = torch.empty_like(a)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    copy_ms, read_ms = [], []
    for _ in range(3):
        tq.tq_hbm_copy(a, bbuf)
        tq.tq_hbm_read(a, sink)
    for _ in range(10):
        e0, e1, e2 = ev(), ev(), ev()
        e0.record()
        tq.tq_hbm_copy(a, bbuf)
        e1.record()
        tq.tq_hbm_read(a, sink)
        e2.record()
        e2.synchronize()
        copy_ms.append(e0.elapsed_time(e1))
        read_ms.append(e1.elapsed_time(e2))
    copy_gbs = 2 * nbytes / (min(copy_ms) * 1e-3) / 1e9
    read_gbs = nbytes / (min(read_ms) * 1e-3) / 1e9
    del a, bbuf
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # ---- clocks: sampled from here through the timed region; an untimed
    # soak of about a second first, so the record covers a busy GPU
    clocks = ClockSampler(local)
    clocks.start()
    t_end = time.perf_counter() + 1.0
    i = 0
    while time.perf_counter() < t_end:
        for _ in range(50):
            append(i)
            dec()
            i += 1
        torch.cuda.synchronize()

    # ---- warm-up
    for i in range(args.warmup):
        append(i)
        dec()
    torch.cuda.synchronize()

    # ---- timed region (device time, CUDA events on the launching stream)
    K = args.steps
    ev_a = [ev() for _ in range(K)]
    ev_b = [ev() for _ in range(K)]
    ev_c = [ev() for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(K):
        ev_a[i].record(stream)
        append(i)
        ev_b[i].record(stream)
        dec()
        ev_c[i].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if clk is not None:
        clk["window"] = "about 1 s of untimed steps, the warm-up steps and the timed steps"
    if world > 1:
        dist.barrier()
    total_ms = ev_a[0].elapsed_time(ev_c[-1])
    append_ms = [ev_a[i].elapsed_time(ev_b[i]) for i in range(K)]
    decode_ms = [ev_b[i].elapsed_time(ev_c[i]) for i in range(K)]

    # ---- end to end through the C ABI with host buffers: every step copies
    # q, the new K/V, their slots, the page table and the lengths from
    # pinned host memory and reads the output back
    e2e_steps = max(3, min(K, 200))

    def pinned(t):
        return torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t.cpu())

    h_q, h_s, h_pt, h_sl = pinned(q), pinned(new_slots), pinned(pt), pinned(sl)
    h_k = [pinned(x) for x in new_k]
    h_v = [pinned(x) for x in new_v]
    h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    d_q, d_k, d_v, d_s = (torch.empty_like(q), torch.empty_like(new_k[0]),
                          torch.empty_like(new_v[0]), torch.empty_like(new_slots))
    d_pt, d_sl = torch.empty_like(pt), torch.empty_like(sl)
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k[0], h_v[0], h_s, h_pt, h_sl))
    d2h = h_out.numel() * 4

    def e2e_step(i):
        j = i % n_variants
        d_q.copy_(h_q, non_blocking=True)
        d_k.copy_(h_k[j], non_blocking=True)
        d_v.copy_(h_v[j], non_blocking=True)
        d_s.copy_(h_s, non_blocking=True)
        d_pt.copy_(h_pt, non_blocking=True)
        d_sl.copy_(h_sl, non_blocking=True)
        fill(d_k, d_v, d_s)
        decode(d_q, cache, d_pt, d_sl, w.q_len, out, max_seq_len=max_len, workspace=ws)
        h_out.copy_(out, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = ev(), ev()
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    err = cache.read_error()
    if err:
        raise SystemExit(f"device error word set: 0x{err:x}")
    del cache, ws, q, pt, sl, out, new_k, new_v
    torch.cuda.empty_cache()

    # ---- reduce over ranks: max of each time
    ms_step, dec_avg, app_avg, e2e_ms = max_over_ranks(
        [total_ms / K, sum(decode_ms) / K, sum(append_ms) / K, e2e_ms], world, dev)

    kv_bytes, app_bytes = step_bytes(w, fmt)
    value = job_throughput(kv_bytes, world, ms_step)
    achieved = kv_bytes / (dec_avg * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": describe(w, fmt), "global_batch": w.batch * world,
                   "seq_len": int(w.seq_lens.max()), "parallelism": f"dp{world}",
                   "l2": f"inputs larger than L2: {kv_bytes / 1e6:.0f} MB of cache read per "
                         f"step vs 126 MB L2, no flush"},
        "seq_per_s": world * w.batch / (ms_step * 1e-3),
        "decode_kv_gbs": achieved,
        "decode_ms": dec_avg,
        "decode_kernel": decode_kernel_label(fmt, w.q_len * w.group),
        "append_gbs": app_bytes / (app_avg * 1e-3) / 1e9,
        "append_ms": app_avg,
        "append_bulk": main_bulk,
        "hbm_inrun_gbs": {"copy": copy_gbs, "read": read_gbs},
        "frac_of_hbm": {"step": (value / world) / peak, "decode_kernel": achieved / peak,
                        "decode_vs_inrun_copy": achieved / copy_gbs,
                        "decode_vs_inrun_read": achieved / read_gbs,
                        "append_bulk": main_bulk["frac_of_hbm"]},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": profiled_traffic(
                         f"{decode_kernel_label(fmt, w.q_len * w.group).split('<')[0]}_"
                         f"{args.workload}_{FORMAT_NAMES[fmt]}"),
                     "peak_source": f"hbm_gbs of {peak_kind}",
                     "algorithmic_bytes_per_launch": kv_bytes},
        "e2e": {"value": world * kv_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": 2 * K,
        "clocks": clk,
    }

    # ================================================== every configuration
    if not args.no_per_config:
        line["per_config"] = per_config(tq, dev, peak, resident_fill_inputs, appender, timed,
                                        bulk_append_report)
        line["extra"] = extra_rows(tq, dev, peak, timed)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, fmt)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def per_config(tq, dev, peak, resident_fill_inputs, appender, timed, bulk_append_report):
    """Decode (and bulk append) of every synthetic workload and format, each
    alone on the GPU with inputs resident and the L2 flushed before every
    timed launch: decode us, KV GB/s, seq/s (tokens/s for verify windows) and
    fractions of the HBM peak; for shared prefixes also the fraction counted
    on unique bytes."""
    import torch
    rows = []
    for name in dict.fromkeys(n for n, _ in PER_CONFIG):
        w = W.make(name)
        s_d, k_d, v_d = resident_fill_inputs(w)
        q = torch.from_numpy(w.queries().view(np.int16)).view(torch.bfloat16).to(dev)
        pt = torch.from_numpy(w.page_table).to(dev)
        sl = torch.from_numpy(w.seq_lens).to(dev)
        out = torch.empty((w.batch, w.q_len, w.num_q_heads, w.head_dim), dtype=torch.float32,
                          device=dev)
        for nm, fmt in PER_CONFIG:
            if nm != name:
                continue
            cache = tq.Cache(fmt, w.num_pages, w.num_kv_heads, w.page_size, device=dev)
            fill = appender(cache, fmt)
            fill(k_d, v_d, s_d)
            bulk = bulk_append_report(w, fmt, fill, s_d, k_d, v_d, flush=True)
            ws = cache.workspace(w.batch, w.q_len, w.num_q_heads, w.max_seq_len)
            fn = tq.tq_paged_decode_bf16 if fmt == 16 else tq.tq_paged_decode

            def dec():
                fn(q, cache, pt, sl, w.q_len, out, max_seq_len=w.max_seq_len, workspace=ws)

            for _ in range(3):
                dec()
            ms, ms_min = timed(dec, 20, flush=True)
            err = cache.read_error()
            if err:
                raise SystemExit(f"{name}/{fmt}: device error word set: 0x{err:x}")
            kv = w.tokens_read() * 2 * W.row_bytes(fmt)
            gbs = kv / (ms * 1e-3) / 1e9
            r = {"workload": name, "format": FORMAT_NAMES[fmt],
                 "kernel": decode_kernel_label(fmt, w.q_len * w.group),
                 "batch": w.batch, "q_len": w.q_len, "q_heads": w.num_q_heads,
                 "kv_heads": w.num_kv_heads, "page_size": w.page_size,
                 "tokens": int(w.seq_lens.sum()),
                 "decode_us": ms * 1e3, "decode_us_min": ms_min * 1e3,
                 "kv_bytes": kv, "kv_gbs": gbs, "frac_of_hbm": gbs / peak,
                 "seq_per_s": w.batch / (ms * 1e-3), "append_bulk": bulk,
                 "l2": "flushed before every timed launch"}
            if w.q_len > 1:
                r["tokens_per_s"] = w.batch * w.q_len / (ms * 1e-3)
            uniq = w.unique_tokens_read() * 2 * W.row_bytes(fmt)
            if uniq != kv:
                r["unique_kv_bytes"] = uniq
                r["unique_frac_of_hbm"] = uniq / (ms * 1e-3) / 1e9 / peak
            rows.append(r)
            del cache, ws
            torch.cuda.empty_cache()
        del s_d, k_d, v_d, q, pt, sl, out
        torch.cuda.empty_cache()
    return rows


def extra_rows(tq, dev, peak, timed):
    """Two measurements beside the per-configuration decodes: a chunk of
    prefill tokens attending causally over a quantised context (q_len 256,
    1024 rows per kv head), and the append + decode step of batch8 eager
    against replayed as one CUDA graph.  L2 flushed before every launch."""
    import torch
    rows = []

    def d_bf16(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(
            torch.bfloat16).to(dev)

    # ---- prefill chunk
    w = W.make("prefill256")
    cache = tq.Cache(4, w.num_pages, w.num_kv_heads, w.page_size, device=dev)
    for slots, k, v in w.iter_fill(1 << 16):
        tq.tq_quantize_append(d_bf16(k), d_bf16(v), torch.from_numpy(slots.astype(np.int64)).to(dev),
                              4, cache)
    q = d_bf16(w.queries())
    pt = torch.from_numpy(w.page_table).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    out = torch.empty((w.batch, w.q_len, w.num_q_heads, w.head_dim), dtype=torch.float32,
                      device=dev)
    ws = cache.workspace(w.batch, w.q_len, w.num_q_heads, w.max_seq_len)

    def dec():
        tq.tq_paged_decode(q, cache, pt, sl, w.q_len, out, max_seq_len=w.max_seq_len, workspace=ws)

    for _ in range(3):
        dec()
    ms, ms_min = timed(dec, 20, flush=True)
    if cache.read_error():
        raise SystemExit("prefill chunk: device error word set")
    G = w.q_len * w.group
    # (row, visible key) pairs: row t of the chunk sees seq_len - q_len + t + 1 keys
    pairs = sum(w.group * (int(L) - w.q_len + t + 1) for L in w.seq_lens for t in range(w.q_len))
    pairs *= w.num_kv_heads
    flops = pairs * 4 * w.head_dim                      # QK and PV, 2 flops per MAC
    uniq = int(w.seq_lens.sum()) * w.num_kv_heads * 2 * W.row_bytes(4)
    rows.append({"workload": "prefill256: batch 4 x 4096-token context, the last 256 tokens "
                             "a prefill chunk, 32 q / 8 kv heads, page 16, turbo4",
                 "kernel": decode_kernel_label(4, G), "rows_per_kv_head": G,
                 "decode_us": ms * 1e3, "decode_us_min": ms_min * 1e3,
                 "chunk_tokens_per_s": w.batch * w.q_len / (ms * 1e-3),
                 "tflops": flops / (ms * 1e-3) / 1e12, "flops": flops,
                 "unique_kv_bytes": uniq, "unique_frac_of_hbm": uniq / (ms * 1e-3) / 1e9 / peak,
                 "l2": "flushed before every timed launch"})
    del cache, ws, q, out
    torch.cuda.empty_cache()

    # ---- batch8 step: eager against one CUDA graph
    w = W.make("batch8")
    cache = tq.Cache(4, w.num_pages, w.num_kv_heads, w.page_size, device=dev)
    for slots, k, v in w.iter_fill(1 << 16, upto=w.seq_lens - 1):
        tq.tq_quantize_append(d_bf16(k), d_bf16(v), torch.from_numpy(slots.astype(np.int64)).to(dev),
                              4, cache)
    new_slots = torch.from_numpy(np.array([w.slots_of(b, [int(w.seq_lens[b]) - 1])[0]
                                           for b in range(w.batch)], np.int64)).to(dev)
    k, v = w.new_tokens(0, w.batch)
    nk, nv = d_bf16(k), d_bf16(v)
    q = d_bf16(w.queries())
    pt = torch.from_numpy(w.page_table).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    out = torch.empty((w.batch, w.q_len, w.num_q_heads, w.head_dim), dtype=torch.float32,
                      device=dev)
    ws = cache.workspace(w.batch, w.q_len, w.num_q_heads, w.max_seq_len)
    side = torch.cuda.Stream(device=dev)
    g = tq.StepGraph(cache, side, q, pt, sl, w.q_len, out, w.max_seq_len, k=nk, v=nv,
                     slot_mapping=new_slots, workspace=ws)

    def eager():
        tq.tq_quantize_append(nk, nv, new_slots, 4, cache)
        tq.tq_paged_decode(q, cache, pt, sl, w.q_len, out, max_seq_len=w.max_seq_len,
                           workspace=ws)

    def graph():
        g.launch(torch.cuda.current_stream())

    for _ in range(3):
        eager()
        graph()
    ms_e, _ = timed(eager, 50, flush=True)
    ms_g, _ = timed(graph, 50, flush=True)
    if cache.read_error():
        raise SystemExit("graph step: device error word set")
    rows.append({"workload": "batch8 step: append 1 token per sequence + decode, 8 x 4096, "
                             "32 q / 8 kv heads, page 16, turbo4",
                 "eager_us": ms_e * 1e3, "graph_us": ms_g * 1e3,
                 "l2": "flushed before every timed step"})
    del g, cache, ws
    torch.cuda.empty_cache()
    return rows


def launch_only(args):
    """Fill the workload's cache (bulk calls of up to 2^18 tokens), then
    launch the decode, or the bulk append of the whole context in one call,
    args.steps times with nothing else in between: the launch sequence an
    ncu capture of one kernel selects from."""
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (libtq.so has no CPU path)")
    from quantized_paged_kv_tq_b200 import build as tqbuild
    tqbuild.build()
    from quantized_paged_kv_tq_b200 import tq
    dev = torch.device("cuda", 0)
    w = W.make(args.workload)
    fmt = args.fmt or w.formats[0]

    def d_bf16(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(
            torch.bfloat16).to(dev)

    cache = tq.Cache(fmt, w.num_pages, w.num_kv_heads, w.page_size, device=dev)

    def fill(k, v, s):
        if fmt == 16:
            tq.tq_append_bf16(k, v, s, cache)
        else:
            tq.tq_quantize_append(k, v, s, fmt, cache)

    if args.launch_only == "append":
        parts = list(w.iter_fill(1 << 18))
        s_d = torch.cat([torch.from_numpy(s.astype(np.int64)) for s, _, _ in parts]).to(dev)
        k_d = torch.cat([d_bf16(k) for _, k, _ in parts])
        v_d = torch.cat([d_bf16(v) for _, _, v in parts])
        del parts
        for _ in range(args.steps):
            fill(k_d, v_d, s_d)
    else:
        for s, k, v in w.iter_fill(1 << 18):
            fill(d_bf16(k), d_bf16(v), torch.from_numpy(s.astype(np.int64)).to(dev))
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        q = d_bf16(w.queries())
        pt = torch.from_numpy(w.page_table).to(dev)
        sl = torch.from_numpy(w.seq_lens).to(dev)
        out = torch.empty((w.batch, w.q_len, w.num_q_heads, w.head_dim), dtype=torch.float32,
                          device=dev)
        ws = cache.workspace(w.batch, w.q_len, w.num_q_heads, w.max_seq_len)
        decode = tq.tq_paged_decode_bf16 if fmt == 16 else tq.tq_paged_decode
        for _ in range(args.steps):
            decode(q, cache, pt, sl, w.q_len, out, max_seq_len=w.max_seq_len, workspace=ws)
    torch.cuda.synchronize()
    err = cache.read_error()
    print(f"launch-only {args.launch_only} {args.workload} format {fmt}: {args.steps} launches, "
          f"device error word {err:#x}")
    return 0 if err == 0 else 1


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=W.ALL)
    ap.add_argument("--fmt", type=int, default=0, help="cache format (default: workload's first)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-configuration decode and bulk-append timings")
    ap.add_argument("--launch-only", choices=("decode", "append"),
                    help="for a profiler: fill the workload's cache, then launch only the "
                         "decode (or the bulk quantise-append of the whole context) --steps "
                         "times, untimed, and print one status line")
    args = ap.parse_args(argv)
    if args.launch_only:
        return launch_only(args)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
