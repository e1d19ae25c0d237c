"""Benchmark of the paged MLA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload v3] [--impl reference]

One step = one pass of the whole hot path over one batch: the split-KV scheduler
(mla_get_metadata), the split kernel and the LSE combine (mla_decode_fwd), all through
the C ABI, captured once as a CUDA graph and replayed per step. The default workload is
DeepSeek-V3-shaped decode: batch 128, s_q 1, 128 query heads, one shared 576-dim latent
head, lengths uniform in [1, 8192], 64-token bf16 pages randomly permuted in the pool.
Inputs are seeded synthetic data.

Rank 0 prints one JSON line. `value` is algorithmic HBM bytes (every visible KV row
once, q, out, lse) of all ranks' steps divided by the max-over-ranks device time. A step
that reads at least twice the 126 MB L2 runs back to back with the others (inputs larger
than L2); smaller ones get an untimed 256 MB L2 write before each, and every workload is
also reported with that flush (`l2_write_flush`);
`roofline` relates the decode call to the measured peaks; `e2e` repeats the measurement
with q, block table and lengths copied from pinned host memory and the outputs read
back every step; `cpu_baseline` times the fp64 CPU oracle on a bounded sample.
With N > 1 each rank decodes its own batch (weak scaling, no data-path collective).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_paged_kv_06_b200 import workloads as wl  # noqa: E402
from mla_paged_kv_06_b200.shard import max_over_ranks, rank_seed  # noqa: E402

L2_FLUSH_BYTES = 256 << 20          # > 126 MB L2
L2_BYTES = 126 << 20                # B200 L2
HEADSTART_CYCLES_PER_STEP = 200_000 # an untimed sleep kernel of ~100 us per queued step
TIMING_NOTE = ("each step is one replay of a CUDA graph of the C-ABI calls mla_get_metadata "
               "+ mla_decode_fwd (metadata, split and combine kernels), between CUDA events "
               "on the launching stream; the decode call and the metadata call are also "
               "timed alone the same way")
kBlockRoom = 64                     # tokens per page
LAUNCHES_PER_STEP = 3               # metadata, split kernel, combine kernel
SPLIT_KV_WORLD = 4                  # ranks of the split-KV-across-devices measurement
SPLIT_KV_LENGTHS = [65536] * 4      # its sequences: long contexts split over the ranks
CONFIG_ORDER = ["tiny", "uniform", "v3", "spec", "skewed"]   # the `configs` entries


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="v3", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--split-kv", type=int, default=SPLIT_KV_WORLD,
                    help="ranks of the split-KV-across-devices timing (<= 1 skips it)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the other workloads after the main one")
    ap.add_argument("--config-cpu-seconds", type=float, default=4.0)
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def metric_name():
    return "MLA decode HBM GB/s, TFLOPS and μs/call at b=128,h_q=128; fraction of roofline"


def workload_config(x, name):
    w = wl.WORKLOADS[name]
    return {"workload": f"{name}: {w.description}", "batch": x.batch, "s_q": x.s_q,
            "h_q": x.h_q, "d": 576, "dv": 512, "block_size": 64, "causal": bool(x.causal),
            "num_blocks": x.num_blocks, "total_tokens": int(x.seqlens.sum()),
            "seed": x.seed}


# ---------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        if not getattr(self, "lines", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [c.strip() for c in ln.split(",")]
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        loaded = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------
def cpu_baseline(x, seconds):
    """Time the fp64 oracle on a bounded sample of the workload's sequences."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
    except Exception:
        cores = os.cpu_count() or 1
    order = sorted(range(x.batch), key=lambda b: int(x.seqlens[b]))
    picked, spent, nbytes = [], 0.0, 0
    g = torch.Generator().manual_seed(123)
    perm = torch.randperm(x.batch, generator=g).tolist()
    for b in perm:
        t0 = time.perf_counter()
        oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, x.causal,
                      batch_indices=[b])
        spent += time.perf_counter() - t0
        picked.append(b)
        nbytes += wl.algorithmic_work(x.seqlens[b:b + 1], x.s_q, x.h_q, x.causal)[0]
        if spent >= seconds:
            break
    del order
    return {"value": nbytes / spent / 1e9, "unit": "GB/s", "cores": int(cores),
            "kind": "oracle",
            "sample": f"{len(picked)} of {x.batch} sequences of the same workload "
                      f"({sum(int(x.seqlens[b]) for b in picked)} tokens), one oracle.decode "
                      f"call each, {spent:.1f} s"}


def run_reference(args):
    """Reference arm: the CPU oracle, timed on the host cores, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    x = wl.make_workload(args.workload, seed=args.seed)
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(x.batch, generator=g).tolist()
    per_step = 2                       # sequences per step: a bounded sample
    try:
        from threadpoolctl import threadpool_info
        cores = max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
    except Exception:
        cores = os.cpu_count() or 1

    def step(k):
        bs = [perm[(k * per_step + j) % x.batch] for j in range(per_step)]
        oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, x.causal,
                      batch_indices=bs)
        return sum(wl.algorithmic_work(x.seqlens[b:b + 1], x.s_q, x.h_q, x.causal)[0]
                   for b in bs)

    for k in range(args.warmup):
        step(k)
    t0 = time.perf_counter()
    nbytes = 0
    for k in range(args.steps):
        nbytes += step(args.warmup + k)
    dt = time.perf_counter() - t0
    val = nbytes / dt / 1e9
    line = {"metric": metric_name(), "value": val, "unit": "GB/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(x, args.workload),
            "cpu_baseline": {"value": val, "unit": "GB/s", "cores": int(cores),
                             "kind": "oracle",
                             "sample": f"{per_step} sequences per step of the same workload"},
            "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------
def time_split_kv(mla, flush, stream, steps, seed):
    """Split-KV across devices, its device work timed on this GPU, on the case it is for:
    a few sequences too long for one GPU's share (SPLIT_KV_LENGTHS tokens, 128 heads).
    Their pages are split over SPLIT_KV_WORLD ranks (splitkv.plan_kv_split); each rank's
    slice is decoded to fp32 partials (mla_get_metadata + mla_decode_fwd_partial, L2
    flushed before each call, as in the main measurement) one rank after another, then
    the stacked parts are merged (mla_combine_partials). The all-gather between the
    ranks' GPUs is not part of it: its size is reported instead."""
    from mla_paged_kv_06_b200 import splitkv
    world = SPLIT_KV_WORLD
    x = wl.make_paged_inputs(SPLIT_KV_LENGTHS, 1, 128, seed=seed + 11)
    plan = splitkv.plan_kv_split(x.seqlens, world, x.s_q, x.causal)
    nsm = mla.default_num_sms()
    rank_us, rank_gbs, parts_o, parts_l = [], [], [], []
    for g in range(world):
        xr = splitkv.make_kv_slice(x, plan, g)
        q, kc, bt, sl = xr.q.cuda(), xr.kcache.cuda(), xr.block_table.cuda(), xr.seqlens.cuda()
        meta = torch.empty(mla.mla_metadata_ints(nsm), dtype=torch.int32, device="cuda")
        ns = torch.empty(mla.mla_num_splits_len(xr.batch, xr.h_q, xr.s_q), dtype=torch.int32,
                         device="cuda")
        ws = torch.empty(mla.mla_workspace_bytes(xr.batch, xr.h_q, xr.s_q, nsm),
                         dtype=torch.uint8, device="cuda")
        o = torch.empty((xr.batch, xr.s_q, xr.h_q, 512), dtype=torch.float32, device="cuda")
        lse = torch.empty((xr.batch, xr.h_q, xr.s_q), dtype=torch.float32, device="cuda")

        def call():
            mla.mla_get_metadata(sl, xr.h_q, xr.s_q, nsm, meta, ns)
            mla.mla_decode_fwd_partial(q, kc, bt, sl, xr.scale, xr.causal, meta, ns, ws, o, lse)

        for _ in range(3):
            flush.zero_()
            call()
        ts = []
        for _ in range(steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        us = statistics.median(ts)
        nb, _ = wl.algorithmic_work(xr.seqlens, xr.s_q, xr.h_q, xr.causal)
        rank_us.append(us)
        rank_gbs.append(nb / (us * 1e-6) / 1e9)
        parts_o.append(o)
        parts_l.append(lse)
        del q, kc, bt, sl, ws
    o_parts, l_parts = torch.stack(parts_o), torch.stack(parts_l)
    out = torch.empty((x.batch, x.s_q, x.h_q, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((x.batch, x.h_q, x.s_q), dtype=torch.float32, device="cuda")
    for _ in range(3):
        mla.mla_combine_partials(o_parts, l_parts, out, lse)
    torch.cuda.synchronize()
    # replayed from a CUDA graph: back-to-back calls from Python would time the host
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(steps):
            mla.mla_combine_partials(o_parts, l_parts, out, lse)
    graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    graph.replay()
    b.record(stream)
    b.synchronize()
    combine_us = a.elapsed_time(b) * 1e3 / steps
    del graph
    st, word = mla.mla_get_last_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the split-KV timing: {mla.status_string(st)} {word:#x}")
    exchange = x.batch * x.s_q * x.h_q * (512 + 1) * 4
    total, _ = wl.algorithmic_work(x.seqlens, x.s_q, x.h_q, x.causal)
    return {"world": world, "workload": f"b={x.batch} s_q=1 h_q=128 L={SPLIT_KV_LENGTHS[0]}",
            "rank_decode_us": rank_us, "rank_GB/s": rank_gbs, "combine_us": combine_us,
            "exchange_bytes_per_rank": exchange,
            "GB/s_without_exchange": total / ((max(rank_us) + combine_us) * 1e-6) / 1e9,
            "note": f"each rank holds about 1/{world} of every sequence's pages; rank decodes "
                    "(fp32 partials, L2 flushed before each) and the merge of the gathered "
                    "parts (replayed from a CUDA graph) timed one after another on this GPU; "
                    "GB/s_without_exchange is "
                    "the whole problem's bytes over the slowest rank plus the merge; the "
                    "all-gather of exchange_bytes_per_rank per rank between GPUs is not "
                    "timed"}


# B200 nominal peaks (HGX HBM3e bandwidth, dense bf16 tensor rate), reported beside the
# measured ones as the stricter reference
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0


def flush_free(nbytes):
    """True when a step reads at least twice L2: then steps run back to back with no flush
    (their inputs exceed L2), otherwise an untimed write of 256 MB flushes L2 before each."""
    return nbytes >= 2 * L2_BYTES


def l2_note(nbytes, no_flush):
    if no_flush:
        return (f"no flush: each step reads {nbytes / 1e6:.0f} MB, "
                f"{nbytes / L2_BYTES:.1f}x the 126 MB L2; the steps run back to back, queued "
                "behind an untimed sleep kernel so that no host gap enters the timing")
    return ("L2 flushed (256 MB write, untimed) before every step")


def capture(parts):
    """A CUDA graph of the calls in `parts`, made in order (their launches through the C
    ABI are recorded once and replayed as one unit, as a serving loop replays its step)."""
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    # thread-local capture: under torchrun the process group's watchdog thread keeps
    # querying its events, which a global-mode capture would refuse
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        for f in parts:
            f()
    torch.cuda.synchronize()
    return g


def time_replays(g, steps, flush, stream, no_flush):
    """Per-step times (ms) of `steps` replays of graph g, each between two CUDA events on
    `stream`. With no_flush the replays run back to back (a sleep kernel queued first lets
    the host enqueue them all before the first starts); otherwise an untimed 256 MB write
    flushes L2 before each."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    if no_flush:
        torch.cuda._sleep(HEADSTART_CYCLES_PER_STEP * steps)
    for a, b in ev:
        if not no_flush:
            flush.zero_()
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


class StepTimer:
    """The step (metadata + decode call), the decode call alone and the metadata call
    alone, each captured as a CUDA graph after `warmup` eager steps."""

    def __init__(self, meta_fn, decode_fn, warmup, flush, stream, no_flush):
        for _ in range(max(warmup, 3)):
            if not no_flush:
                flush.zero_()
            meta_fn()
            decode_fn()
        torch.cuda.synchronize()
        self.graphs = {"step": capture([meta_fn, decode_fn]), "decode": capture([decode_fn]),
                       "metadata": capture([meta_fn])}
        self.flush, self.stream, self.no_flush = flush, stream, no_flush
        for g in self.graphs.values():
            time_replays(g, 3, flush, stream, no_flush)

    def time(self, which, steps, no_flush=None):
        nf = self.no_flush if no_flush is None else no_flush
        return time_replays(self.graphs[which], steps, self.flush, self.stream, nf)

    def release(self):
        self.graphs = {}


def roofline_fracs(nbytes, nflops, seconds, hbm_peak, tf_peak):
    t_bytes = nbytes / (hbm_peak * 1e9)
    t_flops = nflops / (tf_peak * 1e12)
    n_bytes = nbytes / (NOMINAL_HBM_GBS * 1e9)
    n_flops = nflops / (NOMINAL_BF16_TFLOPS * 1e12)
    return {"bound": "hbm" if t_bytes >= t_flops else "tensor",
            "hbm_frac": t_bytes / seconds, "tensor_frac": t_flops / seconds,
            "roofline_frac": max(t_bytes, t_flops) / seconds,
            "roofline_frac_nominal": max(n_bytes, n_flops) / seconds}


def flushed_entry(nbytes, step_ms, decode_ms, hbm_peak):
    """The same workload timed with a 256 MB L2 write before every step. Evicting those
    dirty lines writes up to 126 MB back to HBM inside the timed decode call."""
    t = statistics.mean(decode_ms) / 1e3
    return {"us_per_call": statistics.median(step_ms) * 1e3,
            "us_per_call_decode": statistics.median(decode_ms) * 1e3,
            "GB/s": nbytes / t / 1e9, "hbm_frac": nbytes / t / 1e9 / hbm_peak}


def time_config(mla, name, seed, flush, stream, steps, warmup, hbm_peak, tf_peak,
                cpu_seconds, with_cpu):
    """One workload's decode timed the way the main measurement times it (metadata and
    decode call timed with CUDA events on the launching stream; no flush when the step
    reads at least twice L2, else an untimed L2 flush before each step; the flushed
    timing is also reported), against its own roofline."""
    x = wl.make_workload(name, seed=seed)
    d = dict(q=x.q.cuda(), kcache=x.kcache.cuda(), block_table=x.block_table.cuda(),
             seqlens=x.seqlens.cuda())
    nsm = mla.default_num_sms()
    meta = torch.empty(mla.mla_metadata_ints(nsm), dtype=torch.int32, device="cuda")
    ns = torch.empty(mla.mla_num_splits_len(x.batch, x.h_q, x.s_q), dtype=torch.int32,
                     device="cuda")
    ws = torch.empty(mla.mla_workspace_bytes(x.batch, x.h_q, x.s_q, nsm), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((x.batch, x.s_q, x.h_q, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((x.batch, x.h_q, x.s_q), dtype=torch.float32, device="cuda")
    nbytes, nflops = wl.algorithmic_work(x.seqlens, x.s_q, x.h_q, x.causal)
    no_flush = flush_free(nbytes)
    timer = StepTimer(
        lambda: mla.mla_get_metadata(d["seqlens"], x.h_q, x.s_q, nsm, meta, ns),
        lambda: mla.mla_decode_fwd(d["q"], d["kcache"], d["block_table"], d["seqlens"],
                                   x.scale, x.causal, meta, ns, ws, out, lse),
        warmup, flush, stream, no_flush)
    step_ms, decode_ms, meta_ms = (timer.time(w, steps) for w in ("step", "decode", "metadata"))
    fl = ({w: timer.time(w, steps, no_flush=False) for w in ("step", "decode")} if no_flush
          else {"step": step_ms, "decode": decode_ms})
    timer.release()
    st, word = mla.mla_get_last_device_error()
    if st != 0:
        raise RuntimeError(f"device error in {name}: {mla.status_string(st)} {word:#x}")
    t = statistics.mean(decode_ms) / 1e3
    rows = x.s_q * x.h_q
    entry = {"workload": workload_config(x, name)["workload"], "batch": x.batch,
             "s_q": x.s_q, "h_q": x.h_q, "total_tokens": int(x.seqlens.sum()),
             "kernel": "1-CTA (rows <= 64)" if rows <= 64 else "2-CTA pairs",
             "l2": l2_note(nbytes, no_flush),
             "work_units": mla.mla_num_work_units(nsm, x.h_q, x.s_q),
             "us_per_call": statistics.median(step_ms) * 1e3,
             "us_per_call_decode": statistics.median(decode_ms) * 1e3,
             "us_per_call_metadata": statistics.median(meta_ms) * 1e3,
             "GB/s": nbytes / t / 1e9, "TFLOPS": nflops / t / 1e12,
             "algorithmic_bytes": nbytes, "algorithmic_flops": nflops,
             "roofline": roofline_fracs(nbytes, nflops, t, hbm_peak, tf_peak),
             "l2_write_flush": flushed_entry(nbytes, fl["step"], fl["decode"], hbm_peak)}
    if with_cpu:
        entry["cpu_baseline"] = cpu_baseline(x, cpu_seconds)
    del d, ws, out, lse
    torch.cuda.empty_cache()
    return entry


def time_fp8(mla, seed, flush, stream, steps, warmup, hbm_peak):
    """Decode over an FP8 latent cache (mla_decode_fwd_fp8) on the uniform workload's
    shape, timed like the main measurement. The cache is the uniform pool quantized on the
    GPU by mla_kv_append_fp8 (16 rows per page per call); algorithmic bytes count 656 per
    token (the row format) plus q, out and lse."""
    x = wl.make_workload("uniform", seed=seed)
    nb = x.num_blocks
    kc8 = torch.zeros((nb, 64, mla.MLA_FP8_ROW_BYTES), dtype=torch.uint8, device="cuda")
    rows = x.kcache.view(nb, 64, 576).cuda()
    ident = torch.arange(nb, dtype=torch.int32, device="cuda").view(nb, 1)
    for j in range(4):
        at = torch.full((nb,), 16 * j, dtype=torch.int32, device="cuda")
        mla.mla_kv_append_fp8(rows[:, 16 * j:16 * (j + 1)].contiguous(), ident, at, kc8)
    del rows
    d = dict(q=x.q.cuda(), block_table=x.block_table.cuda(), seqlens=x.seqlens.cuda())
    nsm = mla.default_num_sms()
    meta = torch.empty(mla.mla_metadata_ints(nsm), dtype=torch.int32, device="cuda")
    ns = torch.empty(mla.mla_num_splits_len(x.batch, x.h_q, x.s_q), dtype=torch.int32,
                     device="cuda")
    ws = torch.empty(mla.mla_workspace_bytes(x.batch, x.h_q, x.s_q, nsm), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((x.batch, x.s_q, x.h_q, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((x.batch, x.h_q, x.s_q), dtype=torch.float32, device="cuda")

    # timed like the bf16 decode call: graph replays of the call alone (the schedule is
    # the metadata call's, the same for both formats)
    timer = StepTimer(
        lambda: mla.mla_get_metadata(d["seqlens"], x.h_q, x.s_q, nsm, meta, ns),
        lambda: mla.mla_decode_fwd_fp8(d["q"], kc8, d["block_table"], d["seqlens"], x.scale,
                                       x.causal, meta, ns, ws, out, lse),
        warmup, flush, stream, False)
    ts = [t * 1e3 for t in timer.time("decode", steps)]
    timer.release()
    st, word = mla.mla_get_last_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the FP8 decode: {mla.status_string(st)} {word:#x}")
    tokens = int(x.seqlens.sum())
    rows_total = x.batch * x.s_q * x.h_q
    nbytes = tokens * mla.MLA_FP8_ROW_BYTES + rows_total * (1152 + 1024 + 4)
    us = statistics.median(ts)
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"workload": "uniform shape over an FP8 cache (656-byte rows: E4M3 latent codes, "
                        "four fp32 group scales, bf16 rope)",
            "us_per_call": us, "GB/s": gbs, "hbm_frac": gbs / hbm_peak,
            "algorithmic_bytes": nbytes,
            "bf16_cache_bytes_same_workload": tokens * 1152 + rows_total * (1152 + 1024 + 4),
            "note": "mla_decode_fwd_fp8 alone (graph replays, as the decode call of every "
                    "workload), L2 flushed (256 MB write) before each: "
                    "its reads are under twice L2 (compare the uniform entry's "
                    "l2_write_flush figure); the cache was quantized on the GPU by "
                    "mla_kv_append_fp8"}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    from mla_paged_kv_06_b200 import mla

    # each rank decodes its own batch of the same shape (weak scaling)
    x = wl.make_workload(args.workload, seed=rank_seed(args.seed, rank))
    d = dict(q=x.q.cuda(), kcache=x.kcache.cuda(), block_table=x.block_table.cuda(),
             seqlens=x.seqlens.cuda())
    nsm = mla.default_num_sms()
    meta = torch.empty(mla.mla_metadata_ints(nsm), dtype=torch.int32, device="cuda")
    ns = torch.empty(mla.mla_num_splits_len(x.batch, x.h_q, x.s_q), dtype=torch.int32,
                     device="cuda")
    ws = torch.empty(mla.mla_workspace_bytes(x.batch, x.h_q, x.s_q, nsm), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((x.batch, x.s_q, x.h_q, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((x.batch, x.h_q, x.s_q), dtype=torch.float32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    nbytes, nflops = wl.algorithmic_work(x.seqlens, x.s_q, x.h_q, x.causal)

    no_flush = flush_free(nbytes)
    timer = StepTimer(
        lambda: mla.mla_get_metadata(d["seqlens"], x.h_q, x.s_q, nsm, meta, ns),
        lambda: mla.mla_decode_fwd(d["q"], d["kcache"], d["block_table"], d["seqlens"],
                                   x.scale, x.causal, meta, ns, ws, out, lse),
        args.warmup, flush, stream, no_flush)
    st, word = mla.mla_get_last_device_error()
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {mla.status_string(st)} {word:#x}")

    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_ms = timer.time("step", args.steps)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms = max_over_ranks(sum(step_ms), dist, "cuda")
    # the decode call and the metadata call alone, and the steps with a 256 MB L2 write
    # before each (every rank, in the same order)
    decode_ms = timer.time("decode", args.steps)
    meta_ms = timer.time("metadata", args.steps)
    fl = ({w: timer.time(w, args.steps, no_flush=False) for w in ("step", "decode")}
          if no_flush else {"step": step_ms, "decode": decode_ms})
    timer.release()
    st, word = mla.mla_get_last_device_error()
    if st != 0:
        raise RuntimeError(f"device error during timing: {mla.status_string(st)} {word:#x}")

    # End to end through the public calls with host buffers, run the way a serving loop
    # runs them: every step copies its q, block table and lengths in from pinned host
    # memory and reads its out and lse back, on their own streams, so that step k+1's
    # copy-in and step k-1's copy-out overlap step k's compute. Events order every reuse
    # of the two buffer sets. The KV cache (the step's dominant input) stays resident
    # as decode state and exceeds L2, so no flush separates these steps.
    hq = x.q.pin_memory()
    hbt = x.block_table.pin_memory()
    hsl = x.seqlens.pin_memory()
    dq = [d["q"], torch.empty_like(d["q"])]
    dbt = [d["block_table"], torch.empty_like(d["block_table"])]
    dsl = [d["seqlens"], torch.empty_like(d["seqlens"])]
    douts = [out, torch.empty_like(out)]
    dlses = [lse, torch.empty_like(lse)]
    hout = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    hlse = [torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True) for _ in range(2)]
    h2d = hq.numel() * 2 + hbt.numel() * 4 + hsl.numel() * 4
    d2h = hout[0].numel() * 2 + hlse[0].numel() * 4
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def run_e2e(n):
        ev_comp, ev_out = [], []
        first = torch.cuda.Event(enable_timing=True)
        first.record(s_in)
        for k in range(n):
            i = k % 2
            if k >= 2:
                s_in.wait_event(ev_comp[k - 2])          # step k-2 no longer reads set i
            with torch.cuda.stream(s_in):
                dq[i].copy_(hq, non_blocking=True)
                dbt[i].copy_(hbt, non_blocking=True)
                dsl[i].copy_(hsl, non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
            s_comp.wait_event(ev_in)
            if k >= 2:
                s_comp.wait_event(ev_out[k - 2])         # set i's outputs were read back
            mla.mla_get_metadata(dsl[i], x.h_q, x.s_q, nsm, meta, ns, stream=s_comp)
            mla.mla_decode_fwd(dq[i], d["kcache"], dbt[i], dsl[i], x.scale, x.causal, meta, ns,
                               ws, douts[i], dlses[i], stream=s_comp)
            ec = torch.cuda.Event()
            ec.record(s_comp)
            ev_comp.append(ec)
            s_out.wait_event(ec)
            with torch.cuda.stream(s_out):
                hout[i].copy_(douts[i], non_blocking=True)
                hlse[i].copy_(dlses[i], non_blocking=True)
            eo = torch.cuda.Event(enable_timing=True)
            eo.record(s_out)
            ev_out.append(eo)
        return first, ev_out[-1]

    torch.cuda.synchronize()
    run_e2e(3)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    a, b = run_e2e(args.steps)
    b.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b), dist, "cuda")
    torch.cuda.synchronize()

    # Cache append (the step before each decode): one new latent row per sequence of the
    # batch, into a pool of its own whose last page has room for it.
    ap = wl.make_paged_inputs([kBlockRoom - 1] * x.batch, 1, 8, seed=args.seed + 7)
    ap_kc, ap_bt = ap.kcache.cuda(), ap.block_table.cuda()
    ap_sl = torch.full((x.batch,), kBlockRoom - 1, dtype=torch.int32, device="cuda")
    ap_new = torch.randn((x.batch, 1, 576), generator=torch.Generator().manual_seed(3)).to(
        torch.bfloat16).cuda()
    for _ in range(3):
        mla.mla_kv_append(ap_new, ap_bt, ap_sl, ap_kc)
    torch.cuda.synchronize()
    # replayed from a CUDA graph so the figure is the GPU's, not Python's launch cost
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(args.steps):
            mla.mla_kv_append(ap_new, ap_bt, ap_sl, ap_kc)
    graph.replay()
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    graph.replay()
    eb.record(stream)
    eb.synchronize()
    append_us = ea.elapsed_time(eb) * 1e3 / args.steps
    del graph
    # the same rows quantized into an FP8 cache of the same pages (mla_kv_append_fp8)
    ap_kc8 = torch.zeros((ap_kc.shape[0], kBlockRoom, mla.MLA_FP8_ROW_BYTES), dtype=torch.uint8,
                         device="cuda")
    for _ in range(3):
        mla.mla_kv_append_fp8(ap_new, ap_bt, ap_sl, ap_kc8)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(args.steps):
            mla.mla_kv_append_fp8(ap_new, ap_bt, ap_sl, ap_kc8)
    graph.replay()
    torch.cuda.synchronize()
    ea.record(stream)
    graph.replay()
    eb.record(stream)
    eb.synchronize()
    append_fp8_us = ea.elapsed_time(eb) * 1e3 / args.steps
    del graph
    st, word = mla.mla_get_last_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the cache append: {mla.status_string(st)} {word:#x}")

    split_kv = time_split_kv(mla, flush, stream, args.steps, args.seed) if args.split_kv > 1 else None

    hbm_peak, tf_peak, peak_kind = peaks()
    fp8 = None if args.no_configs else time_fp8(mla, rank_seed(args.seed, rank), flush, stream,
                                                args.steps, args.warmup, hbm_peak)
    # every workload of the benchmark in the same run, each against its own roofline
    configs = {}
    if not args.no_configs:
        for name in CONFIG_ORDER:
            if name == args.workload:
                continue
            configs[name] = time_config(
                mla, name, rank_seed(args.seed, rank), flush, stream, args.steps, args.warmup,
                hbm_peak, tf_peak, args.config_cpu_seconds,
                with_cpu=rank == 0 and world == 1 and not args.no_cpu_baseline)
    avg_decode_s = statistics.mean(decode_ms) / 1e3
    achieved_gbs = nbytes / avg_decode_s / 1e9
    achieved_tf = nflops / avg_decode_s / 1e12
    t_bytes = nbytes / (hbm_peak * 1e9)
    t_flops = nflops / (tf_peak * 1e12)
    bound = "hbm" if t_bytes >= t_flops else "tensor"
    traffic = None
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(prof):
        try:
            with open(prof) as f:
                tj = json.load(f)
            if tj.get("workload") == args.workload and tj.get("kernel_rev") == KERNEL_REV:
                traffic = tj.get("bytes_per_launch")
        except Exception:
            traffic = None
    roof = {"bound": bound, "kernel": "mla_decode_fwd (split kernel + combine kernel)",
            "achieved": achieved_gbs if bound == "hbm" else achieved_tf,
            "peak": hbm_peak if bound == "hbm" else tf_peak,
            "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured"
            else "fallback",
            "frac": (achieved_gbs / hbm_peak) if bound == "hbm" else (achieved_tf / tf_peak),
            "traffic": traffic,
            "hbm_frac": achieved_gbs / hbm_peak, "tensor_frac": achieved_tf / tf_peak,
            "roofline_frac": max(t_bytes, t_flops) / avg_decode_s,
            "roofline_frac_nominal": max(nbytes / (NOMINAL_HBM_GBS * 1e9),
                                         nflops / (NOMINAL_BF16_TFLOPS * 1e12)) / avg_decode_s,
            "algorithmic_bytes": nbytes, "algorithmic_flops": nflops}

    value = nbytes * args.steps * world / (total_ms / 1e3) / 1e9
    line = {"metric": metric_name(), "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 q and cache; seeded lengths and page permutation)",
            "config": dict(workload_config(x, args.workload),
                           l2=l2_note(nbytes, no_flush), parallelism=f"replicas x{world}",
                           timing=TIMING_NOTE),
            "tflops": nflops * args.steps * world / (total_ms / 1e3) / 1e12,
            "us_per_call": statistics.median(step_ms) * 1e3,
            "us_per_call_decode": statistics.median(decode_ms) * 1e3,
            "us_per_call_metadata": statistics.median(meta_ms) * 1e3,
            # 2-CTA clusters (more than 64 query rows) or CTAs the chip runs at once: the
            # clusters a chip fits vary with its SM layout, and the 2-CTA kernel's time with them
            "work_units": mla.mla_num_work_units(nsm, x.h_q, x.s_q),
            "roofline": roof,
            "l2_write_flush": flushed_entry(nbytes, fl["step"], fl["decode"], hbm_peak),
            "e2e": {"value": nbytes * args.steps * world / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / args.steps,
                    "note": "KV cache resident in HBM as decode state; per-step inputs are "
                            "q, block table and lengths, copied in from pinned memory, and "
                            "out + lse read back, every step; copy-in, compute and "
                            "copy-out of consecutive steps overlap on three streams; the "
                            "KV cache exceeds L2 (no flush between these steps)"},
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "kv_append": {"us_per_call": append_us, "rows": x.batch,
                          "GB/s": 2 * 1152 * x.batch / (append_us * 1e-6) / 1e9,
                          "note": "mla_kv_append, one new token per sequence; calls replayed "
                                  "back to back from a CUDA graph on L2-resident rows (a "
                                  "latency figure)"},
            "kv_append_fp8": {"us_per_call": append_fp8_us, "rows": x.batch,
                              "note": "mla_kv_append_fp8: the same rows quantized into the "
                                      "656-byte FP8 row format, replayed from a CUDA graph"},
            "split_kv": split_kv,
            "fp8_cache": fp8,
            "clocks": clk.summary()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(x, args.cpu_seconds)
    if not args.no_configs:
        main_entry = {"workload": line["config"]["workload"], "batch": x.batch, "s_q": x.s_q,
                      "h_q": x.h_q, "total_tokens": int(x.seqlens.sum()),
                      "kernel": "1-CTA (rows <= 64)" if x.s_q * x.h_q <= 64 else "2-CTA pairs",
                      "l2": line["config"]["l2"], "work_units": line["work_units"],
                      "us_per_call": line["us_per_call"],
                      "us_per_call_decode": line["us_per_call_decode"],
                      "us_per_call_metadata": line["us_per_call_metadata"],
                      "GB/s": achieved_gbs, "TFLOPS": achieved_tf,
                      "algorithmic_bytes": nbytes, "algorithmic_flops": nflops,
                      "roofline": roofline_fracs(nbytes, nflops, avg_decode_s, hbm_peak, tf_peak),
                      "l2_write_flush": line["l2_write_flush"]}
        if "cpu_baseline" in line:
            main_entry["cpu_baseline"] = line["cpu_baseline"]
        line["configs"] = {n: (main_entry if n == args.workload else configs[n])
                           for n in CONFIG_ORDER}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# Bumped whenever the split kernel changes, so stale ncu traffic is never reported.
KERNEL_REV = "pair-7"

if __name__ == "__main__":
    sys.exit(main())
