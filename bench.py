"""Benchmark: exact top-k inner-product search on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

The index is built once (K1 normalises the raw corpus, timed on its own and
reported under ``kernels.k1_index_build``). One step is then the query side of
the hot path over one batch: L2-normalise the raw queries, score every query
against every candidate, filter and select the exact top-k (``tt_score_topk``).
Inputs are seeded synthetic data (``workloads.py``) resident in HBM before
timing starts. The default workload is the large-batch contraction (N =
50,000,000, d = 128, B = 1024, k = 1000; 12.8 GB of bf16 rows, larger than L2);
corpora under 1 GB are timed with an L2 flush before every step.

Multi-GPU (torchrun, one process per GPU), two modes:
  --mode replicas (default): every rank runs an independent replica of the
    workload on its own queries - no collective in the data path; the value
    is the total over ranks (weak scaling), timed as the max over ranks.
  --mode shard: the ranks split one corpus by rows; every step each rank
    normalises and scores its shard, the [b, k] lists are all-gathered over
    NCCL and merged (tt_merge_topk) on every rank; the value is the one
    workload's scores per second (strong scaling).

With --op inbatch_softmax the step is instead the in-batch sampled-softmax
training loss (tt_inbatch_softmax: logits, logQ correction, accidental-hit and
padding masks, log-sum-exp, cross-entropy and the mean) over one seeded
training batch (--batch, default 65,536 users x 65,536 candidates, d = 64);
the value is logits per second.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import csv
import dataclasses
import datetime as dt
import json
import math
import os
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "query-candidate scores/sec (exact top-k)"
UNIT = "scores/s"
DEFAULT_WORKLOAD = "large_batch"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PATH_NAMES = {1: "streaming", 2: "tensor-core", 3: "tensor-core (SM pairs)"}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per unit of work
# from ncu captures of a kernel, with the sha256 of the kernel's source file at
# capture time; `traffic` is reported only while that file is unchanged. Units:
# bytes per level row scanned (level-0 capture, applied to every level of a
# step, like `achieved`).
TRAFFIC = {
    # ncu --set full --import-source no --clock-control none -k regex:k3_pair -s 8 -c 1 on `python bench.py
    # --workload large_batch --n 4000000 --steps 3 --warmup 3 --no-e2e --no-cpu-baseline` (level-0 pass,
    # 4,000,000 rows): 1056.253 MB read + 27.411 MB written; scaled to the full corpus by rows scanned
    ("k3_pair", "large_batch"): {"bytes_per_row": 270.916, "src": "exact_inner_product_b200/csrc/k_tensor_pair.cu",
                                 "sha": "8651752c99e9b667e5bf49f551f1fe48623ddfd247f4338868a4988d77e9c7bf"},
    # ncu --set full --import-source no --clock-control none -k regex:k3_tensor -s 8 -c 1 on `python bench.py
    # --workload masked_fused --n 4000000 --steps 3 --warmup 3 --no-e2e --no-cpu-baseline` (level-0 pass,
    # 4,000,000 rows): 4145.305 MB read + 66.409 MB written; scaled to the full corpus by rows scanned
    ("k3_tensor", "masked_fused"): {"bytes_per_row": 1052.929, "src": "exact_inner_product_b200/csrc/k_tensor.cu",
                                    "sha": "d8167680c49f9dea7eb98c71503e446b913a57b8dae7e637926c337aee2309ab"},
}


def source_sha(rel_path):
    import hashlib
    with open(os.path.join(ROOT, rel_path), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def recorded_traffic(kernel: str, workload: str, rows: int):
    rec = TRAFFIC.get((kernel, workload))
    if rec is None:
        return None
    try:
        if source_sha(rec["src"]) != rec["sha"]:
            return None
    except OSError:
        return None
    return rec["bytes_per_row"] * rows


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        out = {k: float(p[k]) for k in FALLBACK_PEAKS}
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"
    # the SM clock seen while the sustained GEMM peak was measured, when recorded
    for key, val in p.items() if isinstance(p, dict) else ():
        if "sustained" in key and "mhz" in key.lower() and isinstance(val, (int, float)):
            out["sustained_mhz"] = float(val)
    return out, "measured"


# ---------------------------------------------------------------------------
# algorithmic work of one step
# ---------------------------------------------------------------------------
def elem_bytes(name):
    return {"f32": 4, "bf16": 2}[name]


def work_model(w: W.Workload, plan: dict, int8: bool = False):
    s_in = elem_bytes(w.raw_dtype)
    if int8:  # normalise + code: read the raw rows, write codes and one scale per row
        k1_bytes = w.n * w.d * s_in + w.n * w.d + w.n * 4
        s_corpus = 1
    elif w.store == "raw":
        k1_bytes = w.n * w.d * s_in + w.n * 4
        s_corpus = s_in
    else:
        s_out = elem_bytes(w.store)
        k1_bytes = w.n * w.d * (s_in + s_out)
        s_corpus = s_out
    rows_scanned = sum(plan["rows"])
    per_row = w.d * s_corpus + (4 if (w.store == "raw" or int8) else 0)
    score_bytes = rows_scanned * per_row + (w.n // 8 if w.masked else 0)
    score_flops = 2.0 * w.b * w.d * rows_scanned
    return {"k1_bytes": k1_bytes, "score_bytes": score_bytes, "score_flops": score_flops,
            "rows_scanned": rows_scanned}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for rec in csv.reader(f):
                if len(rec) < 10:
                    continue
                try:
                    ts = dt.datetime.strptime(rec[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(rec[2]), float(rec[3]), [r.strip() for r in rec[6:10]]))
                except Exception:
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i in range(4) if r[3][i].lower().startswith("active")})
        return {"sm_mhz": float(np.median([r[1] for r in inside])), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":  # host-only arm: no process group, rank 0 works alone
        return world, rank, local
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as tdist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        tdist.init_process_group(backend, timeout=dt.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as tdist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the workload
# ---------------------------------------------------------------------------
def oracle_sample_run(w: W.Workload, raw_c_np, raw_q_np, excl_np, n_s: int, b_s: int):
    import oracle
    corpus = raw_c_np[:n_s]
    qs = raw_q_np[:b_s]
    excl = None if excl_np is None else excl_np[: (n_s + 31) // 32]
    t0 = time.perf_counter()
    if w.store == "raw":
        norms = oracle.row_norms(corpus)
        stored = corpus
    else:
        norms = None
        stored = oracle.normalize(corpus, w.store)
    qn = oracle.normalize(qs, w.query_dtype)
    oracle.topk(qn, stored, min(w.k, n_s), tau=float(np.float32(w.tau)), norms=norms, exclude=excl)
    return time.perf_counter() - t0


def oracle_sample_size(w: W.Workload, raw_c_np, raw_q_np, excl_np, seconds: float):
    """Pick (n_s, b_s) so that one oracle run takes about `seconds`."""
    import oracle
    threads = oracle.max_threads()
    b_s = min(w.b, max(1, threads))
    n_s = min(w.n, 20_000)
    t = oracle_sample_run(w, raw_c_np, raw_q_np, excl_np, n_s, b_s)
    while n_s < w.n and t < seconds / 4:
        n_s = min(w.n, n_s * 4)
        t = oracle_sample_run(w, raw_c_np, raw_q_np, excl_np, n_s, b_s)
    if t > 0 and n_s < w.n:
        n_s = int(min(w.n, max(1000, n_s * seconds / t)))
    return n_s, b_s, threads


def cpu_baseline(w: W.Workload, raw_c_np, raw_q_np, excl_np, seconds=12.0):
    """The oracle on a bounded prefix of the workload (host arrays: the first
    rows of the raw corpus, the raw queries, the packed mask words)."""
    wp = dataclasses.replace(w, n=min(w.n, raw_c_np.shape[0]))
    n_s, b_s, threads = oracle_sample_size(wp, raw_c_np, raw_q_np, excl_np, seconds)
    t = oracle_sample_run(wp, raw_c_np, raw_q_np, excl_np, n_s, b_s)
    return {"value": b_s * n_s / t, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{b_s} queries x first {n_s} candidates of {w.name} (normalise + score + full sort), "
                      f"one run of {t:.2f} s"}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def workload_from_args(args) -> W.Workload:
    """The named workload, resized by --n/--b/--k (smaller cases for profiling)."""
    over = {key: getattr(args, key) for key in ("n", "b", "k") if getattr(args, key)}
    return W.workload(args.workload, **over)


# Rows of the raw corpus kept on the host for the CPU baseline (the oracle
# times a bounded prefix of the corpus, never the whole of a large one).
CPU_SAMPLE_ROWS = 4_000_000
# Corpora smaller than this are scored with an L2 flush before every step
# (the 126 MB L2 could otherwise hold part of them between steps); a corpus of
# at least twice the L2 size, streamed front to back every step, leaves no
# reusable lines behind (ncu: the one-query pass reads its whole 256 MB from
# DRAM in back-to-back steps), and runs without one.
FLUSH_BELOW_BYTES = 2 * 126_000_000
K1_REPS = 3


def run_ours(args, world, rank, local):
    import exact_inner_product_b200 as tt
    from exact_inner_product_b200 import shard

    sharded = args.mode == "shard"
    w = workload_from_args(args)
    if world > 1 and not sharded:  # each rank: its own queries (independent replica)
        w = W.workload(w.name, n=w.n, b=w.b, k=w.k, seed=w.seed + 7919 * rank)
    dev = torch.device("cuda", local)
    raw_c = W.corpus(w, dev)
    raw_q = W.queries(w, dev)
    excl = W.exclusion_bits(w, dev)
    w_all = w
    if sharded:
        # this rank's rows of the one corpus; queries are the same on every rank
        bounds = shard.shard_bounds(w.n, world)
        start, count = bounds[rank]
        raw_c = raw_c[start:start + count].clone()
        excl = shard.exclude_slice(excl, start, count)
        torch.cuda.empty_cache()
        w = dataclasses.replace(w, n=count)
    # the CPU baseline's rows, copied before the raw corpus is released
    host_sample = None
    if rank == 0 and not args.no_cpu_baseline:
        host_sample = (W.to_numpy_rows(raw_c[:min(w.n, CPU_SAMPLE_ROWS)]), raw_q.cpu().numpy(),
                       None if excl is None else excl.cpu().numpy().view(np.uint32))
    int8 = args.quant == "int8"
    if int8:
        prepared = torch.empty((w.n, w.d), dtype=torch.int8, device=dev)
        scales = torch.empty((w.n,), dtype=torch.float32, device=dev)
        mode = None
    elif w.store == "raw":
        prepared = torch.empty((w.n,), dtype=torch.float32, device=dev)
        mode = tt.TT_NORM_FUSED
    else:
        prepared = torch.empty((w.n, w.d), dtype=torch.float32 if w.store == "f32" else torch.bfloat16,
                               device=dev)
        mode = tt.TT_NORM_STORE
    q_torch_dtype = torch.float32 if w.query_dtype == "f32" else torch.bfloat16
    qn = torch.empty((w.b, w.d), dtype=q_torch_dtype, device=dev)
    out_ids = torch.empty((w.b, w.k), dtype=torch.int32, device=dev)
    out_scores = torch.empty((w.b, w.k), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # ---- index time: normalise (or code) the raw corpus once; K1 is timed
    # here, on its own, and reported under `kernels` (it is not part of a step)
    def build_index(make_index):
        if int8:
            return tt.tt_quantize_candidates(raw_c, prepared, scales, make_index=make_index)
        return tt.tt_normalize_candidates(raw_c, prepared, mode, make_index=make_index)

    index = build_index(True)
    k1_evs = []
    for _ in range(K1_REPS):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        build_index(False)
        e1.record(stream)
        k1_evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    k1_ms = sum(a.elapsed_time(b) for a, b in k1_evs) / len(k1_evs)
    if int8 or w.store != "raw":  # the index no longer needs the raw rows
        del raw_c
        torch.cuda.empty_cache()

    # ---- one step: normalise the batch of raw queries, then the exact top-k
    def step():
        tt.tt_normalize_candidates(raw_q, qn, tt.TT_NORM_STORE, make_index=False)
        if sharded:
            shard.sharded_score_topk(index, qn, w.k, bounds, tau=w.tau, exclude_local=excl, path=args.path)
        else:
            tt.tt_score_topk(index, qn, w.k, tau=w.tau, exclude=excl, out_ids=out_ids, out_scores=out_scores,
                             path=args.path)

    corpus_bytes = prepared.numel() * prepared.element_size() + (
        raw_c.numel() * raw_c.element_size() if (not int8 and w.store == "raw") else 0)
    flush = None
    if corpus_bytes < FLUSH_BELOW_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > the 126 MB L2

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    tt.tt_index_check(index)  # raises if a device-side wait expired in the warm-up
    stats = tt.tt_last_stats(index)
    # the plan the searches ran: scored levels, and the sample of the estimate
    # when the small-batch plan replaced the coarse levels with it
    plan = {"rows": stats["level_rows"][:1] if stats["sampled"] else stats["level_rows"],
            "sample_rows": stats["level_rows"][1] if stats["sampled"] else 0}

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = tt.tt_launch_count()

    def timed_steps(n_steps):
        evs = []
        if flush is None:  # inputs larger than L2: steps back to back
            e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e_start.record(stream)
            for _ in range(n_steps):
                step()
            e_stop.record(stream)
            evs.append((e_start, e_stop))
        else:  # L2 flushed before every step, outside the step's events
            for _ in range(n_steps):
                flush.zero_()
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                step()
                b_.record(stream)
                evs.append((a, b_))
        return evs

    t_wall0 = time.time()
    evs = timed_steps(args.steps)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier(world)
    launches = tt.tt_launch_count() - launches0
    clk = clocks.stop(t_wall0, t_wall1)
    tt.tt_index_check(index)
    ms_total = sum(a.elapsed_time(b_) for a, b_ in evs)
    ms_total = max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    # per-kernel device times from a separate pass of the same steps with an
    # event pair around every library launch (kept out of the timed region,
    # where the extra events would lengthen short steps)
    prof_steps = max(1, min(args.steps, 10))
    tt.tt_profile_begin()
    timed_steps(prof_steps)
    torch.cuda.synchronize(dev)
    prof = tt.tt_profile_end()
    barrier(world)

    # replicas: every rank did a whole workload; shards: the ranks did one together
    value = (1 if sharded else world) * w_all.b * w_all.n / (ms_step / 1e3)
    qps = (1 if sharded else world) * w_all.b / (ms_step / 1e3)

    # ---- roofline of the dominant kernel: the scorer over all levels ----
    peaks, peak_src = load_peaks()
    work = work_model(w, plan, int8)
    score_kind = "tensor" if stats["path"] >= 2 else "stream"
    score_kernel = {1: "k2_stream", 2: "k3_tensor", 3: "k3_pair"}[stats["path"]]
    score_ms = prof[score_kind]["ms"] / prof_steps
    qnorm_ms = prof["normalize"]["ms"] / prof_steps
    search_ms = max(1e-9, ms_step - qnorm_ms)  # the tt_score_topk calls of a step
    t_flops = work["score_flops"] / (peaks["bf16_tflops"] * (2.0 if int8 else 1.0) * 1e12)
    t_bytes = work["score_bytes"] / (peaks["hbm_gbs"] * 1e9)
    if stats["path"] >= 2 and t_flops > t_bytes:
        # a kernel of a few ms timed in a short region: the burst peak applies
        # (int8: the bf16 measured peak times the nominal int8 / bf16 ratio, 4.5 / 2.25)
        peak = peaks["bf16_tflops"] * (2.0 if int8 else 1.0)
        achieved = work["score_flops"] / (score_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TOP/s" if int8 else "TFLOP/s", "frac": round(achieved / peak, 4)}
        search_achieved = work["score_flops"] / (search_ms / 1e3) / 1e12
        peak_s = peaks["bf16_tflops_sustained"] * (2.0 if int8 else 1.0)
        roof["peak_sustained"] = peak_s
        roof["frac_sustained"] = round(achieved / peak_s, 4)
        if peaks.get("sustained_mhz"):
            roof["sustained_peak_sm_mhz"] = peaks["sustained_mhz"]
        roof["peak_source"] = peak_src + (" (burst bf16 x 2, the nominal int8 ratio)" if int8 else " (burst bf16)")
    else:
        peak = peaks["hbm_gbs"]
        achieved = work["score_bytes"] / (score_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4)}
        search_achieved = work["score_bytes"] / (search_ms / 1e3) / 1e9
        roof["peak_source"] = peak_src + " (copy)"
    roof["traffic"] = None if int8 else recorded_traffic(score_kernel, w.name, work["rows_scanned"])
    roof["kernel"] = f"{score_kernel} (all levels)"
    roof["kernel_ms"] = round(score_ms, 5)
    roof["launches_per_step"] = prof[score_kind]["launches"] / prof_steps
    # the whole search (every kernel of tt_score_topk: levels, selects, checks)
    # against the same algorithmic work
    roof["search_ms"] = round(search_ms, 5)
    roof["search_frac"] = round(search_achieved / peak, 4)

    kernels = {k: {"ms_per_step": round(v["ms"] / prof_steps, 5), "launches_per_step": v["launches"] / prof_steps}
               for k, v in prof.items() if v["launches"]}
    kernels["profiled_steps"] = prof_steps
    k1_bytes = work["k1_bytes"]
    kernels["k1_index_build"] = {"ms": round(k1_ms, 5), "per": "index build (once, not in a step)",
                                 "gbs": round(k1_bytes / (k1_ms / 1e3) / 1e9, 1),
                                 "frac_hbm": round(k1_bytes / (k1_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}

    # ---- end to end through the public API: host queries in, host results out ----
    e2e = None
    if not args.no_e2e and not sharded:
        host_q = raw_q.cpu().pin_memory()
        host_ids = torch.empty((w.b, w.k), dtype=torch.int32).pin_memory()
        host_scores = torch.empty((w.b, w.k), dtype=torch.float32).pin_memory()
        e2e_steps = max(3, min(args.steps, args.e2e_steps))

        def e2e_step():
            tt.tt_score_topk_host(index, host_q, w.k, tau=w.tau, exclude=excl, normalize=True,
                                  norm_dtype=q_torch_dtype, out_ids=host_ids, out_scores=host_scores)

        e2e_step()
        barrier(world)
        torch.cuda.synchronize(dev)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e2e_steps):
            if flush is not None:
                flush.zero_()
            e2e_step()
        b_.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = a.elapsed_time(b_) / e2e_steps
        if flush is not None:  # take the flushes back out
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for _ in range(e2e_steps):
                flush.zero_()
            f1.record(stream)
            torch.cuda.synchronize(dev)
            e2e_ms -= f0.elapsed_time(f1) / e2e_steps
        e2e_ms = max_over_ranks(e2e_ms, world)
        h2d = host_q.numel() * host_q.element_size()
        e2e = {"value": world * w.b * w.n / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": round(e2e_ms, 4),
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(w.b * w.k * 8), "steps": e2e_steps,
               "call": "tt_score_topk_host (pinned host queries in, host ids and scores out; the index "
                       "is resident in HBM, built once)"}

    l2_note = ("inputs larger than L2 (scored corpus "
               f"{corpus_bytes / 1e6:.0f} MB > 126 MB)") if flush is None else \
        "L2 flushed before every step (256 MB write outside the step's events)"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "strong" if sharded else "weak", "vs_baseline": None,
        "dtype": "i8" if int8 else ("bf16" if w.store != "f32" else "f32"),
        "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": w.name, "n": w_all.n, "d": w.d, "b": w.b, "k": w.k, "tau": w.tau,
                   "corpus_raw": w.raw_dtype, "corpus_store": "i8 codes + f32 scales" if int8 else w.store,
                   "queries": w.query_dtype, "mask_rate": w.mask_rate, "l2": l2_note,
                   "step": "normalise the raw queries + tt_score_topk on the index (built once)",
                   "path": PATH_NAMES[stats["path"]], "levels": plan["rows"],
                   "estimate_sample_rows": plan["sample_rows"],
                   "parallelism": (f"corpus shards x{world} (all-gather of [b, k] lists + merge)" if sharded
                                   else f"replicas x{world}")},
        "topk_queries_per_s": qps,
        "roofline": roof,
        "kernels": kernels,
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": int(launches),
    }
    if host_sample is not None:
        line["cpu_baseline"] = cpu_baseline(w, *host_sample, seconds=args.cpu_seconds)
    return line


# ---------------------------------------------------------------------------
# in-batch sampled softmax
# ---------------------------------------------------------------------------
SOFTMAX_METRIC = "in-batch sampled-softmax logits/sec (fused loss)"
SOFTMAX_UNIT = "logits/s"
# ex2 results per clock per SM (the multi-function unit; CUDA C++ Programming
# Guide, arithmetic instruction throughput, compute capability 10.0)
MUFU_PER_CLK_SM = 16
SM_COUNT = 148
SM_MAX_MHZ = 1965.0


def softmax_oracle_run(inp, rows, tau):
    """fp64 oracle on the listed rows, each against every column."""
    import oracle
    nc = inp["items"].shape[0]
    rest = np.setdiff1d(np.arange(nc), rows)
    cols = np.concatenate([rows, rest])
    users = W.bf16_bits(inp["users"][torch.from_numpy(rows)])
    items = W.bf16_bits(inp["items"][torch.from_numpy(cols)])
    logq = inp["logq"].numpy().astype(np.float64)[cols]
    ids = inp["item_ids"].numpy()[cols]
    valid = inp["valid"].numpy()[cols]
    t0 = time.perf_counter()
    oracle.inbatch_softmax(users, items, tau, logq=logq, item_ids=ids, valid=valid)
    return time.perf_counter() - t0


def softmax_oracle_sample(w, inp, seconds):
    import oracle
    threads = oracle.max_threads()
    r = min(w.b, max(1, threads))
    t = softmax_oracle_run(inp, np.arange(r), w.tau)
    while r < w.b and t < seconds / 4:
        r = min(w.b, r * 4)
        t = softmax_oracle_run(inp, np.arange(r), w.tau)
    if t > 0 and r < w.b:
        r = int(min(w.b, max(1, r * seconds / t)))
    return r, threads


def softmax_cpu_baseline(w, inp, seconds):
    r, threads = softmax_oracle_sample(w, inp, seconds)
    t = softmax_oracle_run(inp, np.arange(r), w.tau)
    return {"value": r * w.nc / t, "unit": SOFTMAX_UNIT, "cores": threads, "kind": "oracle",
            "sample": f"first {r} rows of {w.name} against all {w.nc} columns (fp64 logits, masks, "
                      f"log-sum-exp, loss), one run of {t:.2f} s"}


def run_softmax(args, world, rank, local):
    import exact_inner_product_b200 as tt

    w = W.batch(args.batch)
    if world > 1:  # each rank: its own batch (data parallel; the losses stay per rank)
        w = dataclasses.replace(w, seed=w.seed + 7919 * rank)
    dev = torch.device("cuda", local)
    host = W.batch_inputs(w, "cpu")
    inp = {k: v.to(dev) for k, v in host.items()}
    ws = torch.empty(tt.tt_inbatch_softmax_workspace(w.b, w.nc, w.d, True), dtype=torch.uint8, device=dev)
    out = (torch.empty(w.b, device=dev), torch.empty(w.b, device=dev), torch.empty((), device=dev))
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # larger than the 126 MB L2
    stream = torch.cuda.current_stream(dev)

    def step():
        tt.tt_inbatch_softmax(inp["users"], inp["items"], w.tau, logq=inp["logq"], item_ids=inp["item_ids"],
                              valid=inp["valid"], workspace=ws, out=out, check=False)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    if tt._lib.tt_inbatch_softmax_check(tt._ptr(ws), None) != tt.TT_OK:
        raise RuntimeError("tt_inbatch_softmax: device-side timeout in warm-up")
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = tt.tt_launch_count()
    tt.tt_profile_begin()
    t_wall0 = time.time()
    evs = []
    for _ in range(args.steps):
        flush.zero_()  # L2 flush, outside the step's events
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b_.record(stream)
        evs.append((a, b_))
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier(world)
    recs = tt.tt_profile_launches()
    tt.tt_profile_end()
    launches = tt.tt_launch_count() - launches0
    clk = clocks.stop(t_wall0, t_wall1)
    if tt._lib.tt_inbatch_softmax_check(tt._ptr(ws), None) != tt.TT_OK:
        raise RuntimeError("tt_inbatch_softmax: device-side timeout in the timed steps")
    ms_total = max_over_ranks(sum(a.elapsed_time(b_) for a, b_ in evs), world)
    ms_step = ms_total / args.steps
    logits = w.b * w.nc
    value = world * logits / (ms_step / 1e3)

    # roofline: one ex2 per logit on the multi-function unit (the fused
    # kernel is the longest launch of a step)
    per_step = len(recs) // args.steps
    main_at = int(np.argmax([recs[j][1] for j in range(per_step)]))
    main_ms = [recs[s * per_step + main_at][1] for s in range(args.steps)]
    k5_ms = float(np.mean(main_ms))
    achieved = logits / (k5_ms / 1e3) / 1e12
    peak = MUFU_PER_CLK_SM * SM_COUNT * SM_MAX_MHZ * 1e6 / 1e12
    roof = {"bound": "alu", "achieved": round(achieved, 4), "peak": round(peak, 4), "unit": "Tex2/s",
            "frac": round(achieved / peak, 4), "traffic": recorded_traffic("k5_softmax", w.name, logits),
            "kernel": "k5_softmax", "kernel_ms": round(k5_ms, 5),
            "peak_source": f"derived: {MUFU_PER_CLK_SM} ex2 per clock per SM x {SM_COUNT} SMs x {SM_MAX_MHZ:.0f} MHz "
                           "(clocks.max.sm)"}
    if clk.get("sm_mhz"):
        roof["frac_at_sampled_clock"] = round(achieved / (peak * clk["sm_mhz"] / SM_MAX_MHZ), 4)
    kernels = {}
    names = ["k5_table_clear", "k5_columns", "k5_softmax", "k5_merge"]
    for j in range(per_step):
        kernels[names[j] if per_step == 4 else f"launch{j}"] = {
            "ms_per_step": round(float(np.mean([recs[s * per_step + j][1] for s in range(args.steps)])), 5),
            "launches_per_step": 1}

    # end to end: pinned host batch -> device, the call, the mean back to the host
    e2e = None
    if not args.no_e2e:
        pinned = {k: v.pin_memory() for k, v in host.items()}
        mean_host = torch.empty((), dtype=torch.float32).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in pinned.values())

        def e2e_step():
            d = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
            _, _, mean = tt.tt_inbatch_softmax(d["users"], d["items"], w.tau, logq=d["logq"],
                                               item_ids=d["item_ids"], valid=d["valid"], workspace=ws,
                                               check=False)
            mean_host.copy_(mean, non_blocking=True)

        e2e_step()
        barrier(world)
        torch.cuda.synchronize(dev)
        e2e_steps = max(3, min(args.steps, args.e2e_steps))
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        b_.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(a.elapsed_time(b_) / e2e_steps, world)
        e2e = {"value": world * logits / (e2e_ms / 1e3), "unit": SOFTMAX_UNIT, "ms_per_step": round(e2e_ms, 4),
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": 4, "steps": e2e_steps}

    line = {
        "metric": SOFTMAX_METRIC, "value": value, "unit": SOFTMAX_UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": w.name, "b": w.b, "nc": w.nc, "d": w.d, "tau": w.tau, "catalogue": w.catalogue,
                   "zipf_s": w.zipf_s, "pad_rate": w.pad_rate, "logq": True, "item_ids": True,
                   "l2": "flushed before every step (256 MB write outside the step's events)",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "kernels": kernels,
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": int(launches),
    }
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = softmax_cpu_baseline(w, host, seconds=args.cpu_seconds)
    return line


def run_softmax_reference(args, world, rank):
    """The fp64 oracle as the reference arm of --op inbatch_softmax."""
    if rank != 0:
        return None
    w = W.batch(args.batch)
    host = W.batch_inputs(w, "cpu")
    budget = args.ref_seconds or max(0.05, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    r, threads = softmax_oracle_sample(w, host, budget)
    for _ in range(args.warmup):
        softmax_oracle_run(host, np.arange(r), w.tau)
    t = sum(softmax_oracle_run(host, np.arange(r), w.tau) for _ in range(args.steps))
    ms = t / args.steps * 1e3
    value = r * w.nc / (ms / 1e3)
    sample = f"each step: first {r} rows of {w.name} against all {w.nc} columns (fp64)"
    return {"impl": "reference", "metric": SOFTMAX_METRIC, "value": value, "unit": SOFTMAX_UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, workloads.py)",
            "config": {"workload": w.name, "b": w.b, "nc": w.nc, "d": w.d, "tau": w.tau},
            "cpu_baseline": {"value": value, "unit": SOFTMAX_UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": SOFTMAX_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference(args, world, rank):
    """The fp64 oracle as the reference arm, on this host's cores."""
    if rank != 0:
        return None
    import oracle
    w = w_all = workload_from_args(args)
    # only a prefix of the corpus is ever timed: draw just that (the same rows)
    raw_c = W.corpus(w, "cpu", rows=min(w.n, CPU_SAMPLE_ROWS))
    raw_q = W.queries(w, "cpu")
    excl = W.exclusion_bits(w, "cpu")
    raw_c_np = W.to_numpy_rows(raw_c)
    w = dataclasses.replace(w, n=raw_c_np.shape[0])
    raw_q_np = raw_q.numpy()
    excl_np = None if excl is None else excl.numpy().view(np.uint32)
    budget = args.ref_seconds or max(0.05, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    n_s, b_s, threads = oracle_sample_size(w, raw_c_np, raw_q_np, excl_np, budget)
    for _ in range(args.warmup):
        oracle_sample_run(w, raw_c_np, raw_q_np, excl_np, n_s, b_s)
    t = 0.0
    for _ in range(args.steps):
        t += oracle_sample_run(w, raw_c_np, raw_q_np, excl_np, n_s, b_s)
    ms = t / args.steps * 1e3
    value = b_s * n_s / (ms / 1e3)
    sample = (f"each step: {b_s} queries x first {n_s} candidates of {w.name} "
              "(fp64 normalise + score + full sort)")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, workloads.py)",
            "config": {"workload": w_all.name, "n": w_all.n, "d": w.d, "b": w.b, "k": w.k},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--n", type=int, default=0, help="override the workload's corpus size")
    ap.add_argument("--b", type=int, default=0, help="override the workload's batch size")
    ap.add_argument("--k", type=int, default=0, help="override the workload's k")
    ap.add_argument("--path", type=int, default=0, choices=[0, 1, 2, 3],
                    help="scorer: 0 auto, 1 streaming, 2 tensor-core, 3 tensor-core on SM pairs")
    ap.add_argument("--quant", default="none", choices=["none", "int8"],
                    help="int8: code the normalised corpus in int8 and score int8 codes (tensor cores kind::i8)")
    ap.add_argument("--mode", default="replicas", choices=["replicas", "shard"],
                    help="N > 1: independent replicas (default) or one corpus sharded by rows over the ranks")
    ap.add_argument("--op", default="topk", choices=["topk", "inbatch_softmax"],
                    help="topk: the retrieval step (default); inbatch_softmax: the fused training loss")
    ap.add_argument("--batch", default="inbatch_b65536_d64", choices=sorted(W.BATCHES),
                    help="training batch of --op inbatch_softmax")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=0.0,
                    help="reference arm: oracle seconds per step (default: sized so the run ends in minutes)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup(args)
    try:
        softmax = args.op == "inbatch_softmax"
        if args.impl == "reference":
            line = run_softmax_reference(args, world, rank) if softmax else run_reference(args, world, rank)
        else:
            line = run_softmax(args, world, rank, local) if softmax else run_ours(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as tdist
            tdist.destroy_process_group()


if __name__ == "__main__":
    main()
