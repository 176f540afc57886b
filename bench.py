#!/usr/bin/env python
"""Benchmark: split-KV paged attention (decode / speculative verification).

One step = one pass of the whole hot path over one batch: the partial pass
(lse_attn_run) and the merge pass (lse_attn_merge) through the C ABI, on
resident inputs.  By default every one of the five workloads is timed in
turn (tiny FP32 decode, batched BF16 decode, BF16 chain verify, long-context
FP8, mixed FP16 tree-verify batch); the line's headline ``value``, roofline,
end-to-end and CPU-baseline figures are those of the largest, the
tree-verify batch, and ``per_workload`` holds each workload's own figures.
L2 is flushed (a 256 MiB write) before every timed step, outside the step's
CUDA-event interval.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all|NAME]
                  [--impl ours|reference]

--workload append times the K/V append kernel instead (see run_append);
--workload fragment_ab the fragment-addressing comparison.

Prints one JSON line.  ``value`` is effective GB/s: (K + V + Q + out bytes of
every call on every rank) / (max over ranks of the summed step times).
``--impl reference`` times the float64 CPU oracle on a bounded sample of
the same workload (rank 0 only under torchrun).
Multi-GPU runs are independent replicas (the path needs no exchange).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged attention us/call and effective KV GB/s (% of B200 HBM peak)"
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="all",
                    help="all (the five configurations) or one workload name")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the oracle CPU-baseline sample")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_bf16_tflops():
    """Dense BF16 tensor peak (burst) measured on this machine's B200s."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def attention_flops(w):
    """Algorithmic FLOPs of one call: 4 D per (row, query head, visible key)
    (the score and output products, 2 each); a block row at position C + r
    sees C + r + 1 keys (chain rows, no masks)."""
    lens = np.asarray(w.seq_lens, np.int64)
    offs = np.asarray(w.row_offsets, np.int64)
    vis = 0
    for s in range(len(lens)):
        R = int(offs[s + 1] - offs[s])
        C = int(lens[s]) - R
        vis += R * C + R * (R + 1) // 2
    return 4 * w.head_dim * w.n_q_heads * vis


# the sources each measured kernel (and its launch plan) is built from
KERNEL_SOURCES = {
    "partial": ("lse_host.cpp", "lse_internal.h", "lse_tcgen05.cu", "lse_tc_ptx.h"),
    "prefill": ("lse_host.cpp", "lse_internal.h", "lse_prefill.cu", "lse_tc_ptx.h"),
    "append": ("lse_append.cu", "lse_host.cpp", "lse_internal.h"),
}


def kernel_source_hash(kernel="partial"):
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "verify_attention_paged_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload, kernel="partial"):
    """DRAM bytes per launch of the workload's dominant kernel from the
    committed ncu summary, when it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            pass
        self._stop = threading.Event()

    def active(self, on):
        """Sample only while a timed loop runs (between workloads the box
        is building inputs on the host)."""
        self._on = on

    def _loop(self):
        while not self._stop.is_set():
            if not getattr(self, "_on", True):
                time.sleep(0.002)
                continue
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._loop, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def reduce_max(value, dist, device):
    """Max over ranks of a per-rank float (device time: the slowest rank)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world, bytes_per_call, calls, max_ms):
    """Whole-job effective GB/s: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_call * calls / (max_ms * 1e-3) / 1e9


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _oracle_sample(w, pb, m, outputs, order, budget_s, threads):
    """Oracle outputs (row, head) in `order` on `threads` host threads until
    `budget_s` passes (ctypes releases the GIL for each call, so the threads
    run the C oracle in parallel).  Returns (seconds, outputs done, keys
    visited)."""
    from oracle import oracle as orc
    lock = threading.Lock()
    state = {"next": 0, "done": 0, "keys": 0}
    t0 = time.perf_counter()

    def worker():
        while True:
            with lock:
                if state["next"] >= len(order) or time.perf_counter() - t0 > budget_s:
                    return
                i = int(order[state["next"]])
                state["next"] += 1
            s, r, h = outputs[i]
            orc.attention_one(pb, s, r, h, marshalled=m)
            with lock:
                state["done"] += 1
                state["keys"] += int(w.seq_lens[s])

    pool = [threading.Thread(target=worker) for _ in range(threads)]
    for t in pool:
        t.start()
    for t in pool:
        t.join()
    return time.perf_counter() - t0, state["done"], state["keys"]


def cpu_baseline(w, budget_s, threads=None):
    """The oracle as it stands on the host's cores: a quarter of the budget
    on one thread, the rest on one thread per core, each on a bounded sample
    of the workload's (row, head) outputs, extrapolated to one whole call by
    the keys visited.  `value` is the all-core figure."""
    from oracle import oracle as orc
    threads = threads or os.cpu_count() or 1
    pb = orc.Problem(chunks=w.chunks, chunk_bytes=w.chunk_bytes, fragment_bytes=w.fragment_bytes,
                     dtype=w.dtype, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                     n_q_heads=w.n_q_heads, k_pages=w.k_pages, v_pages=w.v_pages,
                     seq_lens=w.seq_lens, row_offsets=w.row_offsets, row_masks=w.row_masks,
                     q=w.q, scale=w.scale, scales=w.scales)
    m = orc.marshal(pb)
    outputs = [(s, r, h) for s in range(w.n_seqs)
               for r in range(int(w.row_offsets[s + 1] - w.row_offsets[s]))
               for h in range(w.n_q_heads)]
    order = np.random.default_rng(0).permutation(len(outputs))
    all_keys = sum(int(w.seq_lens[s]) for (s, r, h) in outputs)
    res = {}
    for tag, n_thr, budget in (("one", 1, budget_s / 4), ("all", threads, budget_s * 3 / 4)):
        dt, n_done, keys = _oracle_sample(w, pb, m, outputs, order, budget, n_thr)
        call_s = dt * all_keys / max(keys, 1)
        res[tag] = (w.call_bytes() / call_s / 1e9, call_s, n_done, dt)
    gbs, call_s, n_done, dt = res["all"]
    gbs1, call_s1, n_done1, dt1 = res["one"]
    return {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "us_per_call": call_s * 1e6,
            "sample": f"{n_done} of {len(outputs)} (row, head) outputs on {threads} threads in "
                      f"{dt:.1f} s, extrapolated by keys visited to one call",
            "single_core": {"value": gbs1, "us_per_call": call_s1 * 1e6,
                            "sample": f"{n_done1} outputs on 1 thread in {dt1:.1f} s"}}


def run_reference(args, w, world, rank):
    if rank != 0:
        return
    # each step is a bounded sample; the whole run stays within minutes
    per_step = max(0.05, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(w, per_step / 4)
    vals = []
    t_all = 0.0
    for _ in range(args.steps):
        r = cpu_baseline(w, per_step)
        vals.append(r["value"])
        t_all += r["us_per_call"]
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_all / args.steps / 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w),
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": os.cpu_count() or 1,
                             "kind": "oracle",
                             "sample": f"each step: oracle on ~{per_step:.2f} s of "
                                       f"(row, head) outputs (a quarter on one thread, the "
                                       f"rest on every core), extrapolated to one call"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def compute_dtype(kv_dtype, kernel):
    """The arithmetic the partial pass runs in: the tensor-core kernel takes
    16-bit K/V times 16-bit hi + lo terms of Q and P, or 8-bit K/V times 8-bit
    terms, accumulating in FP32; the CUDA-core kernel is FP32 throughout."""
    return f"{kv_dtype}-mma/f32" if kernel in (1, 2) else "f32"


def workload_config(w):
    return {"workload": w.name, "seqs": w.n_seqs, "keys_total": int(np.sum(w.seq_lens)),
            "query_rows": w.total_rows, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "kv_dtype": w.dtype,
            "fragment_bytes": w.fragment_bytes, "chunk_bytes": w.chunk_bytes,
            "bytes_per_call": w.call_bytes(), "l2": "flushed before every step (256 MiB write)",
            "timing": "CUDA events around a CUDA-graph replay of each step"}


HEADLINE = "tree_verify"   # the largest single-GPU workload carries the headline


def time_workload(w, args, flush, dist, clk):
    """Device times of one workload: `args.steps` graph replays of the whole
    step (lse_attn_forward: one launch, the merge inside the partial pass,
    on tensor-core plans; on CUDA-core plans the partial pass and the merge
    as its programmatic dependent) and as many
    of the dominant kernel alone (the partial pass of a two-kernel step; the
    step itself when it is one launch), L2 flushed before each outside the
    CUDA-event interval.
    Returns the DeviceCall (kept for the end-to-end leg) and the per-step
    millisecond lists."""
    import torch
    from verify_attention_paged_b200 import binding as b
    call = b.DeviceCall(w)
    for _ in range(args.warmup):
        flush.fill_(1)
        call.run()
    torch.cuda.synchronize()
    assert call.device_error() == 0, f"{w.name}: device error during warm-up"
    one_kernel = call.info["merge_in_pass"] == 1  # the step is one launch
    g_step, g_part = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    saved = call.stream
    with torch.cuda.graph(g_step):
        call.stream = torch.cuda.current_stream()
        call.run()
    with torch.cuda.graph(g_part):
        call.stream = torch.cuda.current_stream()
        if one_kernel:
            call.run()
        else:
            call.run_partial()
    call.stream = saved
    for _ in range(3):
        flush.fill_(2)
        g_step.replay()
        flush.fill_(3)
        g_part.replay()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clk.active(True)
    for i in range(args.steps):
        flush.fill_(i & 0xff)                  # L2 flush, outside the interval
        ev[i][0].record()
        g_step.replay()
        ev[i][1].record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    for i in range(args.steps):                # the partial pass alone
        flush.fill_(i & 0xff)
        evp[i][0].record()
        g_part.replay()
        evp[i][1].record()
    torch.cuda.synchronize()
    clk.active(False)
    assert call.device_error() == 0, f"{w.name}: device error during the timed steps"
    steps_ms = [e[0].elapsed_time(e[1]) for e in ev]
    part_ms = [e[0].elapsed_time(e[1]) for e in evp]
    del g_step, g_part
    return call, steps_ms, part_ms


def workload_result(w, call, steps_ms, part_ms, world, dist, args, peak, peak_kind):
    """One workload's figures: us per call, whole-job GB/s, and the roofline
    of the dominant kernel (the algorithmic K + V + Q bytes of the partial
    pass over that kernel's CUDA-event time, against the measured copy
    bandwidth)."""
    total_ms = reduce_max(sum(steps_ms), dist, "cuda")
    part_mean = reduce_max(statistics.mean(part_ms), dist, "cuda")
    info = call.info
    fused = info["merge_in_pass"] == 1  # the merge runs inside the partial launch
    bytes_call = w.call_bytes()
    # the dominant kernel's algorithmic bytes: K + V + Q (+ out when the
    # merge is fused into it)
    bytes_partial = w.call_bytes() if fused else (
        w.kv_bytes() + w.total_rows * w.n_q_heads * w.head_dim * 4)
    achieved = bytes_partial / (part_mean * 1e-3) / 1e9
    value = job_gbs(world, bytes_call, args.steps, total_ms)
    bound = "hbm"
    if bytes_call < 4 << 20:
        # a quarter of a megabyte moves in well under a microsecond at HBM
        # speed: launch and dependent-load latency set the time
        bound = "launch"
    roof = {"bound": bound,
            "kernel": "partial pass with the merge fused" if fused else "partial",
            "achieved": achieved, "peak": peak,
            "peak_kind": f"{peak_kind} (copy, burst)", "unit": "GB/s",
            "frac": achieved / peak, "traffic": ncu_traffic(w.name),
            "algorithmic_bytes_per_launch": bytes_partial}
    extra = {}
    if info["kernel_name"] == "prefill":
        # a long query block is a dense contraction: its roofline is the
        # tensor peak (the products carry hi + lo operand terms, so at most
        # half of it counts as algorithmic FLOPs)
        tf_peak, tf_kind = measured_bf16_tflops()
        tflops = attention_flops(w) / (part_mean * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": "long-query-block pass", "achieved": tflops,
                "peak": tf_peak, "peak_kind": f"{tf_kind} (cuBLAS bf16, burst)",
                "unit": "TFLOP/s", "frac": tflops / tf_peak,
                "traffic": ncu_traffic(w.name, "prefill"),
                "algorithmic_flops_per_launch": attention_flops(w)}
        extra = {"tflops": tflops}
    return {
        **extra,
        "value": value, "unit": "GB/s", "us_per_call": total_ms / args.steps * 1e3,
        "us_per_call_median": statistics.median(steps_ms) * 1e3,
        "partial_us_mean": part_mean * 1e3,
        "merge_us_est": (total_ms / args.steps - part_mean) * 1e3,
        "pct_of_8tbs": value / world / 8000.0 * 100.0,
        "pct_of_measured_hbm": value / world / peak * 100.0,
        "bytes_per_call": bytes_call,
        "kernel": info["kernel_name"], "n_splits": info["n_splits"],
        "launches_per_call": 1 if fused else 2,
        "dtype": compute_dtype(w.dtype, info["kernel"]),
        "roofline": roof,
    }


def run_ours(args, names, world, rank, local):
    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from verify_attention_paged_b200 import workloads as wl

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    peak, peak_kind = measured_peaks()
    head = HEADLINE if HEADLINE in names else names[0]
    results, head_w, head_call = {}, None, None
    clk = ClockSampler(local)
    with clk:
        for name in names:
            w = wl.BUILDERS[name]()
            call, steps_ms, part_ms = time_workload(w, args, flush, dist, clk)
            results[name] = workload_result(w, call, steps_ms, part_ms, world, dist, args,
                                            peak, peak_kind)
            if name == head:
                head_w, head_call = w, call
            else:
                call.close()
                del call, w
                torch.cuda.empty_cache()

    # end to end: pinned host inputs -> device -> run -> result back to host
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(head_call, head_w, args, head_call.stream, flush, dist)

    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return
    r = results[head]
    line = {
        "metric": METRIC, "value": r["value"], "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": r["us_per_call"] / 1e3,
        "us_per_call": r["us_per_call"], "us_per_call_median": r["us_per_call_median"],
        "partial_us_mean": r["partial_us_mean"], "merge_us_est": r["merge_us_est"],
        "pct_of_8tbs": r["pct_of_8tbs"], "pct_of_measured_hbm": r["pct_of_measured_hbm"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": r["dtype"], "data": "synthetic",
        "config": {**workload_config(head_w), "parallelism": f"replicas{world}",
                   "kernel": r["kernel"], "n_splits": r["n_splits"]},
        "roofline": r["roofline"],
        "per_workload": {n: {k: v for k, v in res.items()} for n, res in results.items()},
        "gpu_launches": 2 * args.steps * sum(res["launches_per_call"] for res in results.values()),
        "clocks": clk.summary(),
    }
    if e2e:
        line["e2e"] = e2e
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(head_w, args.cpu_seconds)
    print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


def measure_e2e(call, w, args, stream, flush, dist):
    """Same metric through the public API with this step's inputs (Q, page
    tables, lengths, row offsets, masks, packed in one pinned host buffer)
    copied to the device in one copy and the result (out and lse, packed)
    read back in one copy, inside the timed interval."""
    import torch
    host_in = call.host_inputs
    host_out = torch.empty(call.outputs.numel(), dtype=torch.float32).pin_memory()
    h2d = host_in.numel()
    d2h = host_out.numel() * 4
    steps = max(10, args.steps // 5)

    def step():
        call.upload(host_in)
        call.run()
        call.download(host_out)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    if dist:
        dist.barrier()
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush.fill_(i & 0xff)
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
    torch.cuda.synchronize()
    ms = reduce_max(sum(a.elapsed_time(b) for a, b in evs), dist, "cuda")
    world = dist.get_world_size() if dist else 1
    return {"value": job_gbs(world, w.call_bytes(), steps, ms), "unit": "GB/s",
            "us_per_call": ms / steps * 1e3, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "copies_per_step": {"h2d": 1, "d2h": 1}}


APPEND_METRIC = "K/V append us/call and GB/s (FP32 read + stored bytes)"


def run_append(args, world, rank, local):
    """The K/V append (lse_kv_append) of a verify step's drafts: 256
    sequences x 16 new tokens, 24/4 heads, head_dim 128, into a BF16 arena of
    256 KiB fragments.  One step = one append call, captured in a CUDA graph,
    L2 flushed before each step outside the interval."""
    import torch
    torch.cuda.set_device(local)
    from verify_attention_paged_b200 import binding as b
    n_seqs, new, hkv, d = 256, 16, 4, 128
    dtype, esize, frag = "bf16", 2, 256 << 10
    T = frag // (hkv * d * esize)
    rng = np.random.default_rng(1240)
    before = rng.integers(1024, 16384, n_seqs).astype(np.int32)
    pages = (before + new + T - 1) // T
    max_pages = int(pages.max())
    n_frags = int(2 * pages.sum())
    chunk = 256 << 20
    n_chunks = (n_frags * frag + chunk - 1) // chunk
    chunks = [torch.empty(chunk, dtype=torch.uint8, device="cuda") for _ in range(n_chunks)]
    arena = b.lse_kv_arena_create(chunks, chunk, frag, dtype, hkv, d)
    ids = rng.permutation(b.lse_kv_arena_alloc(arena, n_frags)).astype(np.int32)
    kp = np.full((n_seqs, max_pages), -1, np.int32)
    vp = np.full((n_seqs, max_pages), -1, np.int32)
    at = 0
    for s_ in range(n_seqs):
        kp[s_, :pages[s_]] = ids[at:at + pages[s_]]
        vp[s_, :pages[s_]] = ids[at + pages[s_]:at + 2 * pages[s_]]
        at += 2 * pages[s_]
    dev = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    total = n_seqs * new
    gen = torch.Generator().manual_seed(1240)   # seeded on the host, then uploaded
    k_new = torch.randn((total, hkv, d), generator=gen).cuda()
    v_new = torch.randn((total, hkv, d), generator=gen).cuda()
    offs = dev(np.arange(0, total + 1, new, dtype=np.int32))
    kp_d, vp_d, before_d = dev(kp), dev(vp), dev(before)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def step(stream):
        b.lse_kv_append(arena, n_seqs, max_pages, k_new, v_new, kp_d, vp_d, before_d, offs,
                        total, err, stream)

    for _ in range(args.warmup):
        flush.fill_(1)
        step(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(torch.cuda.current_stream())
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xff)
            ev[i][0].record()
            g.replay()
            ev[i][1].record()
        torch.cuda.synchronize()
    assert int(err.item()) == 0, "device error during the append"
    ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = sum(ms)
    nbytes = 2 * total * hkv * d * (4 + esize)  # K and V: FP32 read, BF16 written
    gbs = nbytes * args.steps / (total_ms * 1e-3) / 1e9
    peak, kind = measured_peaks()
    line = {
        "metric": APPEND_METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "us_per_call": total_ms / args.steps * 1e3,
        "us_per_call_median": statistics.median(ms) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32->bf16",
        "data": "synthetic",
        "config": {"workload": "append", "seqs": n_seqs, "new_tokens_per_seq": new,
                   "kv_heads": hkv, "head_dim": d, "kv_dtype": dtype, "fragment_bytes": frag,
                   "bytes_per_call": nbytes, "l2": "flushed before every step (256 MiB write)",
                   "timing": "CUDA events around a CUDA-graph replay of each step"},
        "roofline": {"bound": "hbm", "kernel": "kv_append", "achieved": gbs, "peak": peak,
                     "peak_kind": f"{kind} (copy, burst)", "unit": "GB/s", "frac": gbs / peak,
                     "traffic": ncu_traffic("append", "append"),
                     "algorithmic_bytes_per_launch": nbytes},
        "gpu_launches": args.steps, "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line))
    b.lse_kv_arena_destroy(arena)


FRAG_METRIC = "fragment-addressing overhead, % of the contiguous-cache time (worst case)"


def _step_times(call, steps, flush):
    """Device times (ms) of `steps` graph replays of one partial + merge
    step, L2 flushed before each outside the interval."""
    import torch
    g = torch.cuda.CUDAGraph()
    saved = call.stream
    with torch.cuda.graph(g):
        call.stream = torch.cuda.current_stream()
        call.run()
    call.stream = saved
    for i in range(3):
        flush.fill_(i)
        g.replay()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.fill_(i & 0xff)
        ev[i][0].record()
        g.replay()
        ev[i][1].record()
    torch.cuda.synchronize()
    assert call.device_error() == 0, "device error during the timed steps"
    return [e[0].elapsed_time(e[1]) for e in ev]


def run_frag_ab(args, world, rank, local):
    """The releases page's fragment-addressing measurements on this kernel:
    the same keys through a shuffled page table (256 KiB fragments in random
    order) and through an identity table over a contiguous cache, at 16K
    context with one query row and at 68K with eight; and split attention
    against a forced-unsplit plan (one CTA per kv head) at 65,656 keys with
    four query rows.  Outputs of each pair are compared bit for bit."""
    import torch
    torch.cuda.set_device(local)
    from verify_attention_paged_b200 import binding as b
    from verify_attention_paged_b200 import workloads as wl
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    props = torch.cuda.get_device_properties(local)
    optin = getattr(props, "shared_memory_per_block_optin", 232448)
    cases = []
    with ClockSampler(local) as clk:
        for w in wl.fragment_ab_cases():
            if w.name.startswith("split"):
                variants = [("split", w, None),
                            ("unsplit", w, dict(n_sms=w.n_kv_heads, smem_optin=optin,
                                                ctas_per_sm=0, allow_tcgen05=1))]
            else:
                variants = [("shuffled", w, None), ("contiguous", wl.contiguous_copy(w), None)]
            res = {}
            for tag, wv, limits in variants:
                call = b.DeviceCall(wv, plan_limits=limits)
                for _ in range(args.warmup):
                    flush.fill_(1)
                    call.run()
                t = _step_times(call, args.steps, flush)
                out, lse = call.run()
                torch.cuda.synchronize()
                res[tag] = dict(us=statistics.median(t) * 1e3, kernel=call.info["kernel_name"],
                                ctas=call.info["ctas"], out=out[:wv.total_rows].cpu(),
                                lse=lse[:wv.total_rows].cpu())
                call.close()
            (ta, ra), (tb, rb) = res.items()
            same = bool(torch.equal(ra["out"], rb["out"]) and torch.equal(ra["lse"], rb["lse"]))
            diff = float((ra["out"] - rb["out"]).abs().max())
            case = {"case": w.name, "keys": int(w.seq_lens.sum()), "rows": w.total_rows,
                    "kv_bytes": w.kv_bytes(), "outputs_identical": same,
                    "max_abs_diff": diff}
            for tag, r in res.items():
                case[f"{tag}_us"] = r["us"]
                case[f"{tag}_ctas"] = r["ctas"]
                case["kernel"] = r["kernel"]
            if tb == "contiguous":
                case["overhead_pct"] = (ra["us"] / rb["us"] - 1.0) * 100.0
            else:
                case["unsplit_over_split"] = rb["us"] / ra["us"]
            cases.append(case)
            del res
    worst = max(c["overhead_pct"] for c in cases if "overhead_pct" in c)
    if rank == 0:
        print(json.dumps({
            "metric": FRAG_METRIC, "value": worst, "unit": "%", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "fragment_ab", "fragment_bytes": 256 << 10,
                       "heads": "24/4", "head_dim": 128,
                       "l2": "flushed before every step (256 MiB write)",
                       "timing": "median of CUDA events around graph replays of partial + merge"},
            "cases": cases, "gpu_launches": 2 * args.steps * 2 * len(cases),
            "clocks": clk.summary()}), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.workload == "fragment_ab":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the fragment-addressing A/B has no separate reference arm"}))
            return
        run_frag_ab(args, world, rank, local)
        return
    if args.workload == "append":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the append has no separate reference arm"}))
            return
        run_append(args, world, rank, local)
        return
    from verify_attention_paged_b200 import workloads as wl
    # the five configurations, then the long query block (its own roofline)
    names = list(wl.NAMES) + ["prefill_block"] if args.workload == "all" else [args.workload]
    if args.impl == "reference":
        head = HEADLINE if HEADLINE in names else names[0]
        run_reference(args, wl.BUILDERS[head](), world, rank)
    else:
        run_ours(args, names, world, rank, local)


if __name__ == "__main__":
    main()
