#!/usr/bin/env python
"""Benchmark of absorbed-MLA decode on B200: one JSON line on rank 0.

Workload: paged absorbed decode, B=64 sequences x H=128 heads, every sequence
T=8192 tokens (64-token pages, shuffled block table, latent dims ~N(0, 0.25),
rope dims and q ~N(0,1), bf16), softmax scale 1/sqrt(192), seed 3.  A step is
one mla_decode call: the split-KV decode kernel (whose CTAs derive the split
schedule from the lengths) and the LSE combine.  The 630 MB working set is larger than the 126 MB L2, so consecutive
steps stream the cache from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 it runs under torchrun, one replica per GPU (no data-path
collective; the process group only times the job as the max over ranks).
``--impl reference`` times the fp64 CPU oracle on the host cores instead, on whole steps
of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode µs/step, KV HBM TB/s & % roofline at B=64,H=128,T=8192"
UNIT = "us/step"
B, H, T, PAGE, D, DV = 64, 128, 8192, 64, 576, 512
SEED = 3
WORKLOAD = ("paged absorbed MLA decode, B=64 seqs x H=128 heads, T=8192 tokens each, 576-wide bf16 rows "
            "(512 latent x0.5 + 64 rope), 64-token pages, shuffled block table, softmax_scale=1/sqrt(192), seed 3")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def algorithmic_bytes(b: int, h: int, t: int, max_blocks: int) -> int:
    """Bytes a decode step must move at least once: every cached row (576 bf16),
    q' (576 bf16 per head), out (512 fp32 per head), lse, block table, lengths."""
    per_seq = h * D * 2 + h * DV * 4 + h * 4 + max_blocks * 4 + 4
    return b * t * D * 2 + b * per_seq


def algorithmic_flops(b: int, h: int, t: int) -> int:
    """2 flops per multiply-add: scores over 576 dims and values over 512 dims."""
    return 2 * b * h * t * (D + DV)


def split_pieces(seqlens, workers: int, min_pages: int = 4, granule: int = 4, whole_slack: int = 16,
                 piece_cost: int = 8):
    """The library's split rule for the default knobs, restated on the host: per worker, its
    pieces as (sequence, first page, end page).  Sequences are laid end to end, each as
    piece_cost units of fixed cost followed by its pages; worker w takes the pages inside
    units [w q, (w+1) q), q = max(ceil(units / P), min_pages) rounded up to the granule.
    When batch <= P and the longest sequence is at most whole_slack pages above the
    pages-only share, every sequence runs whole on worker b."""
    pages = [(int(t) + PAGE - 1) // PAGE if 0 <= int(t) else 0 for t in seqlens]
    b_n = len(pages)

    def share(total):
        q = max(-(-total // workers), min_pages, 1)
        return -(-q // granule) * granule

    if whole_slack >= 0 and b_n <= workers and max(pages, default=0) <= share(sum(pages)) + whole_slack:
        return [[(b, 0, n)] if n > 0 else [] for b, n in enumerate(pages)]
    units = [n + piece_cost if n > 0 else 0 for n in pages]
    total = sum(units)
    q = share(total)
    starts = [0]
    for u in units:
        starts.append(starts[-1] + u)
    plan = []
    for w in range(-(-total // q)):
        g0, g1 = w * q, min(w * q + q, total)
        pieces = []
        for b, n in enumerate(pages):
            pos = starts[b] + piece_cost
            lo, hi = max(g0, pos), min(g1, pos + n)
            if n > 0 and lo < hi:
                pieces.append((b, lo - pos, hi - pos))
        plan.append(pieces)
    return plan


def split_partial_bytes(seqlens, heads: int, workers: int) -> int:
    """Bytes of split partials one decode step moves: every piece of a split sequence
    writes its normalised output (512 fp32 per head) and lse, and the combine reads them
    back (the split as `split_pieces` gives it)."""
    pages = [(int(t) + PAGE - 1) // PAGE for t in seqlens]
    split = sum(1 for pieces in split_pieces(seqlens, workers) for (b, lo, hi) in pieces
                if not (lo == 0 and hi == pages[b]))
    return 2 * split * heads * (DV + 1) * 4


def measured_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS}, "fallback"


def strip_comments(src: str) -> str:
    """C++ source without comments and blank space, so that editing a comment does not
    count as changing the code (no string literal in these files contains //)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def decode_source_hash(kernel: str) -> str:
    """Hash of the code of the decode kernel that ran (and the headers it uses), comments
    and layout ignored, to tie an ncu traffic figure to exactly that code."""
    files = {"dimsplit": ["decode_tc.cu", "sm100_ptx.cuh"], "pair": ["decode_pair.cu", "sm100_ptx.cuh"]}[kernel]
    files += ["worker_range.cuh", "mla_device.cuh", "mla_internal.h"]
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_latent_kv_22_b200", "csrc")
    for name in files:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, kernel_hash: str):
    """DRAM bytes per decode launch (headline workload) from the committed ncu summary,
    if it was taken on the current sources of that kernel (else None)."""
    p = os.path.join(ROOT, "profiles", f"decode_{kernel}_headline_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_hash:
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# Distributed plumbing (replicas only: barrier + max over ranks).
# ---------------------------------------------------------------------------

def dist_env() -> tuple[int, int, int]:
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def init_dist(backend: str):
    import torch.distributed as dist
    rank, _, world = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(value: float, dist, device=None) -> float:
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device=None) -> None:
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# Clocks during the timed region (NVML polling thread).
# ---------------------------------------------------------------------------

_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML from a host thread.

    Every sample carries a host timestamp, so the summary can keep only the samples
    taken inside the device-timed region; when that region is too short for three
    samples, it reports all samples of the GPU-busy window (warm-up, timed and
    end-to-end loops, all under the same load) and says so."""

    def __init__(self, device_index: int):
        self.samples: list[tuple[float, int, int]] = []
        self._stop = threading.Event()
        self._ok = False
        self.window = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # no NVML: report that
            self.error = str(e)
            self.max_mhz = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((time.perf_counter(), sm, rs))
            except Exception:
                time.sleep(0.001)

    def start(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def stop(self):
        if self._ok:
            self._stop.set()
            self._t.join()

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def summary(self) -> dict:
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "error": getattr(self, "error", "")}
        picked, where = self.samples, "warm-up + timed + end-to-end loops"
        if self.window is not None:
            inside = [x for x in self.samples if self.window[0] <= x[0] <= self.window[1]]
            if len(inside) >= 3:
                picked, where = inside, "timed region"
        if not picked:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [x[1] for x in picked]
        mask = 0
        for x in picked:
            mask |= x[2]
        reasons = [n for bit, n in _REASONS.items() if mask & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(picked), "sm_mhz_min": min(mhz), "window": where}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the workload.
# ---------------------------------------------------------------------------

def headline_case():
    """The timed workload's inputs (host arrays), the same for both arms."""
    import mla_synth as S
    return S.config_case(3, headline=True, poison=False)


def workload_config(world: int) -> dict:
    """The `config` object of the JSON line; both arms print the same one."""
    return {"workload": WORKLOAD, "global_batch": B * world, "seq_len": T, "heads": H, "page": PAGE,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (630 MB working set, 126 MB L2); no flush"}


def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return os.cpu_count() or 1


def time_oracle_step(case) -> float:
    """Seconds the oracle takes for one whole step: every sequence, every head."""
    import oracle as O
    t0 = time.perf_counter()
    O.mla_decode_ref(case.q, case.kv_cache, case.block_table, case.cache_seqlens, case.softmax_scale)
    return time.perf_counter() - t0


def cpu_baseline(case, budget_s: float = 15.0) -> dict:
    """The oracle timed on whole steps of the workload (all 64 sequences, all heads)."""
    t1 = time_oracle_step(case)
    reps = max(3, min(20, int(budget_s / max(t1, 1e-3))))
    ts = [time_oracle_step(case) for _ in range(reps)]
    return {"value": statistics.median(ts) * 1e6, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle on the whole step (64 sequences x 128 heads, T=8192), "
                      f"median of {reps} steps after one untimed step"}


def run_reference(args) -> None:
    rank, _, world = dist_env()
    if world > 1 and rank != 0:
        return
    case = headline_case()
    for _ in range(args.warmup):
        time_oracle_step(case)
    ts = [time_oracle_step(case) for _ in range(args.steps)]
    us = statistics.mean(ts) * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(world),
        "cpu_baseline": {"value": us, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": "every step runs the fp64 oracle on the whole workload "
                                   "(64 sequences x 128 heads, T=8192); mean over the timed steps"},
        "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Our arm.
# ---------------------------------------------------------------------------

def run_ours(args) -> None:
    import torch

    import mla_latent_kv_22_b200 as M

    rank, local_rank, world = dist_env()
    M.mla_set_knob("decode_kernel", {"auto": 0, "dimsplit": 2, "pair": 3}[args.kernel])
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = init_dist("nccl")

    case = headline_case()
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    q, kv = to_dev(case.q), to_dev(case.kv_cache)
    bt = torch.from_numpy(case.block_table).to(device)
    sl = torch.from_numpy(case.cache_seqlens).to(device)
    out = torch.empty(B, H, DV, device=device)
    lse = torch.empty(B, H, device=device)
    max_blocks = int(case.block_table.shape[1])
    stream = torch.cuda.current_stream(device)

    def step():
        M.mla_decode(q, kv, bt, sl, out, lse, case.softmax_scale, stream=stream)

    clk = ClockSampler(local_rank).start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if M.mla_get_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    # ---- device-timed region: exactly K steps (no per-launch events inside it) ----
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    torch.cuda.synchronize(device)
    h0 = time.perf_counter()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    clk.mark(h0, time.perf_counter())
    barrier(dist, device)
    ms_total = e0.elapsed_time(e1)
    ms_step = max_over_ranks(ms_total / args.steps, dist, device)
    if M.mla_get_device_error() != 0:
        raise RuntimeError("device error during the timed region")

    # ---- per-launch times (decode, combine; the schedule slot is the empty interval the
    # library records where a schedule launch used to be): CUDA events around each launch
    # on the library's stream, in a separate pass of K steps so that they do not break
    # the overlap of consecutive launches in the timed region above ----
    M.mla_timing_enable(True)
    for _ in range(args.steps):
        step()
    kern_ms, calls = M.mla_timing_read()
    M.mla_timing_enable(False)

    # ---- end to end through the public API: host buffers, copies inside the region ----
    # Every step uploads its inputs (q', block table, lengths) from pinned host memory
    # and downloads its result (out, lse), as a serving loop would: upload, decode and
    # download run on three streams over two buffer slots, so step i's upload and step
    # i-1's download overlap step i's decode.  Events keep each slot's reuse ordered
    # (an upload waits for the decode that last read the slot; a decode waits for the
    # download of the output it overwrites).  All decodes stay on one stream, so the
    # library's workspace is never used by two calls at once.
    q_h = torch.from_numpy(np.ascontiguousarray(case.q).view(np.int16)).view(torch.bfloat16).pin_memory()
    bt_h = torch.from_numpy(case.block_table).pin_memory()
    sl_h = torch.from_numpy(case.cache_seqlens).pin_memory()
    out_h = [torch.empty(B, H, DV).pin_memory() for _ in range(2)]
    lse_h = [torch.empty(B, H).pin_memory() for _ in range(2)]
    q_d = [torch.empty_like(q) for _ in range(2)]
    bt_d = [torch.empty_like(bt) for _ in range(2)]
    sl_d = [torch.empty_like(sl) for _ in range(2)]
    out_d = [torch.empty_like(out) for _ in range(2)]
    lse_d = [torch.empty_like(lse) for _ in range(2)]
    s_up, s_down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_dec = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]
    for k in range(2):  # all slots start free
        ev_dec[k].record(stream)
        ev_down[k].record(stream)

    def e2e_step(i):
        k = i & 1
        with torch.cuda.stream(s_up):
            s_up.wait_event(ev_dec[k])
            q_d[k].copy_(q_h, non_blocking=True)
            bt_d[k].copy_(bt_h, non_blocking=True)
            sl_d[k].copy_(sl_h, non_blocking=True)
            ev_up[k].record(s_up)
        stream.wait_event(ev_up[k])
        stream.wait_event(ev_down[k])
        M.mla_decode(q_d[k], kv, bt_d[k], sl_d[k], out_d[k], lse_d[k], case.softmax_scale, stream=stream)
        ev_dec[k].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev_dec[k])
            out_h[k].copy_(out_d[k], non_blocking=True)
            lse_h[k].copy_(lse_d[k], non_blocking=True)
            ev_down[k].record(s_down)

    for i in range(max(3, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    s_up.wait_stream(stream)  # the timed region starts before the first upload
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(ev_down[(args.steps - 1) & 1])  # ... and ends after the last download
    stream.wait_event(ev_down[args.steps & 1])
    f1.record(stream)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    clk.stop()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / args.steps, dist, device)
    if not (torch.equal(out_h[(args.steps - 1) & 1], out.cpu()) and torch.equal(lse_h[(args.steps - 1) & 1], lse.cpu())):
        raise RuntimeError("end-to-end result differs from the device-timed result")
    h2d = q_h.numel() * 2 + bt_h.numel() * 4 + sl_h.numel() * 4
    d2h = out_h[0].numel() * 4 + lse_h[0].numel() * 4

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    peaks, peak_kind = measured_peaks()
    alg_bytes = algorithmic_bytes(B, H, T, max_blocks)
    flops = algorithmic_flops(B, H, T)
    dec_ms = kern_ms[1] / max(calls, 1)
    achieved = alg_bytes / (dec_ms * 1e-3) / 1e9  # GB/s
    hbm_peak = float(peaks["hbm_gbs"])
    roofline_us = max(alg_bytes / (hbm_peak * 1e9), flops / (float(peaks["bf16_tflops"]) * 1e12)) * 1e6
    kernel = {2: "dimsplit", 3: "pair"}[M.mla_selected_decode_kernel(H)]
    workers = torch.cuda.get_device_properties(device).multi_processor_count // 2  # CTA pairs (occupancy 1)
    partial_bytes = split_partial_bytes(case.cache_seqlens, H, workers)
    khash = decode_source_hash(kernel)
    traffic = ncu_traffic(kernel, khash)
    us_step = ms_step * 1e3
    line = {
        "metric": METRIC, "value": us_step, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(world),
        "kv_tbps": B * T * D * 2 / (ms_step * 1e-3) / 1e12,
        "tflops": flops / (ms_step * 1e-3) / 1e12,
        "roofline_us": roofline_us,
        "step_roofline_frac": roofline_us / us_step,
        "launch_us": {"decode": dec_ms * 1e3, "combine": kern_ms[2] / max(calls, 1) * 1e3,
                      "note": "separate pass with CUDA events around each launch; the decode CTAs "
                              "derive the split schedule themselves (no schedule launch)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic,
                     "peak_kind": peak_kind, "kernel": f"decode ({kernel})",
                     "algorithmic_bytes_per_launch": alg_bytes, "source_hash": khash,
                     "partial_bytes": partial_bytes},
        "gpu_launches": 2 * args.steps,
        "e2e": {"value": e2e_ms * 1e3, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clk.summary(),
        "decode_kernel": kernel,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case)
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=["auto", "dimsplit", "pair"], default="auto",
                    help="decode kernel (default: the library's choice)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
