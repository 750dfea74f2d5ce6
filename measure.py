#!/usr/bin/env python
"""Measurement commands for libmla beside the benchmark (one GPU, synthetic seeded inputs).

    python measure.py profile --batch 32 --seqlen 4096 --steps 3 [--kernel 0|2|3]
        runs mla_decode a few times on a paged case smaller than the benchmark's: the
        command to put under ncu.
    python measure.py profile-absorb --batch 64 --steps 2
        runs mla_absorb_q and mla_absorb_o in turn on the layer inputs at that batch (H = 128).
    python measure.py absorb [--batch 64 256] [--calls 40]
        times the two absorption GEMMs against their HBM roofline, L2 emptied between calls.
    python measure.py multi [--batch 64] [--seqlen 8192] [--calls 30]
        times mla_decode_multi (several causal query tokens per sequence) for a few
        (s_q, heads) splits of the 128 rows against the one-token call.
    python measure.py noalloc [--calls 30]
        times mla_decode and mla_decode_noalloc on the headline case (B=64, H=128, T=8192).

Every case is seeded and synthetic (mla_synth: latent dims x0.5, rope dims and q x1,
shuffled 64-token pages).  Times are CUDA-event medians on the current stream after
warm-up; a decode cache of the headline size (604 MB) is larger than L2, so decode
calls need no flush between them.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mla_latent_kv_22_b200 as M  # noqa: E402
import mla_synth as S  # noqa: E402

H = 128


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _decode_tensors(case):
    q, kv = _bf16(case.q), _bf16(case.kv_cache)
    bt = torch.from_numpy(case.block_table).cuda()
    sl = torch.from_numpy(case.cache_seqlens).cuda()
    return q, kv, bt, sl


def _check_device(label: str) -> None:
    status = M.mla_get_device_error()
    if status:
        raise SystemExit(f"{label}: device error {status} ({M.mla_status_string(status)})")


def _median_us(call, calls: int) -> float:
    ts = []
    for _ in range(calls):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1000.0)
    return float(np.median(ts))


def cmd_profile(a) -> None:
    M.mla_set_knob("decode_kernel", a.kernel)
    case = S.make_decode_case(a.batch, a.heads, a.seqlen, seed=3, poison=False, latent_std=0.5)
    q, kv, bt, sl = _decode_tensors(case)
    out = torch.empty(a.batch, a.heads, 512, device="cuda")
    lse = torch.empty(a.batch, a.heads, device="cuda")
    for _ in range(a.steps):
        M.mla_decode(q, kv, bt, sl, out, lse, 1.0 / math.sqrt(192.0))
    torch.cuda.synchronize()
    _check_device("profile")
    print(f"profile: B={a.batch} H={a.heads} T={a.seqlen} steps={a.steps} "
          f"kernel={M.mla_selected_decode_kernel(a.heads)} finite={bool(torch.isfinite(out).all())}")


def _absorb_inputs(batch: int):
    li = S.config_layer_inputs(batch)
    qn, qr, wk, wv = (_bf16(x) for x in (li.q_nope, li.q_rope, li.w_uk, li.w_uv))
    qo = torch.empty(batch, H, 576, dtype=torch.bfloat16, device="cuda")
    ol = torch.randn(batch, H, 512, device="cuda", generator=torch.Generator("cuda").manual_seed(batch))
    out = torch.empty(batch, H, 128, device="cuda")
    return qn, qr, wk, wv, qo, ol, out


def cmd_profile_absorb(a) -> None:
    qn, qr, wk, wv, qo, ol, out = _absorb_inputs(a.batch)
    for _ in range(a.steps):
        M.mla_absorb_q(qn, qr, wk, qo)
        M.mla_absorb_o(ol, wv, out)
    torch.cuda.synchronize()
    _check_device("profile-absorb")
    print(f"profile-absorb: B={a.batch} H={H} steps={a.steps} finite={bool(torch.isfinite(out).all())}")


def cmd_absorb(a) -> None:
    """Every call follows a 256 MB read that evicts the previous call's lines from L2 (a
    read leaves no dirty lines to write back inside the timed call).  The event clock
    moves in steps of about 2 µs, so one round times ten (evict, call) pairs between two
    events and subtracts ten evictions timed the same way; the figure is the median over
    rounds of that difference over ten.  Algorithmic bytes: absorb_q reads q_nope, q_rope
    and W_UK and writes q'; absorb_o reads out_latent (fp32) and W_UV and writes out (fp32)."""
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
        hbm = json.load(f)["hbm_gbs"] * 1e9
    evict = torch.ones(64 * 1024 * 1024, device="cuda")
    sink = torch.empty((), device="cuda")
    print("| kernel | B | µs/call | algorithmic MB | GB/s | roofline µs | fraction of measured copy rate |")
    print("|---|---|---|---|---|---|---|")
    for B in a.batch:
        qn, qr, wk, wv, qo, ol, out = _absorb_inputs(B)
        cases = [
            ("absorb_q", lambda: M.mla_absorb_q(qn, qr, wk, qo),
             B * H * (128 + 64) * 2 + H * 128 * 512 * 2 + B * H * 576 * 2),
            ("absorb_o", lambda: M.mla_absorb_o(ol, wv, out),
             B * H * 512 * 4 + H * 512 * 128 * 2 + B * H * 128 * 4),
        ]

        def span(call, reps=10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                torch.sum(evict, dim=0, out=sink)
                if call is not None:
                    call()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) * 1000.0

        for name, fn, nbytes in cases:
            for _ in range(5):
                fn()
            span(fn)
            us = float(np.median([(span(fn) - span(None)) / 10.0 for _ in range(a.calls)]))
            roof = nbytes / hbm * 1e6
            print(f"| {name} | {B} | {us:.1f} | {nbytes / 1e6:.1f} | {nbytes / us / 1e3:.0f} | {roof:.2f} | "
                  f"{roof / us:.3f} |", flush=True)
    _check_device("absorb")


def cmd_multi(a) -> None:
    B, T = a.batch, a.seqlen
    print("| s_q x heads | rows | µs per call | cache TB/s |")
    print("|---|---|---|---|")
    for sq, h in [(1, 128), (2, 64), (4, 32), (8, 16), (2, 16)]:
        case = S.make_decode_case(B, sq * h, T, seed=3, poison=False, latent_std=0.5)
        q, kv, bt, sl = _decode_tensors(case)
        q = q.view(B, sq, h, -1)
        out = torch.empty(B, sq, h, 512, device="cuda")
        lse = torch.empty(B, sq, h, device="cuda")

        def call():
            M.mla_decode_multi(q, kv, bt, sl, out, lse, case.softmax_scale)

        for _ in range(5):
            call()
        torch.cuda.synchronize()
        us = _median_us(call, a.calls)
        _check_device("multi")
        print(f"| {sq} x {h} | {sq * h} | {us:.1f} | {B * T * 576 * 2 / us / 1e6:.2f} |", flush=True)
        del q, kv, bt, sl, out, lse
        torch.cuda.empty_cache()


def cmd_noalloc(a) -> None:
    B, T = 64, 8192
    case = S.make_decode_case(B, H, T, seed=3, poison=False, latent_std=0.5)
    q, kv, bt, sl = _decode_tensors(case)
    out = torch.empty(B, H, 512, device="cuda")
    lse = torch.empty(B, H, device="cuda")
    calls = {
        "mla_decode": lambda: M.mla_decode(q, kv, bt, sl, out, lse, case.softmax_scale),
        "mla_decode_noalloc": lambda: M.mla_decode_noalloc(q, kv, bt, sl, out, lse, case.softmax_scale),
    }
    print("| entry point | µs per call (CUDA events, median) | kernel |")
    print("|---|---|---|")
    for name, call in calls.items():
        for _ in range(5):
            call()
        torch.cuda.synchronize()
        us = _median_us(call, a.calls)
        _check_device(name)
        print(f"| {name} | {us:.1f} | {M.mla_selected_decode_kernel(H)} |", flush=True)


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    sub = ap.add_subparsers(dest="cmd", required=True)
    p = sub.add_parser("profile")
    p.add_argument("--batch", type=int, default=32)
    p.add_argument("--heads", type=int, default=128)
    p.add_argument("--seqlen", type=int, default=4096)
    p.add_argument("--steps", type=int, default=3)
    p.add_argument("--kernel", type=int, default=0, help="0 auto, 2 dim-split pair, 3 head-split pair")
    p = sub.add_parser("profile-absorb")
    p.add_argument("--batch", type=int, default=64)
    p.add_argument("--steps", type=int, default=2)
    p = sub.add_parser("absorb")
    p.add_argument("--batch", type=int, nargs="+", default=[64, 256])
    p.add_argument("--calls", type=int, default=40)
    p = sub.add_parser("multi")
    p.add_argument("--batch", type=int, default=64)
    p.add_argument("--seqlen", type=int, default=8192)
    p.add_argument("--calls", type=int, default=30)
    p = sub.add_parser("noalloc")
    p.add_argument("--calls", type=int, default=30)
    a = ap.parse_args()
    {"profile": cmd_profile, "profile-absorb": cmd_profile_absorb, "absorb": cmd_absorb, "multi": cmd_multi,
     "noalloc": cmd_noalloc}[a.cmd](a)


if __name__ == "__main__":
    main()
