"""Times the two absorption GEMMs (mla_absorb_q, mla_absorb_o) against their HBM
roofline at H=128 and a few batch sizes, with the L2 emptied between calls.

    python -m mla_latent_kv_22_b200.time_absorb [--batch 64 256] [--calls 40]

Inputs are workload 5's seeded layer inputs (q halves and up-projection weights);
out_latent is random.  Every call follows a 256 MB read that evicts the previous call's
lines from L2 (a read leaves no dirty lines to write back during the timed call).  The
event timer moves in steps of about 2 µs, so one round times ten (evict, call) pairs
between two events and subtracts ten evictions timed the same way; the figure is the
median over rounds of that difference divided by ten.  Algorithmic bytes: absorb_q
reads q_nope, q_rope and W_UK and writes q'; absorb_o reads out_latent (fp32) and W_UV
and writes out (fp32).
"""
import argparse
import json
import os

import numpy as np
import torch

import mla_latent_kv_22_b200 as M
import mla_synth as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--batch", type=int, nargs="+", default=[64, 256])
    ap.add_argument("--calls", type=int, default=40)
    a = ap.parse_args()
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
        hbm = json.load(f)["hbm_gbs"] * 1e9
    evict = torch.ones(64 * 1024 * 1024, device="cuda")  # 256 MB, twice the L2
    sink = torch.empty((), device="cuda")
    H = 128
    print("| kernel | B | µs/call | algorithmic MB | GB/s | roofline µs | fraction of measured copy rate |")
    print("|---|---|---|---|---|---|---|")
    for B in a.batch:
        li = S.config_layer_inputs(B)
        qn, qr, wk, wv = (_bf16(x) for x in (li.q_nope, li.q_rope, li.w_uk, li.w_uv))
        qo = torch.empty(B, H, 576, dtype=torch.bfloat16, device="cuda")
        ol = torch.randn(B, H, 512, device="cuda", generator=torch.Generator("cuda").manual_seed(B))
        out = torch.empty(B, H, 128, device="cuda")
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
            ts = [(span(fn) - span(None)) / 10.0 for _ in range(a.calls)]
            us = float(np.median(ts))
            roof = nbytes / hbm * 1e6
            print(f"| {name} | {B} | {us:.1f} | {nbytes / 1e6:.1f} | {nbytes / us / 1e3:.0f} | {roof:.2f} | "
                  f"{roof / us:.3f} |")


if __name__ == "__main__":
    main()
