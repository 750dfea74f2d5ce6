"""Times mla_decode_multi (several causal query tokens per sequence) on a cache of the
headline size, B=64 sequences of T=8192 tokens, for a few (s_q, heads) splits of the
rows, against the single-token call with 128 heads.

    python -m mla_latent_kv_22_b200.time_multi [--batch 64] [--seqlen 8192] [--calls 30]

Inputs are seeded synthetic cases (the headline recipe: latent x0.5, rope x1, shuffled
64-token pages); each call is timed with CUDA events, median of --calls.  The cache
(604 MB at the default size) is larger than L2, so no flush is needed between calls.
"""
import argparse

import numpy as np
import torch

import mla_latent_kv_22_b200 as M
import mla_synth as S


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--batch", type=int, default=64)
    ap.add_argument("--seqlen", type=int, default=8192)
    ap.add_argument("--calls", type=int, default=30)
    a = ap.parse_args()
    B, T = a.batch, a.seqlen
    print("| s_q x heads | rows | µs per call | cache TB/s |")
    print("|---|---|---|---|")
    for sq, H in [(1, 128), (2, 64), (4, 32), (8, 16), (2, 16)]:
        case = S.make_decode_case(B, sq * H, T, seed=3, poison=False, latent_std=0.5)
        q = _bf16(case.q).view(B, sq, H, -1)
        kv = _bf16(case.kv_cache)
        bt = torch.from_numpy(case.block_table).cuda()
        sl = torch.from_numpy(case.cache_seqlens).cuda()
        out = torch.empty(B, sq, H, 512, device="cuda")
        lse = torch.empty(B, sq, H, device="cuda")

        def call():
            M.mla_decode_multi(q, kv, bt, sl, out, lse, case.softmax_scale)

        for _ in range(5):
            call()
        torch.cuda.synchronize()
        ts = []
        for _ in range(a.calls):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1000.0)
        if M.mla_get_device_error() != 0:
            raise RuntimeError("device error")
        us = float(np.median(ts))
        print(f"| {sq} x {H} | {sq * H} | {us:.1f} | {B * T * 576 * 2 / us / 1e6:.2f} |", flush=True)
        del q, kv, bt, sl, out, lse
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
