"""Runs mla_decode on a synthetic paged case a few times: the command to put
under a profiler (ncu) for a capture smaller than the benchmark workload.

    python -m mla_latent_kv_22_b200.profile_case --batch 32 --seqlen 4096 --steps 3

With --absorb it runs mla_absorb_q and mla_absorb_o instead, `--steps` times each in
turn, on workload 5's seeded layer inputs at --batch (H = 128) and a random fp32
out_latent.
"""
import argparse
import math

import numpy as np
import torch

import mla_latent_kv_22_b200 as M
import mla_synth as S


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--batch", type=int, default=32)
    ap.add_argument("--heads", type=int, default=128)
    ap.add_argument("--seqlen", type=int, default=4096)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--kernel", type=int, default=0, help="0 auto, 2 dim-split pair, 3 head-split pair")
    ap.add_argument("--absorb", action="store_true", help="run the two absorption GEMMs instead")
    a = ap.parse_args()
    if a.absorb:
        absorb_case(a.batch, a.steps)
        return
    M.mla_set_knob("decode_kernel", a.kernel)
    case = S.make_decode_case(a.batch, a.heads, a.seqlen, seed=3, poison=False, latent_std=0.5)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    q, kv = dev(case.q), dev(case.kv_cache)
    bt = torch.from_numpy(case.block_table).cuda()
    sl = torch.from_numpy(case.cache_seqlens).cuda()
    out = torch.empty(a.batch, a.heads, 512, device="cuda")
    lse = torch.empty(a.batch, a.heads, device="cuda")
    for _ in range(a.steps):
        M.mla_decode(q, kv, bt, sl, out, lse, 1.0 / math.sqrt(192.0))
    torch.cuda.synchronize()
    status = M.mla_get_device_error()
    print(f"profile_case: B={a.batch} H={a.heads} T={a.seqlen} steps={a.steps} device_error={status} "
          f"finite={bool(torch.isfinite(out).all())}")
    if status:
        raise SystemExit(1)


def absorb_case(batch: int, steps: int) -> None:
    H = 128
    li = S.config_layer_inputs(batch)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    qn, qr, wk, wv = (dev(x) for x in (li.q_nope, li.q_rope, li.w_uk, li.w_uv))
    qo = torch.empty(batch, H, 576, dtype=torch.bfloat16, device="cuda")
    ol = torch.randn(batch, H, 512, device="cuda", generator=torch.Generator("cuda").manual_seed(batch))
    out = torch.empty(batch, H, 128, device="cuda")
    for _ in range(steps):
        M.mla_absorb_q(qn, qr, wk, qo)
        M.mla_absorb_o(ol, wv, out)
    torch.cuda.synchronize()
    status = M.mla_get_device_error()
    print(f"profile_case: absorb B={batch} H={H} steps={steps} device_error={status} "
          f"finite={bool(torch.isfinite(out).all())}")
    if status:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
