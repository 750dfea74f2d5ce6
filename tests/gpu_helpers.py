"""Shared helpers of the GPU parity tests: upload seeded inputs, run the library,
compare with the oracle under the stated tolerances."""
import numpy as np
import torch

import mla_latent_kv_22_b200 as M

# Tolerances (bf16 inputs, fp32 accumulation): elementwise on out, absolute on lse.
OUT_ATOL, OUT_RTOL, LSE_ATOL = 1e-2, 1e-2, 2e-3


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def upload(case):
    q = bf16_dev(case.q)
    kv = bf16_dev(case.kv_cache)
    bt = None if case.block_table is None else torch.from_numpy(case.block_table).cuda()
    sl = torch.from_numpy(case.cache_seqlens).cuda()
    return q, kv, bt, sl


def run_decode(case, dev=None, scale=None):
    q, kv, bt, sl = dev if dev is not None else upload(case)
    B, H = case.B, case.H
    out = torch.full((B, H, 512), float("nan"), device="cuda")
    lse = torch.full((B, H), float("nan"), device="cuda")
    M.mla_decode(q, kv, bt, sl, out, lse, case.softmax_scale if scale is None else scale)
    err = M.mla_get_device_error()
    return out, lse, err


def assert_close(out, lse, ref_out, ref_lse, what=""):
    o = out.double().cpu().numpy() if isinstance(out, torch.Tensor) else np.asarray(out, np.float64)
    l = lse.double().cpu().numpy() if isinstance(lse, torch.Tensor) else np.asarray(lse, np.float64)
    assert o.shape == ref_out.shape and l.shape == ref_lse.shape, what
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(l), fin), f"{what}: lse finiteness differs"
    d_out = np.abs(o - ref_out)
    bad = d_out > OUT_ATOL + OUT_RTOL * np.abs(ref_out)
    assert not bad.any(), f"{what}: {bad.sum()} out elements off, max |diff| {d_out.max():.3e}"
    d_lse = np.abs(l[fin] - ref_lse[fin]) if fin.any() else np.zeros(1)
    assert d_lse.max() <= LSE_ATOL, f"{what}: max |lse diff| {d_lse.max():.3e}"
    assert np.array_equal(l[~fin], ref_lse[~fin]), f"{what}: non-finite lse values differ"
    rel_l2 = np.linalg.norm(o - ref_out) / max(np.linalg.norm(ref_out), 1e-30)
    return dict(max_abs_out=float(d_out.max()), max_abs_lse=float(d_lse.max()), rel_l2=float(rel_l2))
