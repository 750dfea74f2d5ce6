"""mla_decode_noalloc: the decode for callers that cannot allocate device memory
(a runtime that has reserved all device memory for its own pool, paths that cannot
absorb cudaMalloc's device sync).  It uses
the library's static device scratch instead of the workspace.

Checked through the C ABI against the fp64 oracle (mla_decode_ref) and against
mla_decode, on two calls in a row with different inputs (the scratch keeps the
previous call's contents, so a stale read would show), within the tolerances the
other GPU tests use.  This file is collected last
so that a run stopping at the first failure has run every other test already.
"""
import ctypes

import numpy as np
import pytest
import torch

import mla_latent_kv_22_b200 as M
import mla_synth as S
import oracle as O
from gpu_helpers import LSE_ATOL, OUT_ATOL, OUT_RTOL, assert_close, upload

pytestmark = pytest.mark.gpu


def _call(fn, case, dev):
    q, kv, bt, sl = dev
    B, H = case.B, case.H
    out = torch.full((B, H, 512), float("nan"), device="cuda")
    lse = torch.full((B, H), float("nan"), device="cuda")
    max_blocks = int(bt.shape[1]) if bt is not None else int(kv.shape[1]) // 64
    num_pages = int(kv.shape[0]) if bt is not None else 0
    status = fn(q.data_ptr(), kv.data_ptr(), None if bt is None else bt.data_ptr(), sl.data_ptr(), out.data_ptr(),
                lse.data_ptr(), B, H, num_pages, max_blocks, ctypes.c_float(case.softmax_scale),
                torch.cuda.current_stream().cuda_stream)
    assert status == 0, M.lib.mla_last_error_message().decode()
    assert M.mla_get_device_error() == 0
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def _close(a, b):
    (ao, al), (bo, bl) = a, b
    assert np.isfinite(ao).all() and np.isfinite(al).all()
    assert (np.abs(ao - bo) <= OUT_ATOL + OUT_RTOL * np.abs(bo)).all(), np.abs(ao - bo).max()
    assert np.abs(al - bl).max() <= LSE_ATOL


def _oracle(case):
    return O.mla_decode_ref(case.q, case.kv_cache, case.block_table, case.cache_seqlens, case.softmax_scale)


def test_noalloc_matches_oracle_and_mla_decode_on_two_calls_in_a_row():
    cases = [S.make_decode_case(16, 128, S.uniform_seqlens(3, 16, 100, 4000), seed=71, poison=True),
             S.make_decode_case(5, 128, [4096, 1, 64, 65, 3000], seed=72, poison=True)]
    for i, case in enumerate(cases):
        dev = upload(case)
        got = _call(M.lib.mla_decode_noalloc, case, dev)
        assert_close(*got, *_oracle(case), what=f"noalloc case {i} vs oracle")
        _close(got, _call(M.lib.mla_decode, case, dev))


def test_noalloc_contiguous_and_few_heads():
    case = S.make_decode_case(3, 16, [700, 64, 1], seed=73, paged=False, poison=True)
    dev = upload(case)
    got = _call(M.lib.mla_decode_noalloc, case, dev)
    assert_close(*got, *_oracle(case), what="noalloc contiguous vs oracle")
    _close(got, _call(M.lib.mla_decode, case, dev))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 4M sequences need more schedule metadata than the static scratch holds; the
    # call must refuse before touching the (dummy, aligned) pointers.
    p = 1 << 12
    status = M.lib.mla_decode_noalloc(p, p, p, p, p, p, 4_000_000, 128, 10, 1, ctypes.c_float(0.1), None)
    assert status == 2  # MLA_ERR_UNSUPPORTED
    assert b"static scratch" in M.lib.mla_last_error_message()
