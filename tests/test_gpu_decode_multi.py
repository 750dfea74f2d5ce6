"""GPU parity of mla_decode_multi (s_q causal query tokens per sequence) against the
fp64 oracle on the same seeded inputs.

Same tolerances as the single-token decode: |out - ref| <= 1e-2 + 1e-2 |ref|
elementwise, |lse - ref| <= 2e-3, and rows whose window is empty must be exactly
out = 0, lse = -inf.  The cases cover windows that are empty for some queries
(T < s_q), windows that end inside the previous page, split sequences whose last
piece holds no token of some queries' windows, 8 x 16 = 128 rows, row counts
that are not a multiple of 16, and more than 128 rows (run as groups of 128).
"""
import numpy as np
import pytest
import torch

import mla_latent_kv_22_b200 as M
import mla_synth as S
import oracle as O
from gpu_helpers import assert_close, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=[2, 3], ids=["dimsplit", "pair"])
def kernel(request):
    """Every test runs on both decode kernels."""
    M.mla_set_knob("decode_kernel", request.param)
    yield request.param
    for k in ("num_workers", "min_pages", "decode_kernel"):
        M.mla_set_knob(k, 0)


def _case(B, s_q, H, lens, seed, **kw):
    c = S.make_decode_case(B, s_q * H, lens, seed=seed, **kw)
    return c, c.q.reshape(B, s_q, H, -1)


def _run(c, q_np, s_q, H, dev=None):
    q, kv, bt, sl = dev if dev is not None else upload(c)
    q = q.view(c.B, s_q, H, -1)
    out = torch.full((c.B, s_q, H, 512), float("nan"), device="cuda")
    lse = torch.full((c.B, s_q, H), float("nan"), device="cuda")
    M.mla_decode_multi(q, kv, bt, sl, out, lse, c.softmax_scale)
    return out, lse, M.mla_get_device_error()


def _ref(c, q_np):
    return O.mla_decode_multi_ref(q_np, c.kv_cache, c.block_table, c.cache_seqlens, c.softmax_scale)


@pytest.mark.parametrize("B,s_q,H,lens", [
    (3, 2, 64, [1, 100, 700]),       # T = 1: query 0 sees nothing
    (2, 4, 32, [3, 1000]),           # T < s_q
    (4, 8, 16, [0, 7, 64, 513]),     # 128 rows; an empty sequence; a window ending at a page end
    (2, 3, 40, [130, 2]),            # 120 rows
    (5, 2, 1, [65, 64, 63, 1, 2]),   # one head per query token
    (2, 2, 128, [300, 5]),           # 256 rows: two groups of 128
    (3, 3, 50, [1, 100, 129]),       # 150 rows: groups of 128 and 22
])
def test_multi_matches_oracle(B, s_q, H, lens):
    c, q = _case(B, s_q, H, lens, seed=70 + s_q * H, poison=True)
    out, lse, err = _run(c, q, s_q, H)
    assert err == 0
    ref_o, ref_l = _ref(c, q)
    assert_close(out, lse, ref_o, ref_l, f"s_q={s_q} H={H}")
    empty = np.isneginf(ref_l)
    assert (out.cpu().numpy()[empty] == 0).all()


@pytest.mark.parametrize("workers", [1, 5, 40])
@pytest.mark.parametrize("H", [32, 96])
def test_multi_split_pieces_without_tokens_for_some_queries(workers, H):
    # 65 pages with one token on the last: at 2 pages per worker the last worker's
    # piece holds token 4096 only, which queries 0..2 of s_q = 4 do not see, so their
    # partial for that piece is empty and the combine must give it zero weight.  At
    # H = 96 the 384 rows run as three groups over the same schedule.
    M.mla_set_knob("min_pages", 1)
    M.mla_set_knob("num_workers", workers)
    c, q = _case(2, 4, H, [4097, 300], seed=81, poison=True)
    out, lse, err = _run(c, q, 4, H)
    assert err == 0
    assert_close(out, lse, *_ref(c, q), f"{workers} workers, H={H}")


def test_multi_single_token_is_bit_exact_decode():
    c, q = _case(3, 1, 128, [1, 700, 4096], seed=82, poison=True)
    dev = upload(c)
    out_m, lse_m, err = _run(c, q, 1, 128, dev)
    assert err == 0
    out = torch.full((3, 128, 512), float("nan"), device="cuda")
    lse = torch.full((3, 128), float("nan"), device="cuda")
    M.mla_decode(dev[0], dev[1], dev[2], dev[3], out, lse, c.softmax_scale)
    assert torch.equal(out_m[:, 0], out) and torch.equal(lse_m[:, 0], lse)


def test_multi_paged_equals_contiguous_bit_exact():
    lens = [200, 3, 1000]
    a, qa = _case(3, 4, 16, lens, seed=83, paged=True, poison=True)
    b, qb = _case(3, 4, 16, lens, seed=83, paged=False, poison=True)
    oa, la, ea = _run(a, qa, 4, 16)
    ob, lb, eb = _run(b, qb, 4, 16)
    assert ea == 0 and eb == 0
    assert torch.equal(oa, ob) and torch.equal(la, lb)


def test_multi_rejects_what_it_does_not_handle():
    c, q = _case(2, 2, 64, [100, 5], seed=84, poison=False)
    dev = upload(c)
    too_many = torch.zeros(2, 17, 128, 576, dtype=torch.bfloat16, device="cuda")  # 2176 rows
    out = torch.zeros(2, 17, 128, 512, device="cuda")
    lse = torch.zeros(2, 17, 128, device="cuda")
    with pytest.raises(M.MlaError) as ei:
        M.mla_decode_multi(too_many, dev[1], dev[2], dev[3], out, lse, c.softmax_scale)
    assert ei.value.name == "MLA_ERR_UNSUPPORTED"
    M.mla_set_knob("decode_kernel", 1)  # names no decode kernel
    with pytest.raises(M.MlaError) as ei:
        _run(c, q, 2, 64, dev)
    assert ei.value.name == "MLA_ERR_UNSUPPORTED"
