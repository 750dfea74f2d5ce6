"""GPU parity of mla_decode against the fp64 oracle on the same seeded inputs.

Tolerances: |out - ref| <= 1e-2 + 1e-2 |ref| elementwise and |lse - ref| <= 2e-3.
Full sizes use sampled sequences/heads the oracle computes one by one; reduced
sizes compare every element.  Block-table handling is checked bit-exactly by
comparing paged and contiguous layouts holding the same rows.
"""
import math

import numpy as np
import pytest
import torch

import mla_latent_kv_22_b200 as M
import mla_synth as S
import oracle as O
from gpu_helpers import assert_close, run_decode, upload

pytestmark = pytest.mark.gpu


def oracle_for(case, batch=None, heads=None):
    return O.mla_decode_ref(case.q, case.kv_cache, case.block_table, case.cache_seqlens, case.softmax_scale,
                            batch=batch, heads=heads)


@pytest.fixture(autouse=True, params=[2, 3], ids=["dimsplit", "pair"])
def kernel(request):
    """Every test runs on both decode kernels: 2 = the CTA pair split by latent dims
    (partial scores exchanged through distributed shared memory), 3 = the CTA pair
    split by heads (pair-wide MMAs)."""
    M.mla_set_knob("decode_kernel", request.param)
    yield request.param
    for k in ("num_workers", "min_pages", "decode_kernel", "wait_limit", "withhold_arrive", "split_policy",
              "piece_cost"):
        M.mla_set_knob(k, 0)


def test_config1_tiny_contiguous():
    case = S.config_case(1)
    out, lse, err = run_decode(case)
    assert err == 0
    assert_close(out, lse, *oracle_for(case), "config 1")


def test_config2_paged_full():
    case = S.config_case(2)
    out, lse, err = run_decode(case)
    assert err == 0
    assert_close(out, lse, *oracle_for(case), "config 2")


def test_config3_varlen_full():
    case = S.config_case(3)
    out, lse, err = run_decode(case)
    assert err == 0
    assert_close(out, lse, *oracle_for(case), "config 3 var-len")


@pytest.mark.parametrize("piece_cost", [1, 4, 13, 41])
def test_split_piece_cost_keeps_parity(piece_cost):
    """The split charges each sequence (knob - 1) pages of fixed cost: every charge moves the
    cut points (pieces of 1 to 3 per worker, some workers with none), never the result."""
    M.mla_set_knob("piece_cost", piece_cost)
    case = S.make_decode_case(24, 128, S.uniform_seqlens(41, 24, 1, 3000), seed=41, poison=True)
    out, lse, err = run_decode(case)
    assert err == 0
    assert_close(out, lse, *oracle_for(case), f"piece cost {piece_cost - 1}")


def test_config3_headline_sampled():
    case = S.config_case(3, headline=True)
    out, lse, err = run_decode(case)
    assert err == 0
    bs = [0, 17, 38, 63]
    ref_o, ref_l = oracle_for(case, batch=bs)
    assert_close(out[bs], lse[bs], ref_o, ref_l, "config 3 headline (sampled)")
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


def test_config4_long_context_sampled():
    case = S.config_case(4)
    out, lse, err = run_decode(case)
    assert err == 0
    hs = [0, 5, 64, 127]
    ref_o, ref_l = oracle_for(case, heads=hs)
    assert_close(out[:, hs], lse[:, hs], ref_o, ref_l, "config 4 (sampled heads)")


@pytest.mark.parametrize("lens", [[1, 63, 64, 65, 1000], [0, 7, 0, 129], [4096, 1, 2, 3]])
@pytest.mark.parametrize("H", [16, 128, 1, 100])
def test_edge_lengths_and_heads(lens, H):
    case = S.make_decode_case(len(lens), H, lens, seed=40 + H, poison=True)
    out, lse, err = run_decode(case)
    assert err == 0
    assert_close(out, lse, *oracle_for(case), f"lens {lens} H {H}")
    for b, T in enumerate(lens):
        if T == 0:
            assert (out[b] == 0).all() and torch.isneginf(lse[b]).all()


def test_poison_never_reaches_output():
    case = S.make_decode_case(6, 128, [63, 64, 65, 1, 200, 127], seed=41, poison=True)
    out, lse, err = run_decode(case)
    assert err == 0 and torch.isfinite(out).all() and torch.isfinite(lse).all()
    assert_close(out, lse, *oracle_for(case), "poison")


@pytest.mark.parametrize("scale", [0.0, -0.0625, 0.5])
def test_softmax_scale_zero_negative_large(scale):
    """A zero scale gives uniform weights, a negative one flips the ranking, a large
    one makes the running maximum jump several times within a sequence."""
    case = S.make_decode_case(4, 128, [1, 63, 700, 2000], seed=45, poison=True, softmax_scale=scale)
    out, lse, err = run_decode(case)
    assert err == 0
    assert_close(out, lse, *oracle_for(case), f"scale {scale}")


def test_growing_scores_force_rescales():
    """The rope dims grow along the sequence (factor 1 + 40 t / T): they enter the
    scores but not V, so the running maximum rises 3-9 times per head (by more than
    the lazy-rescale threshold each time) while the values keep their size."""
    lens = [640, 2000, 4100]
    case = S.make_decode_case(3, 128, lens, seed=46, poison=True)
    kv = S.bf16_bits_to_f32(case.kv_cache)
    for b, T in enumerate(lens):
        for t in range(T):
            pg, r = case.block_table[b, t // 64], t % 64
            kv[pg, r, 512:] *= 1.0 + 40.0 * t / T
    case.kv_cache = S.f32_to_bf16_bits(kv)
    out, lse, err = run_decode(case)
    assert err == 0
    assert_close(out, lse, *oracle_for(case), "growing scores")


@pytest.mark.parametrize("workers", [1, 2, 7, 64, 148])
def test_forced_split_counts_and_paged_equals_contiguous(workers):
    lens = [3000, 65, 1, 2048, 777]
    paged = S.make_decode_case(5, 128, lens, seed=42, paged=True)
    contig = S.make_decode_case(5, 128, lens, seed=42, paged=False)
    M.mla_set_knob("num_workers", workers)
    M.mla_set_knob("min_pages", 1)
    po, pl, e1 = run_decode(paged)
    co, cl, e2 = run_decode(contig)
    assert e1 == 0 and e2 == 0
    assert_close(po, pl, *oracle_for(paged), f"{workers} workers")
    assert torch.equal(po, co) and torch.equal(pl, cl), "paged and contiguous differ"


def test_two_piece_merge_deterministic_and_correct():
    """Sequences split into two pieces are merged by whichever piece finishes last
    (tcgen05 kernel); the result must not depend on which one that is.  Lengths of
    15-17 pages over 16 workers give two- and three-piece sequences."""
    lens = [1000, 1100, 900, 1024, 1030, 980, 1010, 1020]
    case = S.make_decode_case(len(lens), 128, lens, seed=47)
    M.mla_set_knob("num_workers", 16)
    M.mla_set_knob("min_pages", 1)
    dev = upload(case)
    runs = [run_decode(case, dev) for _ in range(5)]
    for o, l, e in runs:
        assert e == 0
        assert torch.equal(o, runs[0][0]) and torch.equal(l, runs[0][1])
    assert_close(runs[0][0], runs[0][1], *oracle_for(case), "two-piece merge")


def test_large_batch_crosses_schedule_passes():
    """1,500 sequences (more than the schedule's 1,024-wide prefix-sum pass), lengths
    0..200 with empty ones, few heads: every sequence's output against the oracle, and
    the split counts 1 and 148 agree within rounding."""
    lens = S.uniform_seqlens(48, 1500, 0, 200)
    lens[::37] = 0
    case = S.make_decode_case(1500, 8, lens, seed=48, poison=True)
    dev = upload(case)
    out, lse, err = run_decode(case, dev)
    assert err == 0
    assert_close(out, lse, *oracle_for(case), "B=1500")
    for b in np.flatnonzero(lens == 0):
        assert (out[b] == 0).all() and torch.isneginf(lse[b]).all()
    M.mla_set_knob("num_workers", 1)
    o1, l1, e1 = run_decode(case, dev)
    assert e1 == 0
    assert_close(o1, l1, *oracle_for(case), "B=1500, one worker")


def test_paged_equals_contiguous_default_and_shuffle_invariant():
    lens = S.uniform_seqlens(3, 16, 100, 3000)
    a = S.make_decode_case(16, 128, lens, seed=43, paged=True, shuffle=True)
    b = S.make_decode_case(16, 128, lens, seed=43, paged=True, shuffle=False)
    c = S.make_decode_case(16, 128, lens, seed=43, paged=False)
    ra, rb, rc = run_decode(a), run_decode(b), run_decode(c)
    for r in (rb, rc):
        assert torch.equal(ra[0], r[0]) and torch.equal(ra[1], r[1])


def test_repeat_calls_are_deterministic():
    case = S.config_case(2, T=1000)
    dev = upload(case)
    o1, l1, _ = run_decode(case, dev)
    o2, l2, _ = run_decode(case, dev)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_page_sets_error_and_nan_without_fault():
    case = S.make_decode_case(3, 128, [200, 300, 100], seed=44, poison=True)
    bt = case.block_table.copy()
    bt[1, 2] = case.kv_cache.shape[0] + 5  # outside the pool
    case.block_table = bt
    out, lse, err = run_decode(case)
    assert err == 5  # MLA_ERR_DEVICE_BAD_PAGE
    assert torch.isnan(lse[1]).all()
    ref_o, ref_l = oracle_for(case, batch=[0, 2])
    assert_close(out[[0, 2]], lse[[0, 2]], ref_o, ref_l, "other sequences")
    assert M.mla_get_device_error() == 0  # cleared by the read


def test_invalid_length_sets_error():
    case = S.make_decode_case(2, 16, [100, 64], seed=45)
    q, kv, bt, sl = upload(case)
    sl[1] = 10_000  # beyond max_blocks * 64
    out = torch.empty(2, 16, 512, device="cuda")
    lse = torch.empty(2, 16, device="cuda")
    M.mla_decode(q, kv, bt, sl, out, lse, case.softmax_scale)
    assert M.mla_get_device_error() == 5
    assert torch.isnan(lse[1]).all()
    ref_o, ref_l = oracle_for(case, batch=[0])
    assert_close(out[[0]], lse[[0]], ref_o, ref_l)


def test_external_workspace_and_too_small():
    case = S.config_case(2, T=512)
    need = M.mla_workspace_size(case.B, case.H, case.block_table.shape[1])
    buf = torch.empty(need, dtype=torch.uint8, device="cuda")
    M.mla_set_workspace(buf)
    try:
        out, lse, err = run_decode(case)
        assert err == 0
        assert_close(out, lse, *oracle_for(case))
        small = torch.empty(256, dtype=torch.uint8, device="cuda")
        M.mla_set_workspace(small)
        with pytest.raises(M.MlaError) as ei:
            run_decode(case)
        assert ei.value.status == 3
    finally:
        M.mla_set_workspace(None)


def test_kernel_timing_hook():
    case = S.config_case(2, T=1024)
    dev = upload(case)
    M.mla_timing_enable(True)
    for _ in range(3):
        run_decode(case, dev)
    ms, calls = M.mla_timing_read()
    M.mla_timing_enable(False)
    assert calls == 3 and all(x > 0 for x in ms)


def test_bounded_wait_times_out_and_context_survives(kernel):
    """A wait that nothing will satisfy (the producer withholds one page's arrival)
    must end in MLA_ERR_DEVICE_TIMEOUT within the limit, without a trap or hang,
    and the next call must run normally."""
    if kernel != 2:
        pytest.skip("only the tcgen05 kernel has mbarrier waits")
    case = S.make_decode_case(4, 128, 1000, seed=46, poison=True)
    dev = upload(case)
    M.mla_set_knob("wait_limit", 50)
    M.mla_set_knob("withhold_arrive", 1)
    _, _, err = run_decode(case, dev)
    assert err == 6  # MLA_ERR_DEVICE_TIMEOUT
    M.mla_set_knob("withhold_arrive", 0)
    out, lse, err = run_decode(case, dev)
    assert err == 0
    assert_close(out, lse, *oracle_for(case), "after a timeout")
