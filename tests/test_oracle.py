"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics, not by the
oracle itself.  CPU only.

Each test names what it pins.  Together they are chosen so that a plausible slip in
the oracle (a dropped rope term, a wrong scale, a transposed weight, an off-by-one in
the page gather, values taken from the wrong columns, log base 2 instead of e) fails
at least one of them; ``test_planted_mistakes_are_caught`` checks that claim for a few
such slips by planting them in a copy of the oracle.
"""
import math
import os

import numpy as np
import pytest
import scipy.special

import mla_synth as S
import oracle as O
from oracle import mla_oracle as OM
from oracle.bruteforce import decode_bruteforce, decode_multi_bruteforce

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "toy_expanded_vs_absorbed.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = (x.strip() for x in line.split("="))
            vals[k] = float(v) if any(c in v for c in ".e") else int(v)
    return vals


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# 1. The glossary page's worked example: expanded == absorbed in fp64.
# ---------------------------------------------------------------------------

def _toy(seed=107):
    """The toy of the runnable check, drawn from our own RNG (fp64, not bf16)."""
    g = _golden()
    b, t, hq = g["batch"], g["tokens"], g["heads"]
    hidden, dc, dk, dr, dv = g["hidden"], g["d_c"], g["d_k"], g["d_rope"], g["d_v"]
    r = _rng(seed)
    x = r.standard_normal((b, t, hidden))
    x_new = r.standard_normal((b, 1, hidden))
    w_dkv = r.standard_normal((hidden, dc))
    w_uk_page = r.standard_normal((hq, dc, dk))   # page layout: k = c @ w_uk[h]
    w_uv = r.standard_normal((hq, dc, dv))
    w_qc = r.standard_normal((hidden, hq * dk))
    w_qr = r.standard_normal((hidden, hq * dr))
    w_kr = r.standard_normal((hidden, dr))
    latent = x @ w_dkv                                 # [b, t, dc]
    k_rope = x @ w_kr                                  # [b, t, dr]
    qc = (x_new @ w_qc).reshape(b, hq, dk)             # one query token
    qr = (x_new @ w_qr).reshape(b, hq, dr)
    cache = np.concatenate([latent, k_rope], axis=2)   # contiguous [b, t, dc + dr]
    w_uk = np.transpose(w_uk_page, (0, 2, 1)).copy()   # our layout [H, d_nope, d_c]
    scale = 1.0 / math.sqrt(dk + dr)
    lens = np.full(b, t, dtype=np.int32)
    return dict(qc=qc, qr=qr, w_uk=w_uk, w_uv=w_uv, cache=cache, lens=lens, scale=scale,
                dc=dc, dr=dr, dk=dk, dv=dv, hq=hq, latent=latent, k_rope=k_rope, w_uk_page=w_uk_page)


@pytest.mark.parametrize("seed", [107, 1, 2, 3])
def test_toy_expanded_equals_absorbed(seed):
    g = _golden()
    d = _toy(seed)
    exp_out, exp_lse = O.mla_decode_expanded_ref(d["qc"], d["qr"], d["w_uk"], d["w_uv"], d["cache"], None,
                                                 d["lens"], d["scale"], d_c=d["dc"])
    abs_out, abs_lse = O.mla_layer_absorbed_ref(d["qc"], d["qr"], d["w_uk"], d["w_uv"], d["cache"], None,
                                                d["lens"], d["scale"])
    assert exp_out.shape == (g["batch"], g["heads"], g["d_v"])
    tol_out = g["atol"] + g["rtol"] * np.abs(exp_out)
    assert (np.abs(abs_out - exp_out) <= tol_out).all()
    assert np.abs(abs_lse - exp_lse).max() <= g["atol"] + g["rtol"] * np.abs(exp_lse).max()
    # The page reports ~1e-14 differences for an fp64 run; ours are rounding noise too.
    assert np.abs(abs_out - exp_out).max() < 1e3 * g["reported_output_max_abs_diff"]


def test_toy_absorbed_query_is_page_contraction():
    """Key absorption with the page's weight layout: q_bar_h = q^C_h (W^UK_h)^T, where
    the page stores W^UK_h as [d_c, d_k].  Our W_UK[h] is that matrix transposed, so
    absorb_q must equal the contraction over the page's last axis."""
    d = _toy()
    qp = O.mla_absorb_q_ref(d["qc"], d["qr"], d["w_uk"])
    ref = np.einsum("bhd,hcd->bhc", d["qc"], d["w_uk_page"])
    assert np.allclose(qp[..., :d["dc"]], ref, rtol=1e-13, atol=1e-13)
    assert np.array_equal(qp[..., d["dc"]:], d["qr"])


def test_toy_cache_element_counts():
    g = _golden()
    std, mla = O.cache_elements_per_token(g["heads"], g["d_v"], g["d_c"], g["d_rope"])
    assert (std, mla) == (g["standard_kv_elements"], g["mla_cached_elements"])


def test_capacity_formula_headline_bytes():
    # One layer, B=64 sequences of 8192 tokens, 512+64 bf16 elements: the KV bytes the
    # decode must read once.
    assert O.latent_cache_bytes(1, 64, 8192, 512, 64, 2) == 603_979_776
    std, mla = O.cache_elements_per_token(128, 128, 512, 64)
    assert (std, mla) == (32768, 576)


# ---------------------------------------------------------------------------
# 2. Expanded == absorbed at the real widths (512 latent, 64 rope, 128 nope/v).
# ---------------------------------------------------------------------------

def test_full_width_expanded_equals_absorbed():
    B, H, T = 2, 4, 150
    li = S.make_layer_inputs(B, H, seed=11)
    case = S.make_decode_case(B, H, [T, 77], seed=11, poison=True)
    kw = dict(batch=None, heads=None)
    e_out, e_lse = O.mla_decode_expanded_ref(li.q_nope, li.q_rope, li.w_uk, li.w_uv, case.kv_cache,
                                             case.block_table, case.cache_seqlens, S.SCALE_192, **kw)
    a_out, a_lse = O.mla_layer_absorbed_ref(li.q_nope, li.q_rope, li.w_uk, li.w_uv, case.kv_cache,
                                            case.block_table, case.cache_seqlens, S.SCALE_192, **kw)
    assert np.isfinite(e_out).all() and np.isfinite(a_out).all()
    assert np.abs(a_out - e_out).max() <= 1e-10 + 1e-10 * np.abs(e_out).max()
    assert np.abs(a_lse - e_lse).max() <= 1e-10


# ---------------------------------------------------------------------------
# 3. Softmax facts.
# ---------------------------------------------------------------------------

def test_probs_sum_to_one():
    case = S.make_decode_case(3, 8, [1, 64, 333], seed=21)
    for b in range(3):
        p = O.mla_decode_probs_ref(case.q, case.kv_cache, case.block_table, case.cache_seqlens,
                                   case.softmax_scale, b)
        assert p.shape == (8, int(case.cache_seqlens[b]))
        assert (p >= 0).all()
        assert np.abs(p.sum(axis=1) - 1.0).max() <= 1e-12


def test_single_token_returns_its_value_row():
    case = S.make_decode_case(2, 5, 1, seed=22)
    out, lse = O.mla_decode_ref(case.q, case.kv_cache, case.block_table, case.cache_seqlens,
                                case.softmax_scale)
    for b in range(2):
        row = S.bf16_bits_to_f32(case.kv_cache[case.block_table[b, 0], 0]).astype(np.float64)
        assert np.array_equal(out[b], np.broadcast_to(row[:512], (5, 512)))
        for h in range(5):
            qh = S.bf16_bits_to_f32(case.q[b, h]).astype(np.float64)
            s0 = case.softmax_scale * math.fsum(qh * row)
            assert abs(lse[b, h] - s0) <= 1e-12 * max(1.0, abs(s0))


@pytest.mark.parametrize("how", ["zero_query", "zero_scale"])
def test_equal_scores_give_mean_value_and_log_T(how):
    T = 200
    case = S.make_decode_case(1, 4, T, seed=23)
    q = np.zeros_like(case.q) if how == "zero_query" else case.q
    scale = 0.0 if how == "zero_scale" else case.softmax_scale
    out, lse = O.mla_decode_ref(q, case.kv_cache, case.block_table, case.cache_seqlens, scale)
    rows = np.stack([S.bf16_bits_to_f32(case.kv_cache[case.block_table[0, t // 64], t % 64]).astype(np.float64)
                     for t in range(T)])
    mean = np.array([math.fsum(rows[:, j]) / T for j in range(512)])
    assert np.abs(out[0] - mean).max() <= 1e-14
    assert np.abs(lse[0] - math.log(T)).max() <= 1e-14


def test_empty_sequence():
    case = S.make_decode_case(2, 3, [0, 5], seed=24)
    out, lse = O.mla_decode_ref(case.q, case.kv_cache, case.block_table, case.cache_seqlens,
                                case.softmax_scale)
    assert (out[0] == 0).all() and np.isneginf(lse[0]).all()
    assert np.isfinite(out[1]).all() and np.isfinite(lse[1]).all()


# ---------------------------------------------------------------------------
# 4. A closed form: scores that grow linearly in t.
# ---------------------------------------------------------------------------

def _ramp_case(col, T=200, scale=0.75, value_col=0):
    """One head whose query is 1 at ``col`` and 0 elsewhere; row t holds t/64 at
    ``col`` and t at ``value_col`` (both exact in bf16), the rest random.  Then
    s_t = scale * t / 64 = kappa t, and with Z = sum_t e^{kappa t}:
      lse = ln((e^{kappa T} - 1) / (e^kappa - 1)),
      out[value_col] = d lse / d kappa = T e^{kT}/(e^{kT}-1) - e^k/(e^k-1)."""
    case = S.make_decode_case(1, 1, T, seed=25, poison=True)
    q = np.zeros_like(case.q)
    q[0, 0, col] = S.f32_to_bf16_bits(np.array([1.0], np.float32))[0]
    cache = case.kv_cache.copy()
    for t in range(T):
        p, s = case.block_table[0, t // 64], t % 64
        cache[p, s, col] = S.f32_to_bf16_bits(np.array([t / 64.0], np.float32))[0]
        if value_col != col:
            cache[p, s, value_col] = S.f32_to_bf16_bits(np.array([float(t)], np.float32))[0]
    k = scale / 64.0
    lse = math.log(math.expm1(k * T) / math.expm1(k))
    mean_t = T * math.exp(k * T) / math.expm1(k * T) - math.exp(k) / math.expm1(k)
    return q, cache, case.block_table, case.cache_seqlens, scale, lse, mean_t


@pytest.mark.parametrize("col,value_col", [(540, 0), (600 - 25, 511), (3, 0), (100, 100)])
def test_linear_score_closed_form(col, value_col):
    q, cache, bt, lens, scale, lse_cf, mean_t = _ramp_case(col, value_col=value_col)
    out, lse = O.mla_decode_ref(q, cache, bt, lens, scale)
    assert abs(lse[0, 0] - lse_cf) <= 1e-12 * abs(lse_cf)
    if value_col == col:  # that column holds t/64, not t
        mean_t /= 64.0
    assert abs(out[0, 0, value_col] - mean_t) <= 1e-11 * abs(mean_t)


def test_library_logsumexp_and_softmax():
    """One head over T rows reduces to scipy's logsumexp / softmax of the score row."""
    case = S.make_decode_case(2, 6, [130, 7], seed=26, latent_std=0.5)
    out, lse = O.mla_decode_ref(case.q, case.kv_cache, case.block_table, case.cache_seqlens,
                                case.softmax_scale)
    for b in range(2):
        T = int(case.cache_seqlens[b])
        rows = np.stack([S.bf16_bits_to_f32(case.kv_cache[case.block_table[b, t // 64], t % 64])
                         for t in range(T)]).astype(np.float64)
        for h in range(6):
            qh = S.bf16_bits_to_f32(case.q[b, h]).astype(np.float64)
            s = np.array([case.softmax_scale * math.fsum(qh * rows[t]) for t in range(T)])
            assert abs(lse[b, h] - scipy.special.logsumexp(s)) <= 1e-12 * max(1, abs(lse[b, h]))
            p = scipy.special.softmax(s)
            ref = np.array([math.fsum(p * rows[:, j]) for j in range(512)])
            assert np.abs(out[b, h] - ref).max() <= 1e-13


# ---------------------------------------------------------------------------
# 5. Brute force on tiny inputs (pure Python, no max shift).
# ---------------------------------------------------------------------------

def test_bruteforce_agreement():
    lens = [1, 65, 130]
    case = S.make_decode_case(3, 2, lens, seed=27, poison=True, latent_std=0.5)
    out, lse = O.mla_decode_ref(case.q, case.kv_cache, case.block_table, case.cache_seqlens,
                                case.softmax_scale)
    bo, bl = decode_bruteforce(case.q, case.kv_cache, case.block_table, case.cache_seqlens,
                               case.softmax_scale, 512)
    assert np.abs(out - np.array(bo)).max() <= 1e-13
    assert np.abs(lse - np.array(bl)).max() <= 1e-13


def test_bruteforce_contiguous():
    case = S.make_decode_case(2, 2, [70, 3], seed=28, paged=False, poison=True)
    out, lse = O.mla_decode_ref(case.q, case.kv_cache, None, case.cache_seqlens, case.softmax_scale)
    bo, bl = decode_bruteforce(case.q, case.kv_cache, None, case.cache_seqlens, case.softmax_scale, 512)
    assert np.abs(out - np.array(bo)).max() <= 1e-13
    assert np.abs(lse - np.array(bl)).max() <= 1e-13


# ---------------------------------------------------------------------------
# 5b. Several causal query tokens per sequence (reading taken for s_q > 1).
# ---------------------------------------------------------------------------

def _multi_case(B, s_q, H, lens, seed, **kw):
    """A decode case whose s_q * H query rows are viewed as [B, s_q, H, 576]."""
    c = S.make_decode_case(B, s_q * H, lens, seed=seed, **kw)
    return c, c.q.reshape(B, s_q, H, -1)


def test_multi_query_bruteforce_with_explicit_mask():
    # T = 2 with s_q = 3: query 0 sees nothing, query 1 token 0, query 2 tokens 0..1;
    # T = 70 crosses a page boundary.  Brute force: loops, fsum, no max shift, and the
    # causal mask written as t <= position.
    c, q = _multi_case(2, 3, 2, [2, 70], seed=61, poison=True, latent_std=0.5)
    out, lse = O.mla_decode_multi_ref(q, c.kv_cache, c.block_table, c.cache_seqlens, c.softmax_scale)
    bo, bl = decode_multi_bruteforce(q, c.kv_cache, c.block_table, c.cache_seqlens, c.softmax_scale, 512)
    bo, bl = np.array(bo), np.array(bl)
    assert np.isneginf(lse[0, 0]).all() and (out[0, 0] == 0).all()
    fin = np.isfinite(bl)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.abs(out - bo).max() <= 1e-13
    assert np.abs(lse[fin] - bl[fin]).max() <= 1e-13


def test_multi_query_windows_are_truncated_single_token_decodes():
    # Query i of a sequence of length T is the single-token decode of the same cache cut
    # to its first T - s_q + 1 + i tokens; the last query sees all T.
    B, SQ, H = 3, 4, 2
    lens = [5, 64, 131]
    c, q = _multi_case(B, SQ, H, lens, seed=62, poison=True)
    out, lse = O.mla_decode_multi_ref(q, c.kv_cache, c.block_table, c.cache_seqlens, c.softmax_scale)
    for i in range(SQ):
        cut = np.maximum(np.asarray(lens) - SQ + 1 + i, 0).astype(np.int32)
        ro, rl = O.mla_decode_ref(q[:, i], c.kv_cache, c.block_table, cut, c.softmax_scale)
        assert np.array_equal(out[:, i], ro) and np.array_equal(lse[:, i], rl)


def test_multi_query_single_token_is_decode():
    c, q = _multi_case(3, 1, 4, [1, 64, 300], seed=63, poison=True)
    out, lse = O.mla_decode_multi_ref(q, c.kv_cache, c.block_table, c.cache_seqlens, c.softmax_scale)
    ro, rl = O.mla_decode_ref(c.q, c.kv_cache, c.block_table, c.cache_seqlens, c.softmax_scale)
    assert np.array_equal(out[:, 0], ro) and np.array_equal(lse[:, 0], rl)


# ---------------------------------------------------------------------------
# 6. Invariances: paging, page order, split-and-merge.
# ---------------------------------------------------------------------------

def test_paged_equals_contiguous_and_page_order_is_irrelevant():
    lens = [300, 64, 1, 129]
    a = S.make_decode_case(4, 8, lens, seed=29, paged=True, shuffle=True)
    b = S.make_decode_case(4, 8, lens, seed=29, paged=True, shuffle=False)
    c = S.make_decode_case(4, 8, lens, seed=29, paged=False)
    ra = O.mla_decode_ref(a.q, a.kv_cache, a.block_table, a.cache_seqlens, a.softmax_scale)
    rb = O.mla_decode_ref(b.q, b.kv_cache, b.block_table, b.cache_seqlens, b.softmax_scale)
    rc = O.mla_decode_ref(c.q, c.kv_cache, None, c.cache_seqlens, c.softmax_scale)
    assert not np.array_equal(a.block_table, b.block_table)
    for x, y in ((ra, rb), (ra, rc)):
        assert np.array_equal(x[0], y[0]) and np.array_equal(x[1], y[1])


def test_poison_rows_are_never_read():
    case = S.make_decode_case(3, 4, [63, 64, 65], seed=30, poison=True)
    assert np.isnan(S.bf16_bits_to_f32(case.kv_cache[case.poison_page])).all()
    out, lse = O.mla_decode_ref(case.q, case.kv_cache, case.block_table, case.cache_seqlens,
                                case.softmax_scale)
    assert np.isfinite(out).all() and np.isfinite(lse).all()


@pytest.mark.parametrize("cuts", [[0, 1000], [0, 1, 1000], [0, 64, 128, 640, 999, 1000], [0, 500, 500, 1000]])
def test_split_merge_invariance(cuts):
    T = 1000
    case = S.make_decode_case(1, 6, T, seed=31, paged=False, poison=False)
    full_out, full_lse = O.mla_decode_ref(case.q, case.kv_cache, None, case.cache_seqlens, case.softmax_scale)
    outs, lses = [], []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        part = case.kv_cache[:, lo:hi]
        o, l = O.mla_decode_ref(case.q, part, None, np.array([hi - lo], np.int32), case.softmax_scale)
        outs.append(o)
        lses.append(l)
    mo, ml = O.lse_merge_ref(outs, lses)
    assert np.abs(mo - full_out).max() <= 1e-12
    assert np.abs(ml - full_lse).max() <= 1e-12


def test_lse_merge_all_empty():
    o, l = O.lse_merge_ref([np.zeros((2, 3)), np.zeros((2, 3))], [np.full(2, -np.inf), np.full(2, -np.inf)])
    assert (o == 0).all() and np.isneginf(l).all()


# ---------------------------------------------------------------------------
# 7. Absorption GEMMs: one-hot inputs select a weight row (catches transposes).
# ---------------------------------------------------------------------------

def test_absorb_q_one_hot_selects_weight_row():
    B, H = 2, 3
    li = S.make_layer_inputs(B, H, seed=32)
    qn = np.zeros_like(li.q_nope)
    one = S.f32_to_bf16_bits(np.array([1.0], np.float32))[0]
    sel = [[5, 0, 127], [64, 1, 2]]
    for b in range(B):
        for h in range(H):
            qn[b, h, sel[b][h]] = one
    qp = O.mla_absorb_q_ref(qn, li.q_rope, li.w_uk)
    assert qp.shape == (B, H, 576)
    for b in range(B):
        for h in range(H):
            w = S.bf16_bits_to_f32(li.w_uk[h, sel[b][h], :]).astype(np.float64)
            assert np.array_equal(qp[b, h, :512], w)
            assert np.array_equal(qp[b, h, 512:], S.bf16_bits_to_f32(li.q_rope[b, h]).astype(np.float64))


def test_absorb_o_one_hot_selects_weight_row():
    B, H = 2, 3
    li = S.make_layer_inputs(B, H, seed=33)
    ol = np.zeros((B, H, 512))
    sel = [[0, 511, 17], [256, 3, 4]]
    for b in range(B):
        for h in range(H):
            ol[b, h, sel[b][h]] = 2.0
    out = O.mla_absorb_o_ref(ol, li.w_uv)
    assert out.shape == (B, H, 128)
    for b in range(B):
        for h in range(H):
            w = S.bf16_bits_to_f32(li.w_uv[h, sel[b][h], :]).astype(np.float64)
            assert np.array_equal(out[b, h], 2.0 * w)


# ---------------------------------------------------------------------------
# 8. Planted mistakes in a copy of the oracle must trip the pins above.
# ---------------------------------------------------------------------------

def _pins_pass(monkeypatch_ctx):
    checks = [
        lambda: test_bruteforce_agreement(),
        lambda: test_linear_score_closed_form(540, 0),
        lambda: test_linear_score_closed_form(3, 0),
        lambda: test_equal_scores_give_mean_value_and_log_T("zero_query"),
        lambda: test_single_token_returns_its_value_row(),
    ]
    for c in checks:
        try:
            c()
        except (AssertionError, IndexError, ValueError):
            return False
    return True


def test_planted_mistakes_are_caught(monkeypatch):
    assert _pins_pass(None)
    real_gather = OM.gather_rows

    def off_by_one_gather(kv, bt, b, T, page_size=64):
        rows = real_gather(kv, bt, b, T + 1 if T < 64 else T, page_size)
        return rows[1:] if T < 64 else np.roll(rows, 1, axis=0)

    def dropped_rope_gather(kv, bt, b, T, page_size=64):
        rows = real_gather(kv, bt, b, T, page_size).copy()
        rows[:, 512:] = 0.0
        return rows

    def shifted_value_gather(kv, bt, b, T, page_size=64):
        rows = real_gather(kv, bt, b, T, page_size)
        return np.concatenate([rows[:, 1:], rows[:, :1]], axis=1)

    for bad in (off_by_one_gather, dropped_rope_gather, shifted_value_gather):
        monkeypatch.setattr(OM, "gather_rows", bad)
        assert not _pins_pass(None), bad.__name__
        monkeypatch.setattr(OM, "gather_rows", real_gather)

    real_log = OM.np.log
    monkeypatch.setattr(OM.np, "log", np.log2)
    try:
        assert not _pins_pass(None), "log base 2"
    finally:
        monkeypatch.setattr(OM.np, "log", real_log)
