"""Pins of the fp8-latent-cache oracle (`oracle/fp8_cache.py`), CPU only.

What fixes it independently of itself: PyTorch's own float8_e4m3fn type decodes all 256
codes the same way; the format's landmarks (1, the largest finite value 448, the smallest
normal 2^-6 and subnormal 2^-9, signed zero, the NaN patterns, monotonic codes); a
one-token sequence returns its dequantised latent row, which pins the group scales
(each multiplies exactly its own 128 values and never the rope); and with every scale 1
the fp8 decode is the bf16 decode of the same values (e4m3 values are exact in bf16), bit
for bit.  A planted mistake in a copy of the decoding (exponent bias 8) and in the scale
grouping (groups of 64) is caught.
"""
import numpy as np
import torch

import mla_synth as S
import oracle as O


def test_all_codes_match_torch_float8_e4m3fn():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.signbit(ours[fin]), np.signbit(ref[fin]))


def test_format_landmarks():
    v = O.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    assert v[0x38] == 1.0 and v[0xB8] == -1.0
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9
    assert v[0x00] == 0.0 and np.signbit(v[0x80]) and v[0x80] == 0.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and np.isnan(v).sum() == 2
    assert np.all(np.diff(v[:0x7F]) > 0)  # positive codes increase with the code


def _fp8_case(B, H, lens, seed, scale_lo=0.01, scale_hi=4.0):
    rng = np.random.default_rng(seed)
    base = S.make_decode_case(B, H, lens, seed=seed, poison=False)
    pages = base.kv_cache.shape[0]
    codes = rng.integers(0, 256, size=(pages, 64, 512), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38  # no NaN codes in the cache
    scales = rng.uniform(scale_lo, scale_hi, size=(pages, 64, 4)).astype(np.float32)
    rope = base.kv_cache[..., 512:]
    return base, codes, scales, rope


def test_one_token_returns_the_dequantised_row():
    base, codes, scales, rope = _fp8_case(2, 4, [1, 1], seed=3)
    out, lse = O.mla_decode_fp8_ref(base.q, codes, scales, rope, base.block_table, base.cache_seqlens,
                                    base.softmax_scale)
    for b in range(2):
        page = base.block_table[b][0]
        want = O.e4m3_to_f64(codes[page, 0]) * np.repeat(scales[page, 0].astype(np.float64), 128)
        row = np.concatenate([want, O.bf16_to_f64(rope[page, 0])])  # the rope is never scaled
        for h in range(4):
            assert np.array_equal(out[b, h], want)  # p = 1: out is the dequantised latent row
            s0 = base.softmax_scale * float(O.bf16_to_f64(base.q[b, h]) @ row)
            assert abs(lse[b, h] - s0) <= 1e-12 * max(1.0, abs(s0))  # lse of one token = its score


def test_scale_one_is_the_bf16_decode_of_the_same_values():
    base, codes, scales, rope = _fp8_case(3, 8, [5, 130, 64], seed=4)
    ones = np.ones_like(scales)
    lat = O.e4m3_to_f64(codes).astype(np.float32)  # exact: 3 mantissa bits fit bf16
    bf16_lat = S.f32_to_bf16_bits(lat)
    assert np.array_equal(O.bf16_to_f64(bf16_lat), O.e4m3_to_f64(codes))
    cache = np.concatenate([bf16_lat, rope], axis=-1)
    got = O.mla_decode_fp8_ref(base.q, codes, ones, rope, base.block_table, base.cache_seqlens, base.softmax_scale)
    ref = O.mla_decode_ref(base.q, cache, base.block_table, base.cache_seqlens, base.softmax_scale)
    assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])


def test_planted_mistakes_are_caught():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()

    def wrong_bias(c):  # exponent bias 8 instead of 7
        c = np.asarray(c, dtype=np.int64)
        e, m = (c >> 3) & 0xF, c & 7
        mag = np.where(e == 0, np.ldexp(m / 8.0, -7), np.ldexp(1.0 + m / 8.0, e - 8))
        return np.where((c >> 7) & 1, -mag, mag)

    fin = ~np.isnan(ref)
    assert not np.array_equal(wrong_bias(codes)[fin], ref[fin])

    base, c8, scales, rope = _fp8_case(1, 2, [1], seed=5)
    page = base.block_table[0][0]
    right = O.e4m3_to_f64(c8[page, 0]) * np.repeat(scales[page, 0].astype(np.float64), 128)
    # the four scales applied to groups of 64 values (dims 64-127 would take the second scale)
    grouped_by_64 = O.e4m3_to_f64(c8[page, 0]) * np.repeat(np.tile(scales[page, 0], 2).astype(np.float64), 64)
    assert not np.array_equal(right, grouped_by_64)
    out, _ = O.mla_decode_fp8_ref(base.q, c8, scales, rope, base.block_table, base.cache_seqlens, base.softmax_scale)
    assert np.array_equal(out[0, 0], right)
