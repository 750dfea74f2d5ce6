"""The seeded input generator: determinism, bf16 rounding, page-pool structure."""
import numpy as np
import torch

import mla_synth as S


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(1 << 16).astype(np.float32) * 3
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -0.0, 65504.0]  # ties and exact values
    ours = S.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(S.bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_streams_deterministic_and_chunked():
    n = S.CHUNK * 2 + 123
    a = S.normal_bf16(S.streams(5)["cache"], n)
    b = S.normal_bf16(S.streams(5)["cache"], n)
    c = S.normal_bf16(S.streams(6)["cache"], n)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    # The first chunk does not depend on how many values follow it.
    d = S.normal_bf16(S.streams(5)["cache"], 1000)
    assert np.array_equal(a[:1000], d)


def test_paged_case_structure():
    lens = [0, 1, 63, 64, 65, 200]
    c = S.make_decode_case(6, 4, lens, seed=9, poison=True)
    nblk = [(t + 63) // 64 for t in lens]
    assert c.kv_cache.shape == (sum(nblk) + 1, 64, 576)
    assert c.poison_page == sum(nblk)
    used = []
    for b, n in enumerate(nblk):
        used += list(c.block_table[b, :n])
        assert (c.block_table[b, n:] == c.poison_page).all()
    assert sorted(used) == list(range(sum(nblk)))           # a permutation of the data pages
    f = S.bf16_bits_to_f32(c.kv_cache)
    for b, t in enumerate(lens):
        if t % 64:
            last = c.block_table[b, nblk[b] - 1]
            assert np.isnan(f[last, t % 64:]).all() and np.isfinite(f[last, :t % 64]).all()
    assert np.isnan(f[c.poison_page]).all()


def test_contiguous_holds_same_logical_rows():
    lens = [65, 130]
    p = S.make_decode_case(2, 2, lens, seed=10, paged=True)
    q = S.make_decode_case(2, 2, lens, seed=10, paged=False)
    assert np.array_equal(p.q, q.q)
    for b, T in enumerate(lens):
        for t in range(T):
            assert np.array_equal(p.kv_cache[p.block_table[b, t // 64], t % 64], q.kv_cache[b, t])


def test_timed_case_has_zero_tails():
    c = S.make_decode_case(2, 2, [10, 64], seed=12, poison=False)
    f = S.bf16_bits_to_f32(c.kv_cache)
    assert np.isfinite(f).all()
    assert (f[c.block_table[0, 0], 10:] == 0).all()


def test_workload_distributions():
    lens = S.uniform_seqlens(3, 64, 1024, 8192)
    assert lens.min() >= 1024 and lens.max() <= 8192 and len(set(lens.tolist())) > 32
    c = S.config_case(3, B=4, T=512)
    lat = S.bf16_bits_to_f32(c.kv_cache[c.block_table[0, 0], :, :512]).astype(np.float64)
    rope = S.bf16_bits_to_f32(c.kv_cache[c.block_table[0, 0], :, 512:]).astype(np.float64)
    assert 0.4 < lat.std() < 0.6 and 0.85 < rope.std() < 1.15
    li = S.make_layer_inputs(2, 4, seed=5)
    w = S.bf16_bits_to_f32(li.w_uk).astype(np.float64)
    assert abs(w.std() - 512 ** -0.5) < 0.003
