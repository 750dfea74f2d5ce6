"""Seeded synthetic inputs for absorbed-MLA decode.

This module only *draws* inputs: normal variates, bf16 rounding, page-pool
shuffles and sequence-length samples.  It holds none of the attention
arithmetic, so both the fp64 oracle and the CUDA path can be fed from it
without sharing any of the method's code.

Recipe (the same for every workload):

* every tensor is drawn from its own sub-stream of one integer seed
  (``numpy.random.SeedSequence(seed).spawn``): q, cache, page permutation,
  sequence lengths, weights;
* a stream is consumed in fixed chunks of ``CHUNK`` values, chunk ``i`` seeded
  from ``(stream seed, i)``, so the values do not depend on how many host
  threads draw them;
* normals are drawn in fp32, optionally scaled by a power of two, and rounded
  to bf16 with round-to-nearest-even;  the bf16 bit patterns (``uint16``) are
  what both sides consume;
* a paged cache is a pool of 64-token pages: the data pages of all sequences,
  in a seeded random order, plus one extra *poison* page.  Unused block-table
  slots point at the poison page.  In a correctness case the poison page and
  the rows of each last page beyond the sequence length hold NaN; in a timed
  case they hold zeros.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

PAGE = 64            # tokens per cache page
D_C = 512            # latent width
D_ROPE = 64          # decoupled rope width
D_ROW = D_C + D_ROPE  # one cached row per token
D_NOPE = 128         # per-head no-rope query width (absorb_q input)
D_V = 128            # per-head value width (absorb_o output)

CHUNK = 1 << 22
BF16_NAN = np.uint16(0x7FC0)

_STREAMS = ("q", "cache", "perm", "seqlens", "weights")


def _pool() -> ThreadPoolExecutor:
    n = max(1, min(16, os.cpu_count() or 1))
    return ThreadPoolExecutor(max_workers=n)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round-to-nearest-even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).copy()
    u += ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def streams(seed: int) -> dict:
    """Independent SeedSequences, one per input tensor kind."""
    kids = np.random.SeedSequence(int(seed)).spawn(len(_STREAMS))
    return dict(zip(_STREAMS, kids))


def normal_bf16(ss: np.random.SeedSequence, n: int, std: float = 1.0,
                out: np.ndarray | None = None) -> np.ndarray:
    """``n`` draws of N(0, std^2) rounded to bf16 bits, deterministic in ``ss``.

    ``std`` is applied in fp32 before rounding (exact when it is a power of two).
    """
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    nchunks = (n + CHUNK - 1) // CHUNK
    base = ss.entropy
    key = tuple(ss.spawn_key)

    def work(i: int) -> None:
        lo, hi = i * CHUNK, min(n, (i + 1) * CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(base, spawn_key=key + (i,))))
        x = g.standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[lo:hi] = f32_to_bf16_bits(x)

    if nchunks <= 1:
        for i in range(nchunks):
            work(i)
    else:
        with _pool() as ex:
            list(ex.map(work, range(nchunks)))
    return out


def _gen(ss: np.random.SeedSequence) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(ss))


@dataclass
class DecodeCase:
    """One decode batch: bf16 bit arrays plus int32 metadata (host numpy)."""
    q: np.ndarray                 # [B, H, 576] uint16 (bf16 bits)
    kv_cache: np.ndarray          # paged [num_pages, 64, 576] or contiguous [B, Tcap, 576], uint16
    block_table: np.ndarray | None  # [B, max_blocks] int32, None for a contiguous cache
    cache_seqlens: np.ndarray     # [B] int32
    softmax_scale: float
    poison_page: int | None = None
    meta: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return int(self.q.shape[0])

    @property
    def H(self) -> int:
        return int(self.q.shape[1])


def _logical_pages(ss: np.random.SeedSequence, n_pages: int, latent_std: float, rope_std: float) -> np.ndarray:
    """n_pages * 64 cache rows in logical (sequence-major) order, bf16 bits."""
    rows = n_pages * PAGE
    if latent_std == 1.0 and rope_std == 1.0:
        return normal_bf16(ss, rows * D_ROW).reshape(n_pages, PAGE, D_ROW)
    # Per-part scales: the latent and rope columns come from two sub-streams.
    lat_ss, rope_ss = ss.spawn(2)
    pages = np.empty((n_pages, PAGE, D_ROW), dtype=np.uint16)
    pages[..., :D_C] = normal_bf16(lat_ss, rows * D_C, std=latent_std).reshape(n_pages, PAGE, D_C)
    pages[..., D_C:] = normal_bf16(rope_ss, rows * D_ROPE, std=rope_std).reshape(n_pages, PAGE, D_ROPE)
    return pages


def make_decode_case(B: int, H: int, seqlens, *, seed: int, paged: bool = True,
                     shuffle: bool = True, poison: bool = True, max_blocks: int | None = None,
                     latent_std: float = 1.0, rope_std: float = 1.0, q_std: float = 1.0,
                     softmax_scale: float = 1.0 / math.sqrt(192.0)) -> DecodeCase:
    """A decode batch with the given per-sequence lengths.

    ``seqlens`` is an int or a length-B sequence.  ``max_blocks`` defaults to
    the pages the longest sequence needs (at least 1).  With ``paged=False``
    the cache is contiguous ``[B, max_blocks*64, 576]`` holding the same
    logical rows a paged case of the same seed holds.
    """
    st = streams(seed)
    lens = np.broadcast_to(np.asarray(seqlens, dtype=np.int64), (B,)).astype(np.int32).copy()
    if (lens < 0).any():
        raise ValueError("negative sequence length")
    nblk = (lens.astype(np.int64) + PAGE - 1) // PAGE
    if max_blocks is None:
        max_blocks = max(1, int(nblk.max()) if B else 1)
    if (nblk > max_blocks).any():
        raise ValueError("sequence longer than max_blocks * 64")

    q = normal_bf16(st["q"], B * H * D_ROW, std=q_std).reshape(B, H, D_ROW)
    n_data = int(nblk.sum())
    logical = _logical_pages(st["cache"], n_data, latent_std, rope_std)  # [n_data, 64, 576]
    fill = BF16_NAN if poison else np.uint16(0)
    # Rows at positions >= T in each sequence's last page.
    offs = np.concatenate([[0], np.cumsum(nblk)]).astype(np.int64)
    for b in range(B):
        tail = int(lens[b]) % PAGE
        if nblk[b] and tail:
            logical[offs[b] + nblk[b] - 1, tail:, :] = fill

    meta = dict(seed=seed, latent_std=latent_std, rope_std=rope_std, q_std=q_std,
                n_data_pages=n_data, poison=poison)
    if paged:
        perm = _gen(st["perm"]).permutation(n_data) if shuffle else np.arange(n_data)
        num_pages = n_data + 1
        poison_page = n_data
        cache = np.empty((num_pages, PAGE, D_ROW), dtype=np.uint16)
        cache[perm] = logical
        cache[poison_page] = fill
        table = np.full((B, max_blocks), poison_page, dtype=np.int32)
        for b in range(B):
            table[b, :nblk[b]] = perm[offs[b]:offs[b + 1]]
        return DecodeCase(q, cache, table, lens, softmax_scale, poison_page, meta)

    tcap = max_blocks * PAGE
    cache = np.full((B, tcap, D_ROW), fill, dtype=np.uint16)
    for b in range(B):
        n = int(nblk[b]) * PAGE
        if n:
            cache[b, :n] = logical[offs[b]:offs[b + 1]].reshape(n, D_ROW)
    return DecodeCase(q, cache, None, lens, softmax_scale, None, meta)


def uniform_seqlens(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    """B integer lengths ~ U[lo, hi] inclusive, from the seed's length stream."""
    return _gen(streams(seed)["seqlens"]).integers(lo, hi, size=B, endpoint=True).astype(np.int32)


@dataclass
class LayerInputs:
    """Per-head inputs of the absorbed layer: q halves and up-projection weights."""
    q_nope: np.ndarray   # [B, H, 128] bf16 bits
    q_rope: np.ndarray   # [B, H, 64] bf16 bits
    w_uk: np.ndarray     # [H, 128, 512] bf16 bits  (row i of head h maps latent -> key dim i)
    w_uv: np.ndarray     # [H, 512, 128] bf16 bits  (latent -> value)


def make_layer_inputs(B: int, H: int, *, seed: int, w_std: float = 1.0 / math.sqrt(512.0)) -> LayerInputs:
    st = streams(seed)
    qn_ss, qr_ss = st["q"].spawn(2)
    wk_ss, wv_ss = st["weights"].spawn(2)
    return LayerInputs(
        q_nope=normal_bf16(qn_ss, B * H * D_NOPE).reshape(B, H, D_NOPE),
        q_rope=normal_bf16(qr_ss, B * H * D_ROPE).reshape(B, H, D_ROPE),
        w_uk=normal_bf16(wk_ss, H * D_NOPE * D_C, std=w_std).reshape(H, D_NOPE, D_C),
        w_uv=normal_bf16(wv_ss, H * D_C * D_V, std=w_std).reshape(H, D_C, D_V),
    )


# --------------------------------------------------------------------------
# The five workloads (sizes, seeds and distributions), and the headline.
# --------------------------------------------------------------------------

SCALE_192 = 1.0 / math.sqrt(192.0)


def config_case(n: int, *, poison: bool = True, paged: bool | None = None,
                headline: bool = False, B: int | None = None, T: int | None = None) -> DecodeCase:
    """Decode inputs of workload ``n`` (1..5).  ``B``/``T`` override sizes for
    reduced-size parity cases; the distributions and seeds stay the same."""
    if n == 1:
        return make_decode_case(B or 1, 16, T or 256, seed=1, paged=bool(paged) if paged is not None else False,
                                poison=poison)
    if n == 2:
        return make_decode_case(B or 16, 128, T or 4096, seed=2, paged=True if paged is None else paged,
                                poison=poison)
    if n == 3:
        b = B or 64
        if headline:
            lens = np.full(b, T or 8192, dtype=np.int32)
            mb = (int(lens.max()) + PAGE - 1) // PAGE
        else:
            lens = uniform_seqlens(3, b, 1024, 8192)
            if T is not None:  # reduced size: rescale lengths into [T/8, T]
                lens = np.maximum(1, (lens.astype(np.int64) * T) // 8192).astype(np.int32)
            mb = (int(lens.max()) + PAGE - 1) // PAGE
        return make_decode_case(b, 128, lens, seed=3, paged=True if paged is None else paged, poison=poison,
                                latent_std=0.5, rope_std=1.0, max_blocks=mb)
    if n == 4:
        return make_decode_case(B or 4, 128, T or 131072, seed=4, paged=True if paged is None else paged,
                                poison=poison)
    if n == 5:
        return make_decode_case(B or 64, 128, T or 4096, seed=5, paged=True if paged is None else paged,
                                poison=poison)
    raise ValueError(f"no workload {n}")


def config_layer_inputs(B: int | None = None) -> LayerInputs:
    """Workload 5's q halves and weights (seed 5)."""
    return make_layer_inputs(B or 64, 128, seed=5)
