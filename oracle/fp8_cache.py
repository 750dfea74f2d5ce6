"""fp8 latent cache with scales: the reference a quantised decode is checked against
(test infrastructure, like the rest of this package).

The pages list the quantisation scale among the things a production MLA needs beyond the
teaching version ("Multi-head Latent Attention" glossary entry, the closing note after
the runnable check) and give no format.  Reading taken (the plainest one that keeps the
rest of the path unchanged): each cached token keeps its 512 latent values as OCP FP8
E4M3 codes with one fp32 scale per group of 128 consecutive values (value = decoded code
x the group's scale), and its 64 rope values in bf16 as before, so the part that carries
position keeps bf16 precision.  Decoding dequantises every cached row in float64 and then
computes exactly what ``mla_decode_ref`` computes on those rows.

Layouts: ``lat_codes`` uint8 [..., 512], ``scales`` float32 [..., 4], ``rope`` bf16 bit
patterns uint16 [..., 64], each with the cache's leading dims (paged [num_pages, page]
or contiguous [B, Tcap]).
"""
from __future__ import annotations

import numpy as np

from .mla_oracle import bf16_to_f64, mla_decode_ref

D_LATENT, D_ROPE, GROUP = 512, 64, 128


def e4m3_to_f64(codes) -> np.ndarray:
    """OCP FP8 E4M3 codes -> exact float64.

    Bit 7 is the sign, bits 6..3 the exponent (bias 7), bits 2..0 the mantissa.  An
    exponent field of 0 is subnormal, ``(m / 8) * 2^-6``; otherwise the value is
    ``(1 + m / 8) * 2^(e - 7)``.  The one NaN pattern per sign is exponent 15 with
    mantissa 7; there are no infinities, so exponent 15 with mantissa 0..6 is finite
    (up to 448).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(sign == 1, -mag, mag)


def dequant_rows(lat_codes, scales, rope) -> np.ndarray:
    """float64 rows ``[latent (512) | rope (64)]``: every latent value is its decoded code
    times the fp32 scale of its 128-value group; the rope values are the bf16 values."""
    lat = e4m3_to_f64(lat_codes)
    sc = np.asarray(scales, dtype=np.float32).astype(np.float64)
    assert lat.shape[-1] == D_LATENT and sc.shape[-1] == D_LATENT // GROUP
    lat = lat * np.repeat(sc, GROUP, axis=-1)
    return np.concatenate([lat, bf16_to_f64(rope)], axis=-1)


def mla_decode_fp8_ref(q, lat_codes, scales, rope, block_table, cache_seqlens, softmax_scale: float, *,
                       page_size: int = 64, batch=None, heads=None):
    """Absorbed decode over an fp8 latent cache: ``mla_decode_ref`` on the dequantised
    rows (the value rows are the dequantised latent).  Returns ``(out, lse)``."""
    rows = dequant_rows(lat_codes, scales, rope)
    return mla_decode_ref(q, rows, block_table, cache_seqlens, softmax_scale, page_size=page_size, batch=batch,
                          heads=heads)
