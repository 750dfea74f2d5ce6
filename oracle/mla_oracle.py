"""fp64 reference for absorbed-MLA decode (test infrastructure; see package docstring).

Every function computes a plain definition in float64 from the exact bf16 input
values.  Matrix products (numpy ``@``) are the only library steps; there is no
tiling, no online softmax and no split: softmax is the two-pass form (max, then
sum), exactly as the runnable check on the "Multi-head Latent Attention" glossary
page applies ``torch.softmax`` to the full score row.

Layouts (all row-major):

* ``q``            [B, H, 576]  absorbed query ``[q_nope W_UK (512) | q_rope (64)]``
* ``kv_cache``     paged [num_pages, page, 576] or contiguous [B, Tcap, 576];
                   one row per token: ``[c_KV (512) | k_rope (64)]``
* ``block_table``  [B, max_blocks] int page ids, or ``None`` for a contiguous cache
* ``cache_seqlens``[B] token counts T_b
* ``w_uk``         [H, d_nope, d_c]: row i of head h holds the latent weights of key
                   dim i, so ``k_{h,t} = W_UK[h] c_t`` and ``q'_h = q_nope_h W_UK[h]``
* ``w_uv``         [H, d_c, d_v]:  ``v_{h,t} = c_t W_UV[h]``
"""
from __future__ import annotations

import math

import numpy as np


def bf16_to_f64(x) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64; float input is cast to float64."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def gather_rows(kv_cache, block_table, b: int, T: int, page_size: int = 64) -> np.ndarray:
    """The T cached rows of sequence ``b`` in token order, as float64 [T, D].

    Paged: token t of sequence b is slot ``t % page`` of page ``block_table[b][t // page]``
    (the glossary's note that the latent cache can be paged into blocks).
    Contiguous (``block_table is None``): token t is ``kv_cache[b][t]``.
    """
    t = np.arange(T)
    if block_table is None:
        return bf16_to_f64(kv_cache[b][t])
    pages = np.asarray(block_table[b], dtype=np.int64)[t // page_size]
    if pages.size and (pages.min() < 0 or pages.max() >= kv_cache.shape[0]):
        raise IndexError(f"sequence {b}: page id outside [0, {kv_cache.shape[0]})")
    return bf16_to_f64(kv_cache[pages, t % page_size])


def _select(n: int, which) -> list:
    return list(range(n)) if which is None else [int(i) for i in which]


def mla_decode_ref(q, kv_cache, block_table, cache_seqlens, softmax_scale: float, *,
                   d_v: int = 512, page_size: int = 64, batch=None, heads=None):
    """Absorbed decode: per (b, h), attention of q'_h over the T_b cached rows.

    s_t   = scale * <q'_h, row_t>          over all D = d_c + d_rope dims
            (glossary: content score q^C k^C^T + rope score q^R k^R^T, with the key
            up-projection absorbed into the query, so both parts are one dot product
            against the cached row);
    lse   = m + ln(sum_t exp(s_t - m)),    m = max_t s_t   (natural log, scale included);
    p_t   = exp(s_t - lse);
    out_j = sum_t p_t row_t[j],  j < d_v    (value absorption: the weights multiply the
            latent c_t itself; the W_UV lift happens outside).
    T_b = 0 gives out = 0 and lse = -inf.

    Returns ``(out [nb, nh, d_v], lse [nb, nh])`` for the selected batch rows / heads.
    """
    bs = _select(q.shape[0], batch)
    hs = _select(q.shape[1], heads)
    out = np.zeros((len(bs), len(hs), d_v))
    lse = np.full((len(bs), len(hs)), -np.inf)
    for i, b in enumerate(bs):
        T = int(cache_seqlens[b])
        if T == 0:
            continue
        qb = bf16_to_f64(q[b][hs])                     # [nh, D]
        rows = gather_rows(kv_cache, block_table, b, T, page_size)  # [T, D]
        s = softmax_scale * (qb @ rows.T)              # [nh, T]
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        lse[i] = (m + np.log(l))[:, 0]
        out[i] = (e / l) @ rows[:, :d_v]
    return out, lse


def mla_decode_multi_ref(q, kv_cache, block_table, cache_seqlens, softmax_scale: float, *,
                         d_v: int = 512, page_size: int = 64):
    """Several new query tokens per sequence, each attending causally.

    The pages define decode for one new token.  Reading taken for s_q > 1: the s_q new
    tokens are the last s_q cached rows of sequence b, so query i (0 <= i < s_q) sits at
    position T_b - s_q + i and attends to the rows t <= T_b - s_q + i, i.e. the first
    n_i = T_b - s_q + 1 + i rows; over that window it is the single-token definition of
    ``mla_decode_ref`` (scale on the whole 576-dim dot product, natural-log lse, values =
    the first d_v dims of the rows).  An empty window (n_i <= 0) gives out = 0, lse = -inf.

    q: [B, s_q, H, D].  Returns ``(out [B, s_q, H, d_v], lse [B, s_q, H])``.
    """
    B, SQ, H, _ = q.shape
    out = np.zeros((B, SQ, H, d_v))
    lse = np.full((B, SQ, H), -np.inf)
    for b in range(B):
        T = int(cache_seqlens[b])
        if T <= 0:
            continue
        rows_all = gather_rows(kv_cache, block_table, b, T, page_size)   # [T, D]
        for i in range(SQ):
            n = T - SQ + 1 + i
            if n <= 0:
                continue
            rows = rows_all[:n]
            s = softmax_scale * (bf16_to_f64(q[b, i]) @ rows.T)          # [H, n]
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            lse[b, i] = (m + np.log(l))[:, 0]
            out[b, i] = (e / l) @ rows[:, :d_v]
    return out, lse


def mla_decode_probs_ref(q, kv_cache, block_table, cache_seqlens, softmax_scale: float, b: int, *,
                         page_size: int = 64) -> np.ndarray:
    """The softmax weights p[h, t] of sequence ``b`` (same definition as above)."""
    T = int(cache_seqlens[b])
    rows = gather_rows(kv_cache, block_table, b, T, page_size)
    s = softmax_scale * (bf16_to_f64(q[b]) @ rows.T)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def mla_decode_expanded_ref(q_nope, q_rope, w_uk, w_uv, kv_cache, block_table, cache_seqlens,
                            softmax_scale: float, *, d_c: int = 512, page_size: int = 64,
                            batch=None, heads=None):
    """Expanded (non-absorbed) decode: materialise per-head keys and values.

    From the glossary's teaching abstraction and its runnable check:
      K[h, t, i] = sum_c W_UK[h][i][c] c_t[c]             (content key, i < d_nope)
      V[h, t, j] = sum_c c_t[c] W_UV[h][c][j]             (content value, j < d_v)
      s[h, t]    = scale * (q_nope[h] . K[h, t] + q_rope[h] . k_rope_t)
      out[h]     = sum_t softmax_t(s[h]) V[h, t]
    where row_t = [c_t (d_c) | k_rope_t] and k_rope_t is shared by all heads.
    Returns ``(out [nb, nh, d_v], lse [nb, nh])``.
    """
    bs = _select(q_nope.shape[0], batch)
    hs = _select(q_nope.shape[1], heads)
    wk = bf16_to_f64(w_uk)
    wv = bf16_to_f64(w_uv)
    d_v = wv.shape[2]
    out = np.zeros((len(bs), len(hs), d_v))
    lse = np.full((len(bs), len(hs)), -np.inf)
    for i, b in enumerate(bs):
        T = int(cache_seqlens[b])
        if T == 0:
            continue
        rows = gather_rows(kv_cache, block_table, b, T, page_size)
        c, k_rope = rows[:, :d_c], rows[:, d_c:]
        qn = bf16_to_f64(q_nope[b])
        qr = bf16_to_f64(q_rope[b])
        for k, h in enumerate(hs):
            K = c @ wk[h].T                            # [T, d_nope]
            V = c @ wv[h]                              # [T, d_v]
            s = softmax_scale * (K @ qn[h] + k_rope @ qr[h])
            m = s.max()
            e = np.exp(s - m)
            l = e.sum()
            lse[i, k] = m + math.log(l)
            out[i, k] = (e / l) @ V
    return out, lse


def mla_absorb_q_ref(q_nope, q_rope, w_uk) -> np.ndarray:
    """q'[b, h] = [ q_nope[b, h] W_UK[h]  |  q_rope[b, h] ]   (float64, no rounding).

    Key absorption (glossary, "why absorb in decode"): q^C (W^UK)^T; the absorbed query
    is concatenated with the rope query (FlashMLA issue #16: [bs, H, 512] ++ [bs, H, 64]).
    """
    qn = bf16_to_f64(q_nope)
    qr = bf16_to_f64(q_rope)
    wk = bf16_to_f64(w_uk)
    B, H, _ = qn.shape
    q_lat = np.empty((B, H, wk.shape[2]))
    for h in range(H):
        q_lat[:, h, :] = qn[:, h, :] @ wk[h]
    return np.concatenate([q_lat, qr], axis=2)


def mla_absorb_o_ref(out_latent, w_uv) -> np.ndarray:
    """out[b, h] = out_latent[b, h] W_UV[h]  (value absorption: (sum_t p_t c_t) W^UV)."""
    ol = bf16_to_f64(out_latent)
    wv = bf16_to_f64(w_uv)
    B, H, _ = ol.shape
    out = np.empty((B, H, wv.shape[2]))
    for h in range(H):
        out[:, h, :] = ol[:, h, :] @ wv[h]
    return out


def mla_layer_absorbed_ref(q_nope, q_rope, w_uk, w_uv, kv_cache, block_table, cache_seqlens,
                           softmax_scale: float, *, page_size: int = 64, batch=None, heads=None):
    """absorb_q -> decode against the latent -> absorb_o, all in float64.

    Returns ``(out [nb, nh, d_v], lse [nb, nh])``; the lse is the decode's.
    """
    bs = _select(q_nope.shape[0], batch)
    hs = _select(q_nope.shape[1], heads)
    qp = mla_absorb_q_ref(q_nope[bs][:, hs], q_rope[bs][:, hs], np.asarray(w_uk)[hs])
    d_c = np.asarray(w_uk).shape[2]
    lens = np.asarray(cache_seqlens)[bs]
    bt = None if block_table is None else np.asarray(block_table)[bs]
    kv = kv_cache if block_table is not None else np.asarray(kv_cache)[bs]
    o_lat, lse = mla_decode_ref(qp, kv, bt, lens, softmax_scale, d_v=d_c, page_size=page_size)
    return mla_absorb_o_ref(o_lat, np.asarray(w_uv)[hs]), lse


def lse_merge_ref(outs, lses):
    """Merge attention results over disjoint key sets by their log-sum-exp.

    For parts s with normalised outputs O_s and lse L_s:
      L = ln sum_s exp(L_s),   O = sum_s exp(L_s - L) O_s.
    Parts with L_s = -inf (no keys) carry zero weight; if every part is empty the
    result is O = 0, L = -inf.  This is the same rescaling the glossary's online
    softmax note applies tile by tile.
    """
    lses = np.stack([np.asarray(x, dtype=np.float64) for x in lses])      # [S, ...]
    outs = np.stack([np.asarray(x, dtype=np.float64) for x in outs])      # [S, ..., d_v]
    m = lses.max(axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.exp(lses - m_safe)                                             # exp(-inf) = 0
    tot = w.sum(axis=0)
    L = np.where(finite, m_safe + np.log(np.where(finite, tot, 1.0)), -np.inf)
    wn = np.where(finite, w / np.where(finite, tot, 1.0), 0.0)
    return (wn[..., None] * outs).sum(axis=0), L


def cache_elements_per_token(n_heads_kv: int, d_head: int, d_c: int, d_rope: int):
    """Cached elements per token: standard K/V ``2 H_kv D`` versus latent + rope
    ``d_c + d_rope`` (glossary: layout difference from MHA/GQA, and the runnable
    check's last printed line)."""
    return 2 * n_heads_kv * d_head, d_c + d_rope


def latent_cache_bytes(layers: int, batch: int, tokens: int, d_c: int, d_rope: int,
                       bytes_per_elem: int) -> int:
    """Glossary "capacity and cost": M_MLA ~ L * B * T * (d_c + d_rope) * s."""
    return layers * batch * tokens * (d_c + d_rope) * bytes_per_elem
