"""Second, independent fp64 restatement of paged decode attention in numpy.

TEST INFRASTRUCTURE ONLY (tiny inputs).  It is written the other way round
from ``oracle.c``: it first gathers each sequence's pages into a contiguous
[T, ...] block, materialises explicit per-head K and V, and then applies a
textbook masked softmax with matrix products.  Agreement between the two
pins the C oracle's paging, key/value composition and softmax.
"""
from __future__ import annotations

import numpy as np


def bf16_to_f64(h):
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gather_tokens(cache, block_table_row, T, page_size):
    """Contiguous [T, ...] view of one sequence's first T tokens."""
    n_pages = -(-T // page_size)
    pages = cache[np.asarray(block_table_row[:n_pages])]          # [n_pages, S, ...]
    flat = pages.reshape((n_pages * page_size,) + cache.shape[2:])
    return flat[:T]


def explicit_kv(variant, c0, c1, block_table_row, T, page_size, h_q, h_kv, d, d_r):
    """Per-head explicit K [T, h_q, d_qk] and V [T, h_q, d_v] in float64."""
    g_q = h_q // h_kv
    x0 = bf16_to_f64(gather_tokens(c0, block_table_row, T, page_size))   # [T, h_kv, d]
    x1 = bf16_to_f64(gather_tokens(c1, block_table_row, T, page_size))
    if variant == "gqa":
        K, V = x0, x1                                                       # [T, h_kv, d]
    elif variant == "gta":
        rope = np.broadcast_to(x1[:, None, :], (T, h_kv, d_r))
        K = np.concatenate([x0[:, :, : d - d_r], rope], axis=2)            # [T, h_kv, d]
        V = x0
    else:
        rope = np.broadcast_to(x1[:, None, :], (T, h_kv, d_r))
        K = np.concatenate([x0, rope], axis=2)                              # [T, h_c, d_c + d_r]
        V = x0
    # Expand groups to query heads: head h uses group h // g_q.
    K = np.repeat(K, g_q, axis=1)
    V = np.repeat(V, g_q, axis=1)
    return K, V


def attention(q, K, V, scale, L):
    """Causal decode attention for one sequence.

    q [L, h, d_qk], K [T, h, d_qk], V [T, h, d_v]; row i sees keys t <= T - L + i.
    Returns out [L, h, d_v], lse [L, h].
    """
    T = K.shape[0]
    Lq, H, _ = q.shape
    s = np.einsum("ihd,thd->iht", q, K) * scale                      # [L, h, T]
    pos = T - L + np.arange(Lq)
    visible = np.arange(T)[None, :] <= pos[:, None]                  # [L, T]
    s = np.where(visible[:, None, :], s, -np.inf)
    out = np.zeros((Lq, H, V.shape[2]))
    lse = np.full((Lq, H), -np.inf)
    for i in range(Lq):
        if not visible[i].any():
            continue
        m = s[i].max(axis=1, keepdims=True)
        e = np.exp(s[i] - m)
        den = e.sum(axis=1, keepdims=True)
        p = e / den
        out[i] = np.einsum("ht,thd->hd", p, V)
        lse[i] = (m + np.log(den))[:, 0]
    return out, lse


def decode(variant, q, c0, c1, block_table, seqlens, *, L, h_q, h_kv, d, d_r, page_size, scale):
    B = len(seqlens)
    d_v = d
    out = np.zeros((B, L, h_q, d_v))
    lse = np.zeros((B, L, h_q))
    qf = bf16_to_f64(q)
    for b in range(B):
        T = int(seqlens[b])
        if T == 0:
            lse[b] = -np.inf
            continue
        K, V = explicit_kv(variant, c0, c1, block_table[b], T, page_size, h_q, h_kv, d, d_r)
        out[b], lse[b] = attention(qf[b], K, V, scale, L)
    return out, lse
