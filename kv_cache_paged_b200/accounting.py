"""Algorithmic bytes and FLOPs of one decode step (the roofline numerators).

Bytes: every visible KV element read once (exactly T_b tokens, no rounding up to
whole pages), plus q, out, lse, the block-table entries in use and seqlens.
Split-KV partials are not algorithmic traffic: they count against the kernel.

FLOPs: 2 (d_qk + d_v) per (query row, visible token) pair: the QK^T dot product
and the PV accumulation.  Causally masked pairs and the softmax are excluded.

For q_len 1 the ratio reproduces the paper's intensity I ~= 2 g_q / m_kv
("Hardware-Efficient Attention for Fast Decoding", section 3.1): per token and
KV head, g_q query heads each do 2 * 2 d_h FLOPs on m_kv * d_h * 2 bytes.
"""
from __future__ import annotations

import numpy as np


def kv_elems_per_token(variant: str, h_kv: int, d: int, d_r: int) -> int:
    """Cache elements one token adds (GQA: K and V; GTA: tied + shared rope; GLA: latents + rope)."""
    if variant == "gqa":
        return 2 * h_kv * d
    return h_kv * d + d_r


def dims(variant: str, d: int, d_r: int):
    """(d_qk, d_v)."""
    if variant == "gla":
        return d + d_r, d
    return d, d


def kv_bytes(variant, seqlens, h_kv, d, d_r) -> int:
    return int(np.sum(np.asarray(seqlens, dtype=np.int64))) * kv_elems_per_token(variant, h_kv, d, d_r) * 2


def step_bytes(variant, seqlens, *, L, h_q, h_kv, d, d_r, page_size) -> int:
    sl = np.asarray(seqlens, dtype=np.int64)
    B = sl.shape[0]
    d_qk, d_v = dims(variant, d, d_r)
    pages = int(np.sum((sl + page_size - 1) // page_size))
    return (kv_bytes(variant, sl, h_kv, d, d_r) + B * L * h_q * (d_qk + d_v) * 2
            + B * L * h_q * 4 + pages * 4 + B * 4)


def step_flops(variant, seqlens, *, L, h_q, d, d_r) -> int:
    sl = np.asarray(seqlens, dtype=np.int64)
    d_qk, d_v = dims(variant, d, d_r)
    # row i of sequence b sees max(0, T_b - L + i + 1) tokens
    vis = np.maximum(0, sl[:, None] - L + np.arange(L)[None, :] + 1).sum()
    return int(vis) * h_q * 2 * (d_qk + d_v)


def of_inputs(inp):
    """(bytes, flops, kv_bytes) for a decode-inputs record.  A prefix shared by the batch
    (stored once) is algorithmically read once: its tokens count once, not once per sequence."""
    kw = dict(L=inp.L, h_q=inp.h_q, h_kv=inp.h_kv, d=inp.d, d_r=inp.d_r, page_size=inp.page_size)
    b = step_bytes(inp.variant, inp.seqlens, **kw)
    f = step_flops(inp.variant, inp.seqlens, L=inp.L, h_q=inp.h_q, d=inp.d, d_r=inp.d_r)
    kvb = kv_bytes(inp.variant, inp.seqlens, inp.h_kv, inp.d, inp.d_r)
    shared = getattr(inp, "shared_prefix", 0)
    if shared and inp.B > 1:
        dup = (inp.B - 1) * shared * kv_elems_per_token(inp.variant, inp.h_kv, inp.d, inp.d_r) * 2
        b, kvb = b - dup, kvb - dup
    return b, f, kvb


def roofline_us(nbytes: float, flops: float, hbm_gbs: float, tflops: float) -> float:
    """max(bytes / HBM peak, FLOPs / tensor peak) in microseconds."""
    return max(nbytes / (hbm_gbs * 1e3), flops / (tflops * 1e6))
