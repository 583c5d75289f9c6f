"""Seeded synthetic inputs for paged decode attention.

This module only draws numbers and lays them out; it holds none of the
attention arithmetic.  It serves both the CUDA path (tests, ``bench.py``) and
the fp64 oracle, which never import each other.

Workloads follow the decode settings of "Hardware-Efficient Attention for Fast
Decoding" (Zadouri, Strauss, Dao): GQA and GTA at h_q=32, d_h=128; MLA with one
512-dim latent head plus a 64-dim shared RoPE key; GLA-2 with two 256-dim latent
heads (section 3.3.2 of the paper: h_c = 2, d_c = 2 d_h).

Recipe (every array bf16 unless noted, values i.i.d. N(0, 1) from numpy PCG64):

* draw order: seqlens -> physical page permutation -> caches -> q;
* the pool holds exactly sum_b ceil(T_b / S) pages plus one page that no
  block-table entry names; that page and every slot past T_b in a sequence's
  last page hold bf16 NaN, so any read of memory outside the visible context
  shows up in the output;
* block_table[b, i] is the physical page of logical page i of sequence b, a
  random permutation (or the identity when ``shuffle=False``), and -1 past
  ceil(T_b / S);
* RoPE slices are drawn directly in rotated form: a rotation is orthogonal, so
  rotating an isotropic Gaussian vector gives an isotropic Gaussian vector of
  the same law, and the decode step only ever sees rotated keys and queries;
* ``latent_scale`` multiplies the latent cache before rounding (0.1 for the
  MLA workload); q and the RoPE slices are never scaled.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BF16_NAN = np.uint16(0x7FC0)

# Seeds per named workload.
SEEDS = {"gta_tiny": 0, "gta": 1, "gqa": 2, "mla": 3, "gla2": 4, "gta_prefix": 5, "gta_prefix_long": 6, "gla8": 7}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest even); returns raw uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits to float32."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class DecodeInputs:
    """One decode step's inputs; every array is host memory (numpy).

    ``variant`` is ``"gqa"``, ``"gta"`` or ``"gla"`` (MLA is ``"gla"`` with
    ``h_kv == 1`` latent head).  For GLA, ``h_kv`` holds h_c and ``d`` holds d_c.
    """
    variant: str
    B: int
    L: int
    h_q: int
    h_kv: int          # KV groups (GQA/GTA) or latent heads h_c (GLA/MLA)
    d: int             # d (GQA), d_h (GTA) or d_c (GLA)
    d_r: int           # RoPE slice width (GTA/GLA); 0 for GQA
    page_size: int
    num_pages: int
    max_pages: int
    scale: float
    seqlens: np.ndarray            # int32 [B]
    block_table: np.ndarray        # int32 [B, max_pages]
    q: np.ndarray                  # uint16 (bf16) [B, L, h_q, d_qk]
    caches: dict = field(default_factory=dict)   # name -> uint16 array
    poison_page: int = -1
    name: str = ""
    shared_prefix: int = 0  # tokens at the start of every sequence stored once, in shared pages

    @property
    def d_qk(self) -> int:
        if self.variant == "gqa":
            return self.d
        if self.variant == "gta":
            return self.d
        return self.d + self.d_r

    @property
    def d_v(self) -> int:
        return self.d


def _draw_bf16(rng: np.random.Generator, shape, scale: float = 1.0, chunk: int = 1 << 24) -> np.ndarray:
    """Draw N(0,1) * scale in float32 and round to bf16, in chunks to bound memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = rng.standard_normal(e - s, dtype=np.float32)
        if scale != 1.0:
            x *= np.float32(scale)
        out[s:e] = f32_to_bf16_bits(x)
    return out.reshape(shape)


def draw_seqlens(rng: np.random.Generator, B: int, spec, L: int = 1) -> np.ndarray:
    """Context lengths.

    ``spec`` is an int (fixed length), ``("uniform", lo, hi)`` (integers, both
    ends included), ``("lognormal", median, sigma, cap)`` (rounded to nearest,
    clamped to [max(L, 1), cap]) or an explicit sequence of lengths.
    """
    if isinstance(spec, (int, np.integer)):
        return np.full(B, int(spec), dtype=np.int32)
    if isinstance(spec, tuple) and spec and spec[0] == "uniform":
        _, lo, hi = spec
        return rng.integers(lo, hi + 1, size=B, dtype=np.int64).astype(np.int32)
    if isinstance(spec, tuple) and spec and spec[0] == "lognormal":
        _, median, sigma, cap = spec
        x = rng.lognormal(mean=math.log(median), sigma=sigma, size=B)
        x = np.clip(np.rint(x), max(L, 1), cap)
        return x.astype(np.int32)
    arr = np.asarray(spec, dtype=np.int32)
    assert arr.shape == (B,), "explicit seqlens must have shape [B]"
    return arr


def make_paging(rng: np.random.Generator, seqlens: np.ndarray, page_size: int, shuffle: bool = True,
                prefix_pages: int = 0):
    """Block table over a pool of the used pages plus one unreferenced page.  The first
    ``prefix_pages`` logical pages of every sequence are the same physical pages (a prefix
    shared by the whole batch, stored once); the other pages belong to one sequence each."""
    B = len(seqlens)
    npages = [(int(t) + page_size - 1) // page_size for t in seqlens]
    assert all(n > prefix_pages for n in npages) or prefix_pages == 0, "sequences must extend past the prefix"
    own = [n - prefix_pages for n in npages]
    used = prefix_pages + sum(own)
    max_pages = max(1, max(npages) if npages else 1)
    num_pages = used + 1
    perm = rng.permutation(num_pages).astype(np.int32) if shuffle else np.arange(num_pages, dtype=np.int32)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    k = prefix_pages
    for b in range(B):
        table[b, :prefix_pages] = perm[:prefix_pages]
        table[b, prefix_pages: npages[b]] = perm[k: k + own[b]]
        k += own[b]
    poison = int(perm[used])
    return table, num_pages, max_pages, poison


def poison_cache(cache: np.ndarray, seqlens: np.ndarray, table: np.ndarray, poison_page: int, page_size: int) -> None:
    """Write bf16 NaN into the unreferenced page and into slots past each T_b."""
    cache[poison_page] = BF16_NAN
    for b, t in enumerate(seqlens):
        t = int(t)
        tail = t % page_size
        if tail:
            cache[table[b, t // page_size], tail:] = BF16_NAN


def make_inputs(variant: str, *, B: int, L: int, h_q: int, h_kv: int, d: int, d_r: int = 0,
                page_size: int, seqlens, seed: int, scale: float | None = None,
                latent_scale: float = 1.0, shuffle: bool = True, name: str = "",
                shared_prefix: int = 0) -> DecodeInputs:
    """Draw a full decode step for ``variant`` in ("gqa", "gta", "gla").  With
    ``shared_prefix`` (a multiple of the page size) every sequence starts with the same
    ``shared_prefix`` tokens, stored once; ``seqlens`` then draws the lengths past it."""
    assert variant in ("gqa", "gta", "gla")
    assert shared_prefix % page_size == 0, "the shared prefix covers whole pages"
    rng = np.random.default_rng(seed)
    sl = (draw_seqlens(rng, B, seqlens, L) + shared_prefix).astype(np.int32)
    table, num_pages, max_pages, poison = make_paging(rng, sl, page_size, shuffle, shared_prefix // page_size)
    S = page_size
    caches = {}
    if variant == "gqa":
        caches["k_cache"] = _draw_bf16(rng, (num_pages, S, h_kv, d))
        caches["v_cache"] = _draw_bf16(rng, (num_pages, S, h_kv, d))
        d_qk = d
    elif variant == "gta":
        caches["tied_cache"] = _draw_bf16(rng, (num_pages, S, h_kv, d))
        caches["rope_cache"] = _draw_bf16(rng, (num_pages, S, d_r))
        d_qk = d
    else:
        caches["latent_cache"] = _draw_bf16(rng, (num_pages, S, h_kv, d), latent_scale)
        caches["rope_cache"] = _draw_bf16(rng, (num_pages, S, d_r))
        d_qk = d + d_r
    for c in caches.values():
        poison_cache(c, sl, table, poison, S)
    q = _draw_bf16(rng, (B, L, h_q, d_qk))
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk if variant != "gla" else 192)
    return DecodeInputs(variant=variant, B=B, L=L, h_q=h_q, h_kv=h_kv, d=d, d_r=d_r,
                        page_size=S, num_pages=num_pages, max_pages=max_pages, scale=float(scale),
                        seqlens=sl, block_table=table, q=q, caches=caches, poison_page=poison,
                        name=name, shared_prefix=shared_prefix)


# Named decode workloads (shapes from the paper's decode settings).
WORKLOADS = {
    # GTA tiny: key = tied[0:32] ++ rope(32), value = tied (64); context 128; S = 16.
    "gta_tiny": dict(variant="gta", B=2, h_q=8, h_kv=2, d=64, d_r=32, page_size=16,
                     seqlens=128, scale=1.0 / 8.0),
    "gta": dict(variant="gta", B=32, h_q=32, h_kv=8, d=128, d_r=64, page_size=64,
                seqlens=("uniform", 1024, 8192), scale=1.0 / math.sqrt(128)),
    "gqa": dict(variant="gqa", B=32, h_q=32, h_kv=8, d=128, d_r=0, page_size=64,
                seqlens=8192, scale=1.0 / math.sqrt(128)),
    "mla": dict(variant="gla", B=64, h_q=128, h_kv=1, d=512, d_r=64, page_size=64,
                seqlens=("uniform", 4096, 32768), scale=1.0 / math.sqrt(192), latent_scale=0.1),
    "gla2": dict(variant="gla", B=128, h_q=128, h_kv=2, d=256, d_r=64, page_size=64,
                 seqlens=("lognormal", 8192, 1.0, 65536), scale=1.0 / math.sqrt(192)),
    # GLA-8 (NEXT-3): eight 256-wide latent heads, 16 query heads each, GLA-2's contexts
    "gla8": dict(variant="gla", B=128, h_q=128, h_kv=8, d=256, d_r=64, page_size=64,
                 seqlens=("lognormal", 8192, 1.0, 65536), scale=1.0 / math.sqrt(192)),
    # GTA shape with a 4096-token prefix shared by the batch (stored once) and per-sequence
    # continuations of U[64, 2048] tokens: the shared-prefix decode workload
    "gta_prefix": dict(variant="gta", B=32, h_q=32, h_kv=8, d=128, d_r=64, page_size=64,
                       seqlens=("uniform", 64, 2048), shared_prefix=4096, scale=1.0 / math.sqrt(128)),
    # the same with a 32768-token shared prefix (71 MB of tied state and rope, read once per
    # step by the batched prefix path, 32 times by a one-pass decode)
    "gta_prefix_long": dict(variant="gta", B=32, h_q=32, h_kv=8, d=128, d_r=64, page_size=64,
                            seqlens=("uniform", 64, 2048), shared_prefix=32768, scale=1.0 / math.sqrt(128)),
}

# Query lengths each workload is run at.
WORKLOAD_QLENS = {"gta_tiny": (1,), "gta": (1,), "gqa": (1,), "mla": (1, 2), "gla2": (1, 2, 4), "gta_prefix": (1,), "gta_prefix_long": (1,), "gla8": (1, 2, 4, 8)}


def make_workload(name: str, L: int = 1, seed: int | None = None, **overrides) -> DecodeInputs:
    """Draw a named workload; keyword overrides replace any field (e.g. ``B=4``)."""
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    s = SEEDS[name] if seed is None else seed
    return make_inputs(L=L, seed=s, name=name, **cfg)
