"""The C-ABI library: loads, exports every declared symbol, validates arguments and
plans splits (host logic only; no GPU needed)."""
import ctypes

import numpy as np
import pytest

from kv_cache_paged_b200 import binding


@pytest.fixture(scope="module")
def lib():
    return binding.lib()


def test_every_declared_function_is_exported(lib):
    names = binding.header_functions()
    assert len(names) >= 12
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version(lib):
    for code, text in binding.STATUS.items():
        assert lib.kvd_status_string(code).decode() == text
    assert lib.kvd_version() >= 100


def _gta_params(**kw):
    base = dict(q=16, tied_cache=16, rope_cache=16, block_table=16, seqlens=16, out=16, lse=16,
                B=2, L=1, h_q=8, h_kv=2, d_h=64, d_r=32, page_size=16, num_pages=10, max_pages=8,
                scale=0.125, num_parts=4)
    base.update(kw)
    return binding.GTAParams(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), -1),                 # null pointer
    (dict(q=18), -1),                   # misaligned for TMA
    (dict(h_q=7), -1),                  # h_q % h_kv != 0
    (dict(L=0), -1),
    (dict(d_h=96), -2),                 # head dim outside the compiled set
    (dict(d_r=48), -2),
    (dict(h_q=128, h_kv=2, L=1), -2),   # 64 rows per group: beyond the warp-MMA kernel
    (dict(scale=float("nan")), -1),
])
def test_gta_validation_errors(lib, kw, expect):
    p = _gta_params(**kw)
    assert lib.kvd_gta_workspace_size(ctypes.byref(p)) == 0
    assert lib.kvd_gta_decode(ctypes.byref(p), ctypes.c_void_p(256), 1 << 30, None) == expect


@pytest.mark.parametrize("S", [1, 3, 24, 100])
def test_any_page_size_is_accepted(lib, S):
    """Pages that do not hold whole 16-token tiles are gathered row by row, not rejected."""
    assert lib.kvd_gta_workspace_size(ctypes.byref(_gta_params(page_size=S))) > 0


def test_workspace_size_and_too_small(lib):
    p = _gta_params()
    n = lib.kvd_gta_workspace_size(ctypes.byref(p))
    slots, rows = 2 + 4 - 1, 1 * 8
    assert n == 256 + ((slots * rows * 4 + 255) // 256) * 256 + slots * rows * 64 * 4
    assert lib.kvd_gta_decode(ctypes.byref(p), ctypes.c_void_p(256), n - 1, None) == -3
    assert lib.kvd_gta_decode(ctypes.byref(p), ctypes.c_void_p(8), n, None) == -1   # workspace misaligned


def test_gqa_validation(lib):
    p = binding.GQAParams(q=16, k_cache=16, v_cache=16, block_table=16, seqlens=16, out=16, lse=16,
                          B=1, L=1, h_q=32, h_kv=8, d=80, page_size=64, num_pages=4, max_pages=4,
                          scale=0.1, num_parts=2)
    assert lib.kvd_gqa_decode(ctypes.byref(p), ctypes.c_void_p(256), 1 << 20, None) == -2


def test_debug_knobs_validate(lib):
    assert lib.kvd_debug_set(99, 1) == -1
    assert lib.kvd_debug_set(binding.DEBUG_WAIT_LIMIT_NS, 0) == -1
    assert lib.kvd_debug_set(binding.DEBUG_WAIT_LIMIT_NS, 2_000_000_000) == 0


# ----------------------------------------------------------------------------- split plan (host copy)
def _check_plan(seqlens, tile, parts, max_tokens=1 << 30):
    segs, counts = binding.plan_host(seqlens, tile, max_tokens, parts, cap=max(64, len(seqlens) + 2))
    tiles = [(-(-int(t) // tile)) for t in seqlens]
    N = sum(tiles)
    covered = {b: [] for b in range(len(seqlens))}
    slots = set()
    first_part = {}
    per_part = []
    for c in range(parts):
        n = int(counts[c])
        assert n <= segs.shape[1]
        ntile = 0
        prev_b = -1
        for k in range(n):
            b, t0, t1, split, nsplit, slot = (int(x) for x in segs[c, k])
            assert b > prev_b, "segments of a part are in sequence order"
            prev_b = b
            assert 0 <= t0 < t1 <= tiles[b]
            covered[b].append((t0, t1, split, nsplit))
            assert slot == b + c and slot not in slots
            assert split == c - first_part.setdefault(b, c)
            slots.add(slot)
            ntile += t1 - t0
        per_part.append(ntile)
    for b, segs_b in covered.items():
        segs_b.sort()
        if tiles[b] == 0:
            assert segs_b == []
            continue
        # contiguous, exact cover of [0, tiles_b), split indices 0..n-1, consistent nsplit
        assert segs_b[0][0] == 0 and segs_b[-1][1] == tiles[b]
        for (a0, a1, s0, n0), (b0, b1, s1, n1) in zip(segs_b, segs_b[1:]):
            assert a1 == b0
        assert [s[2] for s in segs_b] == list(range(len(segs_b)))
        assert all(s[3] == len(segs_b) for s in segs_b)
    if N:
        busy = per_part[:min(parts, N)]
        assert min(busy) >= 1, "the first min(parts, N) parts are all non-empty"
        assert all(x == 0 for x in per_part[min(parts, N):])
        assert max(busy) - min(busy) <= 1, "parts differ by at most one tile"
    return per_part


@pytest.mark.parametrize("parts", [1, 2, 7, 148, 1000])
def test_plan_covers_every_tile_once_balanced(parts):
    rng = np.random.default_rng(parts)
    sl = rng.integers(1024, 8193, size=32).astype(np.int32)
    per = _check_plan(sl, 16, parts)
    assert sum(per) == sum(-(-int(t) // 16) for t in sl)


def test_plan_with_empty_and_tiny_sequences():
    sl = np.array([0, 1, 15, 16, 17, 0, 0, 1000, 0], dtype=np.int32)
    for parts in (1, 3, 5, 64):
        _check_plan(sl, 16, parts)


def _plan_reference(seqlens, tile, parts, seg_cost, max_tokens=1 << 30):
    """The plan written out in Python: non-empty sequence b is seg_cost units followed by its tiles;
    the unit stream is cut into min(parts, N) equal parts; a part's segment of b is b's tiles inside
    the part's unit range."""
    tiles = [-(-min(max(int(t), 0), max_tokens) // tile) for t in seqlens]
    units = [n + seg_cost if n else 0 for n in tiles]
    N = sum(units)
    P = min(parts, N)
    out = [[] for _ in range(parts)]
    if N == 0:
        return out
    first_unit, run = [], 0
    for n, u in zip(tiles, units):
        first_unit.append(run + u - n)
        run += u
    part_of = lambda x: ((x + 1) * P - 1) // N
    for c in range(P):
        lo, hi = c * N // P, (c + 1) * N // P
        for b, n in enumerate(tiles):
            cu = first_unit[b]
            if n and cu < hi and cu + n > lo:
                f, l = part_of(cu), part_of(cu + n - 1)
                out[c].append((b, max(lo, cu) - cu, min(hi, cu + n) - cu, c - f, l - f + 1, b + c))
    return out


@pytest.mark.parametrize("seg_cost", [0, 1, 3, 20])
@pytest.mark.parametrize("parts", [1, 3, 74, 148, 1000])
def test_plan_with_a_segment_cost_matches_its_definition(parts, seg_cost):
    rng = np.random.default_rng(parts + seg_cost)
    sl = np.clip(np.round(np.exp(rng.normal(np.log(8192), 1.0, 128))), 1, 65536).astype(np.int32)
    sl[rng.integers(0, 128, 6)] = 0  # a few empty sequences
    segs, counts = binding.plan_host(sl, 96, 1 << 30, parts, cap=160, seg_cost=seg_cost)
    ref = _plan_reference(sl, 96, parts, seg_cost)
    for c in range(parts):
        got = [tuple(int(x) for x in segs[c, k]) for k in range(int(counts[c]))]
        assert got == ref[c], (c, got[:3], ref[c][:3])
    # every tile once, and a part that starts more sequences holds fewer tiles
    tiles = {}
    for c in range(parts):
        for (b, t0, t1, *_r) in ref[c]:
            tiles.setdefault(b, []).append((t0, t1))
    for b, n in enumerate(-(-int(t) // 96) for t in sl):
        got = sorted(tiles.get(b, []))
        assert sum(t1 - t0 for t0, t1 in got) == n and all(a[1] == z[0] for a, z in zip(got, got[1:]))


def test_plan_all_empty():
    segs, counts = binding.plan_host(np.zeros(5, np.int32), 16, 1 << 20, 4)
    assert counts.sum() == 0


def test_plan_clamps_oversized_lengths():
    # lengths above max_tokens are clamped (the decode kernel flags them)
    segs, counts = binding.plan_host(np.array([100, 5000], np.int32), 16, 256, 2)
    tiles = sum(int(segs[c, k, 2] - segs[c, k, 1]) for c in range(2) for k in range(counts[c]))
    assert tiles == 7 + 16


def _gla_params(**kw):
    base = dict(q=16, latent_cache=16, rope_cache=16, block_table=16, seqlens=16, out=16, lse=16,
                B=2, L=1, h_q=128, h_c=2, d_c=256, d_r=64, page_size=64, num_pages=10, max_pages=8,
                scale=0.07, num_parts=4)
    base.update(kw)
    return binding.GLAParams(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(latent_cache=None), -1),
    (dict(out=24), -1),                 # GLA output rows are written as 16-byte vectors
    (dict(h_q=127), -1),
    (dict(d_c=384), -2),                # latent width outside the compiled set
    (dict(d_r=32), -2),
    (dict(h_q=96, h_c=1), -2),          # 96 heads per latent head: neither divides nor is a multiple of 128
])
def test_gla_validation_errors(lib, kw, expect):
    p = _gla_params(**kw)
    assert lib.kvd_gla_workspace_size(ctypes.byref(p)) == 0
    assert lib.kvd_gla_decode(ctypes.byref(p), ctypes.c_void_p(256), 1 << 30, None) == expect


@pytest.mark.parametrize("S,d_c,h_c", [(1, 256, 2), (48, 256, 2), (1, 512, 1), (100, 512, 1)])
def test_gla_any_page_size_is_accepted(lib, S, d_c, h_c):
    """Pages that do not hold whole 64-token tiles are gathered token by token, not rejected."""
    assert lib.kvd_gla_workspace_size(ctypes.byref(_gla_params(page_size=S, d_c=d_c, h_c=h_c))) > 0


@pytest.mark.parametrize("L,S", [(1, 1), (1, 16), (2, 1), (2, 48), (4, 64), (6, 8)])
def test_gla2_every_row_count_and_page_size_is_planned(lib, L, S):
    """GLA-2 at 64, 128, 256 and 384 rows per latent head (the narrow kernel, the 128-row kernel
    in one or several row blocks), with boxed and gathered page sizes: the workspace holds the
    split partials of every row."""
    p = _gla_params(L=L, page_size=S)
    slots, rows = 2 + 4 - 1, L * 128
    assert lib.kvd_gla_workspace_size(ctypes.byref(p)) == (
        256 + ((slots * rows * 4 + 255) // 256) * 256 + slots * rows * 256 * 4)


def test_gla_workspace_size(lib):
    p = _gla_params(L=2, d_c=512, h_c=1, page_size=64)
    n = lib.kvd_gla_workspace_size(ctypes.byref(p))
    slots, rows = 2 + 4 - 1, 2 * 128
    assert n == 256 + ((slots * rows * 4 + 255) // 256) * 256 + slots * rows * 512 * 4
