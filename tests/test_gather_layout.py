"""Index arithmetic of the small-page gather, checked on the CPU.

The gather copies each token's rows with 16-byte cp.async into the layout a tensor-map box load
would produce (128-byte swizzle: unit c of row k of a 64-wide chunk lands at
k * 128 + ((c ^ (k % 8)) * 16)).  This replays, in integers, the lane / loop arithmetic of the
group kernel's producer warps and of gather_tile in the latent kernels for every shape they are
built for, and checks that every 16-byte unit of every token of a tile is written exactly once,
at the box layout's address, from the right source element."""
import itertools

import pytest


def sw128(r, c):
    return r * 128 + ((c ^ (r & 7)) << 4)


def sw64(r, c):
    off = r * 64 + c * 16
    return off ^ (((off >> 7) & 3) << 4)


def group_gather(tied, nch, dr, tt, gw, row_of):
    """Writes (smem offset -> source element) of one tile as the group kernel's producers do."""
    writes = {}
    kv_tile = nch * 64 * tt * 2
    ru = dr * 2 // 16 if tied else 0
    tpw = (tt + gw - 1) // gw
    for pw in range(gw):
        nkw = (tt - pw + gw - 1) // gw
        for lane in range(32):
            dst_l = (lane >> 3) * tt * 128
            c_l = lane & 7
            nj = (nch * 8 - lane + 31) // 32
            for i in range(min(tpw, nkw)):
                k = pw + gw * i
                row = row_of(k)
                dst = dst_l + k * 128 + ((c_l ^ (k & 7)) << 4)
                for j in range(max(nj, 0)):
                    d = dst + 4 * j * tt * 128
                    for arr, base in ((0, 0),) + (() if tied else ((1, kv_tile),)):
                        key = (arr, base + d)
                        assert key not in writes
                        writes[key] = (arr, row, lane * 8 + 256 * j)
            if tied:
                r_u = lane % ru
                for i0 in range(0, tpw, 32 // ru):
                    i = i0 + lane // ru
                    if i < nkw:
                        k = pw + gw * i
                        key = (1, kv_tile + (sw128(k, r_u) if dr == 64 else sw64(k, r_u)))
                        assert key not in writes
                        writes[key] = ("rope", row_of(k), r_u * 8)
    return writes


def group_expected(tied, nch, dr, tt, row_of):
    exp = {}
    kv_tile = nch * 64 * tt * 2
    for k in range(tt):
        for u in range(nch * 8):
            z, c = u >> 3, u & 7
            exp[(0, z * tt * 128 + sw128(k, c))] = (0, row_of(k), u * 8)
            if not tied:
                exp[(1, kv_tile + z * tt * 128 + sw128(k, c))] = (1, row_of(k), u * 8)
        if tied:
            for c in range(dr * 2 // 16):
                exp[(1, kv_tile + (sw128(k, c) if dr == 64 else sw64(k, c)))] = ("rope", row_of(k), c * 8)
    return exp


@pytest.mark.parametrize("tied,d,dr", [(False, 64, 0), (False, 128, 0), (True, 64, 32), (True, 128, 32),
                                       (True, 128, 64), (True, 64, 64)])
@pytest.mark.parametrize("gpc", [1, 2, 4, 8])
@pytest.mark.parametrize("tt,gw", [(16, 4), (32, 4), (32, 6)])
def test_group_gather_covers_the_box_layout(tied, d, dr, gpc, tt, gw):
    nch = gpc * d // 64
    row_of = lambda k: 1000 + 7 * k  # distinct rows per token
    assert group_gather(tied, nch, dr, tt, gw, row_of) == group_expected(tied, nch, dr, tt, row_of)


def gather_tile(nch, rw, chunk_bytes, k0, kstep, nk, row_of):
    writes = {}
    units = nch * 8
    nj = (units + 31) // 32
    tpi = 32 // rw
    rope_dst = nch * chunk_bytes
    for lane in range(32):
        dst_l = (lane >> 3) * chunk_bytes
        c_l = lane & 7
        for i in range(nk):
            k = k0 + i * kstep
            dst = dst_l + k * 128 + ((c_l ^ (k & 7)) << 4)
            for j in range(nj):
                if units % 32 == 0 or lane + 32 * j < units:
                    key = dst + 4 * j * chunk_bytes
                    assert key not in writes
                    writes[key] = ("lat", row_of(k), lane * 8 + 256 * j)
        r_u = lane % rw
        for i0 in range(0, nk, tpi):
            i = i0 + lane // rw
            if i < nk:
                k = k0 + i * kstep
                key = rope_dst + (sw128(k, r_u) if rw == 8 else sw64(k, r_u))
                assert key not in writes
                writes[key] = ("rope", row_of(k), r_u * 8)
    return writes


@pytest.mark.parametrize("nch,rw,tok", [(4, 8, 64), (2, 8, 64), (4, 4, 64), (4, 8, 96)])  # GLA d_c 256 (64- and
@pytest.mark.parametrize("nwarps", [3, 5, 6])                                               # 96-token tiles), GTA
def test_latent_gather_covers_the_box_layout(nch, rw, tok, nwarps):                          # prefix, MLA half
    if (tok + nwarps - 1) // nwarps > 32:
        pytest.skip("one token per gather lane")
    chunk_bytes = tok * 128
    row_of = lambda k: 500 + 3 * k
    writes = {}
    for gw in range(nwarps):  # warps split the tile's tokens k = gw, gw + nwarps, ...
        nk = (tok - gw + nwarps - 1) // nwarps
        w = gather_tile(nch, rw, chunk_bytes, gw, nwarps, nk, row_of)
        assert not (w.keys() & writes.keys())
        writes.update(w)
    exp = {}
    for k in range(tok):
        for u in range(nch * 8):
            exp[(u >> 3) * chunk_bytes + sw128(k, u & 7)] = ("lat", row_of(k), u * 8)
        for c in range(rw):
            exp[nch * chunk_bytes + (sw128(k, c) if rw == 8 else sw64(k, c))] = ("rope", row_of(k), c * 8)
    assert writes == exp


def test_a_wrong_swizzle_is_caught():
    """The check is not vacuous: a copy that forgets the XOR with the row is found."""
    tt, nch = 16, 2
    row_of = lambda k: k
    w = group_gather(False, nch, 0, tt, 4, row_of)
    bad = {(a, off ^ 16 if (off // 128) % 8 == 1 else off): v for (a, off), v in w.items()}
    assert bad != group_expected(False, nch, 0, tt, row_of)
