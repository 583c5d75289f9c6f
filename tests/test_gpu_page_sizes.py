"""Pages smaller than a tile (down to one token per page) and page sizes that are not a
multiple of the tile: the producer gathers cache rows four at a time.  Checked against the
fp64 oracle, with bit-exact indexing (delta attention, page permutation) at page size 1."""
import numpy as np
import pytest

from kv_cache_paged_b200 import workload as wl
from oracle import oracle as orc
from tests import gpu_util as gu
from tests.indexing import decode_digits, make_delta_problem

pytestmark = pytest.mark.gpu


def small(variant, S, **kw):
    base = dict(B=5, L=1, h_q=32, h_kv=8, d=128, d_r=64, page_size=S, seqlens=("uniform", 1, 400), seed=S)
    base.update(kw)
    if variant == "gqa":
        base["d_r"] = 0
    return wl.make_inputs(variant, **base)


def check(inp, num_parts=0, what=""):
    out, lse = gu.run_gpu(inp, num_parts=num_parts)
    o, l = gu.to_np(out, lse)
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(o, l, ref_o, ref_l, what or inp.name)


@pytest.mark.parametrize("variant", ["gta", "gqa"])
@pytest.mark.parametrize("S", [1, 2, 8, 24, 48, 100])
def test_small_and_ragged_page_sizes(cuda_device, variant, S):
    check(small(variant, S), what=f"{variant} S={S}")


@pytest.mark.parametrize("variant", ["gta", "gqa"])
@pytest.mark.parametrize("L,num_parts", [(2, 0), (3, 7), (1, 300)])
def test_page_size_one_q_len_and_splits(cuda_device, variant, L, num_parts):
    inp = small(variant, 1, L=L, seqlens=("uniform", L, 300), seed=40 + L)
    check(inp, num_parts=num_parts, what=f"{variant} S=1 L={L} parts={num_parts}")


def test_page_size_one_short_and_empty_sequences(cuda_device):
    inp = small("gta", 1, B=6, seqlens=[1, 0, 3, 31, 32, 33], seed=44)
    out, lse = gu.run_gpu(inp, num_parts=4)
    o, l = gu.to_np(out, lse)
    assert np.all(o[1] == 0) and np.all(np.isneginf(l[1]))
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(o, l, ref_o, ref_l, "S=1 short")


@pytest.mark.parametrize("variant", ["gqa", "gta"])
def test_delta_attention_exact_at_page_size_one(cuda_device, variant):
    inp, targets = make_delta_problem(variant, seed=23, B=5, h_q=8, h_kv=2, d=64, d_r=32, S=1,
                                      seqlens=("uniform", 20, 500))
    out, lse = gu.run_gpu(inp, num_parts=3)
    assert np.array_equal(decode_digits(inp, gu.to_np(out, lse)[0]), targets)


def test_page_permutation_bit_identical_at_page_size_one(cuda_device):
    import torch
    inp = small("gta", 1, seed=45)
    out1, lse1 = gu.run_gpu(inp)
    rng = np.random.default_rng(1)
    perm = rng.permutation(inp.num_pages)
    inv = np.argsort(perm)
    for k in inp.caches:
        inp.caches[k] = np.ascontiguousarray(inp.caches[k][inv])
    bt = inp.block_table.copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    inp.block_table = bt
    out2, lse2 = gu.run_gpu(inp)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)


def test_page_size_one_full_gta_workload(cuda_device):
    """The GTA decode workload (B 32, contexts U[1024, 8192]) with one token per page."""
    check(wl.make_workload("gta", page_size=1), what="gta workload S=1")


def small_latent(h_c, d_c, S, **kw):
    base = dict(B=4, L=1, h_q=128, h_kv=h_c, d=d_c, d_r=64, page_size=S, seqlens=("uniform", 1, 300), seed=S + d_c,
                scale=0.07, latent_scale=0.1)
    base.update(kw)
    return wl.make_inputs("gla", **base)


@pytest.mark.parametrize("h_c,d_c", [(2, 256), (1, 512)])
@pytest.mark.parametrize("S", [1, 8, 16, 24, 100])
def test_latent_small_and_ragged_page_sizes(cuda_device, h_c, d_c, S):
    check(small_latent(h_c, d_c, S), what=f"h_c={h_c} d_c={d_c} S={S}")


@pytest.mark.parametrize("h_c,d_c", [(2, 256), (1, 512)])
@pytest.mark.parametrize("L,num_parts", [(2, 0), (1, 7)])
def test_latent_page_size_one_q_len_and_splits(cuda_device, h_c, d_c, L, num_parts):
    inp = small_latent(h_c, d_c, 1, L=L, seqlens=("uniform", L, 400), seed=50 + L)
    check(inp, num_parts=num_parts, what=f"h_c={h_c} S=1 L={L} parts={num_parts}")


@pytest.mark.parametrize("h_c,d_c", [(2, 256), (1, 512)])
def test_latent_page_permutation_bit_identical_at_page_size_one(cuda_device, h_c, d_c):
    import torch
    inp = small_latent(h_c, d_c, 1, seed=46)
    out1, lse1 = gu.run_gpu(inp)
    rng = np.random.default_rng(2)
    perm = rng.permutation(inp.num_pages)
    inv = np.argsort(perm)
    for k in inp.caches:
        inp.caches[k] = np.ascontiguousarray(inp.caches[k][inv])
    bt = inp.block_table.copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    inp.block_table = bt
    out2, lse2 = gu.run_gpu(inp)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)
