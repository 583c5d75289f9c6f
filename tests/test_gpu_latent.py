"""GLA / MLA (absorbed) decode on the GPU against the fp64 oracle (the stated output tolerance)."""
import numpy as np
import pytest

from kv_cache_paged_b200 import workload as wl
from oracle import oracle as orc
from tests import gpu_util as gu
from tests.indexing import decode_digits, make_delta_problem

pytestmark = pytest.mark.gpu


def check(inp, num_parts=0, b_sample=None, what="", stress=False):
    """Against the oracle with the flat bound (stress: see gpu_util.assert_close)."""
    out, lse = gu.run_gpu(inp, num_parts=num_parts)
    o, l = gu.to_np(out, lse)
    if b_sample is not None:
        sel = np.asarray(b_sample, dtype=np.int32)
        ref_o, ref_l, _ = orc.decode_inputs(inp, b_list=sel)
        return gu.assert_close(o[sel], l[sel], ref_o, ref_l, what or inp.name, stress=stress)
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    return gu.assert_close(o, l, ref_o, ref_l, what or inp.name, stress=stress)


def small(h_c, d_c, **kw):
    base = dict(B=3, L=1, h_q=128, h_kv=h_c, d=d_c, d_r=64, page_size=64, seqlens=[1, 97, 300], seed=7,
                scale=1.0 / np.sqrt(192), latent_scale=0.1 if h_c == 1 else 1.0)
    base.update(kw)
    return wl.make_inputs("gla", **base)


# ----------------------------------------------------------------------------- small shapes first
@pytest.mark.parametrize("L", [1, 2])
def test_mla_small(cuda_device, L):
    check(small(1, 512, L=L, seqlens=[L, 97, 300]), what=f"MLA L={L}")


@pytest.mark.parametrize("L", [1, 2, 4])
def test_gla2_small(cuda_device, L):
    # stress bound: the first sequence holds exactly L tokens, so its rows see one to L tokens
    check(small(2, 256, L=L, seqlens=[L, 97, 300]), what=f"GLA-2 L={L}", stress=True)


@pytest.mark.parametrize("h_c,d_c", [(1, 512), (2, 256)])
@pytest.mark.parametrize("num_parts", [1, 3, 50])
def test_latent_forced_splits(cuda_device, h_c, d_c, num_parts):
    inp = small(h_c, d_c, B=5, L=2, seqlens=("uniform", 2, 900), seed=11 + num_parts)
    check(inp, num_parts=num_parts, what=f"h_c={h_c} parts={num_parts}")


@pytest.mark.parametrize("h_c,d_c", [(1, 512), (2, 256)])
def test_latent_page_boundaries(cuda_device, h_c, d_c):
    sl = [1, 31, 32, 33, 63, 64, 65, 128, 129]
    check(small(h_c, d_c, B=len(sl), seqlens=sl, seed=13), num_parts=4)


@pytest.mark.parametrize("h_c,h_q,L", [(8, 128, 2), (4, 64, 1), (1, 64, 3), (2, 256, 1)])
def test_latent_group_shapes(cuda_device, h_c, h_q, L):
    """GLA-8 (16 heads per latent head), smaller and larger groups, q_len 3."""
    inp = small(h_c, 256, h_q=h_q, L=L, seqlens=("uniform", L, 500), seed=h_c + h_q + L)
    check(inp, what=f"h_c={h_c} h_q={h_q} L={L}")


def test_latent_peaky_softmax(cuda_device):
    inp = small(2, 256, L=2, seqlens=("uniform", 2, 2000), seed=17)
    inp.scale *= 8
    check(inp, num_parts=9)


def test_latent_empty_sequences(cuda_device):
    inp = small(2, 256, B=4, seqlens=[0, 70, 0, 5], seed=19)
    out, lse = gu.run_gpu(inp, num_parts=3)
    o, l = gu.to_np(out, lse)
    assert np.all(o[[0, 2]] == 0) and np.all(np.isneginf(l[[0, 2]]))
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(o, l, ref_o, ref_l)


# ----------------------------------------------------------------------------- at most 64 rows per latent head
# GLA-2 at q_len 1 and GLA-8 up to q_len 4 run on the narrow kernel (96-token tiles, M = 64).
@pytest.mark.parametrize("num_parts", [1, 3, 50, 148])
def test_narrow_forced_splits(cuda_device, num_parts):
    inp = small(2, 256, B=5, L=1, seqlens=("uniform", 1, 1500), seed=211 + num_parts)
    check(inp, num_parts=num_parts, what=f"GLA-2 L=1 parts={num_parts}")


def test_narrow_tile_boundaries(cuda_device):
    sl = [1, 2, 47, 48, 95, 96, 97, 191, 192, 193, 300]
    inp = small(2, 256, B=len(sl), L=1, seqlens=sl, seed=223)
    for parts in (0, 1, 4, 64):
        # stress bound: the one- and two-token sequences have rows that see one or two tokens
        check(inp, num_parts=parts, what=f"GLA-2 L=1 tile boundaries parts={parts}", stress=True)


@pytest.mark.parametrize("S", [16, 24, 32, 48, 64, 96, 128, 192])
def test_narrow_box_shapes(cuda_device, S):
    """Every box size the box path cuts a 96-token tile into (16, 24, 32, 48 tokens, and one box
    of the whole tile when the page holds whole tiles)."""
    inp = small(2, 256, B=4, L=1, page_size=S, seqlens=("uniform", 30, 700), seed=229 + S)
    check(inp, num_parts=5, what=f"GLA-2 L=1 S={S}")


@pytest.mark.parametrize("h_c,h_q,L", [(4, 32, 3), (8, 128, 1), (2, 8, 1), (1, 64, 1)])
def test_narrow_row_spreads(cuda_device, h_c, h_q, L):
    """R = 24, 16, 4 and 64 rows per latent head: 6, 4, 1 and 16 rows per lane quadrant."""
    inp = small(h_c, 256, h_q=h_q, L=L, seqlens=("uniform", L + 8, 500), seed=233 + h_c + L)
    check(inp, num_parts=3, what=f"h_c={h_c} h_q={h_q} L={L}")


def test_narrow_peaky_softmax(cuda_device):
    inp = small(2, 256, L=1, seqlens=("uniform", 16, 2000), seed=239)
    inp.scale *= 8
    check(inp, num_parts=9)


def _gla_call(d, inp, out, lse, num_parts, ws, stream=None):
    from kv_cache_paged_b200 import binding
    return binding.gla_decode(d["q"], d["latent_cache"], d["rope_cache"], d["block_table"], d["seqlens"], inp.scale,
                              num_parts=num_parts, out=out, lse=lse, workspace=ws, stream=stream)


def _nan_outputs(inp):
    import torch
    out = torch.full((inp.B, inp.L, inp.h_q, inp.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((inp.B, inp.L, inp.h_q), float("nan"), dtype=torch.float32, device="cuda")
    return out, lse


@pytest.mark.parametrize("num_parts", [1, 3, 0])
def test_narrow_empty_sequences(cuda_device, num_parts):
    """Empty sequences have no tiles and no part visits them: the combine writes their rows
    (outputs start as NaN so that nothing passes by chance)."""
    import torch
    inp = small(2, 256, B=6, L=1, seqlens=[0, 70, 0, 5, 300, 0], seed=241)
    d = gu.to_dev(inp)
    out, lse = _nan_outputs(inp)
    _gla_call(d, inp, out, lse, num_parts, torch.zeros(1 << 24, dtype=torch.uint8, device="cuda"))
    o, l = gu.to_np(out, lse)
    assert np.all(o[[0, 2, 5]] == 0) and np.all(np.isneginf(l[[0, 2, 5]]))
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(o, l, ref_o, ref_l)


def test_narrow_all_sequences_empty(cuda_device):
    import torch
    inp = small(2, 256, B=3, L=1, seqlens=[0, 0, 0], seed=243)
    d = gu.to_dev(inp)
    out, lse = _nan_outputs(inp)
    _gla_call(d, inp, out, lse, 0, torch.zeros(1 << 24, dtype=torch.uint8, device="cuda"))
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_narrow_split_merge_ignores_stale_workspace(cuda_device):
    """Arbitrary bytes in the workspace (left by other calls, or never cleared) do not change the
    result of a split call: every partial the combine reads was written by this call.  Only the
    error word has to start at zero."""
    import torch
    inp = small(2, 256, B=7, L=1, seqlens=("uniform", 200, 3000), seed=245)
    d = gu.to_dev(inp)
    clean = torch.zeros(1 << 24, dtype=torch.uint8, device="cuda")
    ref_out, ref_lse = _nan_outputs(inp)
    _gla_call(d, inp, ref_out, ref_lse, 23, clean)
    dirty = torch.randint(0, 256, (1 << 24,), dtype=torch.uint8, device="cuda")
    dirty[:256] = 0
    for call in range(3):
        out, lse = _nan_outputs(inp)
        _gla_call(d, inp, out, lse, 23, dirty)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), f"call {call}"
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32)), f"call {call}"
    o, l = gu.to_np(ref_out, ref_lse)
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(o, l, ref_o, ref_l)


def test_narrow_graph_replay(cuda_device):
    """A captured split call (decode kernel, then the combine as its programmatic dependent)
    replays bit for bit."""
    import torch
    inp = small(2, 256, B=6, L=1, seqlens=("uniform", 100, 2500), seed=247)
    d = gu.to_dev(inp)
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device="cuda")
    out, lse = _nan_outputs(inp)
    _gla_call(d, inp, out, lse, 17, ws)   # eager run (also sets kernel attributes)
    torch.cuda.synchronize()
    ref_out, ref_lse = out.clone(), lse.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            _gla_call(d, inp, out, lse, 17, ws, stream=s)
    for replay in range(3):
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), f"replay {replay}"
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32)), f"replay {replay}"
    from kv_cache_paged_b200 import binding
    assert binding.read_device_error(ws) == 0


def test_narrow_page_permutation_bit_identical(cuda_device):
    import torch
    inp = small(2, 256, B=4, L=1, seqlens=("uniform", 1, 800), seed=251)
    out1, lse1 = gu.run_gpu(inp)
    perm = np.random.default_rng(3).permutation(inp.num_pages)
    inv = np.argsort(perm)
    for k in inp.caches:
        inp.caches[k] = np.ascontiguousarray(inp.caches[k][inv])
    bt = inp.block_table.copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    inp.block_table = bt
    out2, lse2 = gu.run_gpu(inp)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)


# ----------------------------------------------------------------------------- indexing
@pytest.mark.parametrize("h_c,d_c", [(1, 512), (2, 256)])
def test_latent_delta_attention_exact_index(cuda_device, h_c, d_c):
    inp, targets = make_delta_problem("gla", seed=23, B=4, h_q=32 * h_c, h_kv=h_c, d=d_c, d_r=64, S=64,
                                      seqlens=("uniform", 20, 900))
    out, lse = gu.run_gpu(inp, num_parts=5)
    assert np.array_equal(decode_digits(inp, gu.to_np(out, lse)[0]), targets)


def test_latent_page_permutation_bit_identical(cuda_device):
    import torch
    inp = small(2, 256, B=4, L=2, seqlens=("uniform", 2, 800), seed=29)
    out1, lse1 = gu.run_gpu(inp)
    perm = np.random.default_rng(0).permutation(inp.num_pages)
    inv = np.argsort(perm)
    for k in inp.caches:
        inp.caches[k] = np.ascontiguousarray(inp.caches[k][inv])
    bt = inp.block_table.copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    inp.block_table = bt
    out2, lse2 = gu.run_gpu(inp)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)


# ----------------------------------------------------------------------------- more than 64 rows per latent head
# GLA-2 from q_len 2 and GLA-8 from q_len 5 run on the 128-row kernel (64-token tiles, M = 128,
# two softmax warps per lane quadrant that exchange their row maxima every tile; one CTA per
# block of 128 rows).
@pytest.mark.parametrize("num_parts", [1, 3, 50, 148])
def test_m128_forced_splits(cuda_device, num_parts):
    inp = small(2, 256, B=5, L=2, seqlens=("uniform", 16, 1500), seed=311 + num_parts)
    check(inp, num_parts=num_parts, what=f"GLA-2 L=2 parts={num_parts}")


def test_m128_tile_boundaries(cuda_device):
    sl = [2, 3, 31, 32, 63, 64, 65, 127, 128, 129, 300]
    inp = small(2, 256, B=len(sl), L=2, seqlens=sl, seed=323)
    for parts in (0, 1, 4, 64):
        # stress bound: the two- and three-token sequences have rows that see one or two tokens
        check(inp, num_parts=parts, what=f"GLA-2 L=2 tile boundaries parts={parts}", stress=True)


@pytest.mark.parametrize("S", [1, 8, 16, 32, 48, 64, 128])
def test_m128_page_sizes(cuda_device, S):
    """Boxes of 16, 32 and 64 tokens (48: gcd 16), one box of the whole tile, and pages of 1 and 8
    tokens gathered token by token."""
    inp = small(2, 256, B=4, L=2, page_size=S, seqlens=("uniform", 30, 700), seed=329 + S)
    check(inp, num_parts=5, what=f"GLA-2 L=2 S={S}")


@pytest.mark.parametrize("h_c,h_q,L", [(8, 128, 5), (8, 128, 8), (4, 128, 3), (2, 128, 2)])
def test_m128_row_counts(cuda_device, h_c, h_q, L):
    """R = 80, 128, 96 and 128 rows: the last lane quadrants partly or wholly without rows."""
    inp = small(h_c, 256, h_q=h_q, L=L, seqlens=("uniform", L + 8, 500), seed=337 + h_c + L)
    check(inp, num_parts=3, what=f"h_c={h_c} h_q={h_q} L={L}")


@pytest.mark.parametrize("L,parts", [(3, 0), (4, 7), (6, 3)])
def test_m128_row_blocks(cuda_device, L, parts):
    """More than 128 rows per latent head: GLA-2 at q_len 3, 4 and 6 (192, 256 and 384 rows) runs
    one CTA per 128-row block, the last block partly without rows at q_len 3."""
    inp = small(2, 256, L=L, B=4, seqlens=("uniform", L + 16, 900), seed=359 + L)
    check(inp, num_parts=parts, what=f"GLA-2 L={L} parts={parts}")


def test_m128_peaky_softmax(cuda_device):
    inp = small(2, 256, L=2, seqlens=("uniform", 16, 2000), seed=347)
    inp.scale *= 8
    check(inp, num_parts=9)


def test_m128_empty_sequences(cuda_device):
    import torch
    inp = small(2, 256, B=6, L=2, seqlens=[0, 70, 0, 5, 300, 0], seed=349)
    d = gu.to_dev(inp)
    out, lse = _nan_outputs(inp)
    _gla_call(d, inp, out, lse, 3, torch.zeros(1 << 24, dtype=torch.uint8, device="cuda"))
    o, l = gu.to_np(out, lse)
    assert np.all(o[[0, 2, 5]] == 0) and np.all(np.isneginf(l[[0, 2, 5]]))
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(o, l, ref_o, ref_l)


def test_m128_page_permutation_bit_identical(cuda_device):
    import torch
    inp = small(2, 256, B=4, L=2, seqlens=("uniform", 2, 800), seed=353)
    out1, lse1 = gu.run_gpu(inp)
    perm = np.random.default_rng(5).permutation(inp.num_pages)
    inv = np.argsort(perm)
    for k in inp.caches:
        inp.caches[k] = np.ascontiguousarray(inp.caches[k][inv])
    bt = inp.block_table.copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    inp.block_table = bt
    out2, lse2 = gu.run_gpu(inp)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)


# ----------------------------------------------------------------------------- full workloads (sampled)
def check_full(inp, b_sample, what):
    """A sample of sequences (always including the longest) against the oracle, plus every
    sequence against a one-part run of the same kernel: a split or slot error on an unsampled
    sequence changes its result against the unsplit one."""
    import torch
    sel = sorted(set(int(b) for b in b_sample) | {int(np.argmax(inp.seqlens))})
    dev = gu.to_dev(inp)
    out, lse = gu.run_gpu(inp, dev=dev)
    o, l = gu.to_np(out, lse)
    ref_o, ref_l, _ = orc.decode_inputs(inp, b_list=np.asarray(sel, dtype=np.int32))
    gu.assert_close(o[sel], l[sel], ref_o, ref_l, what)
    out1, lse1 = gu.run_gpu(inp, dev=dev, num_parts=1)
    o1, l1 = gu.to_np(out1, lse1)
    # the split result and the unsplit one: both within the oracle bound of the exact result,
    # so within twice that of each other; every row and every sequence is compared
    assert np.isfinite(o).all() and np.array_equal(np.isfinite(l), np.isfinite(l1)), what
    assert np.abs(o - o1).max() <= 2 * gu.TOL_MAX_ABS, f"{what}: split vs unsplit {np.abs(o - o1).max():.3e}"
    fin = np.isfinite(l1)
    assert np.abs(l[fin] - l1[fin]).max() <= 2 * gu.TOL_LSE, what


@pytest.mark.parametrize("L", [1, 2])
def test_mla_workload_full_size(cuda_device, L):
    """B 64, h_q 128, one 512-dim latent head + 64 rope, contexts U[4096, 32768]; 6 sequences and
    the longest checked against the oracle, every sequence against the unsplit run."""
    check_full(wl.make_workload("mla", L=L), [0, 7, 19, 33, 48, 63], f"MLA workload L={L}")


@pytest.mark.parametrize("L", [1, 2, 4])
def test_gla2_workload_full_size(cuda_device, L):
    """B 128, h_q 128 over two 256-dim latent heads + 64 rope, lognormal contexts; 6 sequences and
    the longest checked against the oracle, every sequence against the unsplit run."""
    check_full(wl.make_workload("gla2", L=L), [0, 5, 40, 77, 127], f"GLA-2 workload L={L}")


@pytest.mark.parametrize("L", [1, 2, 3, 4, 8])
def test_gla8_speculation_lengths(cuda_device, L):
    """GLA-8 (16 query heads per latent head) at q_len 1..8: 16 L rows per latent head,
    spread over the lane quadrants when at most 64."""
    inp = small(8, 256, h_q=128, L=L, seqlens=("uniform", L, 400), seed=100 + L)
    check(inp, num_parts=5, what=f"GLA-8 L={L}")


@pytest.mark.parametrize("h_c,d_c", [(2, 256), (1, 512)])
@pytest.mark.parametrize("S", [64, 1])
def test_latent_more_segments_than_one_plan_chunk(cuda_device, h_c, d_c, S):
    """80 short sequences on one part: the CTA walks its plan in chunks of 32 segments."""
    inp = small(h_c, d_c, B=80, page_size=S, seqlens=("uniform", 1, 90), seed=130 + S + h_c)
    check(inp, num_parts=1, what=f"h_c={h_c} 80 sequences S={S}")
