"""GQA / GTA decode on the GPU against the fp64 oracle (the stated output tolerance), plus
bit-exact indexing, split invariance and device error reporting."""
import numpy as np
import pytest

from kv_cache_paged_b200 import workload as wl
from oracle import oracle as orc
from tests import gpu_util as gu
from tests.indexing import decode_digits, make_delta_problem

pytestmark = pytest.mark.gpu


def check(inp, num_parts=0, dev=None, what="", stress=False):
    """Against the oracle with the flat bound (stress: see gpu_util.assert_close)."""
    out, lse = gu.run_gpu(inp, dev=dev, num_parts=num_parts)
    o, l = gu.to_np(out, lse)
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    return gu.assert_close(o, l, ref_o, ref_l, what or inp.name, stress=stress)


def small(variant, **kw):
    base = dict(B=4, L=1, h_q=32, h_kv=8, d=128, d_r=64, page_size=64, seqlens=("uniform", 1, 700), seed=5)
    base.update(kw)
    if variant == "gqa":
        base["d_r"] = 0
    return wl.make_inputs(variant, **base)


# ----------------------------------------------------------------------------- workloads
def test_gta_tiny_workload(cuda_device):
    check(wl.make_workload("gta_tiny"))


def test_gta_workload_full_size(cuda_device):
    """B 32, h_q 32, 8 tied groups, d_h 128, rope 64, contexts U[1024, 8192], page 64."""
    check(wl.make_workload("gta"))


def test_gqa_workload_full_size(cuda_device):
    """B 32, h_q 32, h_kv 8, d 128, context 8192, page 64."""
    check(wl.make_workload("gqa"))


# ----------------------------------------------------------------------------- shapes and edges
@pytest.mark.parametrize("variant", ["gqa", "gta"])
@pytest.mark.parametrize("L", [1, 2, 3])
@pytest.mark.parametrize("num_parts", [0, 1, 5, 300])
def test_ragged_contexts_q_len_and_splits(cuda_device, variant, L, num_parts):
    inp = small(variant, L=L, seqlens=("uniform", L, 700), seed=10 * L + num_parts)
    check(inp, num_parts=num_parts)


@pytest.mark.parametrize("variant", ["gqa", "gta"])
def test_page_boundaries_and_single_token(cuda_device, variant):
    sl = [1, 15, 16, 17, 63, 64, 65, 127, 128, 129, 2]
    inp = small(variant, B=len(sl), seqlens=sl, seed=3)
    for parts in (0, 1, 4, 64):
        check(inp, num_parts=parts, what=f"{variant} parts={parts}")


@pytest.mark.parametrize("variant", ["gqa", "gta"])
def test_empty_sequences_give_zero_and_minus_inf(cuda_device, variant):
    inp = small(variant, B=5, seqlens=[0, 40, 0, 1, 0], seed=4)
    for parts in (0, 2, 9):
        out, lse = gu.run_gpu(inp, num_parts=parts)
        o, l = gu.to_np(out, lse)
        assert np.all(o[[0, 2, 4]] == 0) and np.all(np.isneginf(l[[0, 2, 4]]))
        ref_o, ref_l, _ = orc.decode_inputs(inp)
        gu.assert_close(o, l, ref_o, ref_l)


@pytest.mark.parametrize("h_q,h_kv,L", [(8, 1, 1), (32, 4, 2), (32, 4, 4), (16, 16, 1), (64, 16, 2), (32, 2, 1)])
def test_group_shapes(cuda_device, h_q, h_kv, L):
    for variant in ("gqa", "gta"):
        inp = small(variant, h_q=h_q, h_kv=h_kv, L=L, seqlens=("uniform", L, 400), seed=h_q + h_kv + L)
        check(inp, what=f"{variant} h_q={h_q} h_kv={h_kv} L={L}")


@pytest.mark.parametrize("d,d_r", [(64, 32), (128, 32), (64, 64)])
def test_gta_head_dims(cuda_device, d, d_r):
    check(small("gta", d=d, d_r=d_r, page_size=16, seqlens=("uniform", 1, 300), seed=d + d_r))


def test_gqa_head_dim_64(cuda_device):
    check(small("gqa", d=64, page_size=32, seed=8))


def test_peaky_softmax(cuda_device):
    """Scale x8 makes the softmax nearly one-hot (stresses max tracking and rescaling)."""
    inp = small("gta", seed=12)
    inp.scale *= 8
    check(inp, num_parts=7)


def test_identity_block_table(cuda_device):
    check(small("gqa", shuffle=False, seed=13))


# ----------------------------------------------------------------------------- bit-exact indexing
@pytest.mark.parametrize("variant", ["gqa", "gta"])
@pytest.mark.parametrize("num_parts", [0, 3])
def test_delta_attention_returns_exact_token_index(cuda_device, variant, num_parts):
    inp, targets = make_delta_problem(variant, seed=17, B=6, h_q=8, h_kv=2, d=64, d_r=32, S=16,
                                      seqlens=("uniform", 20, 700))
    out, lse = gu.run_gpu(inp, num_parts=num_parts)
    got = decode_digits(inp, gu.to_np(out, lse)[0])
    assert np.array_equal(got, targets)


@pytest.mark.parametrize("variant", ["gqa", "gta"])
def test_page_permutation_is_bit_identical(cuda_device, variant):
    """Moving physical pages and rewriting block_table accordingly changes no output bit."""
    inp = small(variant, seed=21)
    out1, lse1 = gu.run_gpu(inp)
    rng = np.random.default_rng(0)
    perm = rng.permutation(inp.num_pages)            # new location of physical page p
    inv = np.argsort(perm)
    for k in inp.caches:
        inp.caches[k] = np.ascontiguousarray(inp.caches[k][inv])
    bt = inp.block_table.copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    inp.block_table = bt
    out2, lse2 = gu.run_gpu(inp)
    import torch
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)


def test_nan_poison_never_reaches_output(cuda_device):
    """Tails and the spare page hold NaN; every test already asserts finiteness, this one uses
    lengths that end one token into a page so the tail tile is almost all poison."""
    inp = small("gta", B=6, seqlens=[65, 129, 193, 1, 17, 81], seed=22)
    check(inp)


def test_output_guard_bands_untouched(cuda_device):
    import torch
    from kv_cache_paged_b200 import binding
    inp = small("gta", seed=23)
    d = gu.to_dev(inp)
    B, L, H, D = inp.B, inp.L, inp.h_q, inp.d
    guard = 1024
    big = torch.full((B * L * H * D + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbig = torch.full((B * L * H + 2 * guard,), 7.0, dtype=torch.float32, device="cuda")
    out = big[guard:guard + B * L * H * D].view(B, L, H, D)
    lse = lbig[guard:guard + B * L * H].view(B, L, H)
    binding.gta_decode(d["q"], d["tied_cache"], d["rope_cache"], d["block_table"], d["seqlens"], inp.scale,
                       out=out, lse=lse, num_parts=11)
    torch.cuda.synchronize()
    assert torch.all(big[:guard] == 7) and torch.all(big[-guard:] == 7)
    assert torch.all(lbig[:guard] == 7) and torch.all(lbig[-guard:] == 7)


# ----------------------------------------------------------------------------- plan and errors
def test_device_plan_equals_host_plan(cuda_device):
    import torch
    from kv_cache_paged_b200 import binding
    rng = np.random.default_rng(1)
    sl = rng.integers(0, 3000, size=77).astype(np.int32)
    sl[::7] = 0
    for parts, seg_cost in ((1, 0), (13, 0), (148, 0), (500, 0), (13, 3), (148, 3), (74, 11)):
        hs, hc = binding.plan_host(sl, 16, 1 << 20, parts, cap=96, seg_cost=seg_cost)
        ds, dc = binding.plan_device(torch.from_numpy(sl).cuda(), 16, 1 << 20, parts, cap=96, seg_cost=seg_cost)
        dc = dc.cpu().numpy()
        ds = ds.cpu().numpy()
        assert np.array_equal(hc, dc)
        for c in range(parts):
            n = min(hc[c], 96)
            assert np.array_equal(hs[c, :n], ds[c, :n])


def test_bad_page_is_flagged_not_faulted(cuda_device):
    import torch
    from kv_cache_paged_b200 import binding
    inp = small("gta", seed=30)
    inp.block_table[1, 0] = inp.num_pages + 1000
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device="cuda")
    gu.run_gpu(inp, workspace=ws)
    flags = binding.read_device_error(ws)
    assert flags & binding.DEVERR_BAD_PAGE
    assert binding.read_device_error(ws) == 0      # reading clears it


def test_bad_seqlen_is_flagged_and_clamped(cuda_device):
    import torch
    from kv_cache_paged_b200 import binding
    inp = small("gqa", seed=31)
    inp.seqlens[2] = inp.block_table.shape[1] * inp.page_size + 100
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device="cuda")
    gu.run_gpu(inp, workspace=ws)
    assert binding.read_device_error(ws) & binding.DEVERR_BAD_SEQLEN


def test_clean_run_sets_no_flag(cuda_device):
    import torch
    from kv_cache_paged_b200 import binding
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device="cuda")
    gu.run_gpu(small("gta", seed=32), workspace=ws)
    assert binding.read_device_error(ws) == 0


def test_cuda_graph_capture_and_replay(cuda_device):
    import torch
    from kv_cache_paged_b200 import binding
    inp = small("gta", seed=33)
    d = gu.to_dev(inp)
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device="cuda")
    out = torch.empty((inp.B, inp.L, inp.h_q, inp.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((inp.B, inp.L, inp.h_q), dtype=torch.float32, device="cuda")
    args = (d["q"], d["tied_cache"], d["rope_cache"], d["block_table"], d["seqlens"], inp.scale)
    binding.gta_decode(*args, out=out, lse=lse, workspace=ws)   # warm (sets kernel attributes)
    torch.cuda.synchronize()
    ref = out.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            binding.gta_decode(*args, out=out, lse=lse, workspace=ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("variant", ["gqa", "gta"])
@pytest.mark.parametrize("L", [4, 8])
def test_longer_speculation(cuda_device, variant, L):
    """q_len up to 8 (32 query rows per KV group): the warp-MMA kernel's largest row block."""
    inp = small(variant, L=L, seqlens=("uniform", L, 600), seed=110 + L)
    check(inp, num_parts=7)


@pytest.mark.parametrize("variant", ["gqa", "gta"])
@pytest.mark.parametrize("S", [64, 1])
def test_more_segments_than_one_plan_chunk(cuda_device, variant, S):
    """300 short sequences on 2 parts: each CTA walks its plan in chunks of 128 segments."""
    inp = small(variant, B=300, page_size=S, seqlens=("uniform", 1, 40), seed=120 + S)
    check(inp, num_parts=2, what=f"{variant} 300 sequences S={S}")
