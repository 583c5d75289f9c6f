"""Shared-prefix decode (a prefix stored once and named by every sequence's block table) and
cascade decoding (prefix and continuation decoded separately, then merged by
kvd_merge_states), against the fp64 oracle."""
import numpy as np
import pytest

from kv_cache_paged_b200 import binding, workload as wl
from oracle import oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def prefix_inputs(variant, *, B=6, prefix=256, S=64, L=1, seed=61, **kw):
    base = dict(B=B, L=L, h_q=32, h_kv=8, d=128, d_r=64, page_size=S, seqlens=("uniform", max(L, 1), 300),
                seed=seed, shared_prefix=prefix)
    if variant == "gqa":
        base["d_r"] = 0
    if variant == "gla":
        base.update(h_q=128, h_kv=2, d=256, d_r=64, scale=0.07)
    base.update(kw)
    return wl.make_inputs(variant, **base)


@pytest.mark.parametrize("variant", ["gta", "gqa", "gla"])
@pytest.mark.parametrize("num_parts", [0, 5])
def test_shared_prefix_block_tables(cuda_device, variant, num_parts):
    inp = prefix_inputs(variant)
    assert (inp.block_table[:, :4] == inp.block_table[0, :4]).all()   # the prefix pages are shared
    out, lse = gu.run_gpu(inp, num_parts=num_parts)
    o, l = gu.to_np(out, lse)
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(o, l, ref_o, ref_l, f"{variant} shared prefix")


def _sub(inp, table, seqlens):
    import copy
    s = copy.copy(inp)
    s.block_table = np.ascontiguousarray(table)
    s.seqlens = np.asarray(seqlens, np.int32)
    return s


@pytest.mark.parametrize("variant", ["gta", "gqa"])
def test_cascade_prefix_then_continuation(cuda_device, variant):
    """q_len 1: decode the prefix alone (every block table = the prefix pages, T = prefix), the
    continuation alone (own pages, T = T_b - prefix), merge; equals the one-pass decode."""
    import torch
    P = 256
    inp = prefix_inputs(variant, prefix=P)
    pp = P // inp.page_size
    dev = gu.to_dev(inp)
    pre = _sub(inp, inp.block_table[:, :pp], np.full(inp.B, P))
    suf_table = np.full_like(inp.block_table, -1)
    suf_table[:, : inp.max_pages - pp] = inp.block_table[:, pp:]
    suf = _sub(inp, suf_table, inp.seqlens - P)
    d_pre = dict(dev, block_table=torch.from_numpy(pre.block_table).cuda(), seqlens=torch.from_numpy(pre.seqlens).cuda())
    d_suf = dict(dev, block_table=torch.from_numpy(suf.block_table).cuda(), seqlens=torch.from_numpy(suf.seqlens).cuda())
    o1, l1 = gu.run_gpu(pre, dev=d_pre)
    o2, l2 = gu.run_gpu(suf, dev=d_suf, num_parts=3)
    o, l = binding.merge_states(o1, l1, o2, l2)
    torch.cuda.synchronize()
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(*gu.to_np(o, l), ref_o, ref_l, f"{variant} cascade")


def test_merge_states_matches_oracle_combine(cuda_device):
    import torch
    rng = np.random.default_rng(3)
    rows, d_v = 300, 256
    oa = wl.f32_to_bf16_bits(rng.standard_normal((rows, d_v)).astype(np.float32))
    ob = wl.f32_to_bf16_bits(rng.standard_normal((rows, d_v)).astype(np.float32))
    la = rng.normal(0, 3, rows).astype(np.float32)
    lb = rng.normal(0, 3, rows).astype(np.float32)
    la[:5] = -np.inf                      # empty first state
    lb[3:8] = -np.inf                     # empty second state (rows 3, 4: both empty)
    lb[10] = la[10] + 80.0                # one state dominates completely
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    o, l = binding.merge_states(bf(oa), torch.from_numpy(la).cuda(), bf(ob), torch.from_numpy(lb).cuda())
    torch.cuda.synchronize()
    po = np.stack([wl.bf16_bits_to_f32(oa), wl.bf16_bits_to_f32(ob)]).astype(np.float64)
    pl = np.stack([la, lb]).astype(np.float64)
    ref_o, ref_l = orc.combine(po, pl)
    got_o, got_l = o.float().cpu().numpy().astype(np.float64), l.cpu().numpy().astype(np.float64)
    assert np.all(got_o[3:5] == 0) and np.all(np.isneginf(got_l[3:5]))
    ok = np.isfinite(ref_l)
    assert np.abs(got_o - ref_o)[ok].max() <= 2.0 ** -8 * np.abs(ref_o)[ok].max() + 1e-6
    assert np.abs(got_l[ok] - ref_l[ok]).max() <= 1e-5 * max(1.0, np.abs(ref_l[ok]).max())
    # in place
    oa_t, la_t = bf(oa), torch.from_numpy(la).cuda()
    binding.merge_states(oa_t, la_t, bf(ob), torch.from_numpy(lb).cuda(), out=oa_t, lse=la_t)
    torch.cuda.synchronize()
    assert torch.equal(oa_t.view(torch.int16), o.view(torch.int16)) and torch.equal(la_t, l)


def test_gta_prefix_workload(cuda_device):
    """B 32, a 4096-token shared prefix, continuations U[64, 2048]."""
    inp = wl.make_workload("gta_prefix")
    out, lse = gu.run_gpu(inp)
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(*gu.to_np(out, lse), ref_o, ref_l, "gta_prefix")


def _prefix_only_ref(inp, P):
    """Oracle state of every query row over the prefix alone (no causal mask): each (b, i) row
    becomes a one-row sequence whose block table is the prefix's pages and whose length is P."""
    import copy
    pp = P // inp.page_size
    s = copy.copy(inp)
    s.B, s.L = inp.B * inp.L, 1
    s.q = np.ascontiguousarray(inp.q.reshape(inp.B * inp.L, 1, inp.h_q, -1))
    s.block_table = np.ascontiguousarray(np.repeat(inp.block_table[:1, :pp], s.B, axis=0))
    s.seqlens = np.full(s.B, P, np.int32)
    ref_o, ref_l, _ = orc.decode_inputs(s)
    return ref_o.reshape(inp.B, inp.L, inp.h_q, -1), ref_l.reshape(inp.B, inp.L, inp.h_q)


def _prefix_gpu(inp, dev, P, num_parts=0):
    import torch
    pp = P // inp.page_size if P % inp.page_size == 0 else (P + inp.page_size - 1) // inp.page_size
    bt = torch.from_numpy(np.ascontiguousarray(inp.block_table[:1, :pp])).cuda()
    pl = torch.tensor([P], dtype=torch.int32, device="cuda")
    return binding.gta_prefix_decode(dev["q"], dev["tied_cache"], dev["rope_cache"], bt, pl, inp.scale,
                                     num_parts=num_parts)


@pytest.mark.parametrize("L,num_parts", [(1, 0), (1, 5), (2, 0), (3, 2)])
def test_batched_prefix_decode(cuda_device, L, num_parts):
    P = 256
    inp = prefix_inputs("gta", B=8, prefix=P, L=L, seed=70 + L)
    out, lse = _prefix_gpu(inp, gu.to_dev(inp), P, num_parts)
    ref_o, ref_l = _prefix_only_ref(inp, P)
    gu.assert_close(*gu.to_np(out, lse), ref_o, ref_l, f"prefix-only L={L}")


@pytest.mark.parametrize("S,P", [(1, 77), (16, 96), (64, 64)])
def test_batched_prefix_decode_page_sizes(cuda_device, S, P):
    inp = prefix_inputs("gta", B=6, prefix=P, S=S, seed=80 + S)
    out, lse = _prefix_gpu(inp, gu.to_dev(inp), P)
    ref_o, ref_l = _prefix_only_ref(inp, P)
    gu.assert_close(*gu.to_np(out, lse), ref_o, ref_l, f"prefix-only S={S}")


def test_cascade_batched_prefix_then_continuation(cuda_device):
    import torch
    P = 320
    inp = prefix_inputs("gta", B=16, prefix=P, seed=90)
    pp = P // inp.page_size
    dev = gu.to_dev(inp)
    o1, l1 = _prefix_gpu(inp, dev, P)
    suf_table = np.full_like(inp.block_table, -1)
    suf_table[:, : inp.max_pages - pp] = inp.block_table[:, pp:]
    suf = _sub(inp, suf_table, inp.seqlens - P)
    d_suf = dict(dev, block_table=torch.from_numpy(suf.block_table).cuda(), seqlens=torch.from_numpy(suf.seqlens).cuda())
    o2, l2 = gu.run_gpu(suf, dev=d_suf)
    o, l = binding.merge_states(o1, l1, o2, l2)
    torch.cuda.synchronize()
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(*gu.to_np(o, l), ref_o, ref_l, "batched prefix cascade")


def test_gta_prefix_workload_cascade(cuda_device):
    """The shared-prefix workload through the batched prefix path + continuation + merge."""
    import torch
    inp = wl.make_workload("gta_prefix")
    P = inp.shared_prefix
    pp = P // inp.page_size
    dev = gu.to_dev(inp)
    o1, l1 = _prefix_gpu(inp, dev, P)
    suf_table = np.full_like(inp.block_table, -1)
    suf_table[:, : inp.max_pages - pp] = inp.block_table[:, pp:]
    suf = _sub(inp, suf_table, inp.seqlens - P)
    d_suf = dict(dev, block_table=torch.from_numpy(suf.block_table).cuda(), seqlens=torch.from_numpy(suf.seqlens).cuda())
    o2, l2 = gu.run_gpu(suf, dev=d_suf)
    o, l = binding.merge_states(o1, l1, o2, l2)
    torch.cuda.synchronize()
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(*gu.to_np(o, l), ref_o, ref_l, "gta_prefix cascade")


def test_batched_prefix_more_than_128_rows(cuda_device):
    """48 sequences x 4 heads per KV group = 192 rows: two 128-row blocks per group."""
    P = 128
    inp = prefix_inputs("gta", B=48, prefix=P, seed=95)
    out, lse = _prefix_gpu(inp, gu.to_dev(inp), P)
    ref_o, ref_l = _prefix_only_ref(inp, P)
    gu.assert_close(*gu.to_np(out, lse), ref_o, ref_l, "prefix-only 192 rows")


def test_batched_prefix_empty_prefix(cuda_device):
    import torch
    inp = prefix_inputs("gta", B=4, prefix=64, seed=96)
    dev = gu.to_dev(inp)
    bt = torch.from_numpy(np.ascontiguousarray(inp.block_table[:1, :1])).cuda()
    out, lse = binding.gta_prefix_decode(dev["q"], dev["tied_cache"], dev["rope_cache"], bt,
                                         torch.zeros(1, dtype=torch.int32, device="cuda"), inp.scale)
    torch.cuda.synchronize()
    o, l = gu.to_np(out, lse)
    assert np.all(o == 0) and np.all(np.isneginf(l))
