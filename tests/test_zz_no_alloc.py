"""kvd_gta_decode_noalloc: the GTA decode for callers that cannot allocate a workspace.

Serving engines that have handed all of HBM to KV pages and their own arenas, or
code running under global-mode stream capture (where cudaMalloc is illegal),
cannot pass us a workspace.  The entry point keeps the split-KV scratch in a
fixed device array inside the library instead.  It runs the same kernels on the
same plan as kvd_gta_decode, so the two must agree bit for bit.  This file is
collected last so that a run stopping at the first failure has already run every
other test.
"""
import ctypes

import numpy as np
import pytest

from kv_cache_paged_b200 import binding, workload as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _lib():
    lib = binding.lib()
    lib.kvd_gta_decode_noalloc.restype = ctypes.c_int
    lib.kvd_gta_decode_noalloc.argtypes = [ctypes.POINTER(binding.GTAParams), ctypes.c_void_p]
    return lib


def _params(d, inp, out, lse, num_parts):
    return binding.GTAParams(d["q"].data_ptr(), d["tied_cache"].data_ptr(), d["rope_cache"].data_ptr(),
                             d["block_table"].data_ptr(), d["seqlens"].data_ptr(), out.data_ptr(), lse.data_ptr(),
                             inp.B, inp.L, inp.h_q, inp.h_kv, inp.d, inp.d_r, inp.page_size, inp.num_pages,
                             inp.max_pages, inp.scale, num_parts)


def _noalloc(lib, d, inp, like_out, like_lse, num_parts):
    import torch
    out = torch.full_like(like_out, float("nan"))
    lse = torch.full_like(like_lse, float("nan"))
    p = _params(d, inp, out, lse, num_parts)
    st = lib.kvd_gta_decode_noalloc(ctypes.byref(p), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, binding.STATUS.get(st, st)
    torch.cuda.synchronize()
    return out, lse


def _assert_same_bits(out, lse, ref_out, ref_lse, what):
    import torch
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), f"{what}: out bits differ"
    assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32)), f"{what}: lse bits differ"


@pytest.mark.parametrize("num_parts", [0, 7])
def test_noalloc_matches_workspace_entry_on_two_calls(cuda_device, num_parts):
    """Two calls in a row give exactly the workspace entry's result (and so the oracle's)."""
    lib = _lib()
    inp = wl.make_workload("gta")                        # B 32, contexts 1024..8192
    d = gu.to_dev(inp)
    ref_out, ref_lse = gu.run_gpu(inp, dev=d, num_parts=num_parts)
    ref_o, ref_l = gu.to_np(ref_out, ref_lse)
    from oracle import oracle as orc
    or_o, or_l, _ = orc.decode_inputs(inp)
    gu.assert_close(ref_o, ref_l, or_o, or_l, "workspace entry vs oracle")
    for call in range(2):
        out, lse = _noalloc(lib, d, inp, ref_out, ref_lse, num_parts)
        _assert_same_bits(out, lse, ref_out, ref_lse, f"noalloc call {call}")


def test_noalloc_after_a_larger_call_leaves_no_trace(cuda_device):
    """Partials left in the shared array by a larger call (more sequences, more parts) do not
    leak into a following smaller call, and vice versa."""
    lib = _lib()
    big = wl.make_inputs("gta", B=24, L=2, h_q=32, h_kv=8, d=128, d_r=64, page_size=64,
                         seqlens=("uniform", 2, 3000), seed=41)
    small = wl.make_inputs("gta", B=5, L=1, h_q=32, h_kv=8, d=128, d_r=64, page_size=16,
                           seqlens=("uniform", 1, 900), seed=42)
    cases = [(big, 148), (small, 3), (big, 37), (small, 0)]
    devs = {id(big): gu.to_dev(big), id(small): gu.to_dev(small)}
    for i, (inp, parts) in enumerate(cases):
        d = devs[id(inp)]
        ref_out, ref_lse = gu.run_gpu(inp, dev=d, num_parts=parts)
        out, lse = _noalloc(lib, d, inp, ref_out, ref_lse, parts)
        _assert_same_bits(out, lse, ref_out, ref_lse, f"call {i} (B {inp.B}, parts {parts})")


def test_noalloc_rejects_oversized_calls(cuda_device):
    """A call whose partials need more than the 8 MiB array launches nothing."""
    lib = _lib()
    p = binding.GTAParams(256, 256, 256, 256, 256, 256, 256, 20000, 1, 32, 8, 128, 64, 64, 1000, 16,
                          0.1, 148)
    assert lib.kvd_gta_decode_noalloc(ctypes.byref(p), None) == -3
