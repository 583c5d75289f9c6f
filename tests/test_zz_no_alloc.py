"""kvd_gta_decode_noalloc: the GTA decode for callers that cannot allocate a workspace.

Serving engines that have handed all of HBM to KV pages and their own arenas, or
code running under global-mode stream capture (where cudaMalloc is illegal),
cannot pass us a workspace.  The entry point keeps the split-KV scratch in a
fixed device array inside the library instead.  This file is collected last so
that a run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

from kv_cache_paged_b200 import binding, workload as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _params(d, inp, out, lse, num_parts):
    return binding.GTAParams(d["q"].data_ptr(), d["tied_cache"].data_ptr(), d["rope_cache"].data_ptr(),
                             d["block_table"].data_ptr(), d["seqlens"].data_ptr(), out.data_ptr(), lse.data_ptr(),
                             inp.B, inp.L, inp.h_q, inp.h_kv, inp.d, inp.d_r, inp.page_size, inp.num_pages,
                             inp.max_pages, inp.scale, num_parts)


@pytest.mark.parametrize("num_parts", [0, 7])
def test_noalloc_matches_workspace_entry_on_two_calls(cuda_device, num_parts):
    import torch
    lib = binding.lib()
    lib.kvd_gta_decode_noalloc.restype = ctypes.c_int
    lib.kvd_gta_decode_noalloc.argtypes = [ctypes.POINTER(binding.GTAParams), ctypes.c_void_p]
    inp = wl.make_workload("gta")                        # B 32, contexts 1024..8192
    d = gu.to_dev(inp)
    ref_out, ref_lse = gu.run_gpu(inp, dev=d, num_parts=num_parts)
    ref_o, ref_l = gu.to_np(ref_out, ref_lse)
    stream = torch.cuda.current_stream()
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        p = _params(d, inp, out, lse, num_parts)
        st = lib.kvd_gta_decode_noalloc(ctypes.byref(p), ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, binding.STATUS.get(st, st)
        torch.cuda.synchronize()
        o, l = gu.to_np(out, lse)
        gu.assert_close(o, l, ref_o, ref_l, f"noalloc call {call}")


def test_noalloc_rejects_oversized_calls(cuda_device):
    """A call whose partials need more than the 8 MiB array launches nothing."""
    lib = binding.lib()
    lib.kvd_gta_decode_noalloc.restype = ctypes.c_int
    lib.kvd_gta_decode_noalloc.argtypes = [ctypes.POINTER(binding.GTAParams), ctypes.c_void_p]
    p = binding.GTAParams(256, 256, 256, 256, 256, 256, 256, 20000, 1, 32, 8, 128, 64, 64, 1000, 16,
                          0.1, 148)
    assert lib.kvd_gta_decode_noalloc(ctypes.byref(p), None) == -3
