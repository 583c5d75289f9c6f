"""Failure detection without a GPU fault: a pipeline wait that nothing satisfies runs out,
the kernel reports KVD_DEVERR_TIMEOUT through the workspace's error word and returns, and
the context stays usable.  The missing copy is a test knob of the library (the first tile's
TMA is never issued while its barrier still expects the bytes); the wait limit is lowered to
50 ms so the test is quick."""
import numpy as np
import pytest

from kv_cache_paged_b200 import binding, workload as wl
from oracle import oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture
def short_waits():
    binding.debug_set(binding.DEBUG_WAIT_LIMIT_NS, 50_000_000)
    yield
    binding.debug_set(binding.DEBUG_SKIP_FIRST_LOAD, 0)
    binding.debug_set(binding.DEBUG_WAIT_LIMIT_NS, 2_000_000_000)


CASES = {
    "gta": dict(variant="gta", B=3, L=1, h_q=32, h_kv=8, d=128, d_r=64, page_size=64, seqlens=[300, 70, 500]),
    "gla2": dict(variant="gla", B=2, L=2, h_q=128, h_kv=2, d=256, d_r=64, page_size=64, seqlens=[200, 90],
                 scale=0.07),
    "gla2_q1": dict(variant="gla", B=2, L=1, h_q=128, h_kv=2, d=256, d_r=64, page_size=64, seqlens=[300, 90],
                    scale=0.07),
    "gla2_q4": dict(variant="gla", B=2, L=4, h_q=128, h_kv=2, d=256, d_r=64, page_size=64, seqlens=[300, 90],
                    scale=0.07),
    "mla": dict(variant="gla", B=2, L=1, h_q=128, h_kv=1, d=512, d_r=64, page_size=64, seqlens=[200, 90],
                scale=0.07, latent_scale=0.1),
}


@pytest.mark.parametrize("name", list(CASES))
def test_missing_copy_times_out_and_context_survives(cuda_device, short_waits, name):
    import torch
    inp = wl.make_inputs(seed=5, **CASES[name])
    ws = torch.zeros(1 << 26, dtype=torch.uint8, device="cuda")
    binding.debug_set(binding.DEBUG_SKIP_FIRST_LOAD, 1)
    gu.run_gpu(inp, workspace=ws, num_parts=4)
    flags = binding.read_device_error(ws)          # synchronises: the kernel has returned
    assert flags & binding.DEVERR_TIMEOUT
    binding.debug_set(binding.DEBUG_SKIP_FIRST_LOAD, 0)
    ws.zero_()
    out, lse = gu.run_gpu(inp, workspace=ws, num_parts=4)
    assert binding.read_device_error(ws) == 0
    o, l = gu.to_np(out, lse)
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    gu.assert_close(o, l, ref_o, ref_l, f"{name} after a timed-out call")
