"""The Python binding refuses host tensors: there is no CPU path to fall back to (host logic
only; no GPU needed)."""
import pytest

torch = pytest.importorskip("torch")

from kv_cache_paged_b200 import binding  # noqa: E402


def _bf(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def _paging(B=2, pages=4):
    return torch.zeros(B, pages, dtype=torch.int32), torch.full((B,), 3, dtype=torch.int32)


def test_gta_decode_rejects_host_tensors():
    bt, sl = _paging()
    with pytest.raises(TypeError, match="CUDA"):
        binding.gta_decode(_bf(2, 1, 8, 64), _bf(8, 16, 2, 64), _bf(8, 16, 32), bt, sl, 0.125)


def test_gqa_decode_rejects_host_tensors():
    bt, sl = _paging()
    with pytest.raises(TypeError, match="CUDA"):
        binding.gqa_decode(_bf(2, 1, 8, 64), _bf(8, 16, 2, 64), _bf(8, 16, 2, 64), bt, sl, 0.125)


def test_gla_decode_rejects_host_tensors():
    bt, sl = _paging()
    with pytest.raises(TypeError, match="CUDA"):
        binding.gla_decode(_bf(2, 1, 128, 320), _bf(8, 64, 2, 256), _bf(8, 64, 64), bt, sl, 0.07)


def test_gta_append_rejects_host_tensors():
    with pytest.raises(TypeError, match="CUDA"):
        binding.gta_append(_bf(4, 2, 64), _bf(4, 32), torch.zeros(4, dtype=torch.int32),
                           torch.zeros(4, dtype=torch.int32), _bf(8, 16, 2, 64), _bf(8, 16, 32))


def test_merge_states_rejects_host_tensors():
    out, lse = _bf(2, 4, 64), torch.zeros(2, 4)
    with pytest.raises(TypeError, match="CUDA"):
        binding.merge_states(out, lse, out, lse)
