"""Host-side checks of the cache-append path: the exact rounding used for its expected
values, the rotate-half RoPE of the oracle on the stored layout, and argument validation
of the C entry points (no GPU needed)."""
import ctypes

import numpy as np
import pytest

from kv_cache_paged_b200 import binding
from oracle import oracle as orc
from tests.rounding import bf16_bits_to_f64, f64_to_bf16_bits


def test_f64_to_bf16_single_rounding():
    one = 1.0
    assert f64_to_bf16_bits(one) == 0x3F80
    assert f64_to_bf16_bits(one + 2.0**-8) == 0x3F80            # tie -> even mantissa (1.0)
    assert f64_to_bf16_bits(one + 3 * 2.0**-8) == 0x3F82        # tie between 0x3F81 and 0x3F82 -> even
    assert f64_to_bf16_bits(one + 2.0**-8 + 2.0**-40) == 0x3F81  # just above the tie
    assert f64_to_bf16_bits(-one - 2.0**-8 - 2.0**-40) == 0xBF81
    assert f64_to_bf16_bits(0.0) == 0 and f64_to_bf16_bits(-2.0) == 0xC000
    # a case where rounding through fp32 first would be wrong: fp32 rounds 1 + 2^-8 + 2^-30
    # down to the tie 1 + 2^-8, which then goes to even (1.0); the exact result is 0x3F81
    assert f64_to_bf16_bits(one + 2.0**-8 + 2.0**-30) == 0x3F81


def test_f64_to_bf16_is_nearest():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(20000) * 4
    h = f64_to_bf16_bits(x)
    v = bf16_bits_to_f64(h)
    up = bf16_bits_to_f64(h + np.uint16(1))
    dn = bf16_bits_to_f64(h - np.uint16(1))
    assert np.all(np.abs(v - x) <= np.abs(up - x)) and np.all(np.abs(v - x) <= np.abs(dn - x))


def test_oracle_rope_pairs_rotate_half():
    """The stored convention: pair (j, j + d_r/2) rotated by pos * 10000^(-2j/d_r)."""
    d_r = 8
    x = np.zeros(d_r)
    x[1] = 1.0
    y = orc.rope(x, 3.0)
    th = 10000.0 ** (-2.0 * 1 / d_r)
    assert np.isclose(y[1], np.cos(3 * th)) and np.isclose(y[1 + d_r // 2], np.sin(3 * th))
    assert np.count_nonzero(np.abs(y) > 1e-15) == 2


def _gta_params(**kw):
    base = dict(tied_new=256, rope_new=256, tied_cache=256, rope_cache=256, positions=256, slot_mapping=256,
                error_word=None, N=4, h_kv=8, d_h=128, d_r=64, num_rows=64, rope_base=10000.0)
    base.update(kw)
    return binding.GTAAppendParams(**base)


@pytest.mark.parametrize("kw", [dict(tied_new=None), dict(rope_cache=8), dict(positions=None), dict(slot_mapping=2),
                                dict(N=-1), dict(d_h=100), dict(d_r=0), dict(d_r=30), dict(num_rows=0),
                                dict(rope_base=0.0), dict(rope_base=float("inf"))])
def test_gta_append_validation(kw):
    L = binding.lib()
    assert L.kvd_gta_append(ctypes.byref(_gta_params(**kw)), None) == -1


def test_append_zero_tokens_is_a_no_op():
    L = binding.lib()
    assert L.kvd_gta_append(ctypes.byref(_gta_params(N=0)), None) == 0


def test_gqa_gla_append_and_rope_q_validation():
    L = binding.lib()
    p = binding.GQAAppendParams(256, 256, 256, 256, 256, 256, None, 4, 8, 128, 130, 64, 10000.0)  # d_r > d
    assert L.kvd_gqa_append(ctypes.byref(p), None) == -1
    p = binding.GLAAppendParams(256, 256, 256, 256, 256, 256, None, 4, 1, 512, 63, 64, 10000.0)   # odd d_r
    assert L.kvd_gla_append(ctypes.byref(p), None) == -1
    assert L.kvd_rope_q(ctypes.c_void_p(256), ctypes.c_void_p(256), 2, 1, 8, 128, 100, 64, 10000.0, None) == -1
    assert L.kvd_rope_q(ctypes.c_void_p(8), ctypes.c_void_p(256), 2, 1, 8, 128, 64, 64, 10000.0, None) == -1
    assert L.kvd_rope_q(ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 1, 8, 128, 64, 64, 10000.0, None) == 0
