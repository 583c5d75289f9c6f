"""Byte and FLOP accounting against the paper's layout and intensity statements."""
import numpy as np
import pytest

from kv_cache_paged_b200 import accounting as acc


def test_gta_cache_is_roughly_half_of_gqa():
    """GTA keeps one tied state per group plus one shared rope slice: about half of GQA's
    separate K and V (abstract; section 3.3.1)."""
    gta = acc.kv_elems_per_token("gta", 8, 128, 64)
    gqa = acc.kv_elems_per_token("gqa", 8, 128, 0)
    assert gta == 8 * 128 + 64 and gqa == 2 * 8 * 128
    assert abs(gta / gqa - 0.53125) < 1e-12


def test_gla2_cache_equals_mla():
    """GLA-2 with d_c = 2 d_h keeps the unsharded cache of MLA (4 d_h latent + rope)."""
    assert acc.kv_elems_per_token("gla", 2, 256, 64) == acc.kv_elems_per_token("gla", 1, 512, 64) == 576


@pytest.mark.parametrize("variant,h_q,h_kv,d,d_r,expect", [
    ("gqa", 32, 8, 128, 0, 4.0),          # 2 g_q / m_kv = 2 * 4 / 2
    ("gqa", 32, 32, 128, 0, 1.0),         # MHA: ~1 FLOP per byte
    ("gta", 32, 8, 128, 64, 16384 / 2176),  # ~ 2 g_q / 1, less the rope slice
    ("gla", 128, 1, 512, 64, 278528 / 1152),  # MLA ~ 2 h_q
    ("gla", 128, 2, 256, 64, 128.0),      # GLA-2 ~ h_q
])
def test_intensity_at_q_len_one(variant, h_q, h_kv, d, d_r, expect):
    sl = np.array([4096])
    f = acc.step_flops(variant, sl, L=1, h_q=h_q, d=d, d_r=d_r)
    b = acc.kv_bytes(variant, sl, h_kv, d, d_r)
    assert abs(f / b - expect) < 1e-9


def test_intensity_matches_two_gq_over_mkv_for_gqa_and_mha():
    for g_q in (1, 2, 4, 8, 16):
        f = acc.step_flops("gqa", [1000], L=1, h_q=8 * g_q, d=128, d_r=0)
        b = acc.kv_bytes("gqa", [1000], 8, 128, 0)
        assert abs(f / b - 2 * g_q / 2) < 1e-12


def test_mla_near_two_hq():
    f = acc.step_flops("gla", [4096], L=1, h_q=128, d=512, d_r=64)
    b = acc.kv_bytes("gla", [4096], 1, 512, 64)
    assert 0.9 * 256 < f / b < 256


def test_causal_flops_count_visible_pairs():
    # L = 3, T = 5: rows see 3, 4, 5 tokens
    f = acc.step_flops("gqa", [5], L=3, h_q=1, d=4, d_r=0)
    assert f == (3 + 4 + 5) * 2 * 8


def test_step_bytes_components():
    b = acc.step_bytes("gta", [65, 1], L=1, h_q=4, h_kv=2, d=8, d_r=4, page_size=64)
    kv = 66 * (2 * 8 + 4) * 2
    q_out = 2 * 4 * (8 + 8) * 2
    assert b == kv + q_out + 2 * 4 * 4 + 3 * 4 + 2 * 4
