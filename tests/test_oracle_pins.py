"""Pins for the fp64 oracle: each checks it against something other than itself.

The pages print no worked numeric example, so the pins are identities and
special cases that the definitions in "Hardware-Efficient Attention for Fast
Decoding" (section 3; Figure 2 caption for GTA) fix, closed forms, and a second
independent restatement in numpy.
"""
import math

import numpy as np
import pytest

from kv_cache_paged_b200 import workload as wl
from oracle import numpy_ref
from oracle import oracle as orc

NAMES = {"gqa": ("k_cache", "v_cache"), "gta": ("tied_cache", "rope_cache"),
         "gla": ("latent_cache", "rope_cache")}


def tiny(variant, *, B=3, L=1, h_q=8, h_kv=2, d=32, d_r=16, S=16, seqlens=("uniform", 5, 70),
         seed=11, shuffle=True, scale=None, latent_scale=1.0):
    if variant == "gqa":
        d_r = 0
    return wl.make_inputs(variant, B=B, L=L, h_q=h_q, h_kv=h_kv, d=d, d_r=d_r, page_size=S,
                          seqlens=seqlens, seed=seed, shuffle=shuffle, scale=scale,
                          latent_scale=latent_scale)


def run_c(inp, **kw):
    out, lse, _ = orc.decode_inputs(inp, **kw)
    return out, lse


def run_np(inp):
    c0, c1 = (inp.caches[n] for n in NAMES[inp.variant])
    return numpy_ref.decode(inp.variant, inp.q, c0, c1, inp.block_table, inp.seqlens, L=inp.L,
                            h_q=inp.h_q, h_kv=inp.h_kv, d=inp.d, d_r=inp.d_r,
                            page_size=inp.page_size, scale=inp.scale)


# ---------------------------------------------------------------- P6 brute force
@pytest.mark.parametrize("variant", ["gqa", "gta", "gla"])
@pytest.mark.parametrize("L", [1, 2, 3])
@pytest.mark.parametrize("S", [16, 4])
def test_c_oracle_matches_numpy_restatement(variant, L, S):
    h_kv = 1 if variant == "gla" and S == 4 else 2   # S=4 GLA case is MLA (one latent head)
    inp = tiny(variant, L=L, S=S, h_kv=h_kv, seqlens=("uniform", max(L, 1), 70), seed=100 + L + S)
    o1, l1 = run_c(inp)
    o2, l2 = run_np(inp)
    assert np.isfinite(o1).all() and np.isfinite(l1).all()
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_thread_count_does_not_change_result():
    inp = tiny("gta", B=4, L=2, seed=5)
    o1, l1, n1 = orc.decode_inputs(inp, threads=1)
    o2, l2, n2 = orc.decode_inputs(inp, threads=0)
    assert n1 == 1
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_b_list_selects_sequences():
    inp = tiny("gqa", B=5, seed=6)
    o_all, l_all = run_c(inp)
    sel = np.array([3, 0, 3], dtype=np.int32)
    o, l = run_c(inp, b_list=sel)
    assert np.array_equal(o, o_all[sel]) and np.array_equal(l, l_all[sel])


# ---------------------------------------------------------------- P1 GTA == GQA materialised
@pytest.mark.parametrize("L", [1, 2])
def test_gta_equals_gqa_with_explicit_kv(L):
    """Figure 2: key = [tied[:, :d_h-d_r] ++ rope broadcast to the group], value = tied."""
    inp = tiny("gta", L=L, d=32, d_r=16, seed=21)
    tied, rope = inp.caches["tied_cache"], inp.caches["rope_cache"]
    P, S, H, D = tied.shape
    k = tied.copy()
    k[..., D - inp.d_r:] = np.broadcast_to(rope[:, :, None, :], (P, S, H, inp.d_r))
    g = wl.DecodeInputs(**{**inp.__dict__, "variant": "gqa", "d_r": 0,
                           "caches": {"k_cache": k, "v_cache": tied.copy()}})
    o1, l1 = run_c(inp)
    o2, l2 = run_c(g)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- P2 absorbed == explicit
@pytest.mark.parametrize("h_c", [1, 2])
@pytest.mark.parametrize("L", [1, 2])
def test_absorbed_latent_equals_explicit_up_projection(h_c, L):
    """Section 3.3: per head, k_nope = W_uk^T c and v = W_uv^T c; absorbing W_uk into the
    query and W_uv into the output gives the same scores and outputs."""
    rng = np.random.default_rng(7 + h_c + L)
    h_q, d_c, d_r, d_nope, d_vh = 4, 32, 8, 8, 12
    inp = tiny("gla", L=L, h_q=h_q, h_kv=h_c, d=d_c, d_r=d_r, S=8, seqlens=("uniform", L, 40),
               seed=31 + h_c, latent_scale=0.5)
    W_uk = rng.integers(-2, 3, size=(h_q, d_c, d_nope)).astype(np.float64)
    W_uv = rng.standard_normal((h_q, d_c, d_vh))
    q_nope = rng.integers(-2, 3, size=(inp.B, L, h_q, d_nope)).astype(np.float64)
    q_lat = np.einsum("hcn,blhn->blhc", W_uk, q_nope) / 16.0           # exact in bf16
    assert np.abs(q_lat * 16).max() <= 256
    q_rope = numpy_ref.bf16_to_f64(inp.q[..., d_c:])
    q_abs = np.concatenate([q_lat, q_rope], axis=-1).astype(np.float32)
    inp.q = wl.f32_to_bf16_bits(q_abs)
    assert np.array_equal(numpy_ref.bf16_to_f64(inp.q), q_abs.astype(np.float64))
    out_abs, lse_abs = run_c(inp)

    g_q = h_q // h_c
    for b in range(inp.B):
        T = int(inp.seqlens[b])
        c = numpy_ref.bf16_to_f64(numpy_ref.gather_tokens(inp.caches["latent_cache"],
                                                          inp.block_table[b], T, inp.page_size))
        r = numpy_ref.bf16_to_f64(numpy_ref.gather_tokens(inp.caches["rope_cache"],
                                                          inp.block_table[b], T, inp.page_size))
        K = np.empty((T, h_q, d_nope + d_r))
        V = np.empty((T, h_q, d_vh))
        for h in range(h_q):
            lat = c[:, h // g_q, :]
            K[:, h, :d_nope] = lat @ W_uk[h]
            K[:, h, d_nope:] = r
            V[:, h] = lat @ W_uv[h]
        qe = np.concatenate([q_nope[b] / 16.0, q_rope[b]], axis=-1)
        o_exp, l_exp = numpy_ref.attention(qe, K, V, inp.scale, L)
        o_from_abs = np.einsum("hcv,lhc->lhv", W_uv, out_abs[b])
        np.testing.assert_allclose(o_from_abs, o_exp, rtol=0, atol=1e-10)
        np.testing.assert_allclose(lse_abs[b], l_exp, rtol=0, atol=1e-10)


# ---------------------------------------------------------------- P3 identical keys
@pytest.mark.parametrize("variant", ["gqa", "gta", "gla"])
@pytest.mark.parametrize("L", [1, 3])
def test_identical_keys_give_mean_of_visible_values(variant, L):
    inp = tiny(variant, L=L, seqlens=("uniform", L, 50), seed=41)
    c0n, c1n = NAMES[variant]
    rng = np.random.default_rng(1)
    if variant == "gqa":
        kv = wl.f32_to_bf16_bits(rng.standard_normal((inp.h_kv, inp.d)).astype(np.float32))
        inp.caches[c0n][:] = kv
        kvec = numpy_ref.bf16_to_f64(kv)
    elif variant == "gta":
        # key half of every tied row equal (per group), value half free; rope equal
        half = inp.d - inp.d_r
        kv = wl.f32_to_bf16_bits(rng.standard_normal((inp.h_kv, half)).astype(np.float32))
        inp.caches[c0n][..., :half] = kv
        rp = wl.f32_to_bf16_bits(rng.standard_normal(inp.d_r).astype(np.float32))
        inp.caches[c1n][:] = rp
        kvec = np.concatenate([numpy_ref.bf16_to_f64(kv),
                               np.broadcast_to(numpy_ref.bf16_to_f64(rp), (inp.h_kv, inp.d_r))], 1)
    else:
        # key = [latent ++ rope]: equal keys force equal latents, so V is constant too
        lat = wl.f32_to_bf16_bits(rng.standard_normal((inp.h_kv, inp.d)).astype(np.float32))
        inp.caches[c0n][:] = lat
        rp = wl.f32_to_bf16_bits(rng.standard_normal(inp.d_r).astype(np.float32))
        inp.caches[c1n][:] = rp
        kvec = np.concatenate([numpy_ref.bf16_to_f64(lat),
                               np.broadcast_to(numpy_ref.bf16_to_f64(rp), (inp.h_kv, inp.d_r))], 1)
    out, lse = run_c(inp)
    qf = numpy_ref.bf16_to_f64(inp.q)
    g_q = inp.h_q // inp.h_kv
    vname = "v_cache" if variant == "gqa" else c0n
    for b in range(inp.B):
        T = int(inp.seqlens[b])
        V = numpy_ref.bf16_to_f64(numpy_ref.gather_tokens(inp.caches[vname], inp.block_table[b],
                                                          T, inp.page_size))
        for i in range(L):
            n = T - L + i + 1
            for h in range(inp.h_q):
                g = h // g_q
                s = inp.scale * float(qf[b, i, h] @ kvec[g])
                np.testing.assert_allclose(lse[b, i, h], math.log(n) + s, rtol=0, atol=1e-12)
                np.testing.assert_allclose(out[b, i, h], V[:n, g].mean(axis=0), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- P4 one-token cache, 2-token closed form
@pytest.mark.parametrize("variant", ["gqa", "gta", "gla"])
def test_one_token_cache_returns_its_value(variant):
    inp = tiny(variant, B=2, seqlens=1, seed=51)
    out, lse = run_c(inp)
    o_np, l_np = run_np(inp)
    vname = "v_cache" if variant == "gqa" else NAMES[variant][0]
    qf = numpy_ref.bf16_to_f64(inp.q)
    g_q = inp.h_q // inp.h_kv
    for b in range(inp.B):
        page = inp.block_table[b, 0]
        v0 = numpy_ref.bf16_to_f64(inp.caches[vname][page, 0])
        for h in range(inp.h_q):
            assert np.array_equal(out[b, 0, h], v0[h // g_q])
        np.testing.assert_allclose(lse[b], l_np[b], rtol=0, atol=1e-12)
    # lse = s_0 exactly: recompute the single score by hand for GQA
    if variant == "gqa":
        for b in range(inp.B):
            k0 = numpy_ref.bf16_to_f64(inp.caches["k_cache"][inp.block_table[b, 0], 0])
            for h in range(inp.h_q):
                s0 = inp.scale * float(qf[b, 0, h] @ k0[h // g_q])
                assert abs(lse[b, 0, h] - s0) <= 1e-12


def test_two_token_closed_form():
    inp = tiny("gqa", B=1, seqlens=2, seed=52)
    out, lse = run_c(inp)
    qf = numpy_ref.bf16_to_f64(inp.q)
    page = inp.block_table[0, 0]
    K = numpy_ref.bf16_to_f64(inp.caches["k_cache"][page, :2])
    V = numpy_ref.bf16_to_f64(inp.caches["v_cache"][page, :2])
    g_q = inp.h_q // inp.h_kv
    for h in range(inp.h_q):
        g = h // g_q
        s0 = inp.scale * float(qf[0, 0, h] @ K[0, g])
        s1 = inp.scale * float(qf[0, 0, h] @ K[1, g])
        w0 = 1.0 / (1.0 + math.exp(s1 - s0))
        np.testing.assert_allclose(out[0, 0, h], w0 * V[0, g] + (1 - w0) * V[1, g], atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse[0, 0, h], max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))),
                                   atol=1e-13, rtol=0)


def test_empty_context_gives_zero_and_minus_inf():
    inp = tiny("gta", B=3, seqlens=[0, 7, 0], seed=53)
    out, lse = run_c(inp)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2]))
    assert np.isfinite(lse[1]).all()


# ---------------------------------------------------------------- P5 split combine == unsplit
@pytest.mark.parametrize("variant", ["gqa", "gta", "gla"])
@pytest.mark.parametrize("L", [1, 2])
def test_split_combine_equals_unsplit(variant, L):
    inp = tiny(variant, L=L, B=4, seqlens=("uniform", L, 90), seed=61 + L)
    full, full_lse = run_c(inp)
    rng = np.random.default_rng(3)
    for b in range(inp.B):
        T = int(inp.seqlens[b])
        for nsplit in (1, 2, 5):
            cuts = np.sort(rng.integers(0, T + 1, size=nsplit - 1))
            edges = np.concatenate([[0], cuts, [T]]).astype(np.int32)  # duplicates = empty splits
            lo, hi = edges[:-1], edges[1:]
            part, plse = run_c(inp, b_list=np.full(nsplit, b, np.int32), tok_lo=lo, tok_hi=hi)
            rows = L * inp.h_q
            o, l = orc.combine(part.reshape(nsplit, rows, -1), plse.reshape(nsplit, rows))
            np.testing.assert_allclose(o.reshape(full[b].shape), full[b], rtol=0, atol=1e-12)
            np.testing.assert_allclose(l.reshape(full_lse[b].shape), full_lse[b], rtol=0, atol=1e-12)


def test_combine_with_all_splits_empty():
    o, l = orc.combine(np.ones((3, 2, 4)), np.full((3, 2), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(l))


def test_combine_is_weighted_by_softmax_denominators():
    # Two halves of a two-token softmax: lse_s = s_k, out_s = v_k.
    s = np.array([[0.3], [-1.2]])
    v = np.array([[[1.0, 2.0]], [[-3.0, 5.0]]])
    o, l = orc.combine(v, s)
    w = np.exp(s[:, 0] - np.logaddexp(s[0, 0], s[1, 0]))
    np.testing.assert_allclose(o[0], w[0] * v[0, 0] + w[1] * v[1, 0], atol=1e-15)
    np.testing.assert_allclose(l[0], np.logaddexp(0.3, -1.2), atol=1e-15)


# ---------------------------------------------------------------- P7 indexing (oracle side)
@pytest.mark.parametrize("variant", ["gqa", "gta", "gla"])
def test_delta_attention_recovers_token_index(variant):
    """One-hot keys with a large score pick one token; V carries that token's logical
    index in base-256 digits, exact in bf16, so the output must be that index exactly."""
    from tests.indexing import make_delta_problem, decode_digits
    inp, targets = make_delta_problem(variant, seed=71)
    out, lse = run_c(inp)
    got = decode_digits(inp, out)
    # fp64 and unrounded: non-targets contribute < 1e-25; bf16 rounding on the GPU makes it exact
    assert np.abs(got - targets).max() < 1e-20
    assert np.isfinite(out).all()


# ---------------------------------------------------------------- P9 RoPE
def test_rope_depends_only_on_relative_position():
    rng = np.random.default_rng(9)
    q = rng.standard_normal(64)
    k = rng.standard_normal(64)
    a = orc.rope(q, 1000) @ orc.rope(k, 990)
    b = orc.rope(q, 17) @ orc.rope(k, 7)
    np.testing.assert_allclose(a, b, rtol=1e-10)
    np.testing.assert_allclose(np.linalg.norm(orc.rope(q, 12345)), np.linalg.norm(q), rtol=1e-12)
    assert np.array_equal(orc.rope(q, 0), q)


def test_rope_two_dims_is_a_plane_rotation():
    x = np.array([0.6, -0.8])
    y = orc.rope(x, 0.25, base=10000.0)   # theta_0 = 1, angle 0.25
    c, s = math.cos(0.25), math.sin(0.25)
    np.testing.assert_allclose(y, [0.6 * c + 0.8 * s, -0.8 * c + 0.6 * s], atol=1e-15)
