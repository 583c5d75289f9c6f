"""Delta-attention inputs that make the output an exact token index.

Each query head h of group g points at one target token t*: the target's key
holds 1.0 in a dimension reserved for h and every other key entry in that
dimension is 0, while q holds 2^9 there (scale 1/8, so the target scores 64 and
every other token 0).  The softmax weight of a non-target is e^-64 / (1 + ...)
< 2e-28, far below bf16 resolution, so out = v_{t*} after rounding.  Values hold
the target's logical position in base-256 digits (plus one), which bf16 represents exactly,
so any page or slot addressing error shows up as a wrong integer.
Slots past T_b and the unreferenced page keep their NaN poison.
"""
import numpy as np

from kv_cache_paged_b200 import workload as wl

ONE = wl.f32_to_bf16_bits(np.array([1.0], np.float32))[0]
QVAL = wl.f32_to_bf16_bits(np.array([512.0], np.float32))[0]


def _digits(t, b):
    # digits shifted to 1..256: exact in bf16, and never 0, so the e^-64-weighted
    # contributions of the other tokens (representable next to 0 in bf16, but not
    # next to 1 in fp32) cannot show
    return [t % 256 + 1, (t // 256) % 256 + 1, b % 256 + 1]


def make_delta_problem(variant, seed, *, B=3, L=1, h_q=8, h_kv=2, d=32, d_r=16, S=16,
                       seqlens=("uniform", 20, 100), shuffle=True):
    if variant == "gqa":
        d_r = 0
    inp = wl.make_inputs(variant, B=B, L=L, h_q=h_q, h_kv=h_kv, d=d, d_r=d_r, page_size=S,
                         seqlens=seqlens, seed=seed, scale=1.0 / 8.0, shuffle=shuffle)
    rng = np.random.default_rng(seed + 1000)
    g_q = h_q // h_kv
    names = {"gqa": ("k_cache", "v_cache"), "gta": ("tied_cache", "rope_cache"),
             "gla": ("latent_cache", "rope_cache")}[variant]
    c0, c1 = inp.caches[names[0]], inp.caches[names[1]]
    # dims: key one-hot dims and value digit dims per variant
    if variant == "gqa":
        key_dim0, val_dim0 = 0, 0
    elif variant == "gta":
        key_dim0, val_dim0 = 0, d - d_r          # value digits in the non-key half of tied
        assert g_q <= d - d_r
    else:
        key_dim0, val_dim0 = 0, g_q              # digits after the one-hot dims of the latent
        assert g_q + 3 <= d
    targets = np.zeros((B, L, h_q, 3), dtype=np.float64)
    for b in range(B):
        T = int(inp.seqlens[b])
        for t in range(T):
            page, slot = inp.block_table[b, t // S], t % S
            c0[page, slot] = 0
            if variant != "gqa":
                c1[page, slot] = 0
            else:
                c1[page, slot] = 0
            for g in range(h_kv):
                vals = wl.f32_to_bf16_bits(np.asarray(_digits(t, b), dtype=np.float32))
                if variant == "gqa":
                    c1[page, slot, g, val_dim0:val_dim0 + 3] = vals
                else:
                    c0[page, slot, g, val_dim0:val_dim0 + 3] = vals
        q = np.zeros_like(inp.q)
        for h in range(h_q):
            g, j = h // g_q, h % g_q
            t_star = int(rng.integers(0, T - L + 1))
            page, slot = inp.block_table[b, t_star // S], t_star % S
            c0[page, slot, g, key_dim0 + j] = ONE
            q[:, :, h, key_dim0 + j] = QVAL
            targets[b, :, h] = _digits(t_star, b)
        inp.q[b] = q[b]
    inp._delta_val_dim0 = val_dim0
    return inp, targets


def decode_digits(inp, out):
    v0 = inp._delta_val_dim0
    return np.asarray(out[..., v0:v0 + 3], dtype=np.float64)
