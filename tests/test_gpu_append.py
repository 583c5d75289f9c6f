"""GPU parity of the cache append (+ RoPE) and of the query RoPE against the fp64 oracle:
copied state bit-exact, rotated slices equal to the oracle's rotation rounded once to bf16,
untouched rows unchanged, padding slots skipped, out-of-range slots flagged; and a full
step (append the last token of every sequence, then decode) against the oracle."""
import numpy as np
import pytest

from kv_cache_paged_b200 import binding, workload as wl
from oracle import oracle as orc
from tests import gpu_util as gu
from tests.rounding import f64_to_bf16_bits

pytestmark = pytest.mark.gpu


def _bf(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _bits(t):
    return t.cpu().view(__import__("torch").int16).numpy().view(np.uint16)


def _rand_bf16(rng, shape):
    return wl.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def _expected_rope(x_bits, pos, base=10000.0):
    """Oracle rotation of each row of x (bf16 bits [N, d_r]) to pos[n], rounded once to bf16."""
    x = wl.bf16_bits_to_f32(x_bits).astype(np.float64)
    return np.stack([f64_to_bf16_bits(orc.rope(x[n], float(pos[n]), base)) for n in range(x.shape[0])])


def _slots(rng, N, num_rows, pad=2):
    s = rng.choice(num_rows, size=N, replace=False).astype(np.int32)
    s[rng.choice(N, size=pad, replace=False)] = -1
    return s


@pytest.mark.parametrize("variant,heads,dim,d_r", [("gta", 8, 128, 64), ("gta", 2, 64, 32),
                                                   ("gla", 1, 512, 64), ("gla", 2, 256, 64)])
def test_tied_and_latent_append(cuda_device, variant, heads, dim, d_r):
    import torch
    rng = np.random.default_rng(heads * 7 + dim + d_r)
    P, S, N = 12, 16, 40
    state = _rand_bf16(rng, (N, heads, dim))
    rope = _rand_bf16(rng, (N, d_r))
    pos = rng.integers(0, 65536, N).astype(np.int32)
    slot = _slots(rng, N, P * S)
    c0 = np.full((P, S, heads, dim), 0x1234, np.uint16)
    c1 = np.full((P, S, d_r), 0x4321, np.uint16)
    d0, d1 = _bf(c0), _bf(c1)
    fn = binding.gta_append if variant == "gta" else binding.gla_append
    fn(_bf(state), _bf(rope), torch.from_numpy(pos).cuda(), torch.from_numpy(slot).cuda(), d0, d1)
    torch.cuda.synchronize()
    g0, g1 = _bits(d0).reshape(P * S, heads, dim), _bits(d1).reshape(P * S, d_r)
    e0, e1 = c0.reshape(P * S, heads, dim).copy(), c1.reshape(P * S, d_r).copy()
    ok = slot >= 0
    e0[slot[ok]] = state[ok]
    e1[slot[ok]] = _expected_rope(rope[ok], pos[ok])
    assert np.array_equal(g0, e0)
    assert np.array_equal(g1, e1)


@pytest.mark.parametrize("d_r", [128, 64])
def test_gqa_append_rotates_key_tail(cuda_device, d_r):
    import torch
    rng = np.random.default_rng(d_r)
    P, S, N, H, D = 6, 64, 50, 8, 128
    k = _rand_bf16(rng, (N, H, D))
    v = _rand_bf16(rng, (N, H, D))
    pos = rng.integers(0, 8192, N).astype(np.int32)
    slot = _slots(rng, N, P * S)
    kc, vc = np.zeros((P, S, H, D), np.uint16), np.zeros((P, S, H, D), np.uint16)
    dk, dv = _bf(kc), _bf(vc)
    binding.gqa_append(_bf(k), _bf(v), torch.from_numpy(pos).cuda(), torch.from_numpy(slot).cuda(), dk, dv, d_r)
    torch.cuda.synchronize()
    ek, ev = kc.reshape(P * S, H, D).copy(), vc.reshape(P * S, H, D).copy()
    ok = np.flatnonzero(slot >= 0)
    for n in ok:
        ev[slot[n]] = v[n]
        ek[slot[n], :, :D - d_r] = k[n, :, :D - d_r]
        ek[slot[n], :, D - d_r:] = _expected_rope(k[n, :, D - d_r:], np.full(H, pos[n]))
    assert np.array_equal(_bits(dk).reshape(P * S, H, D), ek)
    assert np.array_equal(_bits(dv).reshape(P * S, H, D), ev)


def test_append_out_of_range_slot_is_flagged(cuda_device):
    import torch
    rng = np.random.default_rng(3)
    P, S, N = 4, 16, 6
    tied, rope = _rand_bf16(rng, (N, 2, 64)), _rand_bf16(rng, (N, 32))
    slot = np.array([0, 5, P * S, 9, P * S + 100, 63], np.int32)
    c0, c1 = _bf(np.zeros((P, S, 2, 64), np.uint16)), _bf(np.zeros((P, S, 32), np.uint16))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.gta_append(_bf(tied), _bf(rope), torch.zeros(N, dtype=torch.int32, device="cuda"),
                       torch.from_numpy(slot).cuda(), c0, c1, error_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == binding.DEVERR_BAD_PAGE
    g0 = _bits(c0).reshape(P * S, 2, 64)
    for n in (0, 1, 3, 5):
        assert np.array_equal(g0[slot[n]], tied[n])
    assert np.count_nonzero(g0.reshape(P * S, -1).any(axis=1)) == 4


@pytest.mark.parametrize("variant", ["gta", "gla", "gqa"])
def test_rope_q_matches_oracle(cuda_device, variant):
    import torch
    rng = np.random.default_rng(11)
    B, L = 5, 3
    heads, d_qk, off, d_r = {"gta": (32, 128, 64, 64), "gla": (16, 576, 512, 64), "gqa": (8, 128, 0, 128)}[variant]
    q = _rand_bf16(rng, (B, L, heads, d_qk))
    seqlens = np.array([3, 100, 2, 70000, 9], np.int32)   # sequence 2 has fewer than L tokens
    dq = _bf(q)
    binding.rope_q(dq, torch.from_numpy(seqlens).cuda(), off, d_r)
    torch.cuda.synchronize()
    got = _bits(dq)
    exp = q.copy()
    for b in range(B):
        for i in range(L):
            p = seqlens[b] - L + i
            if p < 0:
                continue
            exp[b, i, :, off:off + d_r] = _expected_rope(q[b, i, :, off:off + d_r], np.full(heads, p))
    assert np.array_equal(got, exp)


def test_append_then_decode_step(cuda_device):
    """A decode step end to end on the GPU: the last token of every sequence is written by
    the append kernel (tied state as is, rope slice rotated to T_b - 1), then decode; the
    oracle decodes the same cache built on the host with the oracle's rotation."""
    import torch
    inp = wl.make_inputs("gta", B=4, L=1, h_q=32, h_kv=8, d=128, d_r=64, page_size=64,
                         seqlens=[70, 1, 200, 128], seed=21)
    rng = np.random.default_rng(22)
    B = inp.B
    tied_new = _rand_bf16(rng, (B, 8, 128))
    rope_new = _rand_bf16(rng, (B, 64))
    pos = (inp.seqlens - 1).astype(np.int32)
    slot = np.array([inp.block_table[b, pos[b] // 64] * 64 + pos[b] % 64 for b in range(B)], np.int32)
    dev = gu.to_dev(inp)
    binding.gta_append(_bf(tied_new), _bf(rope_new), torch.from_numpy(pos).cuda(), torch.from_numpy(slot).cuda(),
                       dev["tied_cache"], dev["rope_cache"])
    out, lse = gu.run_gpu(inp, dev=dev)
    host_t = inp.caches["tied_cache"].reshape(-1, 8, 128)
    host_r = inp.caches["rope_cache"].reshape(-1, 64)
    host_t[slot] = tied_new
    host_r[slot] = _expected_rope(rope_new, pos)
    ref_o, ref_l, _ = orc.decode_inputs(inp)
    o, l = gu.to_np(out, lse)
    gu.assert_close(o, l, ref_o, ref_l, "append + decode")
