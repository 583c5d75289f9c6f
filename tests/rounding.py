"""Exact rounding of fp64 values to bfloat16 for expected values (test infrastructure).

bf16 keeps 8 significant bits.  With x = m * 2^e (frexp, m in [0.5, 1)), m * 2^8 is exact
in fp64 and numpy's round() rounds half to even, so r * 2^(e - 8) is x rounded once to the
nearest bf16 value, ties to even.  That value is exact in fp32, whose top 16 bits are then
its bf16 encoding.  (Finite values in the normal bf16 range; the tests use |x| < 100.)
"""
import numpy as np


def f64_to_bf16_bits(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    v = np.ldexp(np.round(np.ldexp(m, 8)), e - 8)
    return (v.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(h) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
