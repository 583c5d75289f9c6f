"""Python face of the fp64 C oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  The CUDA library never imports or links
it, and it imports nothing from the CUDA side.

Arrays in, arrays out: caches and q are raw bf16 bit patterns (uint16),
block_table and seqlens int32.  Results are float64 and are not rounded.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

VARIANTS = {"gqa": 0, "gta": 1, "gla": 2}


def build(force: bool = False) -> str:
    """Compile oracle.c with plain gcc -O2 -fopenmp (no fast-math).  KVD_ORACLE_LIB names an
    already-built library to use instead (the tests point it at deliberately broken copies to
    show that the pins catch them)."""
    if os.environ.get("KVD_ORACLE_LIB"):
        return os.environ["KVD_ORACLE_LIB"]
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"],
                   check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i = ctypes.c_int
            lib.orc_decode.restype = ctypes.c_int
            lib.orc_decode.argtypes = [i, i, i, i, i, i, i, i, i, P, P, P, P, P, ctypes.c_double,
                                       P, i, P, P, P, P, i]
            lib.orc_combine.restype = None
            lib.orc_combine.argtypes = [i, i, i, P, P, P, P]
            lib.orc_rope.restype = None
            lib.orc_rope.argtypes = [P, i, ctypes.c_double, ctypes.c_double, P]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def decode(variant: str, q, c0, c1, block_table, seqlens, *, L: int, h_q: int, h_kv: int, d: int,
           d_r: int, page_size: int, scale: float, b_list=None, tok_lo=None, tok_hi=None,
           threads: int = 0):
    """fp64 decode attention.

    variant "gqa": c0 = K cache, c1 = V cache, each [P, S, h_kv, d].
    variant "gta": c0 = tied cache [P, S, h_kv, d_h=d], c1 = rope cache [P, S, d_r].
    variant "gla": c0 = latent cache [P, S, h_c=h_kv, d_c=d], c1 = rope cache [P, S, d_r].
    Returns (out [nb, L, h_q, d], lse [nb, L, h_q], threads_used).
    """
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.uint16)
    c0 = np.ascontiguousarray(c0, dtype=np.uint16)
    c1 = np.ascontiguousarray(c1, dtype=np.uint16)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    B = sl.shape[0]
    assert bt.shape[0] == B and bt.ndim == 2
    assert h_q % h_kv == 0
    if b_list is not None:
        b_list = np.ascontiguousarray(b_list, dtype=np.int32)
        nb = int(b_list.shape[0])
    else:
        nb = B
    if tok_lo is not None:
        tok_lo = np.ascontiguousarray(tok_lo, dtype=np.int32)
        tok_hi = np.ascontiguousarray(tok_hi, dtype=np.int32)
        assert tok_lo.shape == (nb,) and tok_hi.shape == (nb,)
    out = np.zeros((nb, L, h_q, d), dtype=np.float64)
    lse = np.zeros((nb, L, h_q), dtype=np.float64)
    used = lib.orc_decode(VARIANTS[variant], B, L, h_q, h_kv, d, d_r, page_size, bt.shape[1],
                          _ptr(q), _ptr(c0), _ptr(c1), _ptr(bt), _ptr(sl), float(scale),
                          _ptr(b_list), nb, _ptr(tok_lo), _ptr(tok_hi), _ptr(out), _ptr(lse),
                          int(threads))
    return out, lse, used


def decode_inputs(inp, **kw):
    """Run :func:`decode` on an object with the attributes of a decode-inputs record."""
    names = {"gqa": ("k_cache", "v_cache"), "gta": ("tied_cache", "rope_cache"),
             "gla": ("latent_cache", "rope_cache")}[inp.variant]
    return decode(inp.variant, inp.q, inp.caches[names[0]], inp.caches[names[1]], inp.block_table,
                  inp.seqlens, L=inp.L, h_q=inp.h_q, h_kv=inp.h_kv, d=inp.d, d_r=inp.d_r,
                  page_size=inp.page_size, scale=inp.scale, **kw)


def combine(part_out, part_lse):
    """LSE combine: part_out [n, rows, d_v], part_lse [n, rows] -> (out, lse)."""
    lib = _load()
    po = np.ascontiguousarray(part_out, dtype=np.float64)
    pl = np.ascontiguousarray(part_lse, dtype=np.float64)
    n, rows, dv = po.shape
    assert pl.shape == (n, rows)
    out = np.zeros((rows, dv), dtype=np.float64)
    lse = np.zeros(rows, dtype=np.float64)
    lib.orc_combine(n, rows, dv, _ptr(po), _ptr(pl), _ptr(out), _ptr(lse))
    return out, lse


def rope(x, pos: float, base: float = 10000.0):
    """Rotate one d_r-vector to absolute position ``pos`` (rotate-half pairs)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros_like(x)
    lib.orc_rope(_ptr(x), x.shape[0], float(pos), float(base), _ptr(y))
    return y
