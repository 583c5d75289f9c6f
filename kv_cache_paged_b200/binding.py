"""Thin ctypes binding over the C-ABI in include/kvdecode.h and include/kvappend.h.

Argument marshalling only: tensors are checked for dtype/shape/device and their
device pointers, together with torch's current CUDA stream, are handed to the
library; every step of the decode runs in the library's kernels.  There is no
fallback: if the shared library is missing or a call fails, this raises.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "_lib", "libkvdecode.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
HEADER = os.path.join(INCLUDE, "kvdecode.h")

KVD_OK = 0
STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported shape", -3: "workspace too small",
          -4: "CUDA error", -5: "device error flag set"}
DEVERR_TIMEOUT, DEVERR_BAD_PAGE, DEVERR_BAD_SEQLEN = 1, 2, 4
DEBUG_WAIT_LIMIT_NS, DEBUG_SKIP_FIRST_LOAD = 1, 2

_i32 = ctypes.c_int32
_vp = ctypes.c_void_p


class GQAParams(ctypes.Structure):
    _fields_ = [("q", _vp), ("k_cache", _vp), ("v_cache", _vp), ("block_table", _vp), ("seqlens", _vp),
                ("out", _vp), ("lse", _vp),
                ("B", _i32), ("L", _i32), ("h_q", _i32), ("h_kv", _i32), ("d", _i32), ("page_size", _i32),
                ("num_pages", _i32), ("max_pages", _i32), ("scale", ctypes.c_float), ("num_parts", _i32)]


class GTAParams(ctypes.Structure):
    _fields_ = [("q", _vp), ("tied_cache", _vp), ("rope_cache", _vp), ("block_table", _vp), ("seqlens", _vp),
                ("out", _vp), ("lse", _vp),
                ("B", _i32), ("L", _i32), ("h_q", _i32), ("h_kv", _i32), ("d_h", _i32), ("d_r", _i32),
                ("page_size", _i32), ("num_pages", _i32), ("max_pages", _i32), ("scale", ctypes.c_float),
                ("num_parts", _i32)]


class GLAParams(ctypes.Structure):
    _fields_ = [("q", _vp), ("latent_cache", _vp), ("rope_cache", _vp), ("block_table", _vp), ("seqlens", _vp),
                ("out", _vp), ("lse", _vp),
                ("B", _i32), ("L", _i32), ("h_q", _i32), ("h_c", _i32), ("d_c", _i32), ("d_r", _i32),
                ("page_size", _i32), ("num_pages", _i32), ("max_pages", _i32), ("scale", ctypes.c_float),
                ("num_parts", _i32)]


class GQAAppendParams(ctypes.Structure):
    _fields_ = [("k_new", _vp), ("v_new", _vp), ("k_cache", _vp), ("v_cache", _vp), ("positions", _vp),
                ("slot_mapping", _vp), ("error_word", _vp),
                ("N", _i32), ("h_kv", _i32), ("d", _i32), ("d_r", _i32), ("num_rows", _i32),
                ("rope_base", ctypes.c_float)]


class GTAAppendParams(ctypes.Structure):
    _fields_ = [("tied_new", _vp), ("rope_new", _vp), ("tied_cache", _vp), ("rope_cache", _vp), ("positions", _vp),
                ("slot_mapping", _vp), ("error_word", _vp),
                ("N", _i32), ("h_kv", _i32), ("d_h", _i32), ("d_r", _i32), ("num_rows", _i32),
                ("rope_base", ctypes.c_float)]


class GLAAppendParams(ctypes.Structure):
    _fields_ = [("latent_new", _vp), ("rope_new", _vp), ("latent_cache", _vp), ("rope_cache", _vp),
                ("positions", _vp), ("slot_mapping", _vp), ("error_word", _vp),
                ("N", _i32), ("h_c", _i32), ("d_c", _i32), ("d_r", _i32), ("num_rows", _i32),
                ("rope_base", ctypes.c_float)]


_lib = None
_lock = threading.Lock()


class KVDecodeError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status})")
        self.status = status


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                                   "(run `python -m kv_cache_paged_b200.build`)")
            L = ctypes.CDLL(LIB_PATH)
            for name, P in (("gqa", GQAParams), ("gta", GTAParams), ("gla", GLAParams)):
                f = getattr(L, f"kvd_{name}_decode")
                f.restype = ctypes.c_int
                f.argtypes = [ctypes.POINTER(P), _vp, ctypes.c_size_t, _vp]
                w = getattr(L, f"kvd_{name}_workspace_size")
                w.restype = ctypes.c_size_t
                w.argtypes = [ctypes.POINTER(P)]
            L.kvd_plan.restype = ctypes.c_int
            L.kvd_plan.argtypes = [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _vp]
            L.kvd_plan_host.restype = ctypes.c_int
            L.kvd_plan_host.argtypes = [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i32]
            L.kvd_read_device_error.restype = ctypes.c_int
            L.kvd_read_device_error.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
            L.kvd_num_sms.restype = ctypes.c_int
            L.kvd_read_stream.restype = ctypes.c_int
            L.kvd_read_stream.argtypes = [_vp, ctypes.c_size_t, _vp, ctypes.c_int, _vp]
            L.kvd_profile_events.restype = ctypes.c_int
            L.kvd_profile_events.argtypes = [_vp, _vp]
            L.kvd_debug_set.restype = ctypes.c_int
            L.kvd_debug_set.argtypes = [ctypes.c_int, ctypes.c_longlong]
            L.kvd_status_string.restype = ctypes.c_char_p
            L.kvd_status_string.argtypes = [ctypes.c_int]
            L.kvd_version.restype = ctypes.c_int
            for name, P in (("gqa", GQAAppendParams), ("gta", GTAAppendParams), ("gla", GLAAppendParams)):
                f = getattr(L, f"kvd_{name}_append")
                f.restype = ctypes.c_int
                f.argtypes = [ctypes.POINTER(P), _vp]
            L.kvd_gta_prefix_decode.restype = ctypes.c_int
            L.kvd_gta_prefix_decode.argtypes = [ctypes.POINTER(GTAParams), _vp, ctypes.c_size_t, _vp]
            L.kvd_gta_prefix_workspace_size.restype = ctypes.c_size_t
            L.kvd_gta_prefix_workspace_size.argtypes = [ctypes.POINTER(GTAParams)]
            L.kvd_merge_states.restype = ctypes.c_int
            L.kvd_merge_states.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp]
            L.kvd_rope_q.restype = ctypes.c_int
            L.kvd_rope_q.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.c_float, _vp]
            _lib = L
    return _lib


def header_functions():
    """Names of the functions the headers under include/ declare."""
    names = set()
    for h in sorted(os.listdir(INCLUDE)):
        if h.endswith(".h"):
            text = re.sub(r"/\*.*?\*/", "", open(os.path.join(INCLUDE, h)).read(), flags=re.S)
            names.update(re.findall(r"\b(kvd_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def _check(fn, status):
    if status != KVD_OK:
        raise KVDecodeError(fn, status)


# ----------------------------------------------------------------------------- torch helpers
def _torch():
    import torch
    return torch


def _stream_ptr(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name, dtype, ndim=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    return ctypes.c_void_p(t.data_ptr())


_ws_cache: dict = {}


def workspace(nbytes: int, device):
    """A zeroed device workspace of at least nbytes, cached per device (one per process)."""
    torch = _torch()
    key = str(device)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def _outputs(B, L, h_q, d_v, device, out, lse):
    torch = _torch()
    if out is None:
        out = torch.empty((B, L, h_q, d_v), dtype=torch.bfloat16, device=device)
    if lse is None:
        lse = torch.empty((B, L, h_q), dtype=torch.float32, device=device)
    return out, lse


def _run(kind, params, ws, stream):
    L = lib()
    size = getattr(L, f"kvd_{kind}_workspace_size")(ctypes.byref(params))
    if size == 0:
        # let the decode call report the precise status
        _check(f"kvd_{kind}_decode", getattr(L, f"kvd_{kind}_decode")(ctypes.byref(params), None, 0, None))
    torch = _torch()
    if ws is None:
        ws = workspace(size, torch.device("cuda", torch.cuda.current_device()))
    elif ws.numel() * ws.element_size() < size:
        raise ValueError(f"workspace too small: need {size} bytes")
    st = getattr(L, f"kvd_{kind}_decode")(ctypes.byref(params), ctypes.c_void_p(ws.data_ptr()),
                                          ws.numel() * ws.element_size(), _stream_ptr(stream))
    _check(f"kvd_{kind}_decode", st)
    return ws


def gqa_decode(q, k_cache, v_cache, block_table, seqlens, scale, *, num_parts=0, out=None, lse=None,
               workspace=None, stream=None):
    """GQA/MQA/MHA decode.  q [B, L, h_q, d], caches [P, S, h_kv, d] (bf16) -> (out, lse)."""
    torch = _torch()
    B, L, h_q, d = q.shape
    P, S, h_kv, d2 = k_cache.shape
    assert d2 == d and v_cache.shape == k_cache.shape
    out, lse = _outputs(B, L, h_q, d, q.device, out, lse)
    p = GQAParams(_dev(q, "q", torch.bfloat16, 4), _dev(k_cache, "k_cache", torch.bfloat16, 4),
                  _dev(v_cache, "v_cache", torch.bfloat16, 4), _dev(block_table, "block_table", torch.int32, 2),
                  _dev(seqlens, "seqlens", torch.int32, 1), _dev(out, "out", torch.bfloat16, 4),
                  _dev(lse, "lse", torch.float32, 3), B, L, h_q, h_kv, d, S, P, block_table.shape[1],
                  float(scale), int(num_parts))
    _run("gqa", p, workspace, stream)
    return out, lse


def gta_decode(q, tied_cache, rope_cache, block_table, seqlens, scale, *, num_parts=0, out=None, lse=None,
               workspace=None, stream=None):
    """GTA decode.  q [B, L, h_q, d_h], tied [P, S, h_kv, d_h], rope [P, S, d_r] (bf16) -> (out, lse)."""
    torch = _torch()
    B, L, h_q, d_h = q.shape
    P, S, h_kv, d2 = tied_cache.shape
    assert d2 == d_h and rope_cache.shape[:2] == (P, S)
    d_r = rope_cache.shape[2]
    out, lse = _outputs(B, L, h_q, d_h, q.device, out, lse)
    p = GTAParams(_dev(q, "q", torch.bfloat16, 4), _dev(tied_cache, "tied_cache", torch.bfloat16, 4),
                  _dev(rope_cache, "rope_cache", torch.bfloat16, 3), _dev(block_table, "block_table", torch.int32, 2),
                  _dev(seqlens, "seqlens", torch.int32, 1), _dev(out, "out", torch.bfloat16, 4),
                  _dev(lse, "lse", torch.float32, 3), B, L, h_q, h_kv, d_h, d_r, S, P, block_table.shape[1],
                  float(scale), int(num_parts))
    _run("gta", p, workspace, stream)
    return out, lse


def gla_decode(q, latent_cache, rope_cache, block_table, seqlens, scale, *, num_parts=0, out=None, lse=None,
               workspace=None, stream=None):
    """GLA/MLA decode (absorbed).  q [B, L, h_q, d_c + d_r], latent [P, S, h_c, d_c], rope [P, S, d_r]."""
    torch = _torch()
    B, L, h_q, dqk = q.shape
    P, S, h_c, d_c = latent_cache.shape
    d_r = rope_cache.shape[2]
    assert dqk == d_c + d_r and rope_cache.shape[:2] == (P, S)
    out, lse = _outputs(B, L, h_q, d_c, q.device, out, lse)
    p = GLAParams(_dev(q, "q", torch.bfloat16, 4), _dev(latent_cache, "latent_cache", torch.bfloat16, 4),
                  _dev(rope_cache, "rope_cache", torch.bfloat16, 3), _dev(block_table, "block_table", torch.int32, 2),
                  _dev(seqlens, "seqlens", torch.int32, 1), _dev(out, "out", torch.bfloat16, 4),
                  _dev(lse, "lse", torch.float32, 3), B, L, h_q, h_c, d_c, d_r, S, P, block_table.shape[1],
                  float(scale), int(num_parts))
    _run("gla", p, workspace, stream)
    return out, lse


def read_device_error(ws, stream=None):
    """Synchronise, read and clear the workspace's device error word; returns the flag bits."""
    flags = ctypes.c_uint32(0)
    st = lib().kvd_read_device_error(ctypes.c_void_p(ws.data_ptr()), _stream_ptr(stream), ctypes.byref(flags))
    if st not in (KVD_OK, -5):
        raise KVDecodeError("kvd_read_device_error", st)
    return flags.value


def plan_device(seqlens, tile, max_tokens, num_parts, cap=64, stream=None, seg_cost=0):
    """Run the device planner; returns (segments int32 [parts, cap, 6], counts [parts]) on the device."""
    torch = _torch()
    segs = torch.full((num_parts, cap, 6), -1, dtype=torch.int32, device=seqlens.device)
    counts = torch.zeros(num_parts, dtype=torch.int32, device=seqlens.device)
    st = lib().kvd_plan(_dev(seqlens, "seqlens", torch.int32, 1), seqlens.shape[0], tile, seg_cost, max_tokens, num_parts,
                        ctypes.c_void_p(segs.data_ptr()), ctypes.c_void_p(counts.data_ptr()), cap,
                        _stream_ptr(stream))
    _check("kvd_plan", st)
    return segs, counts


def plan_host(seqlens, tile, max_tokens, num_parts, cap=64, seg_cost=0):
    """The same plan computed on the host (numpy int32 in, numpy arrays out)."""
    import numpy as np
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    segs = np.full((num_parts, cap, 6), -1, dtype=np.int32)
    counts = np.zeros(num_parts, dtype=np.int32)
    st = lib().kvd_plan_host(sl.ctypes.data_as(_vp), sl.shape[0], tile, seg_cost, max_tokens, num_parts,
                             segs.ctypes.data_as(_vp), counts.ctypes.data_as(_vp), cap)
    _check("kvd_plan_host", st)
    return segs, counts


def profile_events(before=None, after=None):
    """Record torch.cuda.Event `before`/`after` around each call's main decode kernel (None: off)."""
    b = ctypes.c_void_p(before.cuda_event) if before is not None else None
    a = ctypes.c_void_p(after.cuda_event) if after is not None else None
    _check("kvd_profile_events", lib().kvd_profile_events(b, a))


def read_stream(buf, sink, blocks_per_sm=4, stream=None):
    """Stream-read every byte of the CUDA tensor `buf` once (kvd_read_stream); `sink` is a
    one-element int64 CUDA tensor the kernel may write."""
    _check("kvd_read_stream", lib().kvd_read_stream(_vp(buf.data_ptr()), buf.numel() * buf.element_size(),
                                                     _vp(sink.data_ptr()), int(blocks_per_sm), _stream_ptr(stream)))


def debug_set(knob, value):
    _check("kvd_debug_set", lib().kvd_debug_set(int(knob), int(value)))


def num_sms():
    n = lib().kvd_num_sms()
    if n < 0:
        raise KVDecodeError("kvd_num_sms", n)
    return n


# ----------------------------------------------------------------------------- cache append + RoPE
def _append_common(positions, slot_mapping, N, error_word):
    torch = _torch()
    pos = _dev(positions, "positions", torch.int32, 1)
    slot = _dev(slot_mapping, "slot_mapping", torch.int32, 1)
    if positions.shape[0] != N or slot_mapping.shape[0] != N:
        raise ValueError("positions and slot_mapping need one entry per new token")
    err = _dev(error_word, "error_word", torch.int32) if error_word is not None else None
    return pos, slot, err


def _rows(cache, name):
    return cache.shape[0] * cache.shape[1]


def gqa_append(k_new, v_new, positions, slot_mapping, k_cache, v_cache, d_r, *, rope_base=10000.0,
               error_word=None, stream=None):
    """Write N new tokens: k_new/v_new [N, h_kv, d] -> caches [P, S, h_kv, d] at slot_mapping rows,
    RoPE on the last d_r dims of each K head at `positions`."""
    torch = _torch()
    N, h_kv, d = k_new.shape
    pos, slot, err = _append_common(positions, slot_mapping, N, error_word)
    p = GQAAppendParams(_dev(k_new, "k_new", torch.bfloat16, 3), _dev(v_new, "v_new", torch.bfloat16, 3),
                        _dev(k_cache, "k_cache", torch.bfloat16, 4), _dev(v_cache, "v_cache", torch.bfloat16, 4),
                        pos, slot, err, N, h_kv, d, d_r, _rows(k_cache, "k_cache"), rope_base)
    _check("kvd_gqa_append", lib().kvd_gqa_append(ctypes.byref(p), _stream_ptr(stream)))


def gta_append(tied_new, rope_new, positions, slot_mapping, tied_cache, rope_cache, *, rope_base=10000.0,
               error_word=None, stream=None):
    """Write N new tokens: tied_new [N, h_kv, d_h] as is, rope_new [N, d_r] rotated to `positions`."""
    torch = _torch()
    N, h_kv, d_h = tied_new.shape
    d_r = rope_new.shape[1]
    pos, slot, err = _append_common(positions, slot_mapping, N, error_word)
    p = GTAAppendParams(_dev(tied_new, "tied_new", torch.bfloat16, 3), _dev(rope_new, "rope_new", torch.bfloat16, 2),
                        _dev(tied_cache, "tied_cache", torch.bfloat16, 4),
                        _dev(rope_cache, "rope_cache", torch.bfloat16, 3),
                        pos, slot, err, N, h_kv, d_h, d_r, _rows(tied_cache, "tied_cache"), rope_base)
    _check("kvd_gta_append", lib().kvd_gta_append(ctypes.byref(p), _stream_ptr(stream)))


def gla_append(latent_new, rope_new, positions, slot_mapping, latent_cache, rope_cache, *, rope_base=10000.0,
               error_word=None, stream=None):
    """Write N new tokens: latent_new [N, h_c, d_c] as is, rope_new [N, d_r] rotated to `positions`."""
    torch = _torch()
    N, h_c, d_c = latent_new.shape
    d_r = rope_new.shape[1]
    pos, slot, err = _append_common(positions, slot_mapping, N, error_word)
    p = GLAAppendParams(_dev(latent_new, "latent_new", torch.bfloat16, 3),
                        _dev(rope_new, "rope_new", torch.bfloat16, 2),
                        _dev(latent_cache, "latent_cache", torch.bfloat16, 4),
                        _dev(rope_cache, "rope_cache", torch.bfloat16, 3),
                        pos, slot, err, N, h_c, d_c, d_r, _rows(latent_cache, "latent_cache"), rope_base)
    _check("kvd_gla_append", lib().kvd_gla_append(ctypes.byref(p), _stream_ptr(stream)))


def rope_q(q, seqlens, rope_off, d_r, *, rope_base=10000.0, stream=None):
    """Rotate q [B, L, heads, d_qk] in place: dims [rope_off, rope_off + d_r) of row (b, i) go to
    position seqlens[b] - L + i."""
    torch = _torch()
    B, L, heads, d_qk = q.shape
    st = lib().kvd_rope_q(_dev(q, "q", torch.bfloat16, 4), _dev(seqlens, "seqlens", torch.int32, 1), B, L, heads,
                          d_qk, rope_off, d_r, rope_base, _stream_ptr(stream))
    _check("kvd_rope_q", st)


# ----------------------------------------------------------------------------- cascade
def merge_states(out_a, lse_a, out_b, lse_b, *, out=None, lse=None, stream=None):
    """Merge two attention states (out bf16 [..., d_v], lse fp32 [...]) over disjoint key sets."""
    torch = _torch()
    if out_a.shape != out_b.shape or lse_a.shape != lse_b.shape or out_a.shape[:-1] != lse_a.shape:
        raise ValueError("states must have matching shapes")
    d_v = out_a.shape[-1]
    rows = lse_a.numel()
    out = torch.empty_like(out_a) if out is None else out
    lse = torch.empty_like(lse_a) if lse is None else lse
    st = lib().kvd_merge_states(_dev(out_a, "out_a", torch.bfloat16), _dev(lse_a, "lse_a", torch.float32),
                                _dev(out_b, "out_b", torch.bfloat16), _dev(lse_b, "lse_b", torch.float32),
                                _dev(out, "out", torch.bfloat16), _dev(lse, "lse", torch.float32), rows, d_v,
                                _stream_ptr(stream))
    _check("kvd_merge_states", st)
    return out, lse


def gta_prefix_decode(q, tied_cache, rope_cache, prefix_block_table, prefix_len, scale, *, num_parts=0, out=None,
                      lse=None, workspace=None, stream=None):
    """Attention of every row of q [B, L, h_q, d_h] over one shared prefix (no causal mask).
    prefix_block_table: int32 [1, max_pages] (or [max_pages]); prefix_len: int32 [1] (device)."""
    torch = _torch()
    B, L, h_q, d_h = q.shape
    P, S, h_kv, _ = tied_cache.shape
    bt = prefix_block_table.reshape(1, -1)
    out, lse = _outputs(B, L, h_q, d_h, q.device, out, lse)
    params = GTAParams(_dev(q, "q", torch.bfloat16, 4), _dev(tied_cache, "tied_cache", torch.bfloat16, 4),
                       _dev(rope_cache, "rope_cache", torch.bfloat16, 3), _dev(bt, "block_table", torch.int32, 2),
                       _dev(prefix_len, "prefix_len", torch.int32, 1), _dev(out, "out", torch.bfloat16, 4),
                       _dev(lse, "lse", torch.float32, 3), B, L, h_q, h_kv, d_h, rope_cache.shape[-1], S, P,
                       bt.shape[1], scale, num_parts)
    Lb = lib()
    size = Lb.kvd_gta_prefix_workspace_size(ctypes.byref(params))
    if size == 0:
        _check("kvd_gta_prefix_decode", Lb.kvd_gta_prefix_decode(ctypes.byref(params), None, 0, None))
    if workspace is None:
        workspace = globals()["workspace"](size, q.device)
    st = Lb.kvd_gta_prefix_decode(ctypes.byref(params), ctypes.c_void_p(workspace.data_ptr()),
                                  workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _check("kvd_gta_prefix_decode", st)
    return out, lse
