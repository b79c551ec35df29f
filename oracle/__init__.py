"""Float64 CPU oracle for the MiMo-V2.6-Flash hybrid attention forward (ctypes binding).

TEST INFRASTRUCTURE.  Only tests/, the smoke check in __graft_entry__ and the
bench's CPU-baseline / reference legs may import this package.  The product
path (global_attention_attn_b200) never imports it and shares no code with it.

The arithmetic lives in mimo_oracle.cpp (plain C++, float64).  This module
compiles it with g++ on first use (or from build()), and marshals arguments.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mimo_oracle.cpp")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libmimo_oracle.so")
_lib = None

P_I32 = C.POINTER(C.c_int32)
P_U16 = C.POINTER(C.c_uint16)
P_F32 = C.POINTER(C.c_float)
P_F64 = C.POINTER(C.c_double)


class OracleLayer(C.Structure):
    _fields_ = [
        ("hq", C.c_int), ("hkv", C.c_int), ("dqk", C.c_int), ("dv", C.c_int), ("rope_dim", C.c_int),
        ("rope_base", C.c_double), ("softmax_scale", C.c_double), ("v_scale", C.c_double),
        ("window", C.c_int), ("sink", P_F32),
        ("num_seqs", C.c_int), ("q_row0", P_I32), ("q_len", P_I32), ("q_pos0", P_I32),
        ("k_new", P_U16), ("v_new", P_U16), ("new_row0", P_I32), ("new_pos0", P_I32), ("new_len", P_I32),
        ("cache_kind", C.c_int), ("k_cache", P_U16), ("v_cache", P_U16), ("page_size", C.c_int),
        ("block_table", P_I32), ("max_pages", C.c_int),
        ("cache_dtype", C.c_int), ("k_dequant", P_F32), ("v_dequant", P_F32),
    ]


def build(force: bool = False) -> str:
    """Compile the oracle (g++ -O3, portable x86-64-v2 code) into oracle/_build/."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O3", "-march=x86-64-v2", "-std=c++17", "-shared", "-fPIC", "-pthread",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.oracle_rope.argtypes = [P_F64, C.c_int, C.c_int, C.c_double, C.c_double, P_F64]
        _lib.oracle_rope.restype = None
        _lib.oracle_attention.argtypes = [C.POINTER(OracleLayer), P_U16, C.c_int, P_I32, P_I32, P_F64, P_F64,
                                          C.c_int, C.c_int]
        _lib.oracle_attention.restype = C.c_int
        _lib.oracle_kv_append.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_double, P_U16, P_U16,
                                          P_I32, P_F64, P_F64]
        _lib.oracle_kv_append.restype = C.c_int
        _lib.oracle_e4m3_to_double.argtypes = [C.c_int]
        _lib.oracle_e4m3_to_double.restype = C.c_double
    return _lib


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def _ptr(a, t):
    return None if a is None else a.ctypes.data_as(t)


def rope(x, pos: float, base: float, rope_dim: int) -> np.ndarray:
    """Partial NeoX RoPE of one head vector, in float64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    lib().oracle_rope(_ptr(x, P_F64), x.size, rope_dim, float(base), float(pos), _ptr(out, P_F64))
    return out


def attention(*, q, hq, hkv, dqk, dv, rope_dim, rope_base, softmax_scale, v_scale, window, sink,
              q_row0, q_len, q_pos0, sel_seq, sel_row,
              k_new=None, v_new=None, new_row0=None, new_pos0=None, new_len=None,
              cache_kind=0, k_cache=None, v_cache=None, page_size=0, block_table=None,
              cache_dtype=0, k_dequant=None, v_dequant=None, nthreads=None, online=False):
    """Evaluates the selected rows (sel_seq[i], row sel_row[i] of that sequence) for all heads.
    cache_dtype 1: the caches hold E4M3 bytes with per-KV-head scales k_dequant / v_dequant.

    Returns (out [n, hq, dv] float64, lse [n, hq] float64)."""
    keep = []

    def arr(a, dt):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dtype=dt)
        keep.append(a)
        return a

    B = len(q_len)
    L = OracleLayer()
    L.hq, L.hkv, L.dqk, L.dv, L.rope_dim = hq, hkv, dqk, dv, rope_dim
    L.rope_base, L.softmax_scale, L.v_scale, L.window = float(rope_base), float(softmax_scale), float(v_scale), int(window)
    L.sink = _ptr(arr(sink, np.float32), P_F32)
    L.num_seqs = B
    L.q_row0 = _ptr(arr(q_row0, np.int32), P_I32)
    L.q_len = _ptr(arr(q_len, np.int32), P_I32)
    L.q_pos0 = _ptr(arr(q_pos0, np.int32), P_I32)
    L.k_new = _ptr(arr(k_new, np.uint16), P_U16)
    L.v_new = _ptr(arr(v_new, np.uint16), P_U16)
    zeros = np.zeros(B, np.int32)
    L.new_row0 = _ptr(arr(new_row0 if new_row0 is not None else zeros, np.int32), P_I32)
    L.new_pos0 = _ptr(arr(new_pos0 if new_pos0 is not None else zeros, np.int32), P_I32)
    L.new_len = _ptr(arr(new_len if new_len is not None else zeros, np.int32), P_I32)
    L.cache_kind = int(cache_kind)
    cdt = np.uint8 if cache_dtype == 1 else np.uint16
    L.k_cache = C.cast(_ptr(arr(k_cache, cdt), C.c_void_p), P_U16) if k_cache is not None else None
    L.v_cache = C.cast(_ptr(arr(v_cache, cdt), C.c_void_p), P_U16) if v_cache is not None else None
    L.cache_dtype = int(cache_dtype)
    L.k_dequant = _ptr(arr(k_dequant, np.float32), P_F32)
    L.v_dequant = _ptr(arr(v_dequant, np.float32), P_F32)
    L.page_size = int(page_size)
    bt = arr(block_table, np.int32)
    L.block_table = _ptr(bt, P_I32)
    L.max_pages = 0 if bt is None else int(bt.shape[1])
    qa = arr(q, np.uint16)
    ss = arr(sel_seq, np.int32)
    sr = arr(sel_row, np.int32)
    n = len(ss)
    out = np.empty((n, hq, dv), np.float64)
    lse = np.empty((n, hq), np.float64)
    rc = lib().oracle_attention(C.byref(L), _ptr(qa, P_U16), n, _ptr(ss, P_I32), _ptr(sr, P_I32),
                                _ptr(out, P_F64), _ptr(lse, P_F64), int(nthreads or default_threads()),
                                1 if online else 0)
    if rc != 0:
        raise RuntimeError(f"oracle_attention failed with code {rc}")
    return out, lse


def e4m3_to_double(codes) -> np.ndarray:
    """Values of E4M3 bytes (OCP 8-bit floating point), in float64."""
    codes = np.asarray(codes, np.int64)
    f = lib().oracle_e4m3_to_double
    return np.array([f(int(c)) for c in codes.reshape(-1)], np.float64).reshape(codes.shape)


def kv_append(k_new, v_new, pos, rope_base: float, rope_dim: int = 64):
    """Expected cache rows after appending: (K rotated at pos [n,hkv,dqk], V [n,hkv,dv]) in float64."""
    k_new = np.ascontiguousarray(k_new, np.uint16)
    v_new = np.ascontiguousarray(v_new, np.uint16)
    pos = np.ascontiguousarray(pos, np.int32)
    n, hkv, dqk = k_new.shape
    dv = v_new.shape[2]
    ko = np.empty((n, hkv, dqk), np.float64)
    vo = np.empty((n, hkv, dv), np.float64)
    lib().oracle_kv_append(n, hkv, dqk, dv, rope_dim, float(rope_base), _ptr(k_new, P_U16), _ptr(v_new, P_U16),
                           _ptr(pos, P_I32), _ptr(ko, P_F64), _ptr(vo, P_F64))
    return ko, vo


from . import workload as _workload  # noqa: E402  (adapters for the seeded workloads)

prefill = _workload.prefill
decode = _workload.decode
chunked = _workload.chunked
