"""libmimoattn: MiMo-V2.6-Flash hybrid attention forward on B200 (sm_100a).

Thin ctypes binding over the C ABI in include/mimoattn.h.  It marshals torch
tensors (device memory and streams only) into the argument structs; every step
of the attention runs in the library's CUDA kernels.  There is no fallback: if
the shared library is missing the import of `lib()` raises.
"""
from __future__ import annotations

import ctypes as C
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libmimoattn.so")

MIMO_OK = 0
MIMO_ERR_INVALID_ARG = 1
MIMO_ERR_UNSUPPORTED = 2
MIMO_ERR_WORKSPACE = 3
MIMO_ERR_CUDA = 4
MIMO_ERR_TIMEOUT = 5
MIMO_STATUS_TIMEOUT = 1
MIMO_STATUS_BAD_INDEX = 2
MIMO_STATUS_RANGE = 4
MIMO_STATUS_BAD_SCALE = 8
MIMO_CACHE_NONE = 0
MIMO_CACHE_PAGED = 1
MIMO_CACHE_RING = 2
MIMO_DTYPE_BF16 = 0
MIMO_DTYPE_FP8_E4M3 = 1
MIMO_RING_SLOTS_DEFAULT = 128
MIMO_RING_SLOTS_MAX = 512
MIMO_MAX_DRAFTS = 8

NUM_Q_HEADS = 64
HEAD_DIM_QK = 192
HEAD_DIM_V = 128
ROPE_DIM = 64
SOFTMAX_SCALE = 1.0 / math.sqrt(192.0)
V_SCALE = 0.707

EXPORTS = ("mimo_attn_prefill", "mimo_attn_prefill_workspace_size", "mimo_attn_prefill_stall_test", "mimo_attn_decode",
           "mimo_attn_decode_workspace_size", "mimo_attn_verify_workspace_size", "mimo_attn_decode_noalloc",
           "mimo_kv_append", "mimo_last_error",
           "mimo_status_poll", "mimo_version", "mimo_window_from_left_right")
DECODE_NOALLOC_MAX_BYTES = 16 << 20

_P = C.c_void_p
_PI = C.POINTER(C.c_int32)


class MimoLayer(C.Structure):
    _fields_ = [("num_q_heads", C.c_int), ("num_kv_heads", C.c_int), ("head_dim_qk", C.c_int),
                ("head_dim_v", C.c_int), ("rope_dim", C.c_int), ("rope_base", C.c_double),
                ("softmax_scale", C.c_float), ("v_scale", C.c_float), ("window", C.c_int), ("sink", _P)]


class MimoPrefillArgs(C.Structure):
    _fields_ = [("layer", MimoLayer), ("num_seqs", C.c_int), ("total_q", C.c_int), ("total_k", C.c_int),
                ("q", _P), ("k", _P), ("v", _P), ("cu_seqlens_q", _P), ("cu_seqlens_k", _P), ("cache_lens", _P),
                ("cache_kind", C.c_int), ("k_cache", _P), ("v_cache", _P), ("block_table", _P),
                ("max_pages", C.c_int), ("num_pages", C.c_int), ("out", _P), ("lse", _P), ("workspace", _P),
                ("workspace_bytes", C.c_size_t), ("ev_kernel_begin", _P), ("ev_kernel_end", _P),
                ("ring_slots", C.c_int)]


class MimoDecodeArgs(C.Structure):
    _fields_ = [("layer", MimoLayer), ("batch", C.c_int), ("max_seq_len", C.c_int), ("q", _P),
                ("seq_lens", _P), ("cache_kind", C.c_int), ("k_cache", _P), ("v_cache", _P),
                ("block_table", _P), ("max_pages", C.c_int), ("num_pages", C.c_int), ("out", _P), ("lse", _P),
                ("workspace", _P), ("workspace_bytes", C.c_size_t), ("ev_kernel_begin", _P),
                ("ev_kernel_end", _P), ("cache_dtype", C.c_int), ("k_dequant", _P), ("v_dequant", _P),
                ("ring_slots", C.c_int), ("q_len", C.c_int)]


class MimoAppendArgs(C.Structure):
    _fields_ = [("num_tokens", C.c_int), ("num_kv_heads", C.c_int), ("head_dim_qk", C.c_int),
                ("head_dim_v", C.c_int), ("rope_dim", C.c_int), ("rope_base", C.c_double), ("k_new", _P),
                ("v_new", _P), ("pos", _P), ("seq_idx", _P), ("cache_kind", C.c_int), ("k_cache", _P),
                ("v_cache", _P), ("num_seqs", C.c_int), ("block_table", _P), ("max_pages", C.c_int),
                ("num_pages", C.c_int), ("cache_dtype", C.c_int), ("k_dequant", _P), ("v_dequant", _P),
                ("ring_slots", C.c_int)]


_lib = None


class MimoError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


def lib():
    """The loaded libmimoattn (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmimoattn is not built ({LIB_PATH} missing): run "
                               "python -m global_attention_attn_b200.build")
        L = C.CDLL(LIB_PATH)
        L.mimo_attn_prefill.argtypes = [C.POINTER(MimoPrefillArgs), _P]
        L.mimo_attn_prefill.restype = C.c_int
        L.mimo_attn_prefill_workspace_size.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int]
        L.mimo_attn_prefill_workspace_size.restype = C.c_size_t
        L.mimo_attn_prefill_stall_test.argtypes = [C.POINTER(MimoPrefillArgs), _P, C.c_ulonglong]
        L.mimo_attn_prefill_stall_test.restype = C.c_int
        L.mimo_attn_decode.argtypes = [C.POINTER(MimoDecodeArgs), _P]
        L.mimo_attn_decode.restype = C.c_int
        L.mimo_attn_decode_workspace_size.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int]
        L.mimo_attn_decode_workspace_size.restype = C.c_size_t
        L.mimo_attn_verify_workspace_size.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int]
        L.mimo_attn_verify_workspace_size.restype = C.c_size_t
        L.mimo_attn_decode_noalloc.argtypes = [C.POINTER(MimoDecodeArgs), _P]
        L.mimo_attn_decode_noalloc.restype = C.c_int
        L.mimo_kv_append.argtypes = [C.POINTER(MimoAppendArgs), _P]
        L.mimo_kv_append.restype = C.c_int
        L.mimo_last_error.argtypes = []
        L.mimo_last_error.restype = C.c_char_p
        L.mimo_status_poll.argtypes = [C.POINTER(C.c_uint32)]
        L.mimo_status_poll.restype = C.c_int
        L.mimo_version.argtypes = []
        L.mimo_version.restype = C.c_char_p
        L.mimo_window_from_left_right.argtypes = [C.c_int, C.c_int, C.POINTER(C.c_int)]
        L.mimo_window_from_left_right.restype = C.c_int
        _lib = L
    return _lib


def _check(rc: int):
    if rc != MIMO_OK:
        raise MimoError(rc, lib().mimo_last_error().decode())


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_layer(num_kv_heads: int, rope_base: float, window: int, sink=None, softmax_scale: float = SOFTMAX_SCALE,
               v_scale: float = V_SCALE) -> MimoLayer:
    L = MimoLayer()
    L.num_q_heads, L.num_kv_heads, L.head_dim_qk, L.head_dim_v, L.rope_dim = (NUM_Q_HEADS, num_kv_heads,
                                                                             HEAD_DIM_QK, HEAD_DIM_V, ROPE_DIM)
    L.rope_base, L.softmax_scale, L.v_scale, L.window = float(rope_base), float(softmax_scale), float(v_scale), int(window)
    L.sink = _ptr(sink)
    return L


def prefill_workspace_size(num_seqs: int, total_q: int, total_k: int, num_kv_heads: int, cache_kind: int) -> int:
    return int(lib().mimo_attn_prefill_workspace_size(num_seqs, total_q, total_k, num_kv_heads, cache_kind))


def decode_workspace_size(batch: int, max_seq_len: int, num_kv_heads: int, window: int, q_len: int = 1) -> int:
    if q_len == 1:
        return int(lib().mimo_attn_decode_workspace_size(batch, max_seq_len, num_kv_heads, window))
    return int(lib().mimo_attn_verify_workspace_size(batch, q_len, max_seq_len, num_kv_heads, window))


def _events(pair):
    """cudaEvent_t handles of a (begin, end) pair of torch.cuda.Event (None: no hooks)."""
    if pair is None:
        return None, None
    handles = [int(ev.cuda_event) for ev in pair]
    if len(handles) != 2 or not all(handles):
        raise ValueError("kernel_events: pass two torch.cuda.Event that have been recorded once")
    return handles[0], handles[1]


def mimo_attn_prefill(q, k, v, cu_seqlens_q, cu_seqlens_k, *, num_kv_heads: int, rope_base: float, window: int,
                      sink=None, cache_lens=None, cache_kind: int = MIMO_CACHE_NONE, k_cache=None, v_cache=None,
                      block_table=None, num_pages: int = 0, out=None, lse=None, workspace=None,
                      softmax_scale: float = SOFTMAX_SCALE, v_scale: float = V_SCALE, stream=None,
                      with_lse: bool = True, kernel_events=None, ring_slots: int = 0,
                      stall_test_wait_ns: int | None = None):
    """Varlen prefill (see include/mimoattn.h).  Tensors are CUDA tensors: q/k/v/caches bf16,
    index tensors int32, sink fp32.  kernel_events: optional (begin, end) pair of recorded-once
    torch.cuda.Event placed around the attention kernel.  ring_slots: slots per sequence of a
    ring cache (0 = 128).  stall_test_wait_ns: call mimo_attn_prefill_stall_test instead (the
    failure-detection test whose waits run out after that many ns).  Returns (out, lse)."""
    import torch
    total_q = q.shape[0]
    num_seqs = cu_seqlens_q.shape[0] - 1
    total_k = 0 if k is None else k.shape[0]
    if out is None:
        out = torch.empty((total_q, NUM_Q_HEADS, HEAD_DIM_V), dtype=torch.bfloat16, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty((total_q, NUM_Q_HEADS), dtype=torch.float32, device=q.device)
    need = prefill_workspace_size(num_seqs, total_q, total_k, num_kv_heads, cache_kind)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    a = MimoPrefillArgs()
    a.layer = make_layer(num_kv_heads, rope_base, window, sink, softmax_scale, v_scale)
    a.num_seqs, a.total_q, a.total_k = num_seqs, total_q, total_k
    a.q, a.k, a.v = _ptr(q), _ptr(k), _ptr(v)
    a.cu_seqlens_q, a.cu_seqlens_k, a.cache_lens = _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), _ptr(cache_lens)
    a.cache_kind = cache_kind
    a.k_cache, a.v_cache, a.block_table = _ptr(k_cache), _ptr(v_cache), _ptr(block_table)
    a.max_pages = 0 if block_table is None else block_table.shape[1]
    a.num_pages = num_pages
    a.out, a.lse = _ptr(out), _ptr(lse)
    a.workspace = _ptr(workspace)
    a.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a.ev_kernel_begin, a.ev_kernel_end = _events(kernel_events)
    a.ring_slots = int(ring_slots)
    if stall_test_wait_ns is not None:
        _check(lib().mimo_attn_prefill_stall_test(C.byref(a), _stream(stream), int(stall_test_wait_ns)))
    else:
        _check(lib().mimo_attn_prefill(C.byref(a), _stream(stream)))
    return out, lse


def mimo_attn_decode(q, seq_lens, *, max_seq_len: int, num_kv_heads: int, rope_base: float, window: int,
                     cache_kind: int, k_cache, v_cache, block_table=None, num_pages: int = 0, sink=None, out=None,
                     lse=None, workspace=None, softmax_scale: float = SOFTMAX_SCALE, v_scale: float = V_SCALE,
                     stream=None, with_lse: bool = True, kernel_events=None, cache_dtype: int = MIMO_DTYPE_BF16,
                     k_dequant=None, v_dequant=None, ring_slots: int = 0, q_len: int = 1):
    """Decode step (see include/mimoattn.h).  kernel_events as for mimo_attn_prefill (around the
    split kernel, not the combine).  ring_slots: slots per sequence of a ring cache (0 = 128).
    q_len: query tokens per sequence (draft tokens to verify; q holds batch * q_len rows).
    Returns (out, lse)."""
    import torch
    rows = q.shape[0]
    if rows % q_len:
        raise ValueError("q holds batch * q_len rows")
    B = rows // q_len
    if out is None:
        out = torch.empty((rows, NUM_Q_HEADS, HEAD_DIM_V), dtype=torch.bfloat16, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty((rows, NUM_Q_HEADS), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(B, max_seq_len, num_kv_heads, window, q_len)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    a = MimoDecodeArgs()
    a.layer = make_layer(num_kv_heads, rope_base, window, sink, softmax_scale, v_scale)
    a.batch, a.max_seq_len = B, int(max_seq_len)
    a.q, a.seq_lens = _ptr(q), _ptr(seq_lens)
    a.cache_kind = cache_kind
    a.k_cache, a.v_cache, a.block_table = _ptr(k_cache), _ptr(v_cache), _ptr(block_table)
    a.max_pages = 0 if block_table is None else block_table.shape[1]
    a.num_pages = num_pages
    a.out, a.lse = _ptr(out), _ptr(lse)
    a.workspace = _ptr(workspace)
    a.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a.ev_kernel_begin, a.ev_kernel_end = _events(kernel_events)
    a.cache_dtype, a.k_dequant, a.v_dequant = cache_dtype, _ptr(k_dequant), _ptr(v_dequant)
    a.ring_slots, a.q_len = int(ring_slots), int(q_len)
    _check(lib().mimo_attn_decode(C.byref(a), _stream(stream)))
    return out, lse


def mimo_attn_decode_noalloc(q, seq_lens, *, max_seq_len: int, num_kv_heads: int, rope_base: float, window: int,
                             cache_kind: int, k_cache, v_cache, out, lse=None, block_table=None, num_pages: int = 0,
                             sink=None, softmax_scale: float = SOFTMAX_SCALE, v_scale: float = V_SCALE, stream=None,
                             cache_dtype: int = MIMO_DTYPE_BF16, k_dequant=None, v_dequant=None, ring_slots: int = 0):
    """Decode that allocates nothing (see mimo_attn_decode_noalloc in include/mimoattn.h): the
    caller passes the output buffers; the split-KV partials go to the library's static
    device scratch (16 MiB), so concurrent calls must not overlap on the GPU."""
    a = MimoDecodeArgs()
    a.layer = make_layer(num_kv_heads, rope_base, window, sink, softmax_scale, v_scale)
    a.batch, a.max_seq_len = q.shape[0], int(max_seq_len)
    a.q, a.seq_lens = _ptr(q), _ptr(seq_lens)
    a.cache_kind = cache_kind
    a.k_cache, a.v_cache, a.block_table = _ptr(k_cache), _ptr(v_cache), _ptr(block_table)
    a.max_pages = 0 if block_table is None else block_table.shape[1]
    a.num_pages = num_pages
    a.out, a.lse = _ptr(out), _ptr(lse)
    a.cache_dtype, a.k_dequant, a.v_dequant = cache_dtype, _ptr(k_dequant), _ptr(v_dequant)
    a.ring_slots = int(ring_slots)
    _check(lib().mimo_attn_decode_noalloc(C.byref(a), _stream(stream)))
    return out, lse


def mimo_kv_append(k_new, v_new, pos, seq_idx, *, rope_base: float, cache_kind: int, k_cache, v_cache,
                   num_seqs: int, block_table=None, num_pages: int = 0, stream=None,
                   cache_dtype: int = MIMO_DTYPE_BF16, k_dequant=None, v_dequant=None, ring_slots: int = 0):
    """Rotate and store new keys/values into the ring or paged cache (see include/mimoattn.h);
    an E4M3 cache (cache_dtype) quantises with the per-KV-head scales k_dequant / v_dequant.
    ring_slots: slots per sequence of a ring cache (0 = 128)."""
    a = MimoAppendArgs()
    a.num_tokens, a.num_kv_heads = k_new.shape[0], k_new.shape[1]
    a.head_dim_qk, a.head_dim_v, a.rope_dim, a.rope_base = HEAD_DIM_QK, HEAD_DIM_V, ROPE_DIM, float(rope_base)
    a.k_new, a.v_new, a.pos, a.seq_idx = _ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(seq_idx)
    a.cache_kind = cache_kind
    a.k_cache, a.v_cache = _ptr(k_cache), _ptr(v_cache)
    a.num_seqs = num_seqs
    a.block_table = _ptr(block_table)
    a.max_pages = 0 if block_table is None else block_table.shape[1]
    a.num_pages = num_pages
    a.cache_dtype, a.k_dequant, a.v_dequant = cache_dtype, _ptr(k_dequant), _ptr(v_dequant)
    a.ring_slots = int(ring_slots)
    _check(lib().mimo_kv_append(C.byref(a), _stream(stream)))


def mimo_window_from_left_right(left: int, right: int = 0) -> int:
    """`window` (keys in total including the query) of the (left, right) window form:
    (128, 0) -> 129, (127, 0) -> 128, (-1, 0) -> 0 (global)."""
    w = C.c_int(0)
    _check(lib().mimo_window_from_left_right(int(left), int(right), C.byref(w)))
    return int(w.value)


def status_poll() -> int:
    """Reads and clears the device status word (synchronises the device)."""
    st = C.c_uint32(0)
    rc = lib().mimo_status_poll(C.byref(st))
    if rc not in (MIMO_OK, MIMO_ERR_TIMEOUT):
        _check(rc)
    return int(st.value)
