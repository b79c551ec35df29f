"""Adapters from the seeded workloads (workloads.configs) to the oracle's layer description.

TEST INFRASTRUCTURE (see oracle/__init__.py).
"""
from __future__ import annotations

import numpy as np

from workloads.configs import DQK, DV, HQ, ROPE_DIM, SOFTMAX_SCALE, V_SCALE


def _layer_kw(layer):
    return dict(hq=HQ, hkv=layer.num_kv_heads, dqk=DQK, dv=DV, rope_dim=ROPE_DIM, rope_base=layer.rope_base,
                softmax_scale=SOFTMAX_SCALE, v_scale=V_SCALE, window=layer.window, sink=layer.sink)


def _rows_to_sel(cu, rows):
    """Global query rows -> (sequence, row within sequence)."""
    rows = np.asarray(rows, np.int64)
    seq = np.searchsorted(cu, rows, side="right") - 1
    return seq.astype(np.int32), (rows - cu[seq]).astype(np.int32)


def prefill(cfg, rows=None, nthreads=None, online=False):
    """Oracle for a contiguous varlen prefill (workloads.configs.Prefill).

    rows: global query rows to evaluate (default: all).  Returns (out, lse) for those rows."""
    from . import attention
    cu_q = cfg.cu_q.astype(np.int64)
    if rows is None:
        rows = np.arange(cu_q[-1])
    seq, r = _rows_to_sel(cu_q, rows)
    return attention(q=cfg.q, **_layer_kw(cfg.layer), q_row0=cfg.cu_q[:-1], q_len=cfg.q_lens, q_pos0=cfg.q_pos0,
                     sel_seq=seq, sel_row=r, k_new=cfg.k, v_new=cfg.v, new_row0=cfg.cu_k[:-1],
                     new_pos0=np.zeros(cfg.num_seqs, np.int32), new_len=cfg.k_lens, nthreads=nthreads,
                     online=online)


def decode(cfg, seqs=None, nthreads=None):
    """Oracle for a decode step (workloads.configs.Decode): q_len queries per sequence at
    positions ctx-q_len .. ctx-1, every key from the cache.  Returns the rows of the selected
    sequences in order (q_len rows each)."""
    from . import attention
    B = len(cfg.ctx)
    ql = int(getattr(cfg, "q_len", 1))
    if seqs is None:
        seqs = np.arange(B)
    seqs = np.asarray(seqs, np.int32)
    kw = dict(cache_kind=1, page_size=cfg.k_cache.shape[1], block_table=cfg.block_table) if cfg.paged else \
        dict(cache_kind=2, page_size=cfg.k_cache.shape[1])
    kw.update(cache_dtype=cfg.cache_dtype, k_dequant=cfg.k_dequant, v_dequant=cfg.v_dequant)
    return attention(q=cfg.q, **_layer_kw(cfg.layer), q_row0=(np.arange(B) * ql).astype(np.int32),
                     q_len=np.full(B, ql, np.int32), q_pos0=(cfg.ctx - ql).astype(np.int32),
                     sel_seq=np.repeat(seqs, ql), sel_row=np.tile(np.arange(ql, dtype=np.int32), len(seqs)),
                     new_row0=np.zeros(B, np.int32), new_pos0=cfg.ctx.astype(np.int32),
                     new_len=np.zeros(B, np.int32), k_cache=cfg.k_cache, v_cache=cfg.v_cache, nthreads=nthreads,
                     **kw)


def chunked(cfg, rows=None, nthreads=None):
    """Oracle for a chunked prefill (workloads.configs.Chunked): prefix keys from the cache
    (stored rotated), chunk keys from the raw pre-RoPE chunk arrays."""
    from . import attention
    cu = cfg.cu_new.astype(np.int64)
    if rows is None:
        rows = cfg.sample_rows if cfg.sample_rows is not None else np.arange(cu[-1])
    seq, r = _rows_to_sel(cu, rows)
    lens = np.diff(cfg.cu_new).astype(np.int32)
    kw = dict(cache_kind=1, page_size=cfg.k_cache.shape[1], block_table=cfg.block_table) if cfg.paged else \
        dict(cache_kind=2, page_size=cfg.k_cache.shape[1])
    return attention(q=cfg.q, **_layer_kw(cfg.layer), q_row0=cfg.cu_new[:-1], q_len=lens, q_pos0=cfg.start,
                     sel_seq=seq, sel_row=r, k_new=cfg.k_new, v_new=cfg.v_new, new_row0=cfg.cu_new[:-1],
                     new_pos0=cfg.start, new_len=lens, k_cache=cfg.k_cache, v_cache=cfg.v_cache,
                     nthreads=nthreads, **kw)
