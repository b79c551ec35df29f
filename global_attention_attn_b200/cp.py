"""Context-parallel sliding-window prefill: the window-bounded K/V halo exchange.

Source: the "Model techniques map" page lists, under "training parallelism", a
window-bounded KV exchange under context parallelism (a label without details); the
radixark miles docs "MiMo-V2.6-Flash", section 5.1 "Parallelism", train that model
without context parallelism.  Reading taken here: every sequence is split into
contiguous chunks, chunk r on rank r of the process group.  A sliding-window query at
position p sees the keys p - W + 1 .. p (W <= 129 keys in total), so a rank needs the
rotated keys and the values of at most the 128 positions before its chunk, and nothing
else from any other rank.  That is exactly what the 128-slot ring cache of the chunked
prefill holds (position p of sequence s in slot p % 128), so the exchange moves one
ring per sequence to the next rank:

- when every local chunk holds at least 128 positions, a rank fills its outgoing ring
  from its own last 128 keys and all ranks swap rings in one round;
- otherwise the ring is relayed: a rank receives the ring of the positions before its
  chunk, appends its own keys to a copy and passes that on, so that a short chunk's
  outgoing ring also carries the positions of the chunks before it.

The rings are written by mimo_kv_append (RoPE at each key's position, the cache
format) and read by mimo_attn_prefill with the ring cache; only the point-to-point
transfers go through torch.distributed (NCCL between GPUs): 128 x Hkv x (384 + 256)
bytes per sequence and neighbour, 655 KB for the 8-KV-head layers.
"""
from __future__ import annotations

from typing import Callable, Sequence

import numpy as np

from . import (HEAD_DIM_QK, HEAD_DIM_V, MIMO_CACHE_RING, mimo_attn_prefill, mimo_kv_append)

RING = 128  # ring slots: the positions a window of <= 129 keys reaches before its query


def ring_buffers(num_seqs: int, num_kv_heads: int, device, dtype=None):
    """Zeroed ring caches [num_seqs, 128, Hkv, 192] and [num_seqs, 128, Hkv, 128]."""
    import torch
    dtype = torch.bfloat16 if dtype is None else dtype
    k = torch.zeros((num_seqs, RING, num_kv_heads, HEAD_DIM_QK), dtype=dtype, device=device)
    v = torch.zeros((num_seqs, RING, num_kv_heads, HEAD_DIM_V), dtype=dtype, device=device)
    return k, v


def tail_ranges(chunk_lens: Sequence[int], start_pos: Sequence[int]):
    """For each sequence: (first local row, first position, count) of the last
    min(n, 128) keys of its chunk, the ones a later chunk's window can reach."""
    out, off = [], 0
    for n, st in zip(chunk_lens, start_pos):
        m = min(int(n), RING)
        out.append((off + int(n) - m, int(st) + int(n) - m, m))
        off += int(n)
    return out


def fill_ring_tail(ring_k, ring_v, k, v, chunk_lens, start_pos, *, rope_base: float, stream=None):
    """Rotate and store the last min(n, 128) keys and values of each sequence's chunk into
    slot p % 128 of that sequence's ring (one mimo_kv_append per sequence)."""
    import torch
    for s, (row0, pos0, m) in enumerate(tail_ranges(chunk_lens, start_pos)):
        if m == 0:
            continue
        pos = torch.arange(pos0, pos0 + m, dtype=torch.int32, device=k.device)
        seq = torch.full((m,), s, dtype=torch.int32, device=k.device)
        mimo_kv_append(k[row0:row0 + m], v[row0:row0 + m], pos, seq, rope_base=rope_base,
                       cache_kind=MIMO_CACHE_RING, k_cache=ring_k, v_cache=ring_v,
                       num_seqs=ring_k.shape[0], stream=stream)


def chunks_fill_ring(chunk_lens: Sequence[int]) -> bool:
    """True when every local chunk alone covers the 128 positions a later window reaches,
    so the outgoing ring does not depend on the incoming one."""
    return all(int(n) >= RING for n in chunk_lens)


def outgoing_ring(recv_k, recv_v, send_k, send_v, fill: Callable, independent: bool):
    """The ring this rank passes on: its own last keys, on top of the incoming ring when
    its chunks are too short to cover the 128 positions alone."""
    if not independent:
        send_k.copy_(recv_k)
        send_v.copy_(recv_v)
    fill(send_k, send_v)


def exchange_halo(send_k, send_v, recv_k, recv_v, fill: Callable, *, independent: bool, group=None):
    """Receive the ring of the positions before this rank's chunks from rank - 1 into
    recv_k / recv_v, and send this rank's outgoing ring (built in send_k / send_v by
    `outgoing_ring`) to rank + 1.  Rank 0 receives nothing (its recv ring stays as given,
    zeros); the last rank sends nothing.  Every rank sends at most one message pair to its
    successor and receives at most one from its predecessor, so ranks in either mode pair
    up; relaying ranks wait for their predecessor, which never waits for a later rank."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    prev = dist.get_global_rank(group, rank - 1) if group is not None and rank > 0 else rank - 1
    nxt = dist.get_global_rank(group, rank + 1) if group is not None and rank + 1 < world else rank + 1
    if independent:
        if rank + 1 < world:
            outgoing_ring(recv_k, recv_v, send_k, send_v, fill, True)
        ops = []
        if rank + 1 < world:
            ops += [dist.P2POp(dist.isend, send_k, nxt, group), dist.P2POp(dist.isend, send_v, nxt, group)]
        if rank > 0:
            ops += [dist.P2POp(dist.irecv, recv_k, prev, group), dist.P2POp(dist.irecv, recv_v, prev, group)]
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()
        return
    if rank > 0:
        dist.recv(recv_k, prev, group)
        dist.recv(recv_v, prev, group)
    if rank + 1 < world:
        outgoing_ring(recv_k, recv_v, send_k, send_v, fill, False)
        dist.send(send_k, nxt, group)
        dist.send(send_v, nxt, group)


def prefill_with_halo(q, k, v, chunk_lens, start_pos, ring_k, ring_v, *, rope_base: float, window: int,
                      sink=None, out=None, lse=None, stream=None):
    """Sliding-window prefill of this rank's chunks (queries and keys at positions
    start .. start + n - 1 of each sequence) over the received ring."""
    import torch
    if not 1 <= window <= RING + 1:
        raise ValueError(f"a halo of {RING} positions serves windows of 1..{RING + 1} keys (got {window})")
    cu = torch.as_tensor(np.concatenate([[0], np.cumsum(np.asarray(chunk_lens, np.int64))]).astype(np.int32),
                         device=q.device)
    cache_lens = torch.as_tensor(np.asarray(start_pos, np.int32), device=q.device)
    return mimo_attn_prefill(q, k, v, cu, cu, num_kv_heads=k.shape[1], rope_base=rope_base, window=window,
                             sink=sink, cache_lens=cache_lens, cache_kind=MIMO_CACHE_RING, k_cache=ring_k,
                             v_cache=ring_v, out=out, lse=lse, stream=stream)


def swa_prefill_context_parallel(q, k, v, chunk_lens: Sequence[int], start_pos: Sequence[int], *,
                                 rope_base: float, window: int, sink=None, group=None, out=None, lse=None,
                                 stream=None):
    """This rank's part of a context-parallel sliding-window prefill.

    q [sum(chunk_lens), 64, 192], k [.., Hkv, 192], v [.., Hkv, 128] (pre-RoPE, bf16, on
    this rank's GPU) hold this rank's chunk of each sequence; chunk_lens and start_pos
    (host integers) give each chunk's length and first position.  Rank r's chunk of a
    sequence starts where rank r - 1's ends, and rank 0's at position 0.  Returns
    (out, lse) for the local rows."""
    import contextlib

    import torch.distributed as dist
    if dist.get_rank(group) == 0 and any(int(p) != 0 for p in start_pos):
        raise ValueError("rank 0 holds the first chunk of every sequence (start position 0)")
    rope_base = float(rope_base)
    num_seqs, hkv = len(chunk_lens), k.shape[1]
    # torch.distributed orders its transfers against the current stream, so every step
    # (zeroing the rings, the appends, the send / receive, the prefill) runs with `stream`
    # made current: the send then follows the append that fills the ring, and the prefill
    # follows the receive.  The caller orders q / k / v against `stream`.
    if stream is not None:
        import torch
        scope = torch.cuda.stream(stream)
    else:
        scope = contextlib.nullcontext()
    with scope:
        recv_k, recv_v = ring_buffers(num_seqs, hkv, q.device)
        send_k, send_v = ring_buffers(num_seqs, hkv, q.device)

        def fill(rk, rv):
            fill_ring_tail(rk, rv, k, v, chunk_lens, start_pos, rope_base=rope_base)

        exchange_halo(send_k, send_v, recv_k, recv_v, fill, independent=chunks_fill_ring(chunk_lens), group=group)
        return prefill_with_halo(q, k, v, chunk_lens, start_pos, recv_k, recv_v, rope_base=rope_base,
                                 window=window, sink=sink, out=out, lse=lse)
