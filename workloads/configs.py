"""The five seeded synthetic workloads of the MiMo-V2.6-Flash hybrid attention forward.

Shapes and distributions follow the layer as the model pages state it
(radixark miles docs "MiMo-V2.6-Flash", section 1 "Key highlights"): 64 query
heads, 192-dim Q/K, 128-dim V, partial RoPE on 64 dims, sliding-window layers
with window 128, 8 KV heads, RoPE base 1e4 and a per-head sink; global layers
with 4 KV heads and RoPE base 1e7.  All tensors are bf16 ~N(0,1) (uint16 bit
patterns), sinks are fp32 ~N(0,1).  Cached keys are synthetic values that are
treated as already rotated and are laid out in the library's cache format
(key dims 0..63 as IEEE fp16, dims 64..191 and values as bf16).  This module
draws numbers and lays them out; it computes nothing of the attention itself.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

from . import synth

HQ = 64
DQK = 192
DV = 128
ROPE_DIM = 64
WINDOW = 128
PAGE = 128
RING = 128
SOFTMAX_SCALE = 1.0 / np.sqrt(192.0)
V_SCALE = 0.707
BASE_SEED = 20261202


@dataclass
class Layer:
    kind: str            # "swa" or "global"
    num_kv_heads: int
    rope_base: float
    window: int          # keys in total incl. self; 0 = global causal
    sink: np.ndarray | None  # fp32 [HQ] or None

    @property
    def group(self) -> int:
        return HQ // self.num_kv_heads


def swa_layer(sink: np.ndarray | None) -> Layer:
    return Layer("swa", 8, 1.0e4, WINDOW, sink)


def global_layer() -> Layer:
    return Layer("global", 4, 1.0e7, 0, None)


def _normal_bf16_parallel(key: int, shape) -> np.ndarray:
    """Same values as synth.normal_bf16, drawn on a thread pool (numpy releases the GIL)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    step = 1 << 24
    starts = list(range(0, n, step))

    def work(lo):
        hi = min(n, lo + step)
        out[lo:hi] = synth.f64_to_bf16_bits(synth.normal_f64(synth.stream_seed(key, lo // step), hi - lo))

    if len(starts) <= 1:
        for lo in starts:
            work(lo)
    else:
        nthr = max(1, min(len(starts), len(os.sched_getaffinity(0))))
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(work, starts))
    return out.reshape(shape)


def bf16_normal(seed: int, tag: int, shape) -> np.ndarray:
    return _normal_bf16_parallel(synth.stream_seed(seed, tag), shape)


def fp8_codes(seed: int, tag: int, shape) -> np.ndarray:
    """Synthetic E4M3 cache bytes: sign and 3 mantissa bits uniform, exponent field uniform
    in 4..8, i.e. magnitudes (1 + m/8) * 2^(e-7) in [0.125, 3.75]."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint8)
    step = 1 << 24
    key = synth.stream_seed(seed, tag)

    def work(lo):
        hi = min(n, lo + step)
        u = synth.u64(synth.stream_seed(key, lo // step), hi - lo)
        e = (np.uint64(4) + (u >> np.uint64(4)) % np.uint64(5)).astype(np.uint8)
        out[lo:hi] = ((u & np.uint64(1)).astype(np.uint8) << 7) | (e << 3) | ((u >> np.uint64(1)) & np.uint64(7)).astype(np.uint8)

    with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(work, range(0, n, step)))
    return out.reshape(shape)


def cached_keys(seed: int, tag: int, shape) -> np.ndarray:
    """~N(0,1) key rows [..., 192] in the cache format: dims 0..63 (the rotated part)
    as IEEE fp16 bit patterns, dims 64..191 as bf16 bit patterns."""
    assert shape[-1] == DQK
    rows = int(np.prod(shape[:-1]))
    out = np.empty((rows, DQK), dtype=np.uint16)
    step = 1 << 16
    key = synth.stream_seed(seed, tag)

    def work(lo):
        hi = min(rows, lo + step)
        x = synth.normal_f64(synth.stream_seed(key, lo // step), (hi - lo) * DQK).reshape(hi - lo, DQK)
        out[lo:hi, :ROPE_DIM] = synth.f64_to_f16_bits(x[:, :ROPE_DIM])
        out[lo:hi, ROPE_DIM:] = synth.f64_to_bf16_bits(x[:, ROPE_DIM:])

    starts = list(range(0, rows, step))
    nthr = max(1, min(len(starts), len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(nthr) as ex:
        list(ex.map(work, starts))
    return out.reshape(shape)


@dataclass
class Prefill:
    """Varlen prefill over contiguous (pre-RoPE) K/V: query i of sequence s sits at
    position q_pos0[s] + i and key j at position j (bottom-right aligned)."""
    layer: Layer
    q: np.ndarray            # [total_q, HQ, DQK] bf16 bits
    k: np.ndarray            # [total_k, Hkv, DQK]
    v: np.ndarray            # [total_k, Hkv, DV]
    cu_q: np.ndarray         # int32 [B+1]
    cu_k: np.ndarray         # int32 [B+1]
    name: str = ""

    @property
    def num_seqs(self) -> int:
        return len(self.cu_q) - 1

    @property
    def q_lens(self) -> np.ndarray:
        return np.diff(self.cu_q)

    @property
    def k_lens(self) -> np.ndarray:
        return np.diff(self.cu_k)

    @property
    def q_pos0(self) -> np.ndarray:
        return (self.k_lens - self.q_lens).astype(np.int32)


@dataclass
class Decode:
    """q_len query tokens per sequence (one decode step, or draft tokens to verify): query
    row s * q_len + i at position ctx[s] - q_len + i, over a cache that already holds
    positions 0..ctx-1 (SWA: the last ring_slots of them in a ring)."""
    layer: Layer
    q: np.ndarray            # [B * q_len, HQ, DQK] (pre-RoPE)
    ctx: np.ndarray          # int32 [B]
    # ring cache (SWA): [B, RING, Hkv, D]; paged cache (global): [pages, PAGE, Hkv, D]
    k_cache: np.ndarray
    v_cache: np.ndarray
    block_table: np.ndarray | None = None   # int32 [B, max_pages] (paged only)
    name: str = ""
    cache_dtype: int = 0                     # 0: bf16 rows (fp16 rotated dims); 1: E4M3 bytes
    k_dequant: np.ndarray | None = None      # fp32 [Hkv] dequantisation scales (E4M3 caches)
    v_dequant: np.ndarray | None = None
    q_len: int = 1

    @property
    def paged(self) -> bool:
        return self.block_table is not None


@dataclass
class Chunked:
    """A chunk of new tokens at positions [start, start+n) of each sequence, whose
    prefix [0, start) sits in a cache (paged for global layers, ring for SWA)."""
    layer: Layer
    q: np.ndarray            # [total_new, HQ, DQK] (pre-RoPE)
    k_new: np.ndarray        # [total_new, Hkv, DQK] (pre-RoPE)
    v_new: np.ndarray        # [total_new, Hkv, DV]
    cu_new: np.ndarray       # int32 [B+1]
    start: np.ndarray        # int32 [B] position of the first new token
    k_cache: np.ndarray
    v_cache: np.ndarray
    block_table: np.ndarray | None = None   # paged only; covers start+n positions
    sample_rows: np.ndarray | None = None   # query rows checked against the oracle
    name: str = ""

    @property
    def paged(self) -> bool:
        return self.block_table is not None


def swa_prefill_s512(seed: int = BASE_SEED + 0) -> Prefill:
    """One SWA layer prefill, batch 1, seq 512."""
    S = 512
    L = swa_layer(synth.normal_f32(synth.stream_seed(seed, 4), (HQ,)))
    return Prefill(L, bf16_normal(seed, 1, (S, HQ, DQK)), bf16_normal(seed, 2, (S, 8, DQK)),
                   bf16_normal(seed, 3, (S, 8, DV)), np.array([0, S], np.int32),
                   np.array([0, S], np.int32), name="swa_prefill_s512")


def swa_varlen_lengths(seed: int = BASE_SEED + 1) -> np.ndarray:
    return synth.randint(synth.stream_seed(seed, 0), 8, 1024, 8192)


def swa_varlen_prefill(seed: int = BASE_SEED + 1) -> Prefill:
    """SWA layer varlen prefill: 8 sequences, lengths uniform in [1024, 8192]."""
    lens = swa_varlen_lengths(seed)
    cu = np.zeros(9, np.int32)
    cu[1:] = np.cumsum(lens)
    T = int(cu[-1])
    L = swa_layer(synth.normal_f32(synth.stream_seed(seed, 4), (HQ,)))
    return Prefill(L, bf16_normal(seed, 1, (T, HQ, DQK)), bf16_normal(seed, 2, (T, 8, DQK)),
                   bf16_normal(seed, 3, (T, 8, DV)), cu, cu.copy(), name="swa_varlen_prefill_8x[1024,8192]")


def global_causal_prefill(seed: int = BASE_SEED + 2, S: int = 16384) -> Prefill:
    """Global layer causal prefill, batch 1, seq 16384, no sink."""
    L = global_layer()
    return Prefill(L, bf16_normal(seed, 1, (S, HQ, DQK)), bf16_normal(seed, 2, (S, 4, DQK)),
                   bf16_normal(seed, 3, (S, 4, DV)), np.array([0, S], np.int32),
                   np.array([0, S], np.int32), name=f"global_prefill_s{S}")


def paged_layout(seed: int, tag: int, ctx: np.ndarray, extra_pool: int = 0):
    """Block tables for contexts `ctx`: the needed pages are a seeded permutation of a pool."""
    npages = (ctx + PAGE - 1) // PAGE
    total = int(npages.sum()) + extra_pool
    perm = synth.permutation(synth.stream_seed(seed, tag), total).astype(np.int32)
    maxp = int(npages.max())
    bt = np.zeros((len(ctx), maxp), np.int32)
    off = 0
    for s, n in enumerate(npages):
        bt[s, :n] = perm[off:off + n]
        off += n
    return bt, total


def decode_contexts(seed: int = BASE_SEED + 3, B: int = 64) -> np.ndarray:
    return synth.randint(synth.stream_seed(seed, 0), B, 4096, 65536).astype(np.int32)


def decode_batch(seed: int = BASE_SEED + 3, B: int = 64, ctx_range=(4096, 65536),
                 ring_slots: int = RING) -> tuple[Decode, Decode]:
    """Decode step, batch B: the SWA layer over a ring of `ring_slots` slots per sequence
    (128 by default; every slot holds a key), the global layer over a paged cache (page 128)
    with contexts uniform in ctx_range."""
    if ctx_range == (4096, 65536) and B == 64:
        ctx = decode_contexts(seed, B)
    else:
        ctx = synth.randint(synth.stream_seed(seed, 0), B, *ctx_range).astype(np.int32)
    Ls = swa_layer(synth.normal_f32(synth.stream_seed(seed, 4), (HQ,)))
    swa = Decode(Ls, bf16_normal(seed, 1, (B, HQ, DQK)), ctx,
                 cached_keys(seed, 2, (B, ring_slots, 8, DQK)), bf16_normal(seed, 3, (B, ring_slots, 8, DV)),
                 name=f"swa_decode_b{B}_ring{ring_slots}")
    bt, pool = paged_layout(seed, 10, ctx)
    Lg = global_layer()
    glb = Decode(Lg, bf16_normal(seed, 11, (B, HQ, DQK)), ctx,
                 cached_keys(seed, 12, (pool, PAGE, 4, DQK)), bf16_normal(seed, 13, (pool, PAGE, 4, DV)),
                 block_table=bt, name=f"global_decode_b{B}_paged128")
    return swa, glb


def verify(seed: int = BASE_SEED + 5, B: int = 64, q_len: int = 4, ctx_range=(4096, 65536),
           decode: Decode | None = None) -> tuple[Chunked, Chunked]:
    """Speculative-decoding verification: each sequence scores q_len draft tokens at
    positions [ctx - q_len, ctx) after a cached prefix of ctx - q_len tokens, for the
    global layer (paged cache, the drafts appended first) and the SWA layer (ring holding
    the 128 prefix positions before the drafts).  With `decode` (a global-layer Decode from
    `decode_batch`) its contexts, block tables and cache are reused; the drafts then overwrite
    the cache rows of the last q_len positions when they are appended."""
    if decode is None:
        ctx = synth.randint(synth.stream_seed(seed, 0), B, *ctx_range).astype(np.int32)
        bt, pool = paged_layout(seed, 10, ctx)
        kc = cached_keys(seed, 12, (pool, PAGE, 4, DQK))
        vc = bf16_normal(seed, 13, (pool, PAGE, 4, DV))
    else:
        ctx, bt, kc, vc = decode.ctx, decode.block_table, decode.k_cache, decode.v_cache
    B = len(ctx)
    assert int(ctx.min()) >= q_len
    start = (ctx - q_len).astype(np.int32)
    cu = (np.arange(B + 1) * q_len).astype(np.int32)
    n = B * q_len
    glb = Chunked(global_layer(), bf16_normal(seed, 1, (n, HQ, DQK)), bf16_normal(seed, 2, (n, 4, DQK)),
                  bf16_normal(seed, 3, (n, 4, DV)), cu, start, kc, vc, block_table=bt,
                  name=f"global_verify_b{B}_q{q_len}")
    # every ring slot holds a prefix position (slot p % 128 for p in [start - 128, start));
    # slots of positions below 0 are never visible
    Ls = swa_layer(synth.normal_f32(synth.stream_seed(seed, 24), (HQ,)))
    swa = Chunked(Ls, bf16_normal(seed, 21, (n, HQ, DQK)), bf16_normal(seed, 22, (n, 8, DQK)),
                  bf16_normal(seed, 23, (n, 8, DV)), cu, start, cached_keys(seed, 25, (B, RING, 8, DQK)),
                  bf16_normal(seed, 26, (B, RING, 8, DV)), name=f"swa_verify_b{B}_q{q_len}")
    return glb, swa


def decode_fp8(seed: int = BASE_SEED + 6, B: int = 64, ctx_range=(4096, 65536), ring: bool = False,
               ctx: np.ndarray | None = None) -> Decode:
    """Decode step over an E4M3 KV cache with per-KV-head scales: the global layer over a
    paged cache (contexts uniform in ctx_range, or `ctx`), or the SWA layer over the ring."""
    if ctx is None:
        ctx = synth.randint(synth.stream_seed(seed, 0), B, *ctx_range).astype(np.int32)
    B = len(ctx)
    if ring:
        L = swa_layer(synth.normal_f32(synth.stream_seed(seed, 4), (HQ,)))
        h, shape_k, shape_v, bt = 8, (B, RING, 8, DQK), (B, RING, 8, DV), None
    else:
        L = global_layer()
        bt, pool = paged_layout(seed, 10, ctx)
        h, shape_k, shape_v = 4, (pool, PAGE, 4, DQK), (pool, PAGE, 4, DV)
    ks = (0.5 + synth.uniform01(synth.stream_seed(seed, 7), h)).astype(np.float32)
    vs = (0.5 + synth.uniform01(synth.stream_seed(seed, 8), h)).astype(np.float32)
    return Decode(L, bf16_normal(seed, 1, (B, HQ, DQK)), ctx, fp8_codes(seed, 2, shape_k), fp8_codes(seed, 3, shape_v),
                  block_table=bt, name=f"{'swa' if ring else 'global'}_decode_b{B}_fp8", cache_dtype=1,
                  k_dequant=ks, v_dequant=vs)


def sample_rows(seed: int, n_total: int, n_sample: int, always=()) -> np.ndarray:
    always = [r for r in always if 0 <= r < n_total]
    perm = synth.permutation(synth.stream_seed(seed, 99), n_total)
    rows = list(dict.fromkeys(list(always) + [int(r) for r in perm]))[:max(n_sample, len(always))]
    return np.array(sorted(rows), np.int32)


def chunked_prefill(seed: int = BASE_SEED + 4, prefix: int = 120832, chunk: int = 8192,
            n_sample: int = 1024, ring_slots: int = RING) -> tuple[Chunked, Chunked]:
    """Chunked prefill: `chunk` new tokens after a `prefix`-token cached prefix, for the
    global layer (paged cache) and the matching SWA layer (a ring of `ring_slots` slots
    holding the prefix tail)."""
    start = np.array([prefix], np.int32)
    cu = np.array([0, chunk], np.int32)
    ctx = np.array([prefix + chunk], np.int32)
    bt, pool = paged_layout(seed, 10, ctx)
    Lg = global_layer()
    kc = np.zeros((pool, PAGE, 4, DQK), np.uint16)
    vc = np.zeros((pool, PAGE, 4, DV), np.uint16)
    # the prefix positions hold synthetic (already rotated) keys; the chunk's slots stay zero
    npre = (prefix + PAGE - 1) // PAGE
    pk = cached_keys(seed, 12, (npre * PAGE, 4, DQK))
    pv = bf16_normal(seed, 13, (npre * PAGE, 4, DV))
    for i in range(npre):
        n = min(PAGE, prefix - i * PAGE)
        kc[bt[0, i], :n] = pk[i * PAGE:i * PAGE + n]
        vc[bt[0, i], :n] = pv[i * PAGE:i * PAGE + n]
    rows = sample_rows(seed, chunk, n_sample, always=(0, 126, 127, 128, chunk - 1))
    glb = Chunked(Lg, bf16_normal(seed, 1, (chunk, HQ, DQK)), bf16_normal(seed, 2, (chunk, 4, DQK)),
                  bf16_normal(seed, 3, (chunk, 4, DV)), cu, start, kc, vc, block_table=bt,
                  sample_rows=rows, name=f"global_chunk_{chunk}_on_{prefix}")
    Ls = swa_layer(synth.normal_f32(synth.stream_seed(seed, 24), (HQ,)))
    ring_k = np.zeros((1, ring_slots, 8, DQK), np.uint16)
    ring_v = np.zeros((1, ring_slots, 8, DV), np.uint16)
    tail = min(prefix, ring_slots)
    tk = cached_keys(seed, 25, (tail, 8, DQK))
    tv = bf16_normal(seed, 26, (tail, 8, DV))
    for j in range(tail):
        p = prefix - tail + j
        ring_k[0, p % ring_slots] = tk[j]
        ring_v[0, p % ring_slots] = tv[j]
    swa = Chunked(Ls, bf16_normal(seed, 21, (chunk, HQ, DQK)), bf16_normal(seed, 22, (chunk, 8, DQK)),
                  bf16_normal(seed, 23, (chunk, 8, DV)), cu, start, ring_k, ring_v,
                  sample_rows=rows, name=f"swa_chunk_{chunk}_on_{prefix}")
    return glb, swa


def with_drafts(cfg: Decode, q_len: int, seed: int) -> Decode:
    """The same caches scored by q_len query tokens per sequence: fresh ~N(0,1) queries for
    the last q_len positions of every context (whose keys the cache already holds)."""
    import dataclasses
    B = len(cfg.ctx)
    assert int(cfg.ctx.min()) >= q_len
    return dataclasses.replace(cfg, q=bf16_normal(seed, 77, (B * q_len, HQ, DQK)), q_len=q_len,
                               name=f"{cfg.name}_q{q_len}")


def ring_from_chunk(cfg: Chunked, ring_slots: int) -> tuple[np.ndarray, np.ndarray]:
    """A ring of `ring_slots` slots holding the prefix tail of a sliding-window chunk (the
    positions its 128-slot ring holds, each moved to slot p % ring_slots); other slots zero."""
    B, R0 = cfg.k_cache.shape[0], cfg.k_cache.shape[1]
    rk = np.zeros((B, ring_slots) + cfg.k_cache.shape[2:], cfg.k_cache.dtype)
    rv = np.zeros((B, ring_slots) + cfg.v_cache.shape[2:], cfg.v_cache.dtype)
    for s in range(B):
        st = int(cfg.start[s])
        for p in range(max(0, st - R0), st):
            rk[s, p % ring_slots] = cfg.k_cache[s, p % R0]
            rv[s, p % ring_slots] = cfg.v_cache[s, p % R0]
    return rk, rv
