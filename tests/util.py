"""Shared helpers for the GPU parity tests: device copies of the seeded workloads,
calls through the C ABI, and the parity bar (the tolerances of the attention
output and LSE)."""
from __future__ import annotations

import numpy as np

# Parity bar for the bf16 output (fp32 accumulation) and the fp32 LSE.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def dev_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def dev_u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def dev_i32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.int32))).cuda()


def dev_f32(a):
    import torch
    return None if a is None else torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.float32))).cuda()


def host_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def parity(out, lse, ref_out, ref_lse, what=""):
    """Asserts the parity bar; returns (max_abs, mean_abs, lse_max_abs)."""
    o = host_f64(out).reshape(ref_out.shape)
    d = np.abs(o - ref_out)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    mx, mean = float(d.max()), float(d.mean())
    lmx = 0.0
    if lse is not None and ref_lse is not None:
        l = host_f64(lse).reshape(ref_lse.shape)
        lmx = float(np.abs(l - ref_lse).max())
    assert mx <= O_MAX_ABS, f"{what}: max abs err {mx:.3e} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: mean abs err {mean:.3e} > {O_MEAN_ABS}"
    assert lmx <= LSE_MAX_ABS, f"{what}: lse max abs err {lmx:.3e} > {LSE_MAX_ABS}"
    return mx, mean, lmx


def prefill_cfg(cfg, **kw):
    """GPU prefill of a workloads.configs.Prefill through the C ABI."""
    import global_attention_attn_b200 as M
    L = cfg.layer
    return M.mimo_attn_prefill(dev_bf16(cfg.q), dev_bf16(cfg.k), dev_bf16(cfg.v), dev_i32(cfg.cu_q),
                               dev_i32(cfg.cu_k), num_kv_heads=L.num_kv_heads, rope_base=L.rope_base,
                               window=L.window, sink=dev_f32(L.sink), **kw)


def decode_cfg(cfg, **kw):
    """GPU decode of a workloads.configs.Decode through the C ABI."""
    import global_attention_attn_b200 as M
    L = cfg.layer
    extra = {}
    if cfg.paged:
        extra = dict(cache_kind=M.MIMO_CACHE_PAGED, block_table=dev_i32(cfg.block_table),
                     num_pages=cfg.k_cache.shape[0])
    else:
        extra = dict(cache_kind=M.MIMO_CACHE_RING, ring_slots=cfg.k_cache.shape[1])
    if cfg.cache_dtype == M.MIMO_DTYPE_FP8_E4M3:
        kc, vc = dev_u8(cfg.k_cache), dev_u8(cfg.v_cache)
        extra.update(cache_dtype=cfg.cache_dtype, k_dequant=dev_f32(cfg.k_dequant), v_dequant=dev_f32(cfg.v_dequant))
    else:
        kc, vc = dev_bf16(cfg.k_cache), dev_bf16(cfg.v_cache)
    return M.mimo_attn_decode(dev_bf16(cfg.q), dev_i32(cfg.ctx), max_seq_len=int(cfg.ctx.max()),
                              num_kv_heads=L.num_kv_heads, rope_base=L.rope_base, window=L.window,
                              k_cache=kc, v_cache=vc, sink=dev_f32(L.sink), q_len=cfg.q_len, **extra, **kw)


def chunked_cfg(cfg):
    """GPU chunked prefill of a workloads.configs.Chunked: for a paged (global) layer the chunk
    is appended to the cache first and all keys come from the cache; for a ring (sliding)
    layer the prefix tail comes from the ring and the chunk keys from the new rows."""
    import global_attention_attn_b200 as M
    L = cfg.layer
    q = dev_bf16(cfg.q)
    cu = dev_i32(cfg.cu_new)
    if cfg.paged:
        kc, vc = dev_bf16(cfg.k_cache), dev_bf16(cfg.v_cache)
        n = int(cfg.cu_new[-1])
        seq = np.repeat(np.arange(len(cfg.start)), np.diff(cfg.cu_new)).astype(np.int32)
        pos = np.concatenate([cfg.start[s] + np.arange(cfg.cu_new[s + 1] - cfg.cu_new[s])
                              for s in range(len(cfg.start))]).astype(np.int32)
        bt = dev_i32(cfg.block_table)
        M.mimo_kv_append(dev_bf16(cfg.k_new), dev_bf16(cfg.v_new), dev_i32(pos), dev_i32(seq),
                         rope_base=L.rope_base, cache_kind=M.MIMO_CACHE_PAGED, k_cache=kc, v_cache=vc,
                         num_seqs=len(cfg.start), block_table=bt, num_pages=cfg.k_cache.shape[0])
        ctx = (cfg.start + np.diff(cfg.cu_new)).astype(np.int32)
        assert n == q.shape[0]
        return M.mimo_attn_prefill(q, None, None, cu, None, num_kv_heads=L.num_kv_heads, rope_base=L.rope_base,
                                   window=L.window, sink=dev_f32(L.sink), cache_lens=dev_i32(ctx),
                                   cache_kind=M.MIMO_CACHE_PAGED, k_cache=kc, v_cache=vc, block_table=bt,
                                   num_pages=cfg.k_cache.shape[0])
    return M.mimo_attn_prefill(q, dev_bf16(cfg.k_new), dev_bf16(cfg.v_new), cu, cu, num_kv_heads=L.num_kv_heads,
                               rope_base=L.rope_base, window=L.window, sink=dev_f32(L.sink),
                               cache_lens=dev_i32(cfg.start), cache_kind=M.MIMO_CACHE_RING,
                               k_cache=dev_bf16(cfg.k_cache), v_cache=dev_bf16(cfg.v_cache),
                               ring_slots=cfg.k_cache.shape[1])


def make_prefill(lens, hkv, base, window, sink, seed, klens=None):
    """A seeded contiguous varlen prefill (workloads.configs.Prefill): bf16 ~N(0,1) Q/K/V,
    optional ~N(0,1) sinks; queries bottom-right aligned to their keys."""
    from workloads import configs, synth
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    klens = lens if klens is None else klens
    cuk = np.concatenate([[0], np.cumsum(klens)]).astype(np.int32)
    q = configs.bf16_normal(seed, 1, (int(cu[-1]), 64, 192))
    k = configs.bf16_normal(seed, 2, (int(cuk[-1]), hkv, 192))
    v = configs.bf16_normal(seed, 3, (int(cuk[-1]), hkv, 128))
    s = synth.normal_f32(synth.stream_seed(seed, 4), (64,)) if sink else None
    return configs.Prefill(configs.Layer("swa" if window else "global", hkv, base, window, s), q, k, v, cu, cuk)


def check_prefill(cfg, rows=None, what="", **kw):
    """GPU prefill of cfg against the oracle on `rows` (default all); returns the errors."""
    import oracle
    out, lse = prefill_cfg(cfg, **kw)
    ro, rl = oracle.prefill(cfg, rows=rows)
    if rows is not None:
        import torch
        idx = torch.as_tensor(np.asarray(rows), dtype=torch.long, device=out.device)
        out, lse = out[idx], lse[idx]
    return parity(out, lse, ro, rl, what)


def verify_decode_cfg(cfg, ring_slots=144):
    """Draft verification through the decode kernel for a workloads.configs.Chunked whose new
    rows are q_len draft tokens per sequence: the drafts are appended to the cache (the paged
    cache, or a ring of ring_slots slots built from the chunk's prefix tail), then scored by
    one mimo_attn_decode with q_len query tokens per sequence.  Returns (out, lse) for the
    draft rows in order."""
    import global_attention_attn_b200 as M
    from workloads import configs
    L = cfg.layer
    lens = np.diff(cfg.cu_new)
    q_len = int(lens[0])
    assert np.all(lens == q_len)
    B = len(cfg.start)
    seq = np.repeat(np.arange(B), q_len).astype(np.int32)
    pos = (np.repeat(cfg.start, q_len) + np.tile(np.arange(q_len), B)).astype(np.int32)
    ctx = (cfg.start + q_len).astype(np.int32)
    if cfg.paged:
        kc, vc = dev_bf16(cfg.k_cache), dev_bf16(cfg.v_cache)
        extra = dict(cache_kind=M.MIMO_CACHE_PAGED, block_table=dev_i32(cfg.block_table),
                     num_pages=cfg.k_cache.shape[0])
    else:
        rk, rv = configs.ring_from_chunk(cfg, ring_slots)
        kc, vc = dev_bf16(rk), dev_bf16(rv)
        extra = dict(cache_kind=M.MIMO_CACHE_RING, ring_slots=ring_slots)
    M.mimo_kv_append(dev_bf16(cfg.k_new), dev_bf16(cfg.v_new), dev_i32(pos), dev_i32(seq), rope_base=L.rope_base,
                     k_cache=kc, v_cache=vc, num_seqs=B, **extra)
    return M.mimo_attn_decode(dev_bf16(cfg.q), dev_i32(ctx), max_seq_len=int(ctx.max()), num_kv_heads=L.num_kv_heads,
                              rope_base=L.rope_base, window=L.window, k_cache=kc, v_cache=vc, sink=dev_f32(L.sink),
                              q_len=q_len, **extra)
