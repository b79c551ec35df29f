"""mimo_attn_decode_noalloc: decode for callers that cannot allocate device memory
(for instance code inside a CUDA graph capture, or a runtime that only owns a
fixed arena).  It must give the same results as mimo_attn_decode while using the
library's static scratch instead of a caller workspace.

This file is collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.
"""
import ctypes as C
import gc

import numpy as np
import pytest

import global_attention_attn_b200 as M
from workloads import configs

from .util import LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, dev_bf16, dev_f32, dev_i32, dev_u8, parity


def test_noalloc_rejects_oversize_before_touching_the_device():
    a = M.MimoDecodeArgs()
    a.layer = M.make_layer(4, 1e7, 0)
    a.batch, a.max_seq_len = 64, 65536          # partials far beyond the 16 MiB scratch
    fake = C.c_void_p(1 << 20)
    a.q = a.seq_lens = a.k_cache = a.v_cache = a.block_table = a.out = fake
    a.cache_kind, a.max_pages, a.num_pages = M.MIMO_CACHE_PAGED, 512, 4096
    assert M.decode_workspace_size(64, 65536, 4, 0) > M.DECODE_NOALLOC_MAX_BYTES
    assert M.lib().mimo_attn_decode_noalloc(C.byref(a), None) == M.MIMO_ERR_WORKSPACE
    assert b"static scratch" in M.lib().mimo_last_error()


def _case(seed, B, ctx_range, fp8=False):
    if fp8:
        gl = configs.decode_fp8(seed=seed, B=B, ctx_range=ctx_range)
        kc, vc = dev_u8(gl.k_cache), dev_u8(gl.v_cache)
        extra = dict(cache_dtype=M.MIMO_DTYPE_FP8_E4M3, k_dequant=dev_f32(gl.k_dequant),
                     v_dequant=dev_f32(gl.v_dequant))
    else:
        _, gl = configs.decode_batch(seed=seed, B=B, ctx_range=ctx_range)
        kc, vc = dev_bf16(gl.k_cache), dev_bf16(gl.v_cache)
        extra = {}
    L = gl.layer
    return dict(cfg=gl, q=dev_bf16(gl.q), ctx=dev_i32(gl.ctx), kc=kc, vc=vc, bt=dev_i32(gl.block_table),
                pool=gl.k_cache.shape[0], max_len=int(gl.ctx.max()), L=L, extra=extra)


def _kw(t):
    return dict(max_seq_len=t["max_len"], num_kv_heads=t["L"].num_kv_heads, rope_base=t["L"].rope_base,
                window=t["L"].window, cache_kind=M.MIMO_CACHE_PAGED, k_cache=t["kc"], v_cache=t["vc"],
                block_table=t["bt"], num_pages=t["pool"], sink=dev_f32(t["L"].sink), **t["extra"])


@pytest.mark.gpu
def test_noalloc_decode_matches_decode_on_two_calls(cuda_ok):
    """Two calls in a row with different sizes and cache formats (bf16, then E4M3): the
    second finds the first call's partials in the shared scratch and must not depend on
    them.  Each output equals mimo_attn_decode's with a caller workspace and the oracle's,
    and no device memory is taken: neither torch's allocator nor the device's free memory
    (which also sees a cudaMalloc inside the library) changes across a call."""
    import torch
    import oracle
    M.lib()
    cases = [_case(901, 8, (2000, 3000)), _case(902, 5, (700, 1500), fp8=True)]
    for t in cases:
        assert 0 < M.decode_workspace_size(t["q"].shape[0], t["max_len"], 4, 0) <= M.DECODE_NOALLOC_MAX_BYTES
    refs = [M.mimo_attn_decode(t["q"], t["ctx"], **_kw(t)) for t in cases]
    outs = []
    for t in cases:
        B = t["q"].shape[0]
        out = torch.empty((B, 64, 128), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, 64), dtype=torch.float32, device="cuda")
        kw = _kw(t)  # its device tensors exist before the measurement
        # no garbage collection inside the measured window: a collection there frees
        # earlier tensors and moves torch's count without the call having done anything
        gc.collect()
        gc.disable()
        try:
            torch.cuda.synchronize()
            before, free_before = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
            M.mimo_attn_decode_noalloc(t["q"], t["ctx"], out=out, lse=lse, **kw)
            torch.cuda.synchronize()
            after, free_after = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
        finally:
            gc.enable()
        assert after == before
        assert free_after == free_before
        outs.append((out, lse))
    for t, (ro, rl), (o, l) in zip(cases, refs, outs):
        d = (o.float() - ro.float()).abs()
        assert d.max().item() <= O_MAX_ABS and d.mean().item() <= O_MEAN_ABS
        assert (l - rl).abs().max().item() <= LSE_MAX_ABS
        parity(o, l, *oracle.decode(t["cfg"]), "no-alloc decode against the oracle")
    assert M.status_poll() == 0
