"""Failure detection on the GPU without a GPU fault: the device status word.

- Bounded waits: mimo_attn_prefill_stall_test runs the prefill with its query tiles
  withheld (a barrier that nothing arrives on), so the kernel's waits run out after a
  short limit.  The call must end by itself, mimo_status_poll must return
  MIMO_ERR_TIMEOUT, and the next ordinary call must match the oracle (the stalled kernel
  freed its tensor memory and left no copy in flight).
- Indices outside a cache (a page id beyond the pool) are skipped by the kernels' own
  bounds checks and reported as MIMO_STATUS_BAD_INDEX; the other rows are unaffected.
- An E4M3 dequantisation scale that is not finite and positive is reported as
  MIMO_STATUS_BAD_SCALE and its rows are not written.
"""
import ctypes as C
import time

import numpy as np
import pytest

import oracle
from workloads import configs, synth

from .util import check_prefill, decode_cfg, dev_bf16, dev_f32, dev_i32, make_prefill, parity, prefill_cfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    import global_attention_attn_b200 as M
    M.lib()
    M.status_poll()
    yield


def poll():
    import global_attention_attn_b200 as M
    st = C.c_uint32(0)
    rc = M.lib().mimo_status_poll(C.byref(st))
    return rc, int(st.value)


@pytest.mark.parametrize("kind", ["swa", "global"])
def test_stalled_prefill_times_out_and_the_next_call_works(kind):
    import torch
    import global_attention_attn_b200 as M
    hkv, base, window = (8, 1e4, 128) if kind == "swa" else (4, 1e7, 0)
    cfg = make_prefill([700, 300], hkv, base, window, kind == "swa", 930 + hkv)
    assert poll() == (M.MIMO_OK, 0)
    t0 = time.perf_counter()
    prefill_cfg(cfg, stall_test_wait_ns=50_000_000)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    rc, st = poll()
    assert rc == M.MIMO_ERR_TIMEOUT and st & M.MIMO_STATUS_TIMEOUT, (rc, st)
    assert b"gave up" in M.lib().mimo_last_error()
    assert poll() == (M.MIMO_OK, 0)  # the poll cleared the word
    # every wait gave up within its limit (50 ms) plus the bounded drains of copies in flight
    assert dt < 3.0, dt
    # the context is intact: the same call without the stall matches the oracle
    check_prefill(cfg, what=f"{kind} prefill after a stalled call")
    assert poll() == (M.MIMO_OK, 0)


def test_stall_test_rejects_out_of_range_limits():
    import global_attention_attn_b200 as M
    cfg = make_prefill([16], 8, 1e4, 128, True, 935)
    for ns in (10, 10 ** 11):
        with pytest.raises(M.MimoError) as e:
            prefill_cfg(cfg, stall_test_wait_ns=ns)
        assert e.value.code == M.MIMO_ERR_INVALID_ARG


def test_append_skips_and_reports_pages_outside_the_pool():
    import torch
    import global_attention_attn_b200 as M
    n, hkv = 300, 4
    k = configs.bf16_normal(940, 1, (n, hkv, 192))
    v = configs.bf16_normal(940, 2, (n, hkv, 128))
    seq = (np.arange(n) % 2).astype(np.int32)
    pos = (np.arange(n) // 2).astype(np.int32)          # positions 0..149 of two sequences
    bt = np.array([[0, 1], [2, 3]], np.int32)
    bt[1, 1] = 7                                        # sequence 1's second page: not in the pool of 4
    kc = torch.zeros((4, 128, hkv, 192), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros((4, 128, hkv, 128), dtype=torch.bfloat16, device="cuda")
    M.mimo_kv_append(dev_bf16(k), dev_bf16(v), dev_i32(pos), dev_i32(seq), rope_base=1e7,
                     cache_kind=M.MIMO_CACHE_PAGED, k_cache=kc, v_cache=vc, num_seqs=2,
                     block_table=dev_i32(bt), num_pages=4)
    rc, st = poll()
    assert st == M.MIMO_STATUS_BAD_INDEX, st
    ko, vo = oracle.kv_append(k, v, pos, 1e7)
    vcn = vc.float().cpu().numpy()
    for t in range(n):
        s, p = int(seq[t]), int(pos[t])
        if s == 1 and p >= 128:
            continue                                     # skipped: its page is outside the pool
        np.testing.assert_array_equal(vcn[bt[s, p // 128], p % 128], vo[t].astype(np.float32))
    # nothing was written anywhere for the skipped tokens: page 3 (never referenced) stays zero
    assert not vcn[3].any()
    # a sequence index outside the ring and a negative position are skipped the same way
    rk = torch.zeros((2, 128, hkv, 192), dtype=torch.bfloat16, device="cuda")
    rv = torch.zeros((2, 128, hkv, 128), dtype=torch.bfloat16, device="cuda")
    M.mimo_kv_append(dev_bf16(k[:2]), dev_bf16(v[:2]), dev_i32([5, -1]), dev_i32([2, 0]), rope_base=1e4,
                     cache_kind=M.MIMO_CACHE_RING, k_cache=rk, v_cache=rv, num_seqs=2)
    assert poll()[1] == M.MIMO_STATUS_BAD_INDEX
    assert not rk.float().abs().sum().item() and not rv.float().abs().sum().item()


def test_decode_reports_a_page_outside_the_pool():
    """A block-table entry outside the pool: the kernel reads page 0 in its place and
    reports it; the other sequences are unaffected."""
    import torch
    import global_attention_attn_b200 as M
    _, gl = configs.decode_batch(seed=941, B=6, ctx_range=(300, 2000))
    bt = gl.block_table.copy()
    bt[2, 1] = gl.k_cache.shape[0] + 3
    gl.block_table = bt
    out, lse = decode_cfg(gl)
    assert poll()[1] == M.MIMO_STATUS_BAD_INDEX
    good = np.array([0, 1, 3, 4, 5])
    ro, rl = oracle.decode(gl, seqs=good)
    idx = torch.as_tensor(good, device=out.device)
    parity(out[idx], lse[idx], ro, rl, "decode, other sequences of a batch with a bad page id")


def test_fp8_append_skips_and_reports_bad_scales():
    import torch
    import global_attention_attn_b200 as M
    n, hkv = 64, 4
    k = configs.bf16_normal(942, 1, (n, hkv, 192))
    v = configs.bf16_normal(942, 2, (n, hkv, 128))
    kdq = np.array([0.5, 0.0, 1.0, 1.0], np.float32)        # head 1: zero key scale
    vdq = np.array([0.5, 1.0, np.inf, 1.0], np.float32)     # head 2: infinite value scale
    kc = torch.zeros((1, 128, hkv, 192), dtype=torch.uint8, device="cuda")
    vc = torch.zeros((1, 128, hkv, 128), dtype=torch.uint8, device="cuda")
    M.mimo_kv_append(dev_bf16(k), dev_bf16(v), dev_i32(np.arange(n)), dev_i32(np.zeros(n)), rope_base=1e4,
                     cache_kind=M.MIMO_CACHE_RING, k_cache=kc, v_cache=vc, num_seqs=1,
                     cache_dtype=M.MIMO_DTYPE_FP8_E4M3, k_dequant=dev_f32(kdq), v_dequant=dev_f32(vdq))
    assert poll()[1] == M.MIMO_STATUS_BAD_SCALE
    kb, vb = kc.cpu().numpy(), vc.cpu().numpy()
    assert not kb[0, :n, 1:3].any() and not vb[0, :n, 1:3].any()   # heads 1 and 2 skipped
    assert kb[0, :n, 0].any() and kb[0, :n, 3].any()               # heads 0 and 3 written
    assert not kb[0, n:].any()


def test_draft_rows_beyond_a_short_context_are_reported():
    """A context shorter than the draft rows (seq_lens below q_len) on the tensor-core draft path:
    reported as MIMO_STATUS_BAD_INDEX, nothing attended for it; the other sequences unaffected."""
    import torch
    import global_attention_attn_b200 as M
    _, gl = configs.decode_batch(seed=943, B=5, ctx_range=(600, 3000))
    cfg = configs.with_drafts(gl, 4, seed=944)
    ctx = cfg.ctx.copy()
    ctx[3] = 2
    L = cfg.layer
    out, lse = M.mimo_attn_decode(dev_bf16(cfg.q), dev_i32(ctx), max_seq_len=int(ctx.max()),
                                  num_kv_heads=4, rope_base=L.rope_base, window=0, k_cache=dev_bf16(cfg.k_cache),
                                  v_cache=dev_bf16(cfg.v_cache), cache_kind=M.MIMO_CACHE_PAGED,
                                  block_table=dev_i32(cfg.block_table), num_pages=cfg.k_cache.shape[0], q_len=4)
    assert poll()[1] == M.MIMO_STATUS_BAD_INDEX
    good = np.array([0, 1, 2, 4])
    ro, rl = oracle.decode(cfg, seqs=good)
    idx = torch.as_tensor(np.repeat(good, 4) * 4 + np.tile(np.arange(4), len(good)), device=out.device)
    parity(out[idx], lse[idx], ro, rl, "drafts, other sequences of a batch with a too-short context")
