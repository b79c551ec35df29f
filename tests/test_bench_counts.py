"""The bench's algorithmic FLOP and byte counts (every roofline fraction divides by them),
checked on CPU against brute-force counts of visible (query, key) pairs and against the
tensor sizes they stand for."""
import numpy as np
import pytest

import bench
from workloads import configs

FLOP_PER_PAIR = 2 * 192 + 2 * 128  # QK^T over 192 dims + PV over 128, per (query head, key)


def brute_pairs(q_pos, k_pos, window):
    """Visible (query, key) pairs of one sequence, by enumeration."""
    n = 0
    for p in q_pos:
        for t in k_pos:
            if t <= p and (window == 0 or p - t < window):
                n += 1
    return n


def small_prefill(qlens, klens, hkv, window):
    cu_q = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(klens)]).astype(np.int32)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    L = configs.Layer("swa" if window else "global", hkv, 1e4, window, None)
    z = lambda *s: np.zeros(s, np.uint16)
    return configs.Prefill(L, z(tq, 64, 192), z(tk, hkv, 192), z(tk, hkv, 128), cu_q, cu_k)


@pytest.mark.parametrize("qlens,klens,hkv,window", [
    ([7, 130, 1], [7, 130, 1], 8, 128),
    ([40, 17], [300, 17], 8, 128),      # queries at the end of longer key ranges
    ([33, 200], [400, 200], 4, 0),      # global causal
    ([50], [50], 8, 5),
    ([129], [129], 8, 129),
])
def test_prefill_counts_match_enumeration(qlens, klens, hkv, window):
    cfg = small_prefill(qlens, klens, hkv, window)
    pairs = sum(brute_pairs(range(kl - ql, kl), range(kl), window) for ql, kl in zip(qlens, klens))
    flops, by = bench.prefill_counts(cfg)
    assert flops == pairs * 64 * FLOP_PER_PAIR
    # Q read, O (bf16) and LSE (fp32) written once per query row and head; K and V read
    # once per KV head; the two cu_seqlens arrays
    tq, tk = sum(qlens), sum(klens)
    want = tq * 64 * 192 * 2 + tq * 64 * 128 * 2 + tq * 64 * 4 + tk * hkv * (192 + 128) * 2 \
        + 2 * (len(qlens) + 1) * 4
    assert by == want


def test_swa_prefill_s512_closed_form():
    # positions 0..511 with a 128-key window: sum_{p<128} (p + 1) + 384 * 128 = 57408 pairs
    flops, _ = bench.prefill_counts(configs.swa_prefill_s512())
    assert flops == 57408 * 64 * FLOP_PER_PAIR


def test_decode_counts_match_enumeration():
    sw, gl = configs.decode_batch(seed=5, B=6, ctx_range=(1, 400))
    for cfg in (sw, gl):
        L = cfg.layer
        keys = sum(brute_pairs([c - 1], range(c), L.window) for c in cfg.ctx)
        flops, by = bench.decode_counts(cfg)
        assert flops == keys * 64 * FLOP_PER_PAIR
        want = keys * L.num_kv_heads * (192 + 128) * 2 + len(cfg.ctx) * (64 * (192 + 128) * 2 + 64 * 4 + 4)
        if cfg.paged:
            want += int(sum((c + 127) // 128 for c in cfg.ctx)) * 4  # block-table entries read
        assert by == want


def test_chunked_counts_match_enumeration():
    glb, swa = configs.chunked_prefill(seed=7, prefix=300, chunk=200, n_sample=4)
    for cfg in (glb, swa):
        L = cfg.layer
        st, n = int(cfg.start[0]), int(np.diff(cfg.cu_new)[0])
        pairs = brute_pairs(range(st, st + n), range(st + n), L.window)
        flops, by = bench.chunked_counts(cfg)
        assert flops == pairs * 64 * FLOP_PER_PAIR
        # keys the chunk attends: all st + n (global), or the chunk plus the window - 1
        # positions before it (sliding)
        keys = st + n if not L.window else min(st + n, n + L.window - 1)
        want = n * 64 * (192 * 2 + 128 * 2 + 4) + keys * L.num_kv_heads * (192 + 128) * 2
        if cfg.paged:
            want += n * L.num_kv_heads * (192 + 128) * 2 * 2  # the append: read and write
        assert by == want


def test_verify_counts_match_enumeration():
    """Draft verification through the decode kernel: every draft row's visible keys, the keys
    the drafts attend read once per KV head, queries and outputs once, and the drafts' append
    (read and written) for both layer kinds."""
    glb, swa = configs.verify(seed=9, B=5, q_len=4, ctx_range=(5, 700))
    for cfg in (glb, swa):
        L = cfg.layer
        pairs = keys = 0
        for s, st in enumerate(cfg.start):
            st = int(st)
            pairs += brute_pairs(range(st, st + 4), range(st + 4), L.window)
            keys += st + 4 if not L.window else min(st + 4, 4 + L.window - 1)
        flops, by = bench.verify_counts(cfg)
        assert flops == pairs * 64 * FLOP_PER_PAIR
        n = 5 * 4
        want = n * 64 * (192 * 2 + 128 * 2 + 4) + keys * L.num_kv_heads * (192 + 128) * 2 \
            + n * L.num_kv_heads * (192 + 128) * 2 * 2
        assert by == want
