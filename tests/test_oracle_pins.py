"""Pins for the float64 oracle: values the pages print, closed forms, invariants,
reductions to library routines and brute force on tiny inputs.

Each test is chosen so that a plausible mistake in the oracle (a dropped sink
term, a wrong rotation pairing or frequency, an off-by-one window, a wrong GQA
head map, a transposed operand, wrong cache indexing) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import configs, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(key, shape, scale=1.0):
    x = synth.normal_f64(key, int(np.prod(shape))) * scale
    return synth.f64_to_bf16_bits(x).reshape(shape)


def widen(b):
    return synth.bf16_bits_to_f32(b).astype(np.float64)


def tiny(seed=1, S=20, hq=4, hkv=2, dqk=16, dv=8, rope_dim=8, sink=False):
    q = bf16(synth.stream_seed(seed, 1), (S, hq, dqk))
    k = bf16(synth.stream_seed(seed, 2), (S, hkv, dqk))
    v = bf16(synth.stream_seed(seed, 3), (S, hkv, dv))
    s = synth.normal_f32(synth.stream_seed(seed, 4), (hq,)) if sink else None
    return q, k, v, s


def run(q, k, v, sink, *, hq, hkv, dqk, dv, rope_dim, base=100.0, window=0, scale=None, v_scale=0.707,
        q_pos0=0, online=False, rows=None):
    """Single-sequence prefill through the oracle: keys at positions q_pos0-(Sk-Sq) ... ."""
    Sq, Sk = q.shape[0], k.shape[0]
    scale = 1.0 / math.sqrt(dqk) if scale is None else scale
    rows = np.arange(Sq) if rows is None else np.asarray(rows)
    kpos0 = q_pos0 - (Sk - Sq)
    return oracle.attention(q=q, hq=hq, hkv=hkv, dqk=dqk, dv=dv, rope_dim=rope_dim, rope_base=base,
                            softmax_scale=scale, v_scale=v_scale, window=window, sink=sink,
                            q_row0=[0], q_len=[Sq], q_pos0=[q_pos0], sel_seq=np.zeros(len(rows), np.int32),
                            sel_row=rows, k_new=k, v_new=v, new_row0=[0], new_pos0=[kpos0], new_len=[Sk],
                            online=online)


def rotated(x, positions, base, rope_dim):
    """float64 rotated copy of [S, H, D] bf16 bits using oracle.rope (pinned below)."""
    xf = widen(x)
    out = np.empty_like(xf)
    for i, p in enumerate(positions):
        for h in range(x.shape[1]):
            out[i, h] = oracle.rope(xf[i, h], p, base, rope_dim)
    return out


# ----------------------------------------------------------------------------- RoPE

def test_rope_golden_cos_200000():
    """Page value: cos(200000) = 0.9974 in the fastest rotary dimension (angle = position)."""
    kv = {}
    for line in open(os.path.join(GOLDEN, "rope_cos_200000.txt")):
        if line.strip() and not line.startswith("#"):
            a, b = line.split()
            kv[a] = b
    x = np.zeros(192)
    x[0] = 1.0
    for base in (1.0e4, 1.0e7):
        y = oracle.rope(x, float(kv["position"]), base, 64)
        assert round(y[0], int(kv["decimals"])) == float(kv["dim0"])
        # the partner of dim 0 is dim 32 (rotate-half), and it carries the sine
        assert abs(y[32] - math.sin(200000.0)) < 1e-9
        assert np.all(y[1:32] == 0) and np.all(y[33:] == 0)


def test_rope_two_pair_hand_example():
    """rope_dim 4, base 100: pairs (0,2) at angle p and (1,3) at angle p * 100^(-1/2) = p/10."""
    x = np.array([1.0, 2.0, 3.0, 4.0, 5.0])
    y = oracle.rope(x, 1.0, 100.0, 4)
    c1, s1, c2, s2 = math.cos(1.0), math.sin(1.0), math.cos(0.1), math.sin(0.1)
    expect = [1 * c1 - 3 * s1, 2 * c2 - 4 * s2, 3 * c1 + 1 * s1, 4 * c2 + 2 * s2, 5.0]
    np.testing.assert_allclose(y, expect, rtol=0, atol=1e-14)


def test_rope_invariants():
    x = widen(bf16(7, (192,)))
    np.testing.assert_array_equal(oracle.rope(x, 0.0, 1e4, 64), x)          # position 0 is the identity
    y = oracle.rope(x, 12345.0, 1e4, 64)
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12               # rotation preserves the norm
    np.testing.assert_array_equal(y[64:], x[64:])                           # dims 64..191 pass through
    # relative position: <R(a)x, R(b)y> depends only on a - b
    z = widen(bf16(8, (192,)))
    d1 = oracle.rope(x, 1000.0, 1e7, 64) @ oracle.rope(z, 900.0, 1e7, 64)
    d2 = oracle.rope(x, 51000.0, 1e7, 64) @ oracle.rope(z, 50900.0, 1e7, 64)
    assert abs(d1 - d2) < 1e-9


# ----------------------------------------------------------------------------- library reductions

def _sdpa_reference(q, k, v, sink, *, hq, hkv, rope_dim, base, window, scale, v_scale, q_pos0=None):
    """torch scaled_dot_product_attention (float64) on oracle-rotated inputs.  The sink is an
    extra key whose logit is the additive mask value sink_h and whose value is zero."""
    Sq, Sk = q.shape[0], k.shape[0]
    q_pos0 = Sk - Sq if q_pos0 is None else q_pos0
    qpos = np.arange(Sq) + q_pos0
    kpos = np.arange(Sk) + (q_pos0 - (Sk - Sq))
    qr = torch.from_numpy(rotated(q, qpos, base, rope_dim)).permute(1, 0, 2)          # [H, Sq, D]
    kr = torch.from_numpy(rotated(k, kpos, base, rope_dim)).permute(1, 0, 2)
    vv = torch.from_numpy(widen(v)).permute(1, 0, 2)
    G = hq // hkv
    kr = kr.repeat_interleave(G, dim=0)
    vv = vv.repeat_interleave(G, dim=0)
    vis = (kpos[None, :] <= qpos[:, None])
    if window:
        vis &= (qpos[:, None] - kpos[None, :]) < window
    mask = torch.full((hq, Sq, Sk), float("-inf"), dtype=torch.float64)
    mask[:, torch.from_numpy(vis)] = 0.0
    if sink is not None:
        kr = torch.cat([kr, torch.zeros(hq, 1, kr.shape[2], dtype=torch.float64)], 1)
        vv = torch.cat([vv, torch.zeros(hq, 1, vv.shape[2], dtype=torch.float64)], 1)
        col = torch.from_numpy(sink.astype(np.float64))[:, None, None].expand(hq, Sq, 1)
        mask = torch.cat([mask, col], 2)
    o = torch.nn.functional.scaled_dot_product_attention(qr, kr, vv, attn_mask=mask, scale=scale)
    logits = scale * qr @ kr.transpose(1, 2) + mask
    lse = torch.logsumexp(logits, dim=-1)
    return (v_scale * o).permute(1, 0, 2).numpy(), lse.permute(1, 0).numpy()


@pytest.mark.parametrize("window,sink,Sq", [(0, False, 20), (5, True, 20), (0, True, 7), (128, True, 20)])
def test_matches_torch_sdpa(window, sink, Sq):
    dims = dict(hq=8, hkv=2, dqk=16, dv=8, rope_dim=8)
    q, k, v, s = tiny(seed=11 + window, S=20, sink=sink, **dims)
    q = q[:Sq]
    out, lse = run(q, k, v, s, base=100.0, window=window, q_pos0=20 - Sq, **dims)
    ro, rl = _sdpa_reference(q, k, v, s, base=100.0, window=window, scale=1 / 4.0, v_scale=0.707,
                             hq=8, hkv=2, rope_dim=8)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_brute_force_tiny():
    """Pure-Python loops over a full mask matrix with the sink as a last column, S = 6."""
    hq, hkv, dqk, dv, R = 2, 1, 4, 3, 2
    q, k, v, s = tiny(seed=5, S=6, hq=hq, hkv=hkv, dqk=dqk, dv=dv, rope_dim=R, sink=True)
    out, lse = run(q, k, v, s, hq=hq, hkv=hkv, dqk=dqk, dv=dv, rope_dim=R, base=10.0, window=3, scale=0.5,
                   v_scale=0.707)
    qf, kf, vf = widen(q), widen(k), widen(v)
    for i in range(6):
        for h in range(hq):
            def rot(x, p):  # rope_dim 2: one pair (0, 1), angle p
                return [x[0] * math.cos(p) - x[1] * math.sin(p), x[1] * math.cos(p) + x[0] * math.sin(p), x[2], x[3]]
            qi = rot(qf[i, h], i)
            cols = []
            for t in range(6):
                kt = rot(kf[t, 0], t)
                cols.append(0.5 * sum(a * b for a, b in zip(qi, kt)) if (t <= i and i - t < 3) else -math.inf)
            cols.append(float(s[h]))
            mx = max(cols)
            e = [math.exp(c - mx) for c in cols]
            Z = sum(e)
            for d in range(dv):
                o = sum(e[t] * vf[t, 0, d] for t in range(6)) / Z * 0.707
                assert abs(out[i, h, d] - o) < 1e-12
            assert abs(lse[i, h] - (mx + math.log(Z))) < 1e-12


# ----------------------------------------------------------------------------- closed forms

def test_zero_query_gives_uniform_weights():
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=8)
    q, k, v, s = tiny(seed=3, S=40, sink=True, **dims)
    q[:] = 0
    out, lse = run(q, k, v, s, window=16, **dims)
    vf = widen(v)
    for i in range(40):
        lo = max(0, i - 15)
        n = i - lo + 1
        for h in range(4):
            g = h // 2
            expect = 0.707 * vf[lo:i + 1, g].sum(0) / (n + math.exp(s[h]))
            np.testing.assert_allclose(out[i, h], expect, atol=1e-13)
            assert abs(lse[i, h] - math.log(n + math.exp(s[h]))) < 1e-13


def test_constant_value_and_single_key():
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=8)
    q, k, v, s = tiny(seed=4, S=30, sink=True, **dims)
    c = synth.f64_to_bf16_bits(np.array([1.5]))[0]
    v[:] = c
    out, lse = run(q, k, v, s, window=8, **dims)
    # V == c everywhere: o = 0.707 c (1 - exp(sink - lse))
    np.testing.assert_allclose(out, 0.707 * 1.5 * (1 - np.exp(s[None, :] - lse))[:, :, None] *
                               np.ones((1, 1, 8)), atol=1e-13)
    # first position, no sink: exactly the value of key 0 times 0.707, lse = scale q.k
    q2, k2, v2, _ = tiny(seed=5, S=30, **dims)
    out2, lse2 = run(q2, k2, v2, None, **dims)
    np.testing.assert_allclose(out2[0], 0.707 * widen(v2)[0].repeat(2, axis=0), atol=1e-15)
    # key and query both at position 0 are unrotated
    dot = (widen(q2)[0] * widen(k2)[0].repeat(2, axis=0)).sum(-1) / 4.0
    np.testing.assert_allclose(lse2[0], dot, atol=1e-13)


def test_large_sink_suppresses_output():
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=8)
    q, k, v, _ = tiny(seed=6, S=10, **dims)
    s = np.full(4, 80.0, np.float32)
    out, lse = run(q, k, v, s, window=4, **dims)
    assert np.abs(out).max() < 1e-25
    np.testing.assert_allclose(lse, 80.0, atol=1e-20)


def test_no_sink_equals_very_negative_sink():
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=8)
    q, k, v, _ = tiny(seed=9, S=25, **dims)
    o1, l1 = run(q, k, v, None, window=8, **dims)
    o2, l2 = run(q, k, v, np.full(4, -1.0e4, np.float32), window=8, **dims)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


# ----------------------------------------------------------------------------- window / GQA invariants

@pytest.mark.parametrize("W", [128, 129])
def test_window_sees_exactly_min_pos_plus_one_W_keys(W):
    """W = 128 keys in total (HF / Megatron-Bridge) or 129 (SGLang's (128, 0) window,
    radixark miles docs "MiMo-V2.6-Flash", section 5.4): the key at distance W - 1 is
    visible, the one at distance W is not."""
    dims = dict(hq=2, hkv=1, dqk=8, dv=4, rope_dim=4)
    q, k, v, s = tiny(seed=12, S=300, sink=True, **dims)
    base_out, _ = run(q, k, v, s, window=W, **dims)
    i = 250
    for dist, changes in [(W - 2, True), (W - 1, True), (W, False), (W + 1, False), (0, True)]:
        v2 = v.copy()
        v2[i - dist] = synth.f64_to_bf16_bits(widen(v2[i - dist]) + 3.0)
        o, _ = run(q, k, v2, s, window=W, rows=[i], **dims)
        assert (np.abs(o[0] - base_out[i]).max() > 1e-6) == changes, dist
    # a key after the query is never visible
    v2 = v.copy()
    v2[i + 1] = synth.f64_to_bf16_bits(widen(v2[i + 1]) + 3.0)
    o, _ = run(q, k, v2, s, window=W, rows=[i], **dims)
    assert np.abs(o[0] - base_out[i]).max() == 0
    # early positions see pos + 1 keys: zero query -> lse = ln(min(pos + 1, W) + e^s)
    q0 = q.copy()
    q0[:] = 0
    _, l = run(q0, k, v, s, window=W, **dims)
    for p in (0, 1, 126, 127, 128, 129, 299):
        assert abs(l[p, 0] - math.log(min(p + 1, W) + math.exp(s[0]))) < 1e-12


def test_window_at_least_sequence_is_global():
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=8)
    q, k, v, s = tiny(seed=13, S=50, sink=True, **dims)
    o1, l1 = run(q, k, v, s, window=0, **dims)
    o2, l2 = run(q, k, v, s, window=50, **dims)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_gqa_group_reads_its_own_kv_head():
    dims = dict(hq=8, hkv=2, dqk=16, dv=8, rope_dim=8)
    q, k, v, s = tiny(seed=14, S=24, sink=True, **dims)
    o1, _ = run(q, k, v, s, window=8, **dims)
    k2 = k.copy()
    k2[:, 1] = bf16(99, (24, 16))
    o2, _ = run(q, k2, v, s, window=8, **dims)
    d = np.abs(o1 - o2).max(axis=(0, 2))
    assert np.all(d[:4] == 0) and np.all(d[4:] > 1e-6)   # heads 0-3 -> kv 0, heads 4-7 -> kv 1


def test_position_shift_invariance():
    """Shifting every position by a constant leaves windowed attention unchanged (RoPE is relative)."""
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=8)
    q, k, v, s = tiny(seed=15, S=38, sink=True, **dims)
    q = q[8:]                       # 30 queries, each with a full 8-key window of existing keys
    o1, l1 = run(q, k, v, s, window=8, q_pos0=8, **dims)
    o2, l2 = run(q, k, v, s, window=8, q_pos0=70008, **dims)
    np.testing.assert_allclose(o1, o2, atol=1e-9)
    np.testing.assert_allclose(l1, l2, atol=1e-9)


def test_streaming_form_equals_definition():
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=8)
    for window, sink in [(0, False), (8, True)]:
        q, k, v, s = tiny(seed=16, S=64, sink=sink, **dims)
        o1, l1 = run(q, k, v, s, window=window, **dims)
        o2, l2 = run(q, k, v, s, window=window, online=True, **dims)
        np.testing.assert_allclose(o1, o2, atol=1e-12)
        np.testing.assert_allclose(l1, l2, atol=1e-12)


# ----------------------------------------------------------------------------- cache paths

def _cache_from(k, v, kind, page, B=1, perm_seed=0):
    """Lay rows of sequence 0 into a ring (kind 2) or a permuted paged pool (kind 1)."""
    S, hkv, dqk = k.shape
    if kind == 2:
        kc = np.zeros((1, page, hkv, dqk), np.uint16)
        vc = np.zeros((1, page, hkv, v.shape[2]), np.uint16)
        for p in range(max(0, S - page), S):
            kc[0, p % page], vc[0, p % page] = k[p], v[p]
        return kc, vc, None
    npg = (S + page - 1) // page
    pool = npg + 3
    perm = synth.permutation(perm_seed + 1, pool)[:npg].astype(np.int32)
    kc = np.zeros((pool, page, hkv, dqk), np.uint16)
    vc = np.zeros((pool, page, hkv, v.shape[2]), np.uint16)
    for p in range(S):
        kc[perm[p // page], p % page], vc[perm[p // page], p % page] = k[p], v[p]
    return kc, vc, perm[None, :]


@pytest.mark.parametrize("kind,window", [(2, 8), (1, 0), (1, 8)])
def test_decode_and_chunk_from_cache_equal_prefill_rows(kind, window):
    """rope_dim 0 so that cached and fresh keys hold identical values: decode of the
    last token and a chunk over a cached prefix must equal the matching prefill rows."""
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=0)
    S, page = 37, 8
    q, k, v, s = tiny(seed=17, S=S, sink=window > 0, **dims)
    full, full_lse = run(q, k, v, s, window=window, **dims)
    kc, vc, bt = _cache_from(k, v, kind, page)
    common = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=0, rope_base=1.0, softmax_scale=0.25, v_scale=0.707,
                  window=window, sink=s, cache_kind=kind, k_cache=kc, v_cache=vc, page_size=page, block_table=bt)
    # decode: query = last token, all keys from the cache
    o, l = oracle.attention(q=q[S - 1:], q_row0=[0], q_len=[1], q_pos0=[S - 1], sel_seq=[0], sel_row=[0],
                            new_pos0=[S], new_len=[0], **common)
    np.testing.assert_allclose(o[0], full[S - 1], atol=1e-13)
    np.testing.assert_allclose(l[0], full_lse[S - 1], atol=1e-13)
    if kind == 2:
        return
    # chunk: the last 13 tokens fresh, the prefix from the paged cache
    c0 = S - 13
    o, l = oracle.attention(q=q[c0:], q_row0=[0], q_len=[13], q_pos0=[c0], sel_seq=np.zeros(13, np.int32),
                            sel_row=np.arange(13), k_new=k[c0:], v_new=v[c0:], new_row0=[0], new_pos0=[c0],
                            new_len=[13], **common)
    np.testing.assert_allclose(o, full[c0:], atol=1e-13)
    np.testing.assert_allclose(l, full_lse[c0:], atol=1e-13)


def test_page_permutation_invariance():
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=8)
    q, k, v, _ = tiny(seed=18, S=29, **dims)
    res = []
    for ps in (0, 5):
        kc, vc, bt = _cache_from(k, v, 1, 4, perm_seed=ps)
        res.append(oracle.attention(q=q[28:], hq=4, hkv=2, dqk=16, dv=8, rope_dim=8, rope_base=1e4,
                                    softmax_scale=0.25, v_scale=0.707, window=0, sink=None, q_row0=[0],
                                    q_len=[1], q_pos0=[28], sel_seq=[0], sel_row=[0], new_pos0=[29],
                                    new_len=[0], cache_kind=1, k_cache=kc, v_cache=vc, page_size=4,
                                    block_table=bt))
    np.testing.assert_array_equal(res[0][0], res[1][0])


def test_varlen_equals_separate_calls():
    dims = dict(hq=4, hkv=2, dqk=16, dv=8, rope_dim=8)
    lens = [5, 17, 9]
    parts = [tiny(seed=20 + i, S=n, sink=True, **dims) for i, n in enumerate(lens)]
    s = parts[0][3]
    q = np.concatenate([p[0] for p in parts])
    k = np.concatenate([p[1] for p in parts])
    v = np.concatenate([p[2] for p in parts])
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, l = oracle.attention(q=q, hq=4, hkv=2, dqk=16, dv=8, rope_dim=8, rope_base=1e4, softmax_scale=0.25,
                            v_scale=0.707, window=6, sink=s, q_row0=cu[:-1], q_len=lens, q_pos0=[0, 0, 0],
                            sel_seq=np.repeat(np.arange(3), lens), sel_row=np.concatenate([np.arange(n) for n in lens]),
                            k_new=k, v_new=v, new_row0=cu[:-1], new_pos0=[0, 0, 0], new_len=lens)
    for i, (qq, kk, vv, _) in enumerate(parts):
        oi, li = run(qq, kk, vv, s, window=6, base=1e4, scale=0.25, **dims)
        np.testing.assert_array_equal(o[cu[i]:cu[i + 1]], oi)
        np.testing.assert_array_equal(l[cu[i]:cu[i + 1]], li)


def test_cache_rows_decode_rotated_dims_as_fp16():
    """Cache rows hold key dims < rope_dim as IEEE fp16 bit patterns (the library's cache
    format).  A single cached key at position 0 with no sink: lse = scale * q.k exactly."""
    hq, hkv, dqk, dv, R = 2, 1, 8, 4, 4
    # fp16 bit patterns: 0x3C00 = 1.0, 0xC000 = -2.0, 0x7BFF = 65504, 0x0001 = 2^-24 (subnormal)
    f16 = np.array([0x3C00, 0xC000, 0x7BFF, 0x0001], np.uint16)
    rest = synth.f64_to_bf16_bits(np.array([0.5, -1.5, 3.0, 0.25]))
    kc = np.zeros((1, 4, hkv, dqk), np.uint16)
    kc[0, 0, 0, :4] = f16
    kc[0, 0, 0, 4:] = rest
    vc = np.zeros((1, 4, hkv, dv), np.uint16)
    vc[0, 0, 0] = synth.f64_to_bf16_bits(np.array([1.0, 2.0, 3.0, 4.0]))
    q = synth.f64_to_bf16_bits(np.array([[1.0, 1.0, 1.0, 2.0 ** 10, 1.0, 1.0, 1.0, 1.0],
                                         [0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 1.0]])).reshape(1, hq, dqk)
    o, l = oracle.attention(q=q, hq=hq, hkv=hkv, dqk=dqk, dv=dv, rope_dim=R, rope_base=10.0, softmax_scale=0.5,
                            v_scale=0.707, window=0, sink=None, q_row0=[0], q_len=[1], q_pos0=[0], sel_seq=[0],
                            sel_row=[0], new_pos0=[1], new_len=[0], cache_kind=2, k_cache=kc, v_cache=vc,
                            page_size=4)
    k = [1.0, -2.0, 65504.0, 2.0 ** -24, 0.5, -1.5, 3.0, 0.25]
    assert l[0, 0] == 0.5 * (1.0 - 2.0 + 65504.0 + 2.0 ** -14 + 0.5 - 1.5 + 3.0 + 0.25)
    assert l[0, 1] == 0.5 * 0.25
    np.testing.assert_array_equal(o[0, 0], 0.707 * np.array([1.0, 2.0, 3.0, 4.0]))


def test_kv_append_oracle():
    k = bf16(30, (5, 2, 192))
    v = bf16(31, (5, 2, 128))
    pos = np.array([0, 1, 127, 128, 129023], np.int32)
    ko, vo = oracle.kv_append(k, v, pos, 1e7)
    np.testing.assert_array_equal(vo, widen(v))
    for t in range(5):
        for g in range(2):
            np.testing.assert_array_equal(ko[t, g], oracle.rope(widen(k[t, g]), pos[t], 1e7, 64))


# ----------------------------------------------------------------------------- E4M3 KV caches

def test_e4m3_decoding_matches_torch_and_the_format_definition():
    """The oracle's E4M3 decoding against torch.float8_e4m3fn (an independent library
    implementation) for all 256 bytes, and against the format's fixed points."""
    codes = np.arange(256)
    mine = oracle.e4m3_to_double(codes)
    ref = torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert set(np.flatnonzero(nan)) == {0x7F, 0xFF}
    np.testing.assert_array_equal(np.isnan(mine), nan)
    np.testing.assert_array_equal(mine[~nan], ref[~nan])
    fixed = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
             0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    for c, v in fixed.items():
        assert mine[c] == v, hex(c)


def test_fp8_cache_equals_the_same_values_in_the_bf16_cache():
    """Decoding over an E4M3 cache with power-of-two scales is the decoding over a cache in
    the bf16 format that holds the dequantised values exactly (fp16 for the rotated dims):
    the two paths of the oracle must agree bit for bit."""
    from workloads import configs
    cfg = configs.decode_fp8(seed=41, B=3, ctx_range=(200, 700))
    cfg.k_dequant = np.array([0.5, 2.0, 1.0, 0.25], np.float32)
    cfg.v_dequant = np.array([4.0, 1.0, 0.5, 2.0], np.float32)
    ro, rl = oracle.decode(cfg)
    kv = oracle.e4m3_to_double(cfg.k_cache) * cfg.k_dequant[None, None, :, None]
    vv = oracle.e4m3_to_double(cfg.v_cache) * cfg.v_dequant[None, None, :, None]
    kc = np.empty(kv.shape, np.uint16)
    kc[..., :64] = synth.f64_to_f16_bits(kv[..., :64])
    kc[..., 64:] = synth.f64_to_bf16_bits(kv[..., 64:])
    assert np.array_equal(oracle.e4m3_to_double(cfg.k_cache)[..., 64:] * cfg.k_dequant[None, None, :, None],
                          widen(kc[..., 64:]))
    plain = configs.Decode(cfg.layer, cfg.q, cfg.ctx, kc, synth.f64_to_bf16_bits(vv), block_table=cfg.block_table)
    po, pl = oracle.decode(plain)
    np.testing.assert_array_equal(ro, po)
    np.testing.assert_array_equal(rl, pl)


# ----------------------------------------------------------------------------- regression guard

def test_oracle_snapshot():
    """The oracle still produces the values tests/golden/make_oracle_snapshot.py stored
    (a guard against unintended changes to its arithmetic; correctness is pinned above)."""
    import importlib.util
    import json
    import os
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location("make_oracle_snapshot", os.path.join(here, "make_oracle_snapshot.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    stored = json.load(open(os.path.join(here, "oracle_snapshot.json")))
    now = mod.snapshot()
    assert set(now) == set(stored["cases"])
    for name, vals in stored["cases"].items():
        np.testing.assert_allclose(np.asarray(now[name]["out"]), np.asarray(vals["out"]), rtol=0, atol=1e-12,
                                   err_msg=name)
        np.testing.assert_allclose(np.asarray(now[name]["lse"]), np.asarray(vals["lse"]), rtol=0, atol=1e-12,
                                   err_msg=name)


@pytest.mark.parametrize("paged", [True, False])
def test_decode_adapter_with_drafts_equals_single_token_decodes(paged):
    """The decode adapter with q_len query tokens per sequence: draft i of sequence s (position
    ctx - q_len + i) must equal a one-token decode of the same query over the same cache with
    the context ending at its position (keys after it are invisible to it; for the ring the
    slots that then read as older positions lie outside its window)."""
    import dataclasses
    sw, gl = configs.decode_batch(seed=61, B=3, ctx_range=(130, 600), ring_slots=144)
    base = gl if paged else sw
    q_len = 4
    cfg = configs.with_drafts(base, q_len, seed=62)
    o, l = oracle.decode(cfg)
    assert o.shape[0] == 3 * q_len
    for s in range(3):
        for i in range(q_len):
            one = dataclasses.replace(cfg, q=cfg.q[s * q_len + i:s * q_len + i + 1], q_len=1,
                                      ctx=np.array([cfg.ctx[s] - q_len + i + 1], np.int32),
                                      block_table=None if cfg.block_table is None else cfg.block_table[s:s + 1],
                                      k_cache=cfg.k_cache if paged else cfg.k_cache[s:s + 1],
                                      v_cache=cfg.v_cache if paged else cfg.v_cache[s:s + 1])
            o1, l1 = oracle.decode(one)
            np.testing.assert_array_equal(o[s * q_len + i], o1[0])
            np.testing.assert_array_equal(l[s * q_len + i], l1[0])
