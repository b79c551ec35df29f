"""GPU parity in the softmax's edge regimes, against the float64 oracle.

The "Model techniques map" page ("Learnable attention sink") makes the sink an extra
logit column of the softmax, so a sink far above or below the logits is part of the
method; and nothing bounds the logits themselves.  These cases drive the kernels'
rarely taken paths on inputs built so that the path must be taken:

- sinks of +30 and -30 (the sink dominates / vanishes) on prefill and decode;
- logits about six times wider than ~N(0,1) inputs give (query dims 64..191 scaled by 8,
  exact in bf16; the rotated dims 0..63 are kept as drawn, since their fp16 rounding, a
  property of the cache format, grows with the size of the product they enter);
- one dominant key per stretch of keys (a logit ~55 nats above the rest): in the
  sliding-window kernel its column lies outside the tile's own-position columns that
  set the exponentials' reference, so the chunk sum overflows 2^64 and the reference is
  raised; in the global kernel the running maximum arrives late (a later key tile) and
  the accumulated output is rescaled;
- rotated query / key components at and beyond the fp16 range of the rotated dims.

Bars as everywhere: max-abs 2e-2 and mean-abs 2e-3 on the output, 1e-3 on the LSE.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from workloads import configs, synth

from .util import (check_prefill, chunked_cfg, decode_cfg, make_prefill, parity)

pytestmark = pytest.mark.gpu

SCALE = 1.0 / np.sqrt(192.0)
LN2 = np.log(2.0)


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    import global_attention_attn_b200 as M
    M.lib()
    M.status_poll()
    yield


def _status():
    import global_attention_attn_b200 as M
    return M.status_poll()


def bf16_bits(x):
    return synth.f64_to_bf16_bits(np.asarray(x, np.float64))


def bf16_vals(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def with_sink(layer, values):
    return dataclasses.replace(layer, sink=np.asarray(values, np.float32))


def extreme_sinks(seed, value):
    """Half of the 64 heads at the extreme value, the others ~N(0,1)."""
    s = synth.normal_f32(synth.stream_seed(seed, 4), (64,)).copy()
    s[::2] = value
    return s


# ----------------------------------------------------------------------------- sinks of +-30

@pytest.mark.parametrize("value", [30.0, -30.0])
def test_prefill_swa_extreme_sinks(value):
    cfg = make_prefill([300, 129, 17], 8, 1e4, 128, True, 900)
    cfg.layer = with_sink(cfg.layer, extreme_sinks(900, value))
    check_prefill(cfg, what=f"swa prefill, sinks {value:+}")


@pytest.mark.parametrize("value", [30.0, -30.0])
def test_prefill_global_window_extreme_sinks(value):
    # the global kernel with a wide window and a sink (the layer form with window > 129)
    cfg = make_prefill([700], 4, 1e7, 300, True, 901)
    cfg.layer = with_sink(cfg.layer, extreme_sinks(901, value))
    check_prefill(cfg, what=f"global window 300, sinks {value:+}")


@pytest.mark.parametrize("value", [30.0, -30.0])
def test_decode_extreme_sinks(value):
    sw, gl = configs.decode_batch(seed=902, B=8, ctx_range=(1, 3000))
    sw.layer = with_sink(sw.layer, extreme_sinks(902, value))
    # the paged decode with a window and a sink: splits combined with the sink in the denominator
    gl.layer = dataclasses.replace(gl.layer, window=1000, sink=extreme_sinks(903, value))
    for cfg in (sw, gl):
        out, lse = decode_cfg(cfg)
        parity(out, lse, *oracle.decode(cfg), f"{cfg.name}, sinks {value:+}")


@pytest.mark.parametrize("value", [30.0, -30.0])
def test_chunked_swa_extreme_sinks(value):
    _, swa = configs.chunked_prefill(seed=904, prefix=1000, chunk=300, n_sample=300)
    swa.layer = with_sink(swa.layer, extreme_sinks(904, value))
    out, lse = chunked_cfg(swa)
    parity(out, lse, *oracle.chunked(swa, rows=np.arange(300)), f"swa chunk, sinks {value:+}")


# ----------------------------------------------------------------------------- wide logits

def scaled_q(bits, factor):
    """Query dims 64..191 times a power of two (exact in bf16); dims 0..63 unchanged."""
    out = bits.copy()
    out[..., 64:] = bf16_bits(bf16_vals(bits[..., 64:]) * factor)
    return out


def test_prefill_wide_logits():
    for hkv, base, window in ((8, 1e4, 128), (4, 1e7, 0)):
        cfg = make_prefill([600, 45], hkv, base, window, window > 0, 905 + hkv)
        cfg.q = scaled_q(cfg.q, 8.0)
        check_prefill(cfg, what=f"{'swa' if window else 'global'} prefill, Q dims 64..191 x 8")


def test_decode_wide_logits():
    sw, gl = configs.decode_batch(seed=907, B=8, ctx_range=(100, 5000))
    for cfg in (sw, gl):
        cfg.q = scaled_q(cfg.q, 8.0)
        out, lse = decode_cfg(cfg)
        parity(out, lse, *oracle.decode(cfg), f"{cfg.name}, Q dims 64..191 x 8")


# ----------------------------------------------------------------------------- dominant keys

def dominant_key_prefill(lens, hkv, base, window, sink, seed, every):
    """Q dims 64..191 all equal 2u (u a fixed +-1 pattern), and every `every`-th key (from
    position every // 2) has dims 64..191 equal to 3u: those keys' logits are ~55 nats
    above the ~N(0, 1.6^2) logits of the others.  Returns (cfg, dominant positions)."""
    cfg = make_prefill(lens, hkv, base, window, sink, seed)
    u = np.where(synth.uniform01(synth.stream_seed(seed, 50), 128) < 0.5, -1.0, 1.0)
    q = cfg.q.copy()
    q[:, :, 64:] = bf16_bits(2.0 * u)[None, None, :]
    k = cfg.k.copy()
    pos = np.concatenate([np.arange(n) for n in cfg.k_lens])  # positions of the key rows
    dom = (pos % every) == every // 2
    k[dom, :, 64:] = bf16_bits(3.0 * u)[None, None, :]
    cfg.q, cfg.k = q, k
    return cfg, pos[dom]


def test_swa_dominant_keys_raise_the_reference():
    """Sliding-window kernel: a dominant key in columns 0..127 of a tile (not among the
    tile's 16 own positions) overflows the chunk sum taken against the own-position
    reference, which must then be raised to it."""
    every = 50
    cfg, dom = dominant_key_prefill([1000, 700], 8, 1e4, 128, True, 910, every)
    # rows that see a dominant key outside their tile's own 16 positions (the raise is
    # needed there): position p in tile [q0, q0 + 16), dominant d with p - 127 <= d < q0,
    # while no dominant key sits among the own positions (the reference stays low)
    is_dom = lambda d: d % every == every // 2
    need = 0
    for n in cfg.q_lens:
        for p in range(128, int(n)):
            q0 = p - p % 16  # the tile's first position; its own columns are q0 .. q0 + 15
            own = any(is_dom(d) for d in range(q0, p + 1))          # visible own-position columns
            outside = any(is_dom(d) for d in range(p - 127, q0))   # visible columns 0..127
            need += int(outside and not own)
    assert need > 500
    # the margin: the dominant logit (80 log2 units) over the own-position reference (the
    # largest of 16 ordinary logits with ~1.6-nat spread: a few log2 units) beyond 2^64
    qd = 2.0 * 3.0 * 128 * SCALE / LN2
    assert qd > 64 + 12
    check_prefill(cfg, what="swa prefill, dominant keys outside the own-position columns")


def test_global_late_maximum_rescales():
    """Global kernel: the running maximum jumps by far more than 2^8 at a later key tile
    (the dominant keys sit at positions 500 + 1000 i), so O accumulated over the earlier
    tiles is rescaled; rows before the first dominant key never rescale."""
    cfg, dom = dominant_key_prefill([2500], 4, 1e7, 0, False, 911, 1000)
    assert list(dom[:2]) == [500, 1500]
    check_prefill(cfg, what="global prefill, late maxima")


def test_decode_dominant_keys():
    """Decode: a dominant cached key in the last tile (paged) or anywhere in the ring."""
    sw, gl = configs.decode_batch(seed=912, B=8, ctx_range=(600, 5000))
    for cfg in (sw, gl):
        u = np.where(synth.uniform01(synth.stream_seed(912, 50), 128) < 0.5, -1.0, 1.0)
        cfg.q = cfg.q.copy()
        cfg.q[:, :, 64:] = bf16_bits(2.0 * u)[None, None, :]
        kc = cfg.k_cache.copy()
        for s, c in enumerate(cfg.ctx):
            p = int(c) - 3  # a recent position: visible, and late in the paged order
            if cfg.paged:
                kc[cfg.block_table[s, p // 128], p % 128, :, 64:] = bf16_bits(3.0 * u)[None, :]
            else:
                kc[s, p % 128, :, 64:] = bf16_bits(3.0 * u)[None, :]
        cfg.k_cache = kc
        out, lse = decode_cfg(cfg)
        parity(out, lse, *oracle.decode(cfg), f"{cfg.name}, dominant key")


# ----------------------------------------------------------------------------- fp16 range

def _set_pair(a, j, x, y):
    a = a.copy()
    a[..., j] = bf16_bits(x)
    a[..., j + 32] = bf16_bits(y)
    return a


def test_rotated_keys_beyond_fp16_saturate_and_report():
    """Key dims (0, 32) = (60000, 60000): rotated, their magnitude reaches 84852 > 65504, so
    the rotated-key store saturates and reports MIMO_STATUS_RANGE.  The query's dims 0 and
    32 are zero, so those key dims enter no logit and the output still equals the oracle's."""
    import global_attention_attn_b200 as M
    cfg = make_prefill([400], 8, 1e4, 128, True, 920)
    cfg.k = _set_pair(cfg.k, 0, 60000.0, 60000.0)
    cfg.q = _set_pair(cfg.q, 0, 0.0, 0.0)
    # frequency 0 rotates by the position itself: |60000 (cos p -+ sin p)| > 65504 somewhere
    p = np.arange(400)
    assert np.max(np.abs(60000.0 * (np.cos(p) - np.sin(p)))) > 65504
    assert _status() == 0
    check_prefill(cfg, what="swa prefill, rotated keys beyond fp16")
    assert _status() & M.MIMO_STATUS_RANGE


def test_rotated_queries_beyond_fp16_saturate_and_report():
    import global_attention_attn_b200 as M
    for hkv, base, window in ((8, 1e4, 128), (4, 1e7, 0)):
        cfg = make_prefill([300], hkv, base, window, window > 0, 921 + hkv)
        cfg.q = _set_pair(cfg.q, 0, 60000.0, -60000.0)
        cfg.k = _set_pair(cfg.k, 0, 0.0, 0.0)
        assert _status() == 0
        check_prefill(cfg, what="prefill, rotated queries beyond fp16")
        assert _status() & M.MIMO_STATUS_RANGE


def test_rotated_values_near_the_fp16_limit_are_exact():
    """Rotated key dims near the top of the fp16 range (40000 before rotation, which keeps
    them below 65504; 46000 in the caches) with small query dims (0, 32): they enter every
    logit, through the contiguous prefill's key copy and the ring and paged decode."""
    import global_attention_attn_b200 as M
    cfg = make_prefill([500], 8, 1e4, 128, True, 925)
    cfg.k = _set_pair(cfg.k, 0, 40000.0, 0.0)
    # products of ~5: fp16 rounding of the rotated dims stays far below the LSE bar
    cfg.q = _set_pair(cfg.q, 0, 2.0 ** -13, 2.0 ** -13)
    check_prefill(cfg, what="swa prefill, rotated keys near the fp16 limit")
    sw, gl = configs.decode_batch(seed=926, B=4, ctx_range=(200, 900))
    for d in (sw, gl):
        # the caches hold rotated keys in their format: dims 0..63 as fp16 bit patterns
        kc = d.k_cache.copy()
        kc[..., 0] = synth.f64_to_f16_bits(np.full(kc.shape[:-1], 46000.0))
        kc[..., 32] = synth.f64_to_f16_bits(np.full(kc.shape[:-1], -46000.0))
        d.k_cache = kc
        d.q = _set_pair(d.q, 0, 2.0 ** -14, 0.0)
        out, lse = decode_cfg(d)
        parity(out, lse, *oracle.decode(d), f"{d.name}, cached keys near the fp16 limit")
    assert _status() == 0
    assert M.MIMO_STATUS_RANGE == 4
