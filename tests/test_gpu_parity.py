"""GPU parity: the CUDA path through the C ABI against the float64 oracle, element by
element, on the same seeded inputs.

Bar (bf16 output, fp32 accumulation): max-abs 2e-2 and mean-abs 2e-3 on O, 1e-3
on the LSE.  Small cases are checked on every row; the full-size workloads on
sampled rows (the oracle evaluates rows one by one), always including the rows
at the window edge (126, 127, 128), the first and the last.
"""
import numpy as np
import pytest

import oracle
from workloads import configs, synth

from .util import (check_prefill, chunked_cfg, decode_cfg, dev_bf16, dev_f32, dev_i32, host_f64, make_prefill, parity,
                   prefill_cfg, verify_decode_cfg)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    import global_attention_attn_b200 as M
    M.lib()
    yield
    assert M.status_poll() == 0, "device status word reported a timeout or a bad index"


# ----------------------------------------------------------------------------- KV append

@pytest.mark.parametrize("kind", ["ring", "ring144", "paged"])
def test_kv_append(kind):
    import torch
    import global_attention_attn_b200 as M
    # at most `slots` tokens per sequence for a ring: two tokens of one call must not share a slot
    slots = 144 if kind == "ring144" else 128
    n, hkv, base = (3 * slots, 8, 1e4) if kind.startswith("ring") else (700, 4, 1e7)
    k = configs.bf16_normal(41, 1, (n, hkv, 192))
    v = configs.bf16_normal(41, 2, (n, hkv, 128))
    seq = (np.arange(n) % 3).astype(np.int32)
    pos = (np.arange(n) // 3 + np.array([0, 5, 120000])[seq]).astype(np.int32)
    if kind.startswith("ring"):
        kc = torch.zeros((3, slots, hkv, 192), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros((3, slots, hkv, 128), dtype=torch.bfloat16, device="cuda")
        M.mimo_kv_append(dev_bf16(k), dev_bf16(v), dev_i32(pos), dev_i32(seq), rope_base=base,
                         cache_kind=M.MIMO_CACHE_RING, k_cache=kc, v_cache=vc, num_seqs=3,
                         ring_slots=0 if slots == 128 else slots)
        where = {(int(seq[t]), int(pos[t] % slots)): t for t in range(n)}
    else:
        maxp = (int(pos.max()) // 128) + 1
        bt = (synth.permutation(7, 3 * maxp).reshape(3, maxp)).astype(np.int32)
        kc = torch.zeros((3 * maxp, 128, hkv, 192), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros((3 * maxp, 128, hkv, 128), dtype=torch.bfloat16, device="cuda")
        M.mimo_kv_append(dev_bf16(k), dev_bf16(v), dev_i32(pos), dev_i32(seq), rope_base=base,
                         cache_kind=M.MIMO_CACHE_PAGED, k_cache=kc, v_cache=vc, num_seqs=3,
                         block_table=dev_i32(bt), num_pages=3 * maxp)
        where = {(int(bt[seq[t], pos[t] // 128]), int(pos[t] % 128)): t for t in range(n)}
    ko, vo = oracle.kv_append(k, v, pos, base)
    kcn, vcn = host_f64(kc), host_f64(vc)
    # cache format: key dims 0..63 are IEEE fp16 bit patterns
    kbits = kc.view(torch.int16).cpu().numpy().view(np.uint16)
    kcn[..., :64] = kbits[..., :64].view(np.float16).astype(np.float64)
    touched = np.zeros(kcn.shape[:2], bool)
    for (a, b), t in where.items():
        touched[a, b] = True
        # rotated dims: fp32 rotation of bf16 inputs, rounded to fp16 (11 significant bits)
        assert np.all(np.abs(kcn[a, b, :, :64] - ko[t, :, :64]) <= 2.0 ** -11 * np.abs(ko[t, :, :64]) + 1e-6)
        np.testing.assert_array_equal(kcn[a, b, :, 64:], ko[t, :, 64:])     # pass-through dims: exact
        np.testing.assert_array_equal(vcn[a, b], vo[t])                       # values: exact copy
    assert np.all(kcn[~touched] == 0) and np.all(vcn[~touched] == 0)


def _e4m3_grid(x):
    """Spacing of E4M3 values around |x| (subnormal step 2^-9 below 2^-6)."""
    a = np.maximum(np.abs(x), 2.0 ** -6)
    return 2.0 ** (np.floor(np.log2(a)) - 3)


@pytest.mark.parametrize("kind", ["ring", "paged"])
def test_kv_append_fp8(kind):
    """E4M3 append: every stored byte is a nearest E4M3 value of the oracle's (rotated) element
    divided by its KV head's scale (either neighbour where the element sits within rounding
    noise of a midpoint), saturated at 448; untouched slots stay zero."""
    import torch
    import global_attention_attn_b200 as M
    n, hkv, base = (300, 8, 1e4) if kind == "ring" else (500, 4, 1e7)
    k = configs.bf16_normal(43, 1, (n, hkv, 192))
    v = configs.bf16_normal(43, 2, (n, hkv, 128))
    # scales small enough that some elements saturate
    kdq = np.array([0.004, 0.3, 1.0, 2.5, 0.07, 0.5, 1.5, 0.9][:hkv], np.float32)
    vdq = np.array([0.01, 0.8, 2.0, 0.6, 1.1, 0.25, 3.0, 0.45][:hkv], np.float32)
    seq = (np.arange(n) % 3).astype(np.int32)
    pos = (np.arange(n) // 3 + np.array([0, 5, 120000])[seq]).astype(np.int32)
    extra = dict(cache_dtype=M.MIMO_DTYPE_FP8_E4M3, k_dequant=dev_f32(kdq), v_dequant=dev_f32(vdq))
    if kind == "ring":
        kc = torch.zeros((3, 128, hkv, 192), dtype=torch.uint8, device="cuda")
        vc = torch.zeros((3, 128, hkv, 128), dtype=torch.uint8, device="cuda")
        M.mimo_kv_append(dev_bf16(k), dev_bf16(v), dev_i32(pos), dev_i32(seq), rope_base=base,
                         cache_kind=M.MIMO_CACHE_RING, k_cache=kc, v_cache=vc, num_seqs=3, **extra)
        where = {(int(seq[t]), int(pos[t] % 128)): t for t in range(n)}
    else:
        maxp = (int(pos.max()) // 128) + 1
        bt = (synth.permutation(8, 3 * maxp).reshape(3, maxp)).astype(np.int32)
        kc = torch.zeros((3 * maxp, 128, hkv, 192), dtype=torch.uint8, device="cuda")
        vc = torch.zeros((3 * maxp, 128, hkv, 128), dtype=torch.uint8, device="cuda")
        M.mimo_kv_append(dev_bf16(k), dev_bf16(v), dev_i32(pos), dev_i32(seq), rope_base=base,
                         cache_kind=M.MIMO_CACHE_PAGED, k_cache=kc, v_cache=vc, num_seqs=3,
                         block_table=dev_i32(bt), num_pages=3 * maxp, **extra)
        where = {(int(bt[seq[t], pos[t] // 128]), int(pos[t] % 128)): t for t in range(n)}
    ko, vo = oracle.kv_append(k, v, pos, base)
    kb, vb = kc.cpu().numpy(), vc.cpu().numpy()
    kval, vval = oracle.e4m3_to_double(kb), oracle.e4m3_to_double(vb)
    touched = np.zeros(kb.shape[:2], bool)
    slots = list(where.items())
    for (a, b), t in slots:
        touched[a, b] = True
    rows = np.array([t for _, t in slots])
    ia = np.array([a for (a, _), _ in slots])
    ib = np.array([b for (_, b), _ in slots])
    for got, ref, dq in ((kval[ia, ib], ko[rows], kdq), (vval[ia, ib], vo[rows], vdq)):
        x = ref / dq.astype(np.float64)[None, :, None]
        sat = np.abs(x) >= 448.0
        assert np.all(got[sat] == np.sign(x[sat]) * 448.0)
        err = np.abs(got[~sat] - x[~sat])
        half = 0.5 * _e4m3_grid(x[~sat])
        assert np.all(err <= half * (1 + 2.0 ** -10)), float((err / half).max())
        assert sat.any() or dq is vdq
    assert np.all(kb[~touched] == 0) and np.all(vb[~touched] == 0)


# ----------------------------------------------------------------------------- decode

@pytest.mark.parametrize("ctx_range", [(1, 127), (100, 3000), (4096, 9000)])
def test_decode_small(ctx_range):
    sw, gl = configs.decode_batch(seed=100 + ctx_range[0], B=8, ctx_range=ctx_range)
    for cfg in (sw, gl):
        out, lse = decode_cfg(cfg)
        ro, rl = oracle.decode(cfg)
        parity(out, lse, ro, rl, cfg.name)


def test_decode_split_boundaries():
    # contexts on both sides of the 512-key split length and of one page
    import global_attention_attn_b200 as M
    sw, gl = configs.decode_batch(seed=321, B=8, ctx_range=(1, 2))
    ctx = np.array([1, 127, 128, 129, 511, 512, 513, 1025], np.int32)
    bt, pool = configs.paged_layout(5, 1, ctx)
    gl = configs.Decode(gl.layer, gl.q, ctx, configs.cached_keys(5, 2, (pool, 128, 4, 192)),
                        configs.bf16_normal(5, 3, (pool, 128, 4, 128)), block_table=bt)
    out, lse = decode_cfg(gl)
    ro, rl = oracle.decode(gl)
    parity(out, lse, ro, rl, "global split boundaries")
    sw = configs.Decode(sw.layer, sw.q, ctx, sw.k_cache, sw.v_cache)
    out, lse = decode_cfg(sw)
    ro, rl = oracle.decode(sw)
    parity(out, lse, ro, rl, "swa ring wrap")
    assert M.status_poll() == 0


def _shared_page_decode(seed, B, ctx_range, pool, layer):
    """Decode over a small page pool that the block tables share (prefix-shared pages):
    large batches without a large cache."""
    ctx = synth.randint(synth.stream_seed(seed, 0), B, *ctx_range).astype(np.int32)
    maxp = int((ctx.max() + 127) // 128)
    bt = synth.randint(synth.stream_seed(seed, 1), B * maxp, 0, pool - 1).astype(np.int32).reshape(B, maxp)
    h = layer.num_kv_heads
    return configs.Decode(layer, configs.bf16_normal(seed, 2, (B, 64, 192)), ctx,
                          configs.cached_keys(seed, 3, (pool, 128, h, 192)),
                          configs.bf16_normal(seed, 4, (pool, 128, h, 128)), block_table=bt)


def test_decode_large_batch_shared_pages():
    """More than 1024 sequences with several splits each: the split units are enumerated
    densely instead of from the per-sequence table."""
    import torch
    cfg = _shared_page_decode(601, 1100, (513, 1600), 24, configs.global_layer())
    out, lse = decode_cfg(cfg)
    seqs = np.array(sorted(set([0, 1023, 1024, 1099] + list(synth.permutation(602, 1100)[:8]))), np.int32)
    ro, rl = oracle.decode(cfg, seqs=seqs)
    idx = torch.as_tensor(seqs, dtype=torch.long, device=out.device)
    parity(out[idx], lse[idx], ro, rl, "decode 1100 sequences, shared pages")


def test_decode_paged_window_unaligned_splits():
    """A window on the paged cache: splits start mid-page and mid-tile."""
    sink = synth.normal_f32(synth.stream_seed(603, 9), (64,))
    for window in (1000, 300):
        layer = configs.Layer("swa", 4, 1e7, window, sink)
        cfg = _shared_page_decode(604 + window, 12, (200, 3000), 40, layer)
        out, lse = decode_cfg(cfg)
        ro, rl = oracle.decode(cfg)
        parity(out, lse, ro, rl, f"paged decode, window {window}")


@pytest.mark.parametrize("ring", [False, True])
def test_decode_fp8_small(ring):
    """Decode over an E4M3 cache (per-KV-head scales): ring (sliding layer) and paged (global)."""
    cfg = configs.decode_fp8(seed=810 + ring, B=8, ctx_range=(1, 3000), ring=ring)
    out, lse = decode_cfg(cfg)
    ro, rl = oracle.decode(cfg)
    parity(out, lse, ro, rl, cfg.name)


def test_decode_fp8_split_boundaries_and_window():
    ctx = np.array([1, 127, 128, 129, 511, 512, 513, 1025, 8193], np.int32)
    cfg = configs.decode_fp8(seed=820, ctx=ctx)
    out, lse = decode_cfg(cfg)
    ro, rl = oracle.decode(cfg)
    parity(out, lse, ro, rl, "fp8 split boundaries")
    sink = synth.normal_f32(synth.stream_seed(821, 9), (64,))
    cfg.layer = configs.Layer("swa", 4, 1e7, 1000, sink)
    out, lse = decode_cfg(cfg)
    ro, rl = oracle.decode(cfg)
    parity(out, lse, ro, rl, "fp8 paged, window 1000 with sink")


def test_decode_fp8_b64_full_scale():
    """64 sequences, contexts U[4096, 65536] over an E4M3 paged cache, every sequence checked."""
    cfg = configs.decode_fp8()
    out, lse = decode_cfg(cfg)
    ro, rl = oracle.decode(cfg)
    parity(out, lse, ro, rl, "fp8 64-sequence decode, all sequences")


@pytest.mark.parametrize("ring_slots,window", [(144, 129), (144, 128), (256, 129), (512, 300), (128, 5)])
def test_decode_ring_slots(ring_slots, window):
    """Rings longer than 128 slots: the SGLang window of the query plus 128 previous keys
    (radixark miles docs "MiMo-V2.6-Flash", section 5.4) decoded from a ring that keeps one
    16-key tile more than the window (144 slots), and wider rings and windows."""
    import dataclasses
    sw, _ = configs.decode_batch(seed=330 + ring_slots + window, B=12, ctx_range=(1, 2000), ring_slots=ring_slots)
    sw.layer = dataclasses.replace(sw.layer, window=window)
    sw.ctx[:3] = [1, window - 1, window]
    out, lse = decode_cfg(sw)
    parity(out, lse, *oracle.decode(sw), f"ring {ring_slots} decode, window {window}")


def test_decode_ring_rejects_a_window_beyond_its_slots():
    import global_attention_attn_b200 as M
    sw, _ = configs.decode_batch(seed=340, B=2, ctx_range=(200, 300))
    import dataclasses
    sw.layer = dataclasses.replace(sw.layer, window=129)
    with pytest.raises(M.MimoError) as e:
        decode_cfg(sw)
    assert e.value.code == M.MIMO_ERR_INVALID_ARG


@pytest.fixture(scope="module")
def dec64():
    return configs.decode_batch()


def test_decode_b64_swa_ring(dec64):
    sw, _ = dec64
    out, lse = decode_cfg(sw)
    ro, rl = oracle.decode(sw)
    parity(out, lse, ro, rl, "decode b64 swa ring, all 64 sequences")


def test_decode_b64_global_paged(dec64):
    _, gl = dec64
    out, lse = decode_cfg(gl)
    ro, rl = oracle.decode(gl)
    parity(out, lse, ro, rl, "decode b64 global paged, all 64 sequences")


# ----------------------------------------------------------------------------- prefill: sliding window

def test_prefill_swa_s512():
    check_prefill(configs.swa_prefill_s512(), what="swa prefill s512")


@pytest.mark.parametrize("lens", [[1], [16], [127, 128, 129], [1, 15, 16, 17, 31, 300], [1000]])
def test_prefill_swa_edges(lens):
    check_prefill(make_prefill(lens, 8, 1e4, 128, True, 200 + sum(lens)), what=f"swa {lens}")


def test_prefill_many_sequences():
    """More than 256 sequences: the batch is split over several launches."""
    lens = list((np.arange(300) * 7919) % 37 + 1)
    check_prefill(make_prefill(lens, 8, 1e4, 128, True, 310), what="swa 300 sequences")
    check_prefill(make_prefill(lens, 4, 1e7, 0, False, 311), what="global 300 sequences")


def test_prefill_swa_no_sink():
    check_prefill(make_prefill([513, 77], 8, 1e4, 128, False, 301), what="swa no sink")


def test_prefill_swa_window_129():
    # the SGLang / miles window convention: the query plus 128 previous keys
    check_prefill(make_prefill([400], 8, 1e4, 129, True, 302), what="swa window 129")


def test_prefill_swa_small_window():
    check_prefill(make_prefill([300], 8, 1e4, 5, True, 303), what="swa window 5")


@pytest.mark.parametrize("lens,klens", [([40], [300]), ([40, 17, 130, 1], [300, 17, 500, 64])],
                         ids=["one", "mixed"])
def test_prefill_swa_fewer_queries_than_keys(lens, klens):
    # bottom-right alignment: each sequence's queries sit at the end of its keys, so the
    # query cos/sin rows are at other positions than the key rows of the same index
    check_prefill(make_prefill(lens, 8, 1e4, 128, True, 304, klens=klens), what="swa q<k")


def test_prefill_global_fewer_queries_than_keys():
    check_prefill(make_prefill([33, 200, 7], 4, 1e7, 0, False, 305, klens=[400, 200, 129]), what="global q<k")


def test_prefill_swa_varlen_sampled():
    cfg = configs.swa_varlen_prefill()
    cu = cfg.cu_q
    always = set()
    for s in range(cfg.num_seqs):
        for r in (0, 1, 15, 16, 126, 127, 128, 129):
            always.add(int(cu[s] + r))
        always.add(int(cu[s + 1] - 1))
    rows = configs.sample_rows(11, int(cu[-1]), 1024, always=sorted(always))
    check_prefill(cfg, rows=rows, what="swa varlen prefill (sampled rows)")


# ----------------------------------------------------------------------------- prefill: global

@pytest.mark.parametrize("lens", [[1], [8, 9], [1, 127, 128, 129, 300], [1500]])
def test_prefill_global_small(lens):
    check_prefill(make_prefill(lens, 4, 1e7, 0, False, 400 + sum(lens)), what=f"global {lens}")


def test_prefill_global_with_sink_and_wide_window():
    check_prefill(make_prefill([700], 4, 1e7, 300, True, 410), what="global window 300 + sink")


def test_prefill_global_s16384_sampled():
    cfg = configs.global_causal_prefill()
    rows = configs.sample_rows(22, 16384, 1024, always=(0, 1, 7, 8, 127, 128, 129, 8191, 16383))
    assert len(rows) == 1024
    check_prefill(cfg, rows=rows, what="global prefill s16384 (1024 sampled rows)")


# ----------------------------------------------------------------------------- chunked prefill

def test_chunked_small_unaligned():
    glb, swa = configs.chunked_prefill(seed=55, prefix=1000, chunk=300, n_sample=300)
    for cfg in (glb, swa):
        out, lse = chunked_cfg(cfg)
        ro, rl = oracle.chunked(cfg, rows=np.arange(300))
        parity(out, lse, ro, rl, cfg.name)


def test_chunked_swa_window_left_right_128_0():
    """SGLang's (128, 0) window, i.e. 129 keys, on the ring-cache chunk path: the first rows
    of the chunk reach back over all 128 halo positions of the ring."""
    import dataclasses

    import global_attention_attn_b200 as M
    W = M.mimo_window_from_left_right(128, 0)
    assert W == 129
    _, swa = configs.chunked_prefill(seed=56, prefix=1000, chunk=300, n_sample=300)
    L = swa.layer
    swa = dataclasses.replace(swa, layer=configs.Layer(L.kind, L.num_kv_heads, L.rope_base, W, L.sink),
                              name="swa_chunk_300_on_1000_window_129")
    out, lse = chunked_cfg(swa)
    ro, rl = oracle.chunked(swa, rows=np.arange(300))
    parity(out, lse, ro, rl, swa.name)


@pytest.mark.parametrize("window", [128, 129])
def test_chunked_swa_ring_mixed_lengths(window):
    """Sliding-window chunks over ring caches, many sequences: chunk lengths on both sides of
    the 128-position halo and of the 144 new rows copied next to it, prefixes shorter and
    longer than the ring.  Tiles whose window starts inside the chunk read the new keys
    directly, the others the copy of the halo and the first new keys."""
    lens = np.array([1, 16, 127, 128, 129, 143, 144, 145, 300, 517], np.int32)
    starts = np.array([0, 5, 127, 128, 129, 1000, 3, 200, 4096, 77], np.int32)
    B = len(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    n = int(cu[-1])
    seed = 60 + window
    ring_k = np.zeros((B, 128, 8, 192), np.uint16)
    ring_v = np.zeros((B, 128, 8, 128), np.uint16)
    tk = configs.cached_keys(seed, 5, (B, 128, 8, 192))
    tv = configs.bf16_normal(seed, 6, (B, 128, 8, 128))
    for s in range(B):
        for p in range(max(0, int(starts[s]) - 128), int(starts[s])):
            ring_k[s, p % 128], ring_v[s, p % 128] = tk[s, p % 128], tv[s, p % 128]
    L = configs.Layer("swa", 8, 1e4, window, synth.normal_f32(synth.stream_seed(seed, 4), (64,)))
    cfg = configs.Chunked(L, configs.bf16_normal(seed, 1, (n, 64, 192)), configs.bf16_normal(seed, 2, (n, 8, 192)),
                          configs.bf16_normal(seed, 3, (n, 8, 128)), cu, starts, ring_k, ring_v,
                          name=f"swa ring chunks of mixed lengths, window {window}")
    out, lse = chunked_cfg(cfg)
    parity(out, lse, *oracle.chunked(cfg, rows=np.arange(n)), cfg.name)


def test_chunked_swa_from_a_256_slot_ring_window_129():
    """The sliding-window chunk reads its 128 halo positions from a ring longer than 128."""
    import dataclasses
    _, swa = configs.chunked_prefill(seed=57, prefix=1000, chunk=300, n_sample=300, ring_slots=256)
    swa.layer = dataclasses.replace(swa.layer, window=129)
    out, lse = chunked_cfg(swa)
    parity(out, lse, *oracle.chunked(swa, rows=np.arange(300)), "swa chunk from a 256-slot ring, window 129")


def test_chunked_8192_on_120832():
    glb, swa = configs.chunked_prefill()
    out, lse = chunked_cfg(swa)
    ro, rl = oracle.chunked(swa)
    import torch
    idx = torch.as_tensor(swa.sample_rows, dtype=torch.long, device=out.device)
    parity(out[idx], lse[idx], ro, rl, "swa chunk 8192 on 120832 (1024 sampled rows)")
    out, lse = chunked_cfg(glb)
    # the 1024 seeded rows of the workload (rows 0, 126, 127, 128 and 8191 among them)
    rows = glb.sample_rows
    assert len(rows) == 1024 and {0, 126, 127, 128, 8191} <= set(int(r) for r in rows)
    ro, rl = oracle.chunked(glb, rows=rows)
    idx = torch.as_tensor(rows, dtype=torch.long, device=out.device)
    parity(out[idx], lse[idx], ro, rl, "global chunk 8192 on 120832 (1024 sampled rows)")


# ----------------------------------------------------------------------------- cross-path

# ----------------------------------------------------------------------------- speculative verification

# ----------------------------------------------------------------------------- context parallelism

@pytest.mark.parametrize("splits,window", [
    ([[300, 200, 129], [140, 131, 500]], 128),       # every chunk fills the 128-slot ring alone
    ([[50, 30, 200, 7, 250], [10, 300, 2, 128, 64]], 129),  # short chunks: rings relayed
], ids=["independent", "relay_window_129"])
def test_cp_halo_prefill_emulated_on_one_gpu(splits, window):
    """Context-parallel sliding-window prefill with the ranks run one after another on one
    GPU (no rank waits on another's kernel): each rank's outgoing ring is built by the
    library's key append (on top of its incoming ring when its chunk is short), and its
    chunk is prefilled over the incoming ring.  The rows of all ranks must equal the
    oracle's prefill of the whole sequences."""
    import torch

    from global_attention_attn_b200 import cp
    B, R = len(splits), len(splits[0])
    cfg = make_prefill([sum(sp) for sp in splits], 8, 1e4, window, True, 306 + window)
    cu = cfg.cu_q
    q, k, v, sink = dev_bf16(cfg.q), dev_bf16(cfg.k), dev_bf16(cfg.v), dev_f32(cfg.layer.sink)
    out = torch.empty((int(cu[-1]), 64, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((int(cu[-1]), 64), dtype=torch.float32, device="cuda")
    recv_k, recv_v = cp.ring_buffers(B, 8, "cuda")
    starts = [0] * B
    for r in range(R):
        n = [splits[s][r] for s in range(B)]
        idx = torch.cat([torch.arange(int(cu[s]) + starts[s], int(cu[s]) + starts[s] + n[s]) for s in range(B)]).cuda()
        ql, kl, vl = q[idx].contiguous(), k[idx].contiguous(), v[idx].contiguous()
        send_k, send_v = cp.ring_buffers(B, 8, "cuda")
        st = list(starts)
        cp.outgoing_ring(recv_k, recv_v, send_k, send_v,
                         lambda rk, rv: cp.fill_ring_tail(rk, rv, kl, vl, n, st, rope_base=1e4),
                         cp.chunks_fill_ring(n))
        o, l = cp.prefill_with_halo(ql, kl, vl, n, st, recv_k, recv_v, rope_base=1e4, window=window, sink=sink)
        out[idx], lse[idx] = o, l
        recv_k, recv_v = send_k, send_v
        starts = [starts[s] + n[s] for s in range(B)]
    ro, rl = oracle.prefill(cfg)
    parity(out, lse, ro, rl, f"cp halo ({R} ranks emulated, window {window})")


@pytest.mark.parametrize("q_len", [2, 5, 8])
def test_verify_draft_tokens(q_len):
    """q_len draft tokens per sequence scored against the cache: the global layer appends them
    to the paged cache and runs the chunked prefill over it; the sliding layer reads the prefix
    tail from the ring and the drafts from the new rows."""
    glb, swa = configs.verify(seed=700 + q_len, B=12, q_len=q_len, ctx_range=(q_len + 1, 3000))
    for cfg in (glb, swa):
        out, lse = chunked_cfg(cfg)
        ro, rl = oracle.chunked(cfg, rows=np.arange(int(cfg.cu_new[-1])))
        parity(out, lse, ro, rl, cfg.name)


def test_verify_b64_full_scale(dec64):
    """Verification at the decode workload's scale (64 sequences, contexts up to 64K) on the
    64-sequence decode caches, every draft row of every sequence checked."""
    _, gl = dec64
    glb, swa = configs.verify(B=64, q_len=4, decode=gl)
    for cfg in (glb, swa):
        out, lse = chunked_cfg(cfg)
        ro, rl = oracle.chunked(cfg, rows=np.arange(64 * 4))
        parity(out, lse, ro, rl, cfg.name)


# ----------------------------------------------------------------------------- draft tokens in the decode kernel

@pytest.mark.parametrize("q_len", [2, 3, 4, 5, 8])
def test_decode_drafts_paged(q_len):
    """q_len query tokens per sequence over the paged cache: each draft row with its own
    position, rotary angle and causal limit."""
    _, gl = configs.decode_batch(seed=710 + q_len, B=10, ctx_range=(q_len, 3000))
    gl.ctx[:2] = [q_len, q_len + 1]
    cfg = configs.with_drafts(gl, q_len, seed=711)
    out, lse = decode_cfg(cfg)
    parity(out, lse, *oracle.decode(cfg), cfg.name)


@pytest.mark.parametrize("q_len,ring_slots,window", [(2, 144, 128), (4, 144, 128), (8, 144, 128), (5, 144, 129),
                                                     (8, 256, 129), (3, 128, 100)])
def test_decode_drafts_ring(q_len, ring_slots, window):
    """Draft rows over a ring: the ring keeps window + q_len - 1 positions, so the earliest
    draft's window is whole after the drafts are appended."""
    import dataclasses
    sw, _ = configs.decode_batch(seed=720 + q_len + ring_slots, B=10, ctx_range=(q_len, 3000), ring_slots=ring_slots)
    sw.layer = dataclasses.replace(sw.layer, window=window)
    sw.ctx[:3] = [q_len, window, window + q_len]
    cfg = configs.with_drafts(sw, q_len, seed=721)
    out, lse = decode_cfg(cfg)
    parity(out, lse, *oracle.decode(cfg), cfg.name)


def test_decode_drafts_split_edges_and_window():
    """Draft rows straddling the 512-key split boundaries (the rows' partials of one split may
    be empty), and a paged window with a sink."""
    import dataclasses
    ctx = np.array([4, 5, 511, 512, 513, 515, 516, 1025, 8195, 8196], np.int32)
    _, gl = configs.decode_batch(seed=730, B=len(ctx), ctx_range=(4, 5))
    bt, pool = configs.paged_layout(731, 1, ctx)
    gl = configs.Decode(gl.layer, gl.q, ctx, configs.cached_keys(731, 2, (pool, 128, 4, 192)),
                        configs.bf16_normal(731, 3, (pool, 128, 4, 128)), block_table=bt, name="drafts_split_edges")
    cfg = configs.with_drafts(gl, 4, seed=732)
    out, lse = decode_cfg(cfg)
    parity(out, lse, *oracle.decode(cfg), "drafts at split boundaries")
    sink = synth.normal_f32(synth.stream_seed(733, 9), (64,))
    cfg.layer = dataclasses.replace(cfg.layer, window=1000, sink=sink)
    out, lse = decode_cfg(cfg)
    parity(out, lse, *oracle.decode(cfg), "drafts, paged window 1000 with sink")


def _global_drafts(seed, ctx, q_len, sink=False):
    """A global-layer paged cache over contexts `ctx` scored by q_len draft rows per sequence."""
    import dataclasses
    bt, pool = configs.paged_layout(seed, 1, ctx)
    gl = configs.Decode(configs.global_layer(), None, ctx, configs.cached_keys(seed, 2, (pool, 128, 4, 192)),
                        configs.bf16_normal(seed, 3, (pool, 128, 4, 128)), block_table=bt,
                        name=f"global_drafts_{len(ctx)}")
    if sink:
        gl.layer = dataclasses.replace(gl.layer, sink=synth.normal_f32(synth.stream_seed(seed, 9), (64,)))
    return configs.with_drafts(gl, q_len, seed=seed + 1)


@pytest.mark.parametrize("q_len", [2, 4, 8])
def test_decode_drafts_global_tensor_core(q_len):
    """Draft rows of a global layer on a bf16 paged cache go through the tensor-core kernel
    (the q_len x 16 rows of a KV head in one 128-row tile) with page-aligned splits and the
    decode's combine pass: contexts that end just before, at and after a split boundary, a
    sink (the combine adds it once), and a batch whose longest context needs one split only
    (no workspace, final rows written by the kernel itself)."""
    ctx = np.array([q_len, q_len + 1, 127, 128, 129, 511, 512, 513, 512 + q_len - 1, 1024 + q_len, 2047, 3001],
                   np.int32)
    for sink in (False, True):
        cfg = _global_drafts(760 + q_len, ctx, q_len, sink)
        out, lse = decode_cfg(cfg)
        parity(out, lse, *oracle.decode(cfg), f"{cfg.name} sink={sink}")
    cfg = _global_drafts(765 + q_len, np.array([q_len, 100, 200, 256], np.int32), q_len, True)
    out, lse = decode_cfg(cfg)
    parity(out, lse, *oracle.decode(cfg), f"{cfg.name}: one split")


def test_decode_drafts_global_more_sequences_than_one_launch():
    """300 sequences: the tensor-core path launches per group of 256 sequences; rows of the
    second launch keep their global row numbers in the partials and the output."""
    ctx = synth.randint(synth.stream_seed(770, 0), 300, 2, 1400).astype(np.int32)
    cfg = _global_drafts(771, ctx, 2)
    out, lse = decode_cfg(cfg)
    sel = np.array([0, 1, 2, 127, 254, 255, 256, 257, 298, 299], np.int32)
    ro, rl = oracle.decode(cfg, seqs=sel)
    import torch
    rows = torch.as_tensor(np.repeat(sel, 2) * 2 + np.tile([0, 1], len(sel)), device=out.device)
    parity(out[rows], lse[rows], ro, rl, "300 sequences x 2 drafts")


def test_decode_kernels_by_route():
    """Which kernels a decode call launches: draft rows of a global layer on a bf16 paged cache
    run the tensor-core prefill kernel and the combine pass, not the decode kernel; one token
    per sequence runs the decode kernel."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    cfg = _global_drafts(780, np.array([700, 3000, 5000], np.int32), 4)
    one = configs.with_drafts(cfg, 1, seed=781)
    decode_cfg(cfg)
    decode_cfg(one)
    torch.cuda.synchronize()
    names = []
    for c in (cfg, one):
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            decode_cfg(c)
            torch.cuda.synchronize()
        names.append(" ".join(e.name for e in prof.events() if "mimo" in e.name))
    assert "prefill_kernel" in names[0] and "decode_combine_kernel" in names[0], names[0]
    assert "decode_kernel<" not in names[0], names[0]
    assert "decode_kernel<" in names[1] and "prefill_kernel" not in names[1], names[1]


@pytest.mark.parametrize("ring", [False, True])
def test_decode_drafts_fp8(ring):
    import dataclasses
    cfg = configs.decode_fp8(seed=740 + ring, B=8, ctx_range=(4, 3000), ring=ring)
    if ring:  # 128 slots: window + q_len - 1 <= 128
        cfg.layer = dataclasses.replace(cfg.layer, window=125)
    cfg = configs.with_drafts(cfg, 4, seed=742)
    out, lse = decode_cfg(cfg)
    parity(out, lse, *oracle.decode(cfg), cfg.name)


@pytest.mark.parametrize("q_len", [2, 4, 8])
def test_verify_through_the_decode_kernel(q_len):
    """The verification workloads scored by the decode kernel (drafts appended to the paged
    cache or to a 144-slot ring, one decode call with q_len rows per sequence) equal the
    oracle's chunked prefill of the drafts."""
    glb, swa = configs.verify(seed=750 + q_len, B=12, q_len=q_len, ctx_range=(q_len + 1, 3000))
    for cfg in (glb, swa):
        out, lse = verify_decode_cfg(cfg)
        parity(out, lse, *oracle.chunked(cfg, rows=np.arange(int(cfg.cu_new[-1]))), cfg.name + " (decode kernel)")


def test_verify_b64_through_the_decode_kernel(dec64):
    _, gl = dec64
    glb, swa = configs.verify(B=64, q_len=4, decode=gl)
    for cfg in (glb, swa):
        out, lse = verify_decode_cfg(cfg)
        parity(out, lse, *oracle.chunked(cfg, rows=np.arange(64 * 4)), cfg.name + " (decode kernel)")


def test_decode_matches_last_prefill_row():
    """Appending a sequence to the caches and decoding its last token gives the last prefill row."""
    import torch
    import global_attention_attn_b200 as M
    for hkv, base, window, sink, slots in [(8, 1e4, 128, True, 128), (8, 1e4, 129, True, 144),
                                           (4, 1e7, 0, False, 0)]:
        S = 700
        cfg = make_prefill([S], hkv, base, window, sink, 500 + hkv + window)
        out, lse = prefill_cfg(cfg)
        # the ring keeps the last `slots` positions: append only those (one call may not reuse a slot)
        first = S - slots if window else 0
        pos = np.arange(first, S, dtype=np.int32)
        seq = np.zeros(S - first, np.int32)
        if window:
            kc = torch.zeros((1, slots, hkv, 192), dtype=torch.bfloat16, device="cuda")
            vc = torch.zeros((1, slots, hkv, 128), dtype=torch.bfloat16, device="cuda")
            extra = dict(cache_kind=M.MIMO_CACHE_RING, ring_slots=slots)
        else:
            npg = (S + 127) // 128
            bt = dev_i32(synth.permutation(3, npg)[None, :])
            kc = torch.zeros((npg, 128, hkv, 192), dtype=torch.bfloat16, device="cuda")
            vc = torch.zeros((npg, 128, hkv, 128), dtype=torch.bfloat16, device="cuda")
            extra = dict(cache_kind=M.MIMO_CACHE_PAGED, block_table=bt, num_pages=npg)
        M.mimo_kv_append(dev_bf16(cfg.k[first:]), dev_bf16(cfg.v[first:]), dev_i32(pos), dev_i32(seq),
                         rope_base=base, k_cache=kc, v_cache=vc, num_seqs=1, **extra)
        dout, dlse = M.mimo_attn_decode(dev_bf16(cfg.q[S - 1:]), dev_i32([S]), max_seq_len=S, num_kv_heads=hkv,
                                        rope_base=base, window=window, sink=dev_f32(cfg.layer.sink), k_cache=kc,
                                        v_cache=vc, **extra)
        d = (dout.float() - out[S - 1:].float()).abs()
        assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3
        assert (dlse - lse[S - 1:]).abs().max().item() <= 1e-3
