#!/usr/bin/env python
"""Benchmark of the MiMo-V2.6-Flash hybrid attention forward (libmimoattn) on B200.

A step is one pass of the hot path over one batch: the sliding-window layer's
varlen prefill of 8 sequences with lengths uniform in [1024, 8192] (RoPE on Q/K,
QK^T, window-128 mask, online softmax with the per-head sink, PV, epilogue).
`value` is algorithmic TFLOP/s (640 FLOP per visible (query head, key) pair)
over all GPUs; each GPU runs its own replica of the workload (the path has no
exchange step: "weak" scaling, replicas only).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--main-only]

With --gpus N > 1 launch it under torchrun (one process per GPU).  Rank 0
prints one JSON line.  Besides the contract keys the line carries `per_config`:
the other four workloads measured the same way (prefill TFLOP/s, decode GB/s,
fraction of the roofline max(FLOP / bf16 peak, bytes / HBM peak)).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import configs  # noqa: E402

METRIC = "SWA+sink / global attn prefill TFLOP/s, decode KV GB/s; % of B200 roofline"
FLOP_PER_PAIR = 2 * 192 + 2 * 128  # QK^T and PV per visible (query head, key) pair

# The step's dominant kernel (about 96% of the step's device time in the ncu launch list).
DOMINANT = "prefill_swa_kernel"
# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant kernel on the timed
# workload, from one ncu capture of the kernel on a 2 x 4096-token sliding-window prefill
# (inputs larger than L2) scaled by tokens to the 40696-token workload (the kernel's traffic
# is proportional to tokens): 249.64 MB read + 101.57 MB written.  None whenever the kernel
# changes after the capture.
TRAFFIC_BYTES = {"prefill_swa_kernel": int((249644800 + 101571328) * 40696 / 8192)}


# ----------------------------------------------------------------------------- roofline inputs

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def prefill_counts(cfg):
    """Algorithmic FLOP and bytes of a contiguous prefill (workloads.configs.Prefill)."""
    pairs = 0
    for s in range(cfg.num_seqs):
        ql, kl = int(cfg.q_lens[s]), int(cfg.k_lens[s])
        pos = np.arange(kl - ql, kl, dtype=np.int64)
        vis = np.minimum(pos + 1, cfg.layer.window) if cfg.layer.window else pos + 1
        pairs += int(vis.sum())
    tq, tk, h = int(cfg.cu_q[-1]), int(cfg.cu_k[-1]), cfg.layer.num_kv_heads
    by = tq * 64 * (192 * 2 + 128 * 2 + 4) + tk * h * (192 + 128) * 2 + 4 * (2 * cfg.num_seqs + 2)
    return pairs * 64 * FLOP_PER_PAIR, by


def decode_counts(cfg):
    L = cfg.layer
    vis = np.minimum(cfg.ctx, L.window) if L.window else cfg.ctx
    keys = int(vis.astype(np.int64).sum())
    B = len(cfg.ctx)
    esize = 1 if getattr(cfg, "cache_dtype", 0) == 1 else 2  # E4M3 or bf16 cache elements
    by = keys * L.num_kv_heads * (192 + 128) * esize + B * 64 * (192 * 2 + 128 * 2 + 4) + B * 4
    if cfg.paged:
        by += int(((cfg.ctx + 127) // 128).sum()) * 4
    return keys * 64 * FLOP_PER_PAIR, by


def chunked_counts(cfg):
    """Algorithmic FLOP and bytes of a chunked prefill (workloads.configs.Chunked), any number
    of sequences: queries and outputs once, every key the chunk attends once per KV head, and
    for a paged layer the append (the chunk's keys and values read and written)."""
    L = cfg.layer
    lens = np.diff(cfg.cu_new).astype(np.int64)
    pairs = keys_read = 0
    for s in range(len(lens)):
        start, n = int(cfg.start[s]), int(lens[s])
        pos = start + np.arange(n, dtype=np.int64)
        vis = np.minimum(pos + 1, L.window) if L.window else pos + 1
        pairs += int(vis.sum())
        ctx = start + n
        keys_read += min(ctx, n + L.window - 1) if L.window else ctx
    n = int(lens.sum())
    by = n * 64 * (192 * 2 + 128 * 2 + 4) + keys_read * L.num_kv_heads * (192 + 128) * 2
    if cfg.paged:
        by += n * L.num_kv_heads * (192 + 128) * 2 * 2
    return pairs * 64 * FLOP_PER_PAIR, by


def verify_counts(cfg):
    """Draft verification: the chunk's counts (queries and outputs once, every key the drafts
    attend once per KV head) plus the append of the drafts' keys and values to the cache."""
    flops, by = chunked_counts(cfg)
    if not cfg.paged:  # chunked_counts already counts the append of a paged layer
        by += int(cfg.cu_new[-1]) * cfg.layer.num_kv_heads * (192 + 128) * 2 * 2
    return flops, by


def roofline_us(flops, by, hbm, tf):
    return max(flops / (tf * 1e12), by / (hbm * 1e9)) * 1e6


# ----------------------------------------------------------------------------- clocks

_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x10: "sync_boost"}


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML every ~0.2 ms (the
    timed region of the default step count lasts about 10 ms), in a thread."""

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz, self.err = [], set(), None, None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report it, never guess
            self.h, self.err = None, f"nvml unavailable: {e}"

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_reasons(self.h)
                for bit, name in _REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(0.0002)

    def __enter__(self):
        # the launching thread holds the interpreter lock between calls; hand it over every
        # 0.1 ms (the default is 5 ms) so that the sampler runs during a ~10 ms timed region
        self._switch = sys.getswitchinterval()
        sys.setswitchinterval(1e-4)
        if self.h is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.h is not None:
            self.t.join()
        sys.setswitchinterval(self._switch)

    def summary(self):
        d = {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
             "reasons": sorted(self.reasons), "samples": len(self.samples)}
        if self.err:
            d["note"] = self.err
        return d


# ----------------------------------------------------------------------------- helpers

def dev_bf16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def dev_i32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.int32))).cuda()


def dev_f32(a):
    import torch
    return None if a is None else torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.float32))).cuda()


def event_time_ms(fn, iters, flush=None):
    """Device time of `iters` calls of fn on the current stream (CUDA events, synchronised on
    both sides).  With `flush`, L2 is flushed before each call and only the calls are timed."""
    import torch
    s = torch.cuda.current_stream()
    if flush is None:
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(iters):
            fn()
        b.record(s)
        torch.cuda.synchronize()
        return a.elapsed_time(b)
    tot = 0.0
    for _ in range(iters):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        fn()
        b.record(s)
        torch.cuda.synchronize()
        tot += a.elapsed_time(b)
    return tot


def timed_steps_ms(step, iters):
    """Device time of `iters` back-to-back steps, and the summed device time of the attention
    kernel inside them (events the library records on the launching stream around that
    kernel's launch).  Returns (step total ms, kernel total ms)."""
    import torch
    s = torch.cuda.current_stream()
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for a, b in pairs:  # create the event handles before the timed region
        a.record(s)
        b.record(s)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s)
    for ev in pairs:
        step(kernel_events=ev)
    t1.record(s)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1), sum(a.elapsed_time(b) for a, b in pairs)


class Prefill:
    """Device-resident prefill workload plus the call through the C ABI."""

    def __init__(self, cfg):
        import torch
        import global_attention_attn_b200 as M
        self.cfg, self.M = cfg, M
        L = cfg.layer
        self.q, self.k, self.v = dev_bf16(cfg.q), dev_bf16(cfg.k), dev_bf16(cfg.v)
        self.cq, self.ck, self.sink = dev_i32(cfg.cu_q), dev_i32(cfg.cu_k), dev_f32(L.sink)
        T = self.q.shape[0]
        self.out = torch.empty((T, 64, 128), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty((T, 64), dtype=torch.float32, device="cuda")
        n = M.prefill_workspace_size(cfg.num_seqs, T, self.k.shape[0], L.num_kv_heads, M.MIMO_CACHE_NONE)
        self.ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")

    def __call__(self, kernel_events=None):
        L = self.cfg.layer
        self.M.mimo_attn_prefill(self.q, self.k, self.v, self.cq, self.ck, num_kv_heads=L.num_kv_heads,
                                 rope_base=L.rope_base, window=L.window, sink=self.sink, out=self.out, lse=self.lse,
                                 workspace=self.ws, kernel_events=kernel_events)


class HostPipeline:
    """End-to-end prefill from pinned host buffers through the C ABI, one call per sequence
    on the caller's stream: the inputs of later sequences travel host -> device on one copy
    stream while a sequence computes, and the outputs of earlier ones travel back on another
    (PCIe carries both directions at once).  Every step copies all of its inputs in and
    all of its outputs out.  Sequences go longest first, so the output copy left after the
    last call (the step's tail) is the shortest one."""

    def __init__(self, step):
        import torch
        cfg = step.cfg
        if list(cfg.cu_q) != list(cfg.cu_k):
            raise ValueError("contiguous prefill with as many queries as keys per sequence")
        self.step, self.M = step, step.M
        self.cu = [int(x) for x in cfg.cu_q]
        pin = lambda t: t.cpu().pin_memory()
        self.q_h, self.k_h, self.v_h, self.s_h = pin(step.q), pin(step.k), pin(step.v), pin(step.sink)
        self.out_h = torch.empty_like(step.out, device="cpu").pin_memory()
        self.lse_h = torch.empty_like(step.lse, device="cpu").pin_memory()
        lens = np.diff(np.asarray(self.cu))
        self.order = [int(i) for i in np.argsort(-lens, kind="stable")]
        self.cu1_h = [pin(torch.tensor([0, int(n)], dtype=torch.int32)) for n in lens]
        self.cu1_d = [torch.empty(2, dtype=torch.int32, device="cuda") for _ in lens]
        self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def bytes(self):
        ins = [self.q_h, self.k_h, self.v_h, self.s_h] + self.cu1_h
        return (sum(t.numel() * t.element_size() for t in ins),
                sum(t.numel() * t.element_size() for t in (self.out_h, self.lse_h)))

    def __call__(self):
        import torch
        st, M, L, cu = self.step, self.M, self.step.cfg.layer, self.cu
        cur = torch.cuda.current_stream()
        self.s_in.wait_stream(cur)   # the previous step's calls and copies are done
        self.s_out.wait_stream(cur)
        arrived = {}
        with torch.cuda.stream(self.s_in):
            st.sink.copy_(self.s_h, non_blocking=True)
            for s in self.order:
                a, b = cu[s], cu[s + 1]
                st.q[a:b].copy_(self.q_h[a:b], non_blocking=True)
                st.k[a:b].copy_(self.k_h[a:b], non_blocking=True)
                st.v[a:b].copy_(self.v_h[a:b], non_blocking=True)
                self.cu1_d[s].copy_(self.cu1_h[s], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.s_in)
                arrived[s] = ev
        for s in self.order:
            a, b = cu[s], cu[s + 1]
            cur.wait_event(arrived[s])
            M.mimo_attn_prefill(st.q[a:b], st.k[a:b], st.v[a:b], self.cu1_d[s], self.cu1_d[s],
                                num_kv_heads=L.num_kv_heads, rope_base=L.rope_base, window=L.window,
                                sink=st.sink, out=st.out[a:b], lse=st.lse[a:b], workspace=st.ws)
            done = torch.cuda.Event()
            done.record(cur)
            self.s_out.wait_event(done)
            with torch.cuda.stream(self.s_out):
                self.out_h[a:b].copy_(st.out[a:b], non_blocking=True)
                self.lse_h[a:b].copy_(st.lse[a:b], non_blocking=True)
        cur.wait_stream(self.s_out)


class Decode:
    def __init__(self, cfg):
        import torch
        import global_attention_attn_b200 as M
        self.cfg, self.M = cfg, M
        L = cfg.layer
        self.q, self.ctx = dev_bf16(cfg.q), dev_i32(cfg.ctx)
        self.fp8 = {}
        if cfg.cache_dtype == M.MIMO_DTYPE_FP8_E4M3:
            self.kc = torch.from_numpy(np.ascontiguousarray(cfg.k_cache)).cuda()
            self.vc = torch.from_numpy(np.ascontiguousarray(cfg.v_cache)).cuda()
            self.fp8 = dict(cache_dtype=cfg.cache_dtype, k_dequant=dev_f32(cfg.k_dequant), v_dequant=dev_f32(cfg.v_dequant))
        else:
            self.kc, self.vc = dev_bf16(cfg.k_cache), dev_bf16(cfg.v_cache)
        self.sink = dev_f32(L.sink)
        self.extra = dict(cache_kind=M.MIMO_CACHE_PAGED, block_table=dev_i32(cfg.block_table),
                          num_pages=cfg.k_cache.shape[0]) if cfg.paged else \
            dict(cache_kind=M.MIMO_CACHE_RING, ring_slots=cfg.k_cache.shape[1])
        B = self.q.shape[0]
        self.out = torch.empty((B, 64, 128), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty((B, 64), dtype=torch.float32, device="cuda")
        n = M.decode_workspace_size(B, int(cfg.ctx.max()), L.num_kv_heads, L.window)
        self.ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")

    def __call__(self, kernel_events=None):
        L = self.cfg.layer
        self.M.mimo_attn_decode(self.q, self.ctx, max_seq_len=int(self.cfg.ctx.max()), num_kv_heads=L.num_kv_heads,
                                rope_base=L.rope_base, window=L.window, k_cache=self.kc, v_cache=self.vc,
                                sink=self.sink, out=self.out, lse=self.lse, workspace=self.ws,
                                kernel_events=kernel_events, **self.extra, **self.fp8)


class Chunked:
    """Global layer: append the chunk to the paged cache, then prefill from the cache.
    Sliding layer: prefill from the ring (prefix tail) plus the new rows."""

    def __init__(self, cfg):
        import torch
        import global_attention_attn_b200 as M
        self.cfg, self.M = cfg, M
        L = cfg.layer
        n = int(cfg.cu_new[-1])
        self.q, self.k, self.v = dev_bf16(cfg.q), dev_bf16(cfg.k_new), dev_bf16(cfg.v_new)
        self.cu = dev_i32(cfg.cu_new)
        self.kc, self.vc = dev_bf16(cfg.k_cache), dev_bf16(cfg.v_cache)
        self.sink = dev_f32(L.sink)
        self.out = torch.empty((n, 64, 128), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty((n, 64), dtype=torch.float32, device="cuda")
        lens = np.diff(cfg.cu_new)
        B = len(lens)
        if cfg.paged:
            self.bt = dev_i32(cfg.block_table)
            self.pos = dev_i32(np.concatenate([cfg.start[s] + np.arange(lens[s]) for s in range(B)]))
            self.seq = dev_i32(np.repeat(np.arange(B), lens))
            self.ctx = dev_i32(cfg.start + lens)
            self.ws = None
        else:
            self.start = dev_i32(cfg.start)
            w = M.prefill_workspace_size(B, n, n, L.num_kv_heads, M.MIMO_CACHE_RING)
            self.ws = torch.empty(w, dtype=torch.uint8, device="cuda")

    def __call__(self):
        M, L, cfg = self.M, self.cfg.layer, self.cfg
        if cfg.paged:
            M.mimo_kv_append(self.k, self.v, self.pos, self.seq, rope_base=L.rope_base, cache_kind=M.MIMO_CACHE_PAGED,
                             k_cache=self.kc, v_cache=self.vc, num_seqs=len(cfg.start), block_table=self.bt,
                             num_pages=cfg.k_cache.shape[0])
            M.mimo_attn_prefill(self.q, None, None, self.cu, None, num_kv_heads=L.num_kv_heads, rope_base=L.rope_base,
                                window=L.window, sink=self.sink, cache_lens=self.ctx, cache_kind=M.MIMO_CACHE_PAGED,
                                k_cache=self.kc, v_cache=self.vc, block_table=self.bt,
                                num_pages=cfg.k_cache.shape[0], out=self.out, lse=self.lse)
        else:
            M.mimo_attn_prefill(self.q, self.k, self.v, self.cu, self.cu, num_kv_heads=L.num_kv_heads,
                                rope_base=L.rope_base, window=L.window, sink=self.sink, cache_lens=self.start,
                                cache_kind=M.MIMO_CACHE_RING, k_cache=self.kc, v_cache=self.vc, out=self.out,
                                lse=self.lse, workspace=self.ws)


class Verify:
    """Draft verification through the decode kernel: the q_len draft tokens of every sequence
    are appended to the cache (the paged cache, or a ring of 144 slots holding the prefix tail
    and the drafts), then scored by one decode call with q_len query rows per sequence."""

    def __init__(self, cfg, ring_slots=144):
        import torch
        import global_attention_attn_b200 as M
        self.cfg, self.M = cfg, M
        L = cfg.layer
        lens = np.diff(cfg.cu_new)
        self.q_len = int(lens[0])
        B = len(cfg.start)
        self.q, self.k, self.v = dev_bf16(cfg.q), dev_bf16(cfg.k_new), dev_bf16(cfg.v_new)
        self.pos = dev_i32(np.repeat(cfg.start, self.q_len) + np.tile(np.arange(self.q_len), B))
        self.seq = dev_i32(np.repeat(np.arange(B), self.q_len))
        ctx = (cfg.start + self.q_len).astype(np.int32)
        self.ctx, self.max_len = dev_i32(ctx), int(ctx.max())
        if cfg.paged:
            self.kc, self.vc = dev_bf16(cfg.k_cache), dev_bf16(cfg.v_cache)
            self.extra = dict(cache_kind=M.MIMO_CACHE_PAGED, block_table=dev_i32(cfg.block_table),
                              num_pages=cfg.k_cache.shape[0])
        else:
            rk, rv = configs.ring_from_chunk(cfg, ring_slots)
            self.kc, self.vc = dev_bf16(rk), dev_bf16(rv)
            self.extra = dict(cache_kind=M.MIMO_CACHE_RING, ring_slots=ring_slots)
        self.sink = dev_f32(L.sink)
        n = B * self.q_len
        self.out = torch.empty((n, 64, 128), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty((n, 64), dtype=torch.float32, device="cuda")
        w = M.decode_workspace_size(B, self.max_len, L.num_kv_heads, L.window, self.q_len)
        self.ws = torch.empty(max(w, 256), dtype=torch.uint8, device="cuda")

    def __call__(self):
        M, L = self.M, self.cfg.layer
        M.mimo_kv_append(self.k, self.v, self.pos, self.seq, rope_base=L.rope_base, k_cache=self.kc, v_cache=self.vc,
                         num_seqs=len(self.cfg.start), **self.extra)
        M.mimo_attn_decode(self.q, self.ctx, max_seq_len=self.max_len, num_kv_heads=L.num_kv_heads,
                           rope_base=L.rope_base, window=L.window, k_cache=self.kc, v_cache=self.vc, sink=self.sink,
                           out=self.out, lse=self.lse, workspace=self.ws, q_len=self.q_len, **self.extra)


def host_call_us(call, n=50):
    """Host wall time of one call (the Python binding's marshalling, the library's validation,
    tensor-map encoding and launches), the device kept busy by nothing else."""
    import torch
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(n):
        call()
    dt = (time.perf_counter() - t0) / n
    torch.cuda.synchronize()
    return dt * 1e6


def graph_replay_us(call, flush_buf, n=100):
    """Device time of one call when n calls are replayed from a CUDA graph (no host launch
    overhead between them), each after an L2 flush: a graph of n x (flush + call) minus a
    graph of n flushes, divided by n.  The library neither allocates nor synchronises, so a
    call can be captured as it is."""
    import torch
    torch.cuda.synchronize()
    graphs = []
    for with_call in (True, False):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n):
                flush_buf.fill_(1)
                if with_call:
                    call()
        graphs.append(g)
    times = []
    for g in graphs:
        g.replay()  # warm
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1e3)
    del graphs
    return (times[0] - times[1]) / n


def graph_entry(call, flush_buf, troof_us, n=100):
    """graph_replay_us as a bench entry; a capture that fails is reported, not raised."""
    try:
        us = graph_replay_us(call, flush_buf, n)
        return {"us": us, "frac": troof_us / us, "launches_replayed": n,
                "method": f"CUDA graph of {n} x (L2 flush + call) minus a graph of {n} flushes"}
    except Exception as ex:  # report and go on: the event-timed number stands
        return {"error": f"{type(ex).__name__}: {str(ex)[:200]}"}


def l2_flusher():
    import torch
    buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    return lambda: buf.fill_(1)


# ----------------------------------------------------------------------------- CPU baseline (oracle)

def cpu_baseline(cfg, max_seconds=12.0):
    """The float64 oracle, as it stands, on a bounded sample of the workload's query rows."""
    import oracle
    cores = oracle.default_threads()
    total = int(cfg.cu_q[-1])
    # calibrate on a small sample, then size the sample to about max_seconds
    probe = configs.sample_rows(7, total, 256)
    oracle.prefill(cfg, rows=probe[:16], nthreads=cores)  # load the library, start the threads
    t0 = time.perf_counter()
    oracle.prefill(cfg, rows=probe, nthreads=cores)
    dt = time.perf_counter() - t0
    n = int(min(total, max(256, 256 * max_seconds / max(dt, 1e-3))))
    for attempt in range(2):
        rows = configs.sample_rows(8 + attempt, total, n)
        t0 = time.perf_counter()
        oracle.prefill(cfg, rows=rows, nthreads=cores)
        dt = time.perf_counter() - t0
        if dt >= max_seconds / 3 or n >= total:
            break
        n = int(min(total, n * max_seconds / max(dt, 1e-3)))
    flops = _rows_flops(cfg, rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(rows)} of {total} query rows (all 64 heads), float64, {dt:.1f} s"}


def _rows_flops(cfg, rows):
    cu = cfg.cu_q.astype(np.int64)
    seq = np.searchsorted(cu, rows, side="right") - 1
    pos = (cfg.q_pos0[seq] + (rows - cu[seq])).astype(np.int64)
    vis = np.minimum(pos + 1, cfg.layer.window) if cfg.layer.window else pos + 1
    return int(vis.sum()) * 64 * FLOP_PER_PAIR


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is a bounded sample of the same workload."""
    if rank != 0:
        return 0
    import oracle
    cfg = configs.swa_varlen_prefill()
    cores = oracle.default_threads()
    total = int(cfg.cu_q[-1])
    # size each step's sample so that warmup + steps take about two minutes of CPU time
    probe = configs.sample_rows(7, total, 256)
    t0 = time.perf_counter()
    oracle.prefill(cfg, rows=probe, nthreads=cores)
    per_row = (time.perf_counter() - t0) / 256
    n = int(min(4096, max(64, 120.0 / max(1, args.steps + args.warmup) / max(per_row, 1e-7))))
    rows = configs.sample_rows(9, total, n)
    flops = _rows_flops(cfg, rows)
    for _ in range(args.warmup):
        oracle.prefill(cfg, rows=rows, nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.prefill(cfg, rows=rows, nthreads=cores)
    dt = (time.perf_counter() - t0) / args.steps
    value = flops / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "num_seqs": cfg.num_seqs, "total_tokens": int(cfg.cu_q[-1]),
                       "window": 128, "parallelism": "replicas"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{len(rows)} of {int(cfg.cu_q[-1])} query rows per step (all 64 heads)"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- main arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--main-only", action="store_true", help="skip the per-config details and the CPU baseline")
    ap.add_argument("--profile", choices=["swa", "global", "decode", "decode_fp8", "decode_ring", "swa_chunk"],
                    help="run only a small case of one kernel (inputs > L2, < 1 GB on the device) for ncu captures")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    import torch
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    import global_attention_attn_b200 as M
    M.lib()
    hbm, tf_burst, tf_sust, peak_src = peaks()
    if args.profile:
        return run_profile_case(args)

    def barrier():
        if pg:
            pg.barrier()

    # ---------------- the timed workload: sliding-window varlen prefill
    cfg = configs.swa_varlen_prefill()
    flops, by = prefill_counts(cfg)
    step = Prefill(cfg)
    for _ in range(args.warmup):
        step()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_ms, k_ms = timed_steps_ms(step, args.steps)
    barrier()
    if pg:
        t_ms, k_ms = max_over_ranks([t_ms, k_ms], pg, "cuda")
    ms_step = t_ms / args.steps
    ms_kernel = k_ms / args.steps
    value = whole_job_rate(flops, world, ms_step) / 1e12
    achieved = by / (ms_kernel * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "traffic": TRAFFIC_BYTES.get(DOMINANT),
            "kernel": DOMINANT, "kernel_ms_per_launch": ms_kernel,
            "peak_source": f"{peak_src} hbm_gbs (burst copy)", "algorithmic_bytes_per_launch": by,
            "algorithmic_flop_per_launch": flops,
            "tensor_frac": flops / (ms_kernel * 1e-3) / 1e12 / tf_burst}

    # ---------------- end to end through the C ABI: host buffers, copies inside the timed region
    # (one call per sequence, with the next sequence's inputs and the previous one's outputs
    # crossing PCIe while a sequence computes)
    e2e_step = HostPipeline(step)
    h2d, d2h = e2e_step.bytes()
    for _ in range(2):
        e2e_step()
    ke = max(3, min(args.steps, 10))
    barrier()
    te = event_time_ms(e2e_step, ke) / ke
    if pg:
        te, = max_over_ranks([te], pg, "cuda")
    e2e = {"value": whole_job_rate(flops, world, te) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": te,
           "method": "pinned host buffers; per-sequence calls with H2D / D2H on two copy streams overlapping the calls"}
    del e2e_step

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg.name, "num_seqs": cfg.num_seqs, "total_tokens": int(cfg.cu_q[-1]),
                       "q_heads": 64, "kv_heads": 8, "head_dim_qk": 192, "head_dim_v": 128, "window": 128,
                       "sink": True, "rope_base": 1e4, "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2 ({by / 1e9:.2f} GB moved per step)"},
            "roofline": roof, "e2e": e2e, "gpu_launches": 2 * args.steps, "clocks": clk.summary()}

    # ---------------- per-config details and the CPU baseline (rank 0, one GPU)
    if rank == 0 and world == 1 and not args.main_only:
        del step
        torch.cuda.empty_cache()
        per = {}
        flush = l2_flusher()
        flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

        def measure(name, call, counts, iters, small, sustained=False):
            """One per-config entry: event-timed calls (L2 flushed before each call for the
            small workloads, whose inputs fit in L2), and for the microsecond-scale ones also
            the device time per call in a CUDA-graph replay and the host time the Python call
            itself takes (marshalling, tensor-map encoding, launches).  Every entry is set
            against the burst peaks (each call is timed on its own); sustained: a call long
            enough to reach the power cap's clocks also gets its fraction of the sustained
            bf16 peak, and the clocks it ran at."""
            flops, by = counts
            for _ in range(3):
                call()
            if small:
                ms = event_time_ms(call, iters, flush=flush) / iters
            else:
                with ClockSampler(local) as ck:  # the clocks the longer calls ran at
                    ms = event_time_ms(call, iters) / iters
            e = _entry(flops, by, ms, hbm, tf_burst, "L2 flushed before each call" if small else "inputs larger than L2")
            if sustained:  # the same call against the sustained peak, beside the burst one
                e["frac_sustained"] = roofline_us(flops, by, hbm, tf_sust) / (ms * 1e3)
            if not small:
                e["clocks"] = ck.summary()
            if small:
                e["graph_replay"] = graph_entry(call, flush_buf, e["roofline_us"])
                e["host_us_per_call"] = host_call_us(call)
            per[name] = e

        c0 = configs.swa_prefill_s512()
        measure("swa_prefill_s512", Prefill(c0), prefill_counts(c0), 50, True)
        c2 = configs.global_causal_prefill()
        measure("global_prefill_s16384", Prefill(c2), prefill_counts(c2), 10, False)
        del c2
        torch.cuda.empty_cache()
        sw, gl = configs.decode_batch()
        measure("swa_decode_b64_ring128", Decode(sw), decode_counts(sw), 20, True)
        measure("global_decode_b64_paged128", Decode(gl), decode_counts(gl), 20, False)
        # the SGLang window of the query plus 128 previous keys, decoded from 144-slot rings
        sw144, _ = configs.decode_batch(ring_slots=144)
        sw144.layer = dataclasses.replace(sw144.layer, window=129)
        measure("swa_decode_b64_ring144_window129", Decode(sw144), decode_counts(sw144), 20, True)
        del sw144
        # the same global decode over an E4M3 cache (per-KV-head scales)
        c8 = configs.decode_fp8(ctx=gl.ctx)
        measure("global_decode_b64_paged128_fp8", Decode(c8), decode_counts(c8), 20, False)
        del c8
        torch.cuda.empty_cache()
        # speculative verification: 4 draft tokens per sequence on the 64-sequence decode caches,
        # appended to the cache and scored by the decode kernel in one call
        vg, vs = configs.verify(B=64, q_len=4, decode=gl)
        measure("global_verify_b64_q4", Verify(vg), verify_counts(vg), 10, False)
        measure("swa_verify_b64_q4", Verify(vs), verify_counts(vs), 20, True)
        del sw, gl, vg, vs
        torch.cuda.empty_cache()
        g4, s4 = configs.chunked_prefill()
        # ~50 ms of tensor work per call: it reaches the power cap's clocks (the same kernel's
        # softmax takes 1.5x longer per key tile than in the 5 ms global prefill)
        measure("global_chunk_8192_on_120832", Chunked(g4), chunked_counts(g4), 5, False, sustained=True)
        measure("swa_chunk_8192_on_120832", Chunked(s4), chunked_counts(s4), 10, True)
        line["per_config"] = per
        line["cpu_baseline"] = cpu_baseline(cfg)
    print(json.dumps(line), flush=True) if rank == 0 else None
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def max_over_ranks(values, dist_mod, device):
    """Elementwise maximum of per-rank times over all ranks (every rank receives it): a
    replica run is as slow as its slowest GPU."""
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_rate(units_per_rank, world, ms):
    """Units all ranks processed per second, over the slowest rank's time."""
    return units_per_rank * world / (ms * 1e-3)


def profile_case(name):
    """Small workloads of each kernel for profiler captures: inputs larger than L2 (126 MB),
    well under a gigabyte on the device."""
    if name == "swa":
        lens = np.array([4096, 4096])
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        L = configs.swa_layer(configs.synth.normal_f32(configs.synth.stream_seed(5, 4), (64,)))
        T = int(cu[-1])
        return Prefill(configs.Prefill(L, configs.bf16_normal(5, 1, (T, 64, 192)), configs.bf16_normal(5, 2, (T, 8, 192)),
                                       configs.bf16_normal(5, 3, (T, 8, 128)), cu, cu.copy(), name="swa_prefill_2x4096"))
    if name == "global":
        return Prefill(configs.global_causal_prefill(S=4096))
    if name == "decode_fp8":
        return Decode(configs.decode_fp8(B=16))
    if name == "swa_chunk":
        return Chunked(configs.chunked_prefill(n_sample=8)[1])
    if name == "decode_ring":
        # the 64-sequence sliding-window decode over its 128-slot rings (44.6 MB, below L2;
        # ncu's default cache control flushes the caches before each captured pass)
        return Decode(configs.decode_batch()[0])
    sw, gl = configs.decode_batch(B=16)
    return Decode(gl)


def run_profile_case(args):
    import torch
    w = profile_case(args.profile)
    for _ in range(args.warmup + args.steps):
        w()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": args.profile, "launch_calls": args.warmup + args.steps}))
    return 0


def _entry(flops, by, ms, hbm, tf, l2):
    troof = roofline_us(flops, by, hbm, tf)
    return {"us": ms * 1e3, "TFLOP/s": flops / (ms * 1e-3) / 1e12, "GB/s": by / (ms * 1e-3) / 1e9,
            "roofline_us": troof, "frac": troof / (ms * 1e3),
            "bound": "tensor" if flops / (tf * 1e12) > by / (hbm * 1e9) else "hbm", "l2": l2}


if __name__ == "__main__":
    sys.exit(main())
