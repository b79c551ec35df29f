"""Multi-process host logic on CPU (gloo): the replica bench's max-over-ranks timing and the
context-parallel halo exchange of the sliding-window layers.  No GPU: the exchange is
checked on float32 rings whose slots carry position markers, written by a stand-in for
the key-append kernel."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

RING = 128


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank: int, world: int, port: int):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _run(fn, world: int, *args):
    mp.spawn(fn, args=(world, _free_port()) + args, nprocs=world, join=True)


# ----------------------------------------------------------------------------- replica timing

def _bench_worker(rank, world, port):
    _init(rank, world, port)
    try:
        import bench
        mx = bench.max_over_ranks([10.0 + rank, 5.0 - rank], dist, "cpu")
        assert mx == [10.0 + world - 1, 5.0], mx
        # value = units of all ranks over the slowest rank's time
        assert bench.whole_job_rate(100.0, world, mx[0]) == pytest.approx(100.0 * world / (mx[0] * 1e-3))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_bench_times_are_the_max_over_ranks(world):
    _run(_bench_worker, world)


# ----------------------------------------------------------------------------- CP halo exchange

def _marker(s: int, p: int) -> float:
    return float(p + 1 + 1000 * s)


def _cp_worker(rank, world, port, splits):
    _init(rank, world, port)
    try:
        from global_attention_attn_b200 import cp
        B, hkv = len(splits), 2
        lens = [splits[s][rank] for s in range(B)]
        starts = [sum(splits[s][:rank]) for s in range(B)]
        recv_k, recv_v = cp.ring_buffers(B, hkv, "cpu", torch.float32)
        send_k, send_v = cp.ring_buffers(B, hkv, "cpu", torch.float32)
        fills = []

        def fill(rk, rv):
            # stand-in for fill_ring_tail: slot p % 128 of sequence s gets marker(s, p)
            fills.append(1)
            for s, (row0, pos0, m) in enumerate(cp.tail_ranges(lens, starts)):
                assert row0 == sum(lens[:s]) + lens[s] - m and pos0 == starts[s] + lens[s] - m
                for p in range(pos0, pos0 + m):
                    rk[s, p % RING] = _marker(s, p)
                    rv[s, p % RING] = -_marker(s, p)

        cp.exchange_halo(send_k, send_v, recv_k, recv_v, fill, independent=cp.chunks_fill_ring(lens))
        assert len(fills) == (1 if rank + 1 < world else 0)
        # the received ring holds exactly the 128 positions before this rank's chunk
        for s in range(B):
            st = starts[s]
            for slot in range(RING):
                p = st - RING + (slot - (st - RING)) % RING
                want = _marker(s, p) if p >= 0 else 0.0
                assert torch.all(recv_k[s, slot] == want), (rank, s, slot, p, recv_k[s, slot, 0, 0].item())
                assert torch.all(recv_v[s, slot] == -want), (rank, s, slot, p)
        if rank == 0:
            with pytest.raises(ValueError):
                cp.swa_prefill_context_parallel(None, None, None, [5], [3], rope_base=1e4, window=128)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("splits", [
    # every chunk >= 128 positions: one round, no rank waits for another's ring
    [[200, 150], [300, 129]],
    # short chunks: the rings are relayed and a ring carries positions of several chunks
    [[50, 30, 200, 7], [300, 10, 5, 60]],
    # mixed: rank 1 relays, ranks 0 and 2 fill their rings alone
    [[130, 40, 500]],
], ids=["independent", "relay", "mixed"])
def test_cp_halo_exchange(splits):
    _run(_cp_worker, len(splits[0]), splits)


def _cp_subgroup_worker(rank, world, port):
    """Ranks 1 and 2 of 3 form the context-parallel group: group ranks map to global ranks."""
    _init(rank, world, port)
    try:
        from global_attention_attn_b200 import cp
        group = dist.new_group([1, 2])  # every rank takes part in creating it
        if rank in (1, 2):
            g = rank - 1
            lens, starts = [200 if g == 0 else 50], [0 if g == 0 else 200]
            recv_k, recv_v = cp.ring_buffers(1, 1, "cpu", torch.float32)
            send_k, send_v = cp.ring_buffers(1, 1, "cpu", torch.float32)

            def fill(rk, rv):
                for _, pos0, m in cp.tail_ranges(lens, starts):
                    for p in range(pos0, pos0 + m):
                        rk[0, p % RING] = _marker(0, p)
                        rv[0, p % RING] = -_marker(0, p)

            cp.exchange_halo(send_k, send_v, recv_k, recv_v, fill, independent=cp.chunks_fill_ring(lens), group=group)
            if g == 1:  # positions 72..199 from group rank 0
                for slot in range(RING):
                    p = 200 - RING + (slot - (200 - RING)) % RING
                    assert torch.all(recv_k[0, slot] == _marker(0, p)), (slot, p)
            else:
                assert torch.all(recv_k == 0)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_cp_halo_exchange_in_a_subgroup():
    _run(_cp_subgroup_worker, 3)


# ----------------------------------------------------------------------------- CP host logic

def test_cp_tail_ranges_and_modes():
    from global_attention_attn_b200 import cp
    # (first local row, first position, count) of the keys a later chunk's window reaches
    assert cp.tail_ranges([300, 50, 128], [1000, 0, 7]) == [(172, 1172, 128), (300, 0, 50), (350, 7, 128)]
    assert cp.chunks_fill_ring([128, 500]) and not cp.chunks_fill_ring([128, 127])


def test_cp_rejects_windows_beyond_the_halo():
    from global_attention_attn_b200 import cp
    q = torch.zeros((4, 64, 192), dtype=torch.bfloat16)
    for w in (0, 130):
        with pytest.raises(ValueError):
            cp.prefill_with_halo(q, None, None, [4], [0], None, None, rope_base=1e4, window=w)


def _cp_stream_worker(rank, world, port):
    """With a caller stream, every step of the context-parallel prefill (the ring appends,
    the NCCL transfers, the prefill) runs while that stream is the current one, because
    torch.distributed orders its transfers against the current stream."""
    _init(rank, world, port)
    from global_attention_attn_b200 import cp
    state = {"inside": False, "calls": []}

    class Scope:
        def __init__(self, s):
            assert s == "caller-stream"

        def __enter__(self):
            state["inside"] = True

        def __exit__(self, *a):
            state["inside"] = False

    saved = (torch.cuda.stream, cp.fill_ring_tail, cp.exchange_halo, cp.prefill_with_halo)
    try:
        torch.cuda.stream = Scope

        def fake_fill(rk, rv, k, v, chunk_lens, start_pos, *, rope_base, stream=None):
            state["calls"].append(("append", state["inside"], stream))

        def rec_exchange(*a, **kw):
            state["calls"].append(("exchange", state["inside"], None))
            return saved[2](*a, **kw)

        def fake_prefill(*a, stream=None, **kw):
            state["calls"].append(("prefill", state["inside"], stream))
            return "out", "lse"

        cp.fill_ring_tail, cp.exchange_halo, cp.prefill_with_halo = fake_fill, rec_exchange, fake_prefill
        q = torch.zeros((300, 64, 192), dtype=torch.bfloat16)
        k = torch.zeros((300, 2, 192), dtype=torch.bfloat16)
        res = cp.swa_prefill_context_parallel(q, k, k, [300], [300 * rank], rope_base=1e4, window=128,
                                              stream="caller-stream")
        assert res == ("out", "lse")
        names = [c[0] for c in state["calls"]]
        assert names == (["exchange", "append", "prefill"] if rank + 1 < world else ["exchange", "prefill"]), names
        # inside the caller's stream scope, with no other stream handed down
        assert all(inside and s is None for _, inside, s in state["calls"]), state["calls"]
        assert not state["inside"]
    finally:
        torch.cuda.stream, cp.fill_ring_tail, cp.exchange_halo, cp.prefill_with_halo = saved
        dist.destroy_process_group()


def test_cp_runs_every_step_on_the_caller_stream():
    _run(_cp_stream_worker, 2)
