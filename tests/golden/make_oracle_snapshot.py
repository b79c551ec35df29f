"""Writes oracle_snapshot.json beside this file: float64 oracle outputs (a few rows, heads
and dims) on small seeded workloads of every kind the oracle serves (sliding-window and
global prefill, ring and paged decode, chunked prefill over a ring and a paged cache).

A regression guard, not a correctness pin: the oracle's correctness is pinned by
tests/test_oracle_pins.py.  tests/test_oracle_pins.py::test_oracle_snapshot recomputes
these values, so any later change to the oracle's arithmetic fails it until this script
is re-run, and that commit has to name the passage (or the reading of it) behind the
change.  Calls only oracle/ and the seeded generators.

    python tests/golden/make_oracle_snapshot.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import configs, synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_snapshot.json")
HEADS, DIMS = [0, 7, 8, 63], [0, 1, 64, 127]


def small_prefill(lens, hkv, base, window, sink, seed):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    s = synth.normal_f32(synth.stream_seed(seed, 4), (64,)) if sink else None
    L = configs.Layer("swa" if window else "global", hkv, base, window, s)
    return configs.Prefill(L, configs.bf16_normal(seed, 1, (T, 64, 192)), configs.bf16_normal(seed, 2, (T, hkv, 192)),
                           configs.bf16_normal(seed, 3, (T, hkv, 128)), cu, cu.copy())


def cases():
    """(name, oracle call) pairs; each returns (out [rows, 64, 128], lse [rows, 64])."""
    swa = small_prefill([5, 140], 8, 1e4, 128, True, 901)
    glb = small_prefill([70], 4, 1e7, 0, False, 902)
    dsw, dgl = configs.decode_batch(seed=903, B=3, ctx_range=(1, 300))
    cg, cs = configs.chunked_prefill(seed=904, prefix=200, chunk=40, n_sample=40)
    return [
        ("swa_prefill", lambda: oracle.prefill(swa, rows=[0, 4, 5, 132, 144])),
        ("global_prefill", lambda: oracle.prefill(glb, rows=[0, 1, 69])),
        ("swa_decode_ring", lambda: oracle.decode(dsw)),
        ("global_decode_paged", lambda: oracle.decode(dgl)),
        ("swa_chunk_ring", lambda: oracle.chunked(cs, rows=[0, 39])),
        ("global_chunk_paged", lambda: oracle.chunked(cg, rows=[0, 39])),
    ]


def snapshot():
    snap = {}
    for name, call in cases():
        out, lse = call()
        snap[name] = {"out": out[:, HEADS][:, :, DIMS].tolist(), "lse": lse[:, HEADS].tolist()}
    return snap


if __name__ == "__main__":
    with open(OUT, "w") as f:
        json.dump({"heads": HEADS, "dims": DIMS, "cases": snapshot()}, f, indent=1)
    print("wrote", OUT)
