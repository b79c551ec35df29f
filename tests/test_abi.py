"""CPU tests of the C-ABI boundary: the library loads, exports every entry point
that include/mimoattn.h declares, and rejects bad arguments on the host before
touching a device."""
import ctypes as C
import os
import re

import pytest

import global_attention_attn_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mimoattn.h")


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"MIMO_API\s+[\w\s\*]+?\b(mimo_\w+)\s*\(", src)


def test_header_declares_the_api():
    names = declared_functions()
    assert set(names) == set(M.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = M.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert b"sm_100a" in L.mimo_version()


def test_constants_match_header():
    src = open(HEADER).read()
    for name in ["MIMO_OK", "MIMO_ERR_INVALID_ARG", "MIMO_ERR_UNSUPPORTED", "MIMO_ERR_WORKSPACE", "MIMO_ERR_CUDA",
                 "MIMO_ERR_TIMEOUT", "MIMO_CACHE_NONE", "MIMO_CACHE_PAGED", "MIMO_CACHE_RING"]:
        m = re.search(rf"#define {name} (\d+)", src)
        assert m and int(m.group(1)) == getattr(M, name), name


def test_struct_layouts_match_c(tmp_path):
    """ctypes mirrors of the argument structs have the C compiler's sizes and field offsets."""
    import subprocess
    structs = {"mimo_layer": M.MimoLayer, "mimo_prefill_args": M.MimoPrefillArgs,
               "mimo_decode_args": M.MimoDecodeArgs, "mimo_append_args": M.MimoAppendArgs}
    lines = ["#include <stdio.h>", "#include <stddef.h>", f'#include "{HEADER}"', "int main(void) {"]
    for cname, py in structs.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-o", str(exe), str(src)])
    out = subprocess.check_output([str(exe)]).decode().split("\n")
    for line in filter(None, out):
        cname, field, val = line.split()
        py = structs[cname]
        got = C.sizeof(py) if field == "size" else getattr(py, field).offset
        assert got == int(val), (cname, field, got, val)


def test_workspace_sizes():
    # rotated key dims (fp16) + a cos/sin table of 32 float2 per query row
    assert M.prefill_workspace_size(1, 512, 512, 8, M.MIMO_CACHE_NONE) == 512 * 8 * 64 * 2 + 512 * 32 * 8
    assert M.prefill_workspace_size(3, 100, 100, 4, M.MIMO_CACHE_PAGED) == 0
    ring = M.prefill_workspace_size(1, 8192, 8192, 8, M.MIMO_CACHE_RING)
    assert ring >= (8192 + 128) * 8 * (192 + 128) * 2 + 8192 * 32 * 8
    assert M.decode_workspace_size(64, 128, 8, 128) == 0          # one split: no partials
    ns = (65536 + 1023) // 1024                                   # 1024-key splits past 8192 keys
    assert M.decode_workspace_size(64, 65536, 4, 0) >= 64 * 64 * ns * (128 + 2) * 4


FAKE = 1 << 20  # an aligned non-null address: validation runs before any device access


def _prefill_args(**over):
    a = M.MimoPrefillArgs()
    a.layer = M.make_layer(8, 1e4, 128)
    a.num_seqs, a.total_q, a.total_k = 1, 16, 16
    a.q = a.k = a.v = a.cu_seqlens_q = a.cu_seqlens_k = a.out = C.c_void_p(FAKE)
    a.workspace = C.c_void_p(FAKE)
    a.workspace_bytes = 1 << 30
    for k, v in over.items():
        if k.startswith("layer."):
            setattr(a.layer, k[6:], v)
        else:
            setattr(a, k, v)
    return a


@pytest.mark.parametrize("over,code", [
    ({"layer.num_q_heads": 32}, M.MIMO_ERR_UNSUPPORTED),
    ({"layer.head_dim_qk": 128}, M.MIMO_ERR_UNSUPPORTED),
    ({"layer.num_kv_heads": 2}, M.MIMO_ERR_UNSUPPORTED),
    ({"layer.window": -1}, M.MIMO_ERR_INVALID_ARG),
    ({"layer.rope_base": 0.0}, M.MIMO_ERR_INVALID_ARG),
    ({"layer.softmax_scale": float("nan")}, M.MIMO_ERR_INVALID_ARG),
    ({"num_seqs": 0}, M.MIMO_ERR_INVALID_ARG),
    ({"q": None}, M.MIMO_ERR_INVALID_ARG),
    ({"q": C.c_void_p(FAKE + 2)}, M.MIMO_ERR_INVALID_ARG),
    ({"out": None}, M.MIMO_ERR_INVALID_ARG),
    ({"workspace_bytes": 10}, M.MIMO_ERR_WORKSPACE),
    ({"workspace": None}, M.MIMO_ERR_WORKSPACE),
    ({"cache_kind": 7}, M.MIMO_ERR_INVALID_ARG),
    ({"cache_kind": M.MIMO_CACHE_PAGED}, M.MIMO_ERR_INVALID_ARG),          # paged: k/v must be NULL
    ({"cache_kind": M.MIMO_CACHE_RING, "layer.window": 0}, M.MIMO_ERR_INVALID_ARG),
    ({"layer.sink": C.c_void_p(FAKE + 2)}, M.MIMO_ERR_INVALID_ARG),
    ({"ring_slots": 96}, M.MIMO_ERR_INVALID_ARG),                          # below 128
    ({"ring_slots": 136}, M.MIMO_ERR_INVALID_ARG),                         # not a multiple of 16
    ({"ring_slots": 528}, M.MIMO_ERR_INVALID_ARG),                         # above 512
    ({"cache_kind": M.MIMO_CACHE_RING, "layer.window": 130, "k_cache": C.c_void_p(FAKE),
      "v_cache": C.c_void_p(FAKE), "cache_lens": C.c_void_p(FAKE)}, M.MIMO_ERR_INVALID_ARG),
])
def test_prefill_validation(over, code):
    a = _prefill_args(**over)
    rc = M.lib().mimo_attn_prefill(C.byref(a), None)
    assert rc == code, M.lib().mimo_last_error()
    assert M.lib().mimo_last_error().startswith(b"mimo_attn_prefill")


def test_prefill_empty_is_a_no_op():
    a = _prefill_args(total_q=0)
    assert M.lib().mimo_attn_prefill(C.byref(a), None) == M.MIMO_OK


def _decode_args(**over):
    a = M.MimoDecodeArgs()
    a.layer = M.make_layer(4, 1e7, 0)
    a.batch, a.max_seq_len = 4, 4096
    a.q = a.seq_lens = a.k_cache = a.v_cache = a.block_table = a.out = C.c_void_p(FAKE)
    a.cache_kind = M.MIMO_CACHE_PAGED
    a.max_pages, a.num_pages = 32, 128
    a.workspace = C.c_void_p(FAKE)
    a.workspace_bytes = 1 << 30
    for k, v in over.items():
        if k.startswith("layer."):
            setattr(a.layer, k[6:], v)
        else:
            setattr(a, k, v)
    return a


@pytest.mark.parametrize("over,code", [
    ({"batch": -1}, M.MIMO_ERR_INVALID_ARG),
    ({"max_seq_len": 0}, M.MIMO_ERR_INVALID_ARG),
    ({"cache_kind": M.MIMO_CACHE_NONE}, M.MIMO_ERR_INVALID_ARG),
    ({"cache_kind": M.MIMO_CACHE_RING}, M.MIMO_ERR_INVALID_ARG),         # ring needs window 1..128
    ({"block_table": None}, M.MIMO_ERR_INVALID_ARG),
    ({"max_pages": 8}, M.MIMO_ERR_INVALID_ARG),                           # 8 * 128 < 4096
    ({"workspace_bytes": 64}, M.MIMO_ERR_WORKSPACE),
    ({"layer.head_dim_v": 64}, M.MIMO_ERR_UNSUPPORTED),
    ({"seq_lens": None}, M.MIMO_ERR_INVALID_ARG),
    ({"cache_dtype": 5}, M.MIMO_ERR_INVALID_ARG),
    ({"cache_dtype": M.MIMO_DTYPE_FP8_E4M3}, M.MIMO_ERR_INVALID_ARG),     # E4M3 needs dequant scales
    ({"cache_dtype": M.MIMO_DTYPE_FP8_E4M3, "k_dequant": C.c_void_p(FAKE), "v_dequant": C.c_void_p(FAKE + 2)},
     M.MIMO_ERR_INVALID_ARG),                                             # misaligned scales
    ({"cache_kind": M.MIMO_CACHE_RING, "layer.window": 129}, M.MIMO_ERR_INVALID_ARG),   # 128 slots < 129 keys
    ({"cache_kind": M.MIMO_CACHE_RING, "layer.window": 145, "ring_slots": 144}, M.MIMO_ERR_INVALID_ARG),
    ({"ring_slots": 100}, M.MIMO_ERR_INVALID_ARG),
    ({"ring_slots": 1024}, M.MIMO_ERR_INVALID_ARG),
    ({"q_len": 9}, M.MIMO_ERR_INVALID_ARG),                                # beyond MIMO_MAX_DRAFTS
    ({"q_len": -1}, M.MIMO_ERR_INVALID_ARG),
    ({"q_len": 4, "max_seq_len": 3}, M.MIMO_ERR_INVALID_ARG),             # fewer positions than drafts
    ({"q_len": 4, "workspace_bytes": 64}, M.MIMO_ERR_WORKSPACE),           # the draft route's partials
    ({"q_len": 4, "workspace": None, "workspace_bytes": 0}, M.MIMO_ERR_WORKSPACE),
    ({"q_len": 4, "cache_kind": M.MIMO_CACHE_RING, "layer.window": 128, "ring_slots": 128},
     M.MIMO_ERR_INVALID_ARG),                                             # 128 + 4 - 1 keys > 128 slots
])
def test_decode_validation(over, code):
    a = _decode_args(**over)
    assert M.lib().mimo_attn_decode(C.byref(a), None) == code, M.lib().mimo_last_error()


def test_append_validation():
    a = M.MimoAppendArgs()
    a.num_tokens, a.num_kv_heads, a.head_dim_qk, a.head_dim_v, a.rope_dim, a.rope_base = 4, 8, 192, 128, 64, 1e4
    a.k_new = a.v_new = a.pos = a.seq_idx = a.k_cache = a.v_cache = C.c_void_p(FAKE)
    a.cache_kind, a.num_seqs = M.MIMO_CACHE_PAGED, 1
    assert M.lib().mimo_kv_append(C.byref(a), None) == M.MIMO_ERR_INVALID_ARG   # paged without a block table
    a.cache_kind = 9
    assert M.lib().mimo_kv_append(C.byref(a), None) == M.MIMO_ERR_INVALID_ARG
    a.cache_kind, a.rope_dim = M.MIMO_CACHE_RING, 32
    assert M.lib().mimo_kv_append(C.byref(a), None) == M.MIMO_ERR_UNSUPPORTED
    a.rope_dim, a.num_tokens = 64, 0
    assert M.lib().mimo_kv_append(C.byref(a), None) == M.MIMO_OK                 # nothing to append


def test_ring_slots_constants_match_header():
    src = open(HEADER).read()
    for name in ["MIMO_RING_SLOTS_DEFAULT", "MIMO_RING_SLOTS_MAX", "MIMO_STATUS_TIMEOUT", "MIMO_STATUS_BAD_INDEX",
                 "MIMO_STATUS_RANGE", "MIMO_STATUS_BAD_SCALE"]:
        m = re.search(rf"#define {name} (\d+)", src)
        assert m and int(m.group(1)) == getattr(M, name), name


@pytest.mark.parametrize("ns", [0, 999_999, 10_000_000_001])
def test_stall_test_rejects_limits_outside_its_range(ns):
    a = _prefill_args()
    assert M.lib().mimo_attn_prefill_stall_test(C.byref(a), None, ns) == M.MIMO_ERR_INVALID_ARG
    assert M.lib().mimo_last_error().startswith(b"mimo_attn_prefill_stall_test")


def test_append_rejects_bad_ring_slots():
    a = M.MimoAppendArgs()
    a.num_tokens, a.num_kv_heads, a.head_dim_qk, a.head_dim_v, a.rope_dim, a.rope_base = 4, 8, 192, 128, 64, 1e4
    a.k_new = a.v_new = a.pos = a.seq_idx = a.k_cache = a.v_cache = C.c_void_p(FAKE)
    a.cache_kind, a.num_seqs, a.ring_slots = M.MIMO_CACHE_RING, 1, 200
    assert M.lib().mimo_kv_append(C.byref(a), None) == M.MIMO_ERR_INVALID_ARG


def test_status_poll_rejects_null():
    assert M.lib().mimo_status_poll(None) == M.MIMO_ERR_INVALID_ARG


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "global_attention_attn_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in src.replace("Oracle", ""), f


@pytest.mark.parametrize("left,window", [(128, 129), (127, 128), (0, 1), (-1, 0), (2**31 - 2, 2**31 - 1)])
def test_window_from_left_right(left, window):
    assert M.mimo_window_from_left_right(left, 0) == window


@pytest.mark.parametrize("left,right,code", [(128, 1, "MIMO_ERR_UNSUPPORTED"), (127, -1, "MIMO_ERR_UNSUPPORTED"),
                                             (-2, 0, "MIMO_ERR_INVALID_ARG"), (2**31 - 1, 0, "MIMO_ERR_INVALID_ARG")])
def test_window_from_left_right_rejects(left, right, code):
    with pytest.raises(M.MimoError) as e:
        M.mimo_window_from_left_right(left, right)
    assert e.value.code == getattr(M, code)
    L = M.lib()
    assert L.mimo_window_from_left_right(128, 0, None) == M.MIMO_ERR_INVALID_ARG
