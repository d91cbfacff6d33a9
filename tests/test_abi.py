"""The C-ABI library loads and exports what include/pkv.h declares (CPU only).

These tests make no compute call: they check symbols, status strings and the
host-side argument checks, which return before any launch.
"""
import ctypes
import os
import re

import pytest

from paged_kv_gqa_scatter_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_calls():
    names = declared_functions()
    for required in ("pkv_store_kv", "pkv_decode_attn", "pkv_extend_attn", "pkv_gather_kv"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in pkv.h but not exported"
    assert set(declared_functions()) == set(_lib.SIGNATURES), "binding signatures out of sync"


def test_library_is_sm100a_build():
    # The build step compiles for sm_100a only.
    from paged_kv_gqa_scatter_b200 import build
    assert "arch=compute_100a,code=sm_100a" in build.ARCH


def test_status_strings():
    lib = _lib.load()
    assert lib.pkv_status_string(0) == b"ok"
    assert b"argument" in lib.pkv_status_string(1)
    assert lib.pkv_status_string(999) == b"unknown status"
    assert lib.pkv_version().startswith(b"pkv")


def _pool(**kw):
    base = dict(k=16, v=32, num_layers=1, num_slots=64, layer_stride=64 * 1024, slot_stride=1024,
                num_kv_heads=8, head_dim=128, page_size=1, dtype=0)
    base.update(kw)
    return _lib.PkvPool(**base)


def test_host_validation_rejects_bad_arguments():
    lib = _lib.load()
    dummy = 4096  # never dereferenced: every case fails validation first
    P = ctypes.byref
    # null pool
    assert lib.pkv_store_kv(None, 0, dummy, 1024, dummy, 1024, dummy, 0, 1, None, None) == 1
    # unsupported head_dim
    assert lib.pkv_store_kv(P(_pool(head_dim=64)), 0, dummy, 1024, dummy, 1024, dummy, 0, 1, None, None) == 2
    # unsupported dtype
    assert lib.pkv_store_kv(P(_pool(dtype=7)), 0, dummy, 1024, dummy, 1024, dummy, 0, 1, None, None) == 2
    # layer out of range
    assert lib.pkv_store_kv(P(_pool()), 3, dummy, 1024, dummy, 1024, dummy, 0, 1, None, None) == 1
    # misaligned pool pointer
    assert lib.pkv_store_kv(P(_pool(k=4104)), 0, dummy, 1024, dummy, 1024, dummy, 0, 1, None, None) == 3
    # misaligned slot stride (bf16: 1028 elements = 2056 bytes)
    assert lib.pkv_store_kv(P(_pool(slot_stride=1028, layer_stride=1028 * 64)), 0, dummy, 1024, dummy, 1024,
                            dummy, 0, 1, None, None) == 3
    # row stride shorter than a row
    assert lib.pkv_store_kv(P(_pool()), 0, dummy, 512, dummy, 1024, dummy, 0, 1, None, None) == 1
    # negative count
    assert lib.pkv_store_kv(P(_pool()), 0, dummy, 1024, dummy, 1024, dummy, 0, -1, None, None) == 1
    # zero tokens is a no-op that launches nothing
    assert lib.pkv_store_kv(P(_pool()), 0, dummy, 1024, dummy, 1024, dummy, 0, 0, None, None) == 0
    t = _lib.PkvPageTable(entries=dummy, rows=4, cols=64, row_stride=64)
    # GQA group size 3 is not built
    assert lib.pkv_decode_attn(P(_pool()), 0, dummy, 24, P(t), dummy, dummy, 2, 0.1, dummy, dummy,
                               1 << 20, None, None) == 2
    # Hq not a multiple of Hkv
    assert lib.pkv_decode_attn(P(_pool()), 0, dummy, 12, P(t), dummy, dummy, 2, 0.1, dummy, dummy,
                               1 << 20, None, None) == 1
    # batch beyond the documented maximum
    assert lib.pkv_decode_attn(P(_pool()), 0, dummy, 16, P(t), dummy, dummy, 5000, 0.1, dummy, dummy,
                               1 << 30, None, None) == 6
    # workspace too small
    assert lib.pkv_decode_attn(P(_pool()), 0, dummy, 16, P(t), dummy, dummy, 2, 0.1, dummy, dummy,
                               16, None, None) == 4
    # empty batch is a no-op
    assert lib.pkv_decode_attn(P(_pool()), 0, dummy, 16, P(t), dummy, dummy, 0, 0.1, dummy, dummy,
                               0, None, None) == 0
    # GQA group 16: decode on bf16 and E4M3 pools passes the head check (an empty
    # batch then launches nothing); fp32 pools, extend and groups of 32 are not built
    assert lib.pkv_decode_attn(P(_pool()), 0, dummy, 128, P(t), dummy, dummy, 0, 0.1, dummy, dummy,
                               0, None, None) == 0
    assert lib.pkv_decode_attn(P(_pool(dtype=2, k_scale=0.5, v_scale=0.5)), 0, dummy, 128, P(t), dummy, dummy, 0, 0.1,
                               dummy, dummy, 0, None, None) == 0
    assert lib.pkv_decode_attn(P(_pool(dtype=1, layer_stride=64 * 1024)), 0, dummy, 128, P(t), dummy, dummy, 2,
                               0.1, dummy, dummy, 1 << 20, None, None) == 2
    assert lib.pkv_decode_attn(P(_pool()), 0, dummy, 256, P(t), dummy, dummy, 2, 0.1, dummy, dummy,
                               1 << 20, None, None) == 2
    assert lib.pkv_extend_attn(P(_pool()), 0, dummy, 128, P(t), dummy, dummy, dummy, dummy, 2, 10,
                               5, 0.1, dummy, None, 0, None, None) == 2
    # bad table (row stride < cols)
    tb = _lib.PkvPageTable(entries=dummy, rows=4, cols=64, row_stride=8)
    assert lib.pkv_extend_attn(P(_pool()), 0, dummy, 16, P(tb), dummy, dummy, dummy, dummy, 2, 10,
                               5, 0.1, dummy, None, 0, None, None) == 1
    # slots not a multiple of page_size
    assert lib.pkv_gather_kv(P(_pool(page_size=16, num_slots=40, layer_stride=40 * 1024)), 0, P(t), dummy,
                             dummy, dummy, 2, dummy, dummy, None, None) == 1


def test_workspace_size_grows_with_batch_and_heads():
    lib = _lib.load()
    a = lib.pkv_decode_workspace_bytes(64, 16)
    b = lib.pkv_decode_workspace_bytes(256, 16)
    c = lib.pkv_decode_workspace_bytes(64, 32)
    assert 0 < a < b and a < c
    assert lib.pkv_decode_workspace_bytes(-1, 16) == 0


def test_host_validation_of_the_newer_calls():
    lib = _lib.load()
    dummy = 4096
    P = ctypes.byref
    t = _lib.PkvPageTable(entries=dummy, rows=4, cols=64, row_stride=64)
    row = (16 + 2 * 8) * 128
    # qk_norm_rope_store: (pool, layer, qkv, stride, hq, pos, pos64, cache, maxpos, qw, kw, eps,
    #                      loc, loc64, n, q_out, err, stream)
    rope = lambda **kw: lib.pkv_qk_norm_rope_store(
        P(kw.get("pool", _pool())), 0, kw.get("qkv", dummy), kw.get("stride", row), 16, dummy, 0, dummy,
        kw.get("maxpos", 4096), None, None, kw.get("eps", 1e-6), dummy, 0, kw.get("n", 4), dummy, None, None)
    assert rope(qkv=None) == 1
    assert rope(eps=-1.0) == 1
    assert rope(maxpos=0) == 1
    assert rope(stride=row - 8) == 1
    assert rope(qkv=dummy + 2) == 3
    assert rope(n=0) == 0
    # cascade decode: (pool, layer, q, hq, table, ti, sl, batch, off, pre, groups, maxp, scale, out,
    #                  ws, ws_bytes, err, stream)
    cas = lambda **kw: lib.pkv_decode_attn_cascade(
        P(kw.get("pool", _pool())), 0, dummy, 16, P(t), dummy, dummy, kw.get("batch", 4), dummy, dummy,
        kw.get("groups", 1), kw.get("maxp", 32), 0.1, dummy, dummy, kw.get("ws", 1 << 30), None, None)
    assert cas(pool=_pool(dtype=1, slot_stride=1024, layer_stride=64 * 1024)) == 2  # fp32 pool
    assert cas(groups=0) == 1
    assert cas(groups=5) == 1          # more groups than requests
    assert cas(maxp=65) == 6           # prefix longer than the table
    assert cas(ws=16) == 4
    assert cas(batch=0) == 0
    # FP8 pools need finite positive scales; rows written into them are bf16.
    f8 = lambda ks, vs: _pool(dtype=2, slot_stride=1024, layer_stride=64 * 1024, k_scale=ks, v_scale=vs)
    for ks, vs in ((0.0, 1.0), (1.0, -2.0), (float("inf"), 1.0), (float("nan"), 1.0)):
        assert lib.pkv_store_kv(P(f8(ks, vs)), 0, dummy, 1024, dummy, 1024, dummy, 0, 1, None, None) == 1
    assert lib.pkv_store_kv(P(f8(0.05, 0.09)), 0, dummy, 1024, dummy, 1024, dummy, 0, 0, None, None) == 0
    # bf16 rows of 1024 elements: a stride of 1028 bf16 elements breaks 16-byte rows
    assert lib.pkv_store_kv(P(f8(0.05, 0.09)), 0, dummy, 1028, dummy, 1024, dummy, 0, 1, None, None) == 3
    # self-test and workspace objects
    assert lib.pkv_selftest_wait_timeout(None, None) == 1
    h = ctypes.c_void_p()
    assert lib.pkv_workspace_create(0, 16, 0, P(h)) == 1 and not h.value
    assert lib.pkv_workspace_create(4, 16, -1, P(h)) == 1
    assert lib.pkv_workspace_create(4, 16, 0, None) == 1
    code = ctypes.c_int32()
    assert lib.pkv_read_device_error(None, None, P(code)) == 1
    n = ctypes.c_size_t(7)
    assert lib.pkv_workspace_buffer(None, P(n)) is None and n.value == 0
    assert lib.pkv_workspace_error_word(None) is None
    lib.pkv_workspace_destroy(None)  # a no-op


def test_cascade_workspace_size():
    lib = _lib.load()
    a = lib.pkv_decode_cascade_workspace_bytes(64, 16, 0)
    b = lib.pkv_decode_cascade_workspace_bytes(64, 16, 4096)
    c = lib.pkv_decode_cascade_workspace_bytes(64, 16, 32768)
    assert lib.pkv_decode_workspace_bytes(64, 16) <= a < b < c
    assert lib.pkv_decode_cascade_workspace_bytes(64, 16, -1) == 0
