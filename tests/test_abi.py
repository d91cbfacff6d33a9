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
