"""pkv_decode_attn_noalloc against pkv_decode_attn and the oracle (needs a B200).

The no-allocation decode serves callers that cannot allocate device memory:
an engine that has already handed almost all free memory to its KV pool, or
code hosted by a framework that owns every allocation.  It runs the same
split and combine kernels, with the same grid, as the workspace version, so
its output must be bit-identical to that version's; it is also checked
against the float64 oracle.  The calls run in the order a, b, a on two
different workloads, so partial results that workload b leaves in the shared
scratch array would show up in the second result of a.  The call must not
change the device memory in use.  This file is collected last so that a
failure here cannot stop the rest of the suite under -x.
"""
import ctypes

import pytest
import torch

from gpu_helpers import DeviceDecode, from_dev, oracle_decode, tol_check
from paged_kv_gqa_scatter_b200 import _lib, api
from paged_kv_gqa_scatter_b200 import workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _reference(d: DeviceDecode) -> torch.Tensor:
    """Store the step's rows, then the existing entry point (caller-provided workspace)."""
    wl = d.wl
    api.store_kv(d.pool, wl.layer, d.k_new, d.v_new, d.out_loc, d.err)
    ref = torch.empty_like(d.q)
    api.decode_attn(d.pool, wl.layer, d.q, d.table, d.table_idx, d.seq_lens, ref, d.ws,
                    scale=wl.scale, dev_err=d.err)
    return ref


def _noalloc_c_call(d: DeviceDecode, out: torch.Tensor) -> int:
    """Call pkv_decode_attn_noalloc straight through the C ABI."""
    lib = _lib.load()
    wl = d.wl
    B, Hq, _ = d.q.shape
    return lib.pkv_decode_attn_noalloc(
        ctypes.byref(d.pool.c), wl.layer, d.q.data_ptr(), Hq, ctypes.byref(d.table.c),
        d.table_idx.data_ptr(), d.seq_lens.data_ptr(), B, ctypes.c_float(wl.scale), out.data_ptr(),
        d.err.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _memory():
    torch.cuda.synchronize()
    free, _ = torch.cuda.mem_get_info()
    return free, torch.cuda.memory_allocated()


def test_noalloc_matches_workspace_decode_bit_for_bit_in_order_a_b_a():
    # a: long contexts split across CTAs (partials go through the scratch);
    # b: a page_size-16 batch with other lengths, so the split points differ.
    a = DeviceDecode(W.decode_qwen3_06b(num_layers=1, layer=0))
    b = DeviceDecode(W.decode_paged_small())
    ref_a = _reference(a)
    ref_b = _reference(b)
    out_a1 = torch.full_like(a.q, float("nan"))
    out_b = torch.full_like(b.q, float("nan"))
    out_a2 = torch.full_like(a.q, float("nan"))
    assert _noalloc_c_call(a, out_a1) == 0
    before = _memory()
    assert _noalloc_c_call(b, out_b) == 0
    assert _noalloc_c_call(a, out_a2) == 0
    after = _memory()
    assert before == after, f"device memory changed across no-alloc calls: {before} -> {after}"
    assert torch.equal(out_a1, ref_a), "no-alloc call 1 (a) differs from the workspace decode"
    assert torch.equal(out_b, ref_b), "no-alloc call 2 (b) differs from the workspace decode"
    assert torch.equal(out_a2, out_a1), "no-alloc call 3 (a again) differs from call 1"
    exp_a, _ = oracle_decode(a.wl)
    exp_b, _ = oracle_decode(b.wl)
    tol_check(from_dev(out_a2), exp_a, W.BF16, "no-alloc decode a vs oracle")
    tol_check(from_dev(out_b), exp_b, W.BF16, "no-alloc decode b vs oracle")
    assert int(a.err.item()) == 0 and int(b.err.item()) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = _lib.load()
    limit = lib.pkv_decode_noalloc_max_scratch_bytes()
    assert limit == 16 << 20
    # 4096 requests x 64 query heads need far more partial space than the array holds.
    assert lib.pkv_decode_workspace_bytes(4096, 64) > limit
    st = lib.pkv_decode_attn_noalloc(None, 0, None, 64, None, None, None, 4096, ctypes.c_float(0.1),
                                     None, None, None)
    assert st == 6  # PKV_ERR_TOO_LARGE
    assert b"maximum" in lib.pkv_status_string(st)
