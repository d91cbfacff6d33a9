"""pkv_decode_attn_noalloc against pkv_decode_attn (needs a B200).

The no-allocation decode serves callers that cannot allocate device memory:
an engine that has already handed almost all free memory to its KV pool, or
code hosted by a framework that owns every allocation.  It must give the same
results as the workspace version.  Two calls in a row on different workloads
check that the shared scratch array carries nothing harmful from one call to
the next.  This file is collected last so that a failure here cannot stop the
rest of the suite under -x.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_helpers import DeviceDecode, from_dev, tol_check
from paged_kv_gqa_scatter_b200 import _lib, api
from paged_kv_gqa_scatter_b200 import workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _reference(d: DeviceDecode) -> torch.Tensor:
    """Output of the existing entry point (caller-provided workspace)."""
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


def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row():
    # Long contexts split across CTAs (partials go through the scratch), then a
    # page_size-16, G = 4 batch with different shapes.
    a = DeviceDecode(W.decode_qwen3_06b(num_layers=1, layer=0))
    b = DeviceDecode(W.decode_paged_small())
    ref_a = _reference(a)
    ref_b = _reference(b)
    out_a = torch.full_like(a.q, float("nan"))
    out_b = torch.full_like(b.q, float("nan"))
    assert _noalloc_c_call(a, out_a) == 0
    assert _noalloc_c_call(b, out_b) == 0
    torch.cuda.synchronize()
    tol_check(from_dev(out_a), from_dev(ref_a), W.BF16, "no-alloc call 1 vs workspace decode")
    tol_check(from_dev(out_b), from_dev(ref_b), W.BF16, "no-alloc call 2 vs workspace decode")
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
