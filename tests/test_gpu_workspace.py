"""Library-owned workspace objects: decode and cascade decode run with the
workspace buffer and its error word; pkv_read_device_error returns the
accumulated bits and clears them."""
import numpy as np
import pytest
import torch

from gpu_helpers import DeviceDecode, from_dev, i32, oracle_decode, tol_check
from paged_kv_gqa_scatter_b200 import api
from paged_kv_gqa_scatter_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_workspace_object_decode_cascade_and_error_word():
    gd = W.grouped_decode(groups=((64, 3), (300, 5)), max_suffix=60, seed=81)
    wl = gd.decode
    d = DeviceDecode(wl)
    mp = int(gd.group_prefix_lens.max())
    ws = api.Workspace(wl.batch, wl.num_q_heads, mp)
    ptr, nbytes = ws.buffer()
    assert ptr != 0 and nbytes >= api.decode_workspace_bytes(wl.batch, wl.num_q_heads)
    assert nbytes >= api.decode_cascade_workspace_bytes(wl.batch, wl.num_q_heads, mp)

    api.store_kv(d.pool, 0, d.k_new, d.v_new, d.out_loc, ws)
    api.decode_attn(d.pool, 0, d.q, d.table, d.table_idx, d.seq_lens, d.out, ws, scale=wl.scale,
                    dev_err=ws)
    assert ws.read_device_error() == 0
    exp, _ = oracle_decode(wl)
    tol_check(from_dev(d.out), exp, W.BF16, "decode with a workspace object")

    out2 = torch.empty_like(d.out)
    api.decode_attn_cascade(d.pool, 0, d.q, d.table, d.table_idx, d.seq_lens, i32(gd.group_offsets),
                            i32(gd.group_prefix_lens), mp, out2, ws, scale=wl.scale, dev_err=ws)
    assert ws.read_device_error() == 0
    tol_check(from_dev(out2), exp, W.BF16, "cascade with a workspace object")

    # An out-of-range slot is flagged; reading clears the word.
    bad = d.out_loc.clone()
    bad[0] = wl.pool.num_slots + 5
    api.store_kv(d.pool, 0, d.k_new, d.v_new, bad, ws)
    assert ws.read_device_error() & api.DEV_ERR_SLOT_RANGE
    assert ws.read_device_error() == 0
    ws.close()
    ws.close()  # idempotent


def test_workspace_create_rejects_bad_sizes():
    with pytest.raises(RuntimeError, match="invalid"):
        api.Workspace(0, 16)
    with pytest.raises(RuntimeError, match="invalid"):
        api.Workspace(4, 16, -1)
