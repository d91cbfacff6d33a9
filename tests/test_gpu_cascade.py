"""GPU parity for cascade (shared-prefix aware) decode against the oracle.

The cascade call must produce decode attention over each request's whole
context, so its expectation is the oracle's plain decode_attn on the same
inputs; tolerance as for decode (|err| <= 1e-2 + 1e-2 |ref|, bf16).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_helpers import DeviceDecode, from_dev, i32, oracle_decode, tol_check
from paged_kv_gqa_scatter_b200 import api
from paged_kv_gqa_scatter_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _run_cascade(dd: DeviceDecode, off, plen, max_prefix=None, store=True, out=None):
    wl = dd.wl
    if store:
        api.store_kv(dd.pool, wl.layer, dd.k_new, dd.v_new, dd.out_loc, dd.err)
    mp = int(np.max(plen)) if max_prefix is None else int(max_prefix)
    ws = api.decode_cascade_workspace(wl.batch, wl.num_q_heads, mp)
    out = torch.empty_like(dd.q) if out is None else out
    api.decode_attn_cascade(dd.pool, wl.layer, dd.q, dd.table, dd.table_idx, dd.seq_lens,
                            i32(off), i32(plen), mp, out, ws, scale=wl.scale, dev_err=dd.err)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("hq,hkv", [(16, 8), (32, 8), (8, 8), (64, 8)])
def test_cascade_grouped_matches_oracle(hq, hkv):
    """Seven groups: prefixes 0, 1, 63, 64, 65, 1000, 2500 tokens with 3, 1,
    2, 5, 1, 70 and 4 members; suffixes U{0..300} plus the stored token."""
    gd = W.grouped_decode(num_q_heads=hq, num_kv_heads=hkv)
    dd = DeviceDecode(gd.decode)
    out = _run_cascade(dd, gd.group_offsets, gd.group_prefix_lens)
    assert int(dd.err.item()) == 0
    exp, _ = oracle_decode(gd.decode)
    tol_check(from_dev(out), exp, W.BF16, f"cascade hq={hq}")


@pytest.mark.parametrize("page_size", [16, 64])
def test_cascade_paged(page_size):
    gd = W.grouped_decode(page_size=page_size, seed=21)
    dd = DeviceDecode(gd.decode)
    out = _run_cascade(dd, gd.group_offsets, gd.group_prefix_lens)
    assert int(dd.err.item()) == 0
    exp, _ = oracle_decode(gd.decode)
    tol_check(from_dev(out), exp, W.BF16, f"cascade page_size {page_size}")


def test_cascade_whole_context_shared():
    """Members whose every context token is the shared prefix (empty suffix
    pass): here the prefix covers all but the stored token, and one group's
    prefix is declared to include that token too (a single-member group)."""
    gd = W.grouped_decode(groups=((200, 3), (700, 1)), min_suffix=0, max_suffix=0, seed=22)
    d = gd.decode
    plen = gd.group_prefix_lens.copy()
    plen[1] = d.seq_lens[gd.group_offsets[1]]  # the lone member: prefix == context
    dd = DeviceDecode(d)
    out = _run_cascade(dd, gd.group_offsets, plen)
    assert int(dd.err.item()) == 0
    exp, _ = oracle_decode(d)
    tol_check(from_dev(out), exp, W.BF16, "cascade empty suffix")


def test_cascade_max_prefix_above_need():
    """A larger max_prefix_len (up to the table width) only changes the split
    plan, not the result."""
    gd = W.grouped_decode(seed=23)
    dd = DeviceDecode(gd.decode)
    cols = gd.decode.page_table.shape[1]
    out = _run_cascade(dd, gd.group_offsets, gd.group_prefix_lens, max_prefix=cols)
    assert int(dd.err.item()) == 0
    exp, _ = oracle_decode(gd.decode)
    tol_check(from_dev(out), exp, W.BF16, f"cascade max_prefix {cols}")


def test_cascade_no_prefix_equals_decode():
    """All prefixes 0 with max_prefix_len 0: the call is the plain decode."""
    gd = W.grouped_decode(groups=((0, 9), (0, 4)), seed=24)
    dd = DeviceDecode(gd.decode)
    out = _run_cascade(dd, gd.group_offsets, gd.group_prefix_lens, max_prefix=0)
    assert int(dd.err.item()) == 0
    exp, _ = oracle_decode(gd.decode)
    tol_check(from_dev(out), exp, W.BF16, "cascade without prefix")


def test_cascade_radix_serving_decode():
    """The radix workload's decode (256 requests on one shared 4096-token
    prefix, Hq 32): steps 1 and 3 through the cascade call, eight sampled
    requests against the oracle and every request against plain decode."""
    rs = W.radix_shared_prefix(decode_steps=3)
    ext = rs.extend
    from gpu_helpers import DeviceExtend, oracle_extend
    de = DeviceExtend(ext)
    de.run()
    rng = np.random.default_rng(5)
    req = sorted(rng.choice(ext.batch, 8, replace=False).tolist())
    _, planes = oracle_extend(ext, rows=np.zeros(0, dtype=np.int64))
    off = np.array([0, ext.batch], dtype=np.int32)
    plen = np.array([4096], dtype=np.int32)
    for t in range(1, 4):
        dwl = rs.decode_step(t)
        dd = DeviceDecode(dwl, pool=de.pool, table=de.table)
        out = _run_cascade(dd, off, plen)
        plain = torch.empty_like(out)
        api.decode_attn(dd.pool, dwl.layer, dd.q, dd.table, dd.table_idx, dd.seq_lens, plain,
                        dd.ws, scale=dwl.scale, dev_err=dd.err)
        torch.cuda.synchronize()
        assert int(dd.err.item()) == 0
        want = req if t in (1, 3) else []
        exp, planes = oracle_decode(dwl, requests=want, planes=planes)
        if want:
            tol_check(from_dev(out)[want], exp[want], W.BF16, f"radix cascade t={t}")
        # Both GPU paths approximate the same value: within twice the bound.
        a, b = from_dev(out), from_dev(plain)
        assert np.all(np.abs(a - b) <= 2e-2 + 2e-2 * np.abs(b))


def test_cascade_bad_prefix_flagged():
    gd = W.grouped_decode(groups=((100, 3),), seed=25)
    d = gd.decode
    plen = np.array([int(d.seq_lens[:3].min()) + 5], dtype=np.int32)  # beyond a member's context
    dd = DeviceDecode(d)
    out = _run_cascade(dd, gd.group_offsets, plen)
    assert int(dd.err.item()) & api.DEV_ERR_BAD_LENGTH
    assert torch.isfinite(out.float()).all()


def test_cascade_bad_offsets_flagged():
    gd = W.grouped_decode(groups=((100, 3), (50, 2)), seed=26)
    off = gd.group_offsets.copy()
    off[-1] = off[-1] - 1  # does not end at batch
    dd = DeviceDecode(gd.decode)
    out = _run_cascade(dd, off, gd.group_prefix_lens)
    assert int(dd.err.item()) & api.DEV_ERR_BAD_LENGTH
    assert torch.isfinite(out.float()).all()


def test_cascade_host_checks():
    gd = W.grouped_decode(groups=((64, 2),), seed=27)
    dd = DeviceDecode(gd.decode)
    wl = gd.decode
    off, plen = i32(gd.group_offsets), i32(gd.group_prefix_lens)
    out = torch.empty_like(dd.q)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="workspace"):
        api.decode_attn_cascade(dd.pool, 0, dd.q, dd.table, dd.table_idx, dd.seq_lens, off, plen,
                                64, out, small, scale=wl.scale)
    ws = api.decode_cascade_workspace(wl.batch, wl.num_q_heads, 64)
    with pytest.raises(RuntimeError, match="beyond"):
        api.decode_attn_cascade(dd.pool, 0, dd.q, dd.table, dd.table_idx, dd.seq_lens, off, plen,
                                wl.page_table.shape[1] + 1, out, ws, scale=wl.scale)
    with pytest.raises(RuntimeError, match="invalid"):
        api.decode_attn_cascade(dd.pool, 0, dd.q, dd.table, dd.table_idx, dd.seq_lens, off,
                                plen[:0], 64, out, ws, scale=wl.scale)


def test_cascade_two_host_threads():
    """Two host threads, each on its own stream, call the cascade at the same
    time.  Each batch is one group of 256 requests, so both calls run the
    prefix pass beside the suffix pass on the library's shared auxiliary
    stream; every result must equal (bit for bit) the same call made alone."""
    import threading
    cases = []
    for seed in (81, 82):
        gd = W.grouped_decode(groups=((1000, 256),), max_suffix=150, seed=seed)
        dd = DeviceDecode(gd.decode)
        ref = _run_cascade(dd, gd.group_offsets, gd.group_prefix_lens).clone()
        exp, _ = oracle_decode(gd.decode, requests=[0, 255])
        tol_check(from_dev(ref)[[0, 255]], exp[[0, 255]], W.BF16, f"cascade seed {seed}")
        cases.append((gd, dd, ref))
    torch.cuda.synchronize()
    failures = []

    def worker(gd, dd, ref):
        try:
            st = torch.cuda.Stream()
            wl = dd.wl
            mp = int(np.max(gd.group_prefix_lens))
            ws = api.decode_cascade_workspace(wl.batch, wl.num_q_heads, mp)
            off, plen = i32(gd.group_offsets), i32(gd.group_prefix_lens)
            torch.cuda.synchronize()
            with torch.cuda.stream(st):
                out = torch.empty_like(dd.q)
                for _ in range(20):
                    out.fill_(0)
                    api.decode_attn_cascade(dd.pool, wl.layer, dd.q, dd.table, dd.table_idx, dd.seq_lens,
                                            off, plen, mp, out, ws, scale=wl.scale, dev_err=dd.err)
                    st.synchronize()
                    if not torch.equal(out, ref):
                        failures.append("a threaded call differs from the same call made alone")
                        return
        except Exception as exc:  # surfaced below
            failures.append(repr(exc))

    threads = [threading.Thread(target=worker, args=c) for c in cases]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads), "a worker thread did not finish"
    assert not failures, failures[0]
    assert all(int(c[1].err.item()) == 0 for c in cases)
