"""CUDA path vs the float64 oracle, element by element (needs a B200).

Tolerances (stated by the acceptance criteria of the method):
  * store_kv and gather: bit-exact;
  * attention, bf16 pool (fp32 accumulation): |gpu - oracle| <= 1e-2 + 1e-2 |oracle|;
  * attention, fp32 check build: |gpu - oracle| <= 1e-4.
Every call goes through the C ABI via the thin ``api`` binding.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (DeviceDecode, DeviceExtend, device_pool, from_dev, host_planes_copy, i32,
                         poison_unreferenced, referenced_slots,
                         oracle_decode, oracle_extend, to_dev, tol_check)
from paged_kv_gqa_scatter_b200 import api
from paged_kv_gqa_scatter_b200 import workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DTYPES = [W.BF16, W.F32]


def test_cuda_present_and_library_loaded():
    from paged_kv_gqa_scatter_b200 import _lib
    lib = _lib.load()
    assert torch.cuda.get_device_capability()[0] == 10, "expects an sm_100 device"
    assert lib.pkv_version().startswith(b"pkv")


def _err(t):
    return int(t.item())


# ---------------------------------------------------------------------------
# store_kv / gather: bit-exact.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("loc64", [False, True])
def test_store_kv_bit_exact(dtype, loc64):
    wl = W.decode_small(dtype=dtype)
    d = DeviceDecode(wl)
    loc = d.out_loc.long() if loc64 else d.out_loc
    api.store_kv(d.pool, 0, d.k_new, d.v_new, loc, d.err)
    torch.cuda.synchronize()
    kp, vp = host_planes_copy(wl.k_planes), host_planes_copy(wl.v_planes)
    oracle.store_kv(kp, vp, 0, wl.k_new, wl.v_new, wl.out_loc, 8, 128)
    st = np.uint16 if dtype == W.BF16 else np.float32
    gk = d.pool.k[0].cpu().view(torch.int16 if dtype == W.BF16 else torch.float32).numpy().view(st)
    gv = d.pool.v[0].cpu().view(torch.int16 if dtype == W.BF16 else torch.float32).numpy().view(st)
    assert np.array_equal(gk.view(np.uint8), kp[0].view(np.uint8))
    assert np.array_equal(gv.view(np.uint8), vp[0].view(np.uint8))
    assert _err(d.err) == 0


def test_store_kv_strided_rows_from_fused_qkv():
    """k and v as column slices of one [N][Hq*d + 2*Hkv*d] qkv buffer (row-strided)."""
    wl = W.decode_small()
    d = DeviceDecode(wl)
    N, Hq, row = wl.batch, wl.num_q_heads, wl.pool.row_elems
    qkv = torch.zeros(N, Hq * 128 + 2 * row, dtype=torch.bfloat16, device="cuda")
    qkv[:, Hq * 128:Hq * 128 + row] = d.k_new
    qkv[:, Hq * 128 + row:] = d.v_new
    api.store_kv(d.pool, 0, qkv[:, Hq * 128:Hq * 128 + row], qkv[:, Hq * 128 + row:], d.out_loc, d.err)
    torch.cuda.synchronize()
    kp, vp = host_planes_copy(wl.k_planes), host_planes_copy(wl.v_planes)
    oracle.store_kv(kp, vp, 0, wl.k_new, wl.v_new, wl.out_loc, 8, 128)
    gk = d.pool.k[0].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(gk, kp[0])


def test_store_kv_out_of_range_slot_is_skipped_and_flagged():
    wl = W.decode_small()
    d = DeviceDecode(wl)
    before = d.pool.k[0].clone()
    bad = d.out_loc.clone()
    bad[1] = wl.pool.num_slots + 5
    bad[2] = -3
    api.store_kv(d.pool, 0, d.k_new, d.v_new, bad, d.err)
    torch.cuda.synchronize()
    assert _err(d.err) & 1  # PKV_DEV_ERR_SLOT_RANGE
    after = d.pool.k[0]
    changed = (after != before).flatten(1).any(1).nonzero().flatten().tolist()
    assert sorted(changed) == sorted([int(wl.out_loc[0]), int(wl.out_loc[3])])


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("maker", ["decode_small", "decode_paged_small"])
def test_gather_bit_exact(dtype, maker):
    wl = getattr(W, maker)(dtype=dtype)
    d = DeviceDecode(wl)
    lens = wl.seq_lens.astype(np.int64)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    ko = torch.empty(int(offs[-1]), wl.pool.row_elems, dtype=d.q.dtype, device="cuda")
    vo = torch.empty_like(ko)
    api.gather_kv(d.pool, 0, d.table, d.table_idx, d.seq_lens,
                  torch.from_numpy(offs).cuda(), ko, vo, d.err)
    torch.cuda.synchronize()
    exp = oracle.gather_kv(wl.k_planes, wl.v_planes, 0, wl.page_table, wl.table_idx, wl.seq_lens,
                           wl.pool.page_size)
    st = torch.int16 if dtype == W.BF16 else torch.float32
    gk = ko.cpu().view(st).numpy()
    gv = vo.cpu().view(st).numpy()
    for r in range(wl.batch):
        ek = exp[r][0].reshape(lens[r], -1).view(np.uint8)
        ev = exp[r][1].reshape(lens[r], -1).view(np.uint8)
        assert np.array_equal(gk[offs[r]:offs[r + 1]].view(np.uint8), ek)
        assert np.array_equal(gv[offs[r]:offs[r + 1]].view(np.uint8), ev)
    assert _err(d.err) == 0


# ---------------------------------------------------------------------------
# decode_attn.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", DTYPES)
def test_decode_small(dtype):
    wl = W.decode_small(dtype=dtype)
    d = DeviceDecode(wl)
    d.run()
    exp, _ = oracle_decode(wl)
    tol_check(from_dev(d.out), exp, dtype, "decode-small")
    assert _err(d.err) == 0


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("page_size,num_slots", [(16, 4096), (64, 4096), (3, 4095)])
def test_decode_paged_small(dtype, page_size, num_slots):
    """page_size 16, the TRT-LLM-style 64, and a non-power-of-two size."""
    wl = W.decode_paged_small(dtype=dtype, page_size=page_size, num_slots=num_slots)
    d = DeviceDecode(wl)
    d.run()
    exp, _ = oracle_decode(wl)
    tol_check(from_dev(d.out), exp, dtype, f"decode-paged P={page_size}")
    assert _err(d.err) == 0


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (64, 8), (4, 1), (16, 2), (32, 4)])
def test_decode_group_sizes(dtype, hq, hkv):
    wl = W.decode_small(dtype=dtype, num_q_heads=hq, num_kv_heads=hkv, seq_lens=(1, 2, 31, 97, 240),
                        seed=1200 + hq + hkv)
    d = DeviceDecode(wl)
    d.run()
    exp, _ = oracle_decode(wl)
    tol_check(from_dev(d.out), exp, dtype, f"decode hq={hq} hkv={hkv}")


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("hq,hkv", [(4, 1), (16, 2), (32, 4), (64, 8)])
def test_decode_paged_group_sizes(dtype, hq, hkv):
    """page_size 16 (page-box stages for bf16) with 1, 2, 4 and 8 KV heads:
    boxes of 4 to 32 KB per plane."""
    wl = W.decode_paged_small(dtype=dtype, num_q_heads=hq, num_kv_heads=hkv, seed=1400 + hq + hkv)
    d = DeviceDecode(wl)
    d.run()
    exp, _ = oracle_decode(wl)
    tol_check(from_dev(d.out), exp, dtype, f"decode P=16 hq={hq} hkv={hkv}")
    assert _err(d.err) == 0


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("page_size,hq,hkv", [(16, 32, 8), (16, 8, 2), (64, 16, 8), (1, 16, 8)])
def test_decode_nan_in_unreferenced_slots(dtype, page_size, hq, hkv):
    """Every slot no context reads holds NaN.  Page boxes load whole 16-slot
    groups, so the tails of last pages and the rows before a CTA's first token
    reach shared memory; they must be masked out of the scores and the PV
    product (p = 0 does not clear NaN)."""
    wl = W.decode_paged_small(dtype=dtype, page_size=page_size, num_q_heads=hq, num_kv_heads=hkv,
                              seq_lens=(1, 15, 17, 33, 300, 1029, 47), seed=1500 + page_size)
    nan = np.uint16(0x7FC0) if dtype == W.BF16 else np.float32("nan")
    keep = referenced_slots(wl)
    assert keep.shape[0] < wl.pool.num_slots
    for planes in (wl.k_planes, wl.v_planes):
        poison_unreferenced(planes, 0, keep, nan)
    d = DeviceDecode(wl)
    d.run()
    torch.cuda.synchronize()
    assert torch.isfinite(d.out.float()).all(), "a masked NaN row reached the output"
    exp, _ = oracle_decode(wl)
    tol_check(from_dev(d.out), exp, dtype, f"decode with NaN in unreferenced slots P={page_size}")
    assert _err(d.err) == 0


@pytest.mark.parametrize("page_size,hq,hkv", [(1, 16, 1), (1, 64, 4), (16, 128, 8), (16, 32, 2)])
def test_decode_group_16(page_size, hq, hkv):
    """GQA groups of 16 query heads per KV head (two 8-head column tiles of
    the tensor-core consumers), row copies and page boxes, ragged lengths
    spread over many CTAs so that most requests go through the merge."""
    wl = W.decode_paged_small(dtype=W.BF16, page_size=page_size, num_q_heads=hq, num_kv_heads=hkv,
                              seed=1800 + hq + page_size)
    d = DeviceDecode(wl)
    d.run()
    exp, _ = oracle_decode(wl)
    tol_check(from_dev(d.out), exp, W.BF16, f"decode G=16 P={page_size} hq={hq} hkv={hkv}")
    assert _err(d.err) == 0


def test_decode_one_token_returns_v_exactly():
    wl = W.decode_small(seq_lens=(1, 1, 1))
    d = DeviceDecode(wl)
    d.run()
    got = d.out.cpu().view(torch.int16).numpy().view(np.uint16)
    G = wl.num_q_heads // wl.pool.num_kv_heads
    for r in range(3):
        v = wl.v_new[r].reshape(wl.pool.num_kv_heads, 128)
        for h in range(wl.num_q_heads):
            assert np.array_equal(got[r, h], v[h // G])


def test_decode_empty_context_zero_and_flagged():
    wl = W.decode_small(seq_lens=(5, 9, 3))
    d = DeviceDecode(wl)
    api.store_kv(d.pool, 0, d.k_new, d.v_new, d.out_loc, d.err)
    sl = d.seq_lens.clone()
    sl[1] = 0
    d.out.fill_(7.0)
    api.decode_attn(d.pool, 0, d.q, d.table, d.table_idx, sl, d.out, d.ws, dev_err=d.err)
    torch.cuda.synchronize()
    assert _err(d.err) & 4  # PKV_DEV_ERR_EMPTY_CONTEXT
    assert torch.all(d.out[1] == 0)
    wl2 = W.decode_small(seq_lens=(5, 9, 3))
    exp, _ = oracle_decode(wl2, requests=[0, 2])
    got = from_dev(d.out)
    tol_check(got[[0, 2]], exp[[0, 2]], W.BF16, "neighbours of an empty context")


def test_decode_bad_table_entry_flagged_and_finite():
    wl = W.decode_small()
    d = DeviceDecode(wl)
    bad = wl.page_table.copy()
    bad[wl.table_idx[2], 4] = wl.pool.num_slots + 100
    d.table = api.PageTable(i32(bad))
    d.run()
    torch.cuda.synchronize()
    assert _err(d.err) & 1
    assert torch.isfinite(d.out.float()).all()
    exp, _ = oracle_decode(wl, requests=[0, 1, 3])
    tol_check(from_dev(d.out)[[0, 1, 3]], exp[[0, 1, 3]], W.BF16, "requests with good tables")


def test_decode_empty_batch_is_noop():
    wl = W.decode_small()
    d = DeviceDecode(wl)
    api.decode_attn(d.pool, 0, d.q[:0], d.table, d.table_idx[:0], d.seq_lens[:0], d.out[:0], d.ws)
    torch.cuda.synchronize()


def test_decode_max_batch_short_contexts():
    """The largest batch the decode call accepts (4096), ragged short contexts."""
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 40, size=4096).astype(np.int32)
    wl = W.decode_small(seq_lens=lens, num_slots=int(lens.sum()) + 64, seed=1300)
    d = DeviceDecode(wl)
    d.run()
    req = list(range(0, 4096, 97)) + [4095]
    exp, _ = oracle_decode(wl, requests=req)
    tol_check(from_dev(d.out)[req], exp[req], W.BF16, "batch 4096")
    assert _err(d.err) == 0


def test_decode_qwen3_06b_full():
    """The 64-request, 300k-slot, 28-layer workload at full size; every output compared."""
    wl = W.decode_qwen3_06b()
    d = DeviceDecode(wl)
    d.run()
    exp, _ = oracle_decode(wl)
    tol_check(from_dev(d.out), exp, W.BF16, "decode-qwen3-0.6b")
    assert _err(d.err) == 0


def test_decode_qwen3_8b_sampled():
    """Batch 256, log-uniform 1k-32k, page_size 16, on the pool the benchmark
    builds (36 layers of W.QWEN3_8B_POOL_PAGES pages, so the same aliased
    pages); layers 0 and 35; 16 sampled requests (longest and shortest
    included) compared on each."""
    wl = W.decode_qwen3_8b()
    assert wl.pool.num_slots == W.QWEN3_8B_POOL_PAGES * 16 and wl.pool.num_layers == 36
    pool = device_pool(wl.pool, wl.k_planes, wl.v_planes, layers=[0, 35])
    lens = wl.seq_lens
    req = sorted(set([int(np.argmax(lens)), int(np.argmin(lens))] +
                     np.random.default_rng(3).choice(wl.batch, 14, replace=False).tolist()))
    table = None
    for layer in (0, 35):
        wl.layer = layer
        d = DeviceDecode(wl, pool=pool, table=table)
        table = d.table
        d.run()
        exp, _ = oracle_decode(wl, requests=req)
        tol_check(from_dev(d.out)[req], exp[req], W.BF16, f"decode-qwen3-8b layer {layer}")
        assert _err(d.err) == 0
    del pool
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# extend_attn.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("page_size,num_slots", [(1, 1024), (4, 1024), (64, 1024), (3, 1023)])
def test_extend_small(dtype, page_size, num_slots):
    wl = W.extend_small(dtype=dtype, page_size=page_size, num_slots=num_slots)
    d = DeviceExtend(wl)
    d.run()
    exp, _ = oracle_extend(wl)
    tol_check(from_dev(d.out), exp, dtype, f"extend-small P={page_size}")
    assert _err(d.err) == 0


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (64, 8), (8, 2)])
def test_extend_group_sizes(dtype, hq, hkv):
    wl = W.extend_small(dtype=dtype, num_q_heads=hq, num_kv_heads=hkv, prefix_lens=(0, 129, 7, 300),
                        extend_lens=(130, 64, 1, 257), num_slots=2048, seed=1400 + hq + hkv)
    d = DeviceExtend(wl)
    d.run()
    exp, _ = oracle_extend(wl)
    tol_check(from_dev(d.out), exp, dtype, f"extend hq={hq} hkv={hkv}")
    assert _err(d.err) == 0


def test_extend_zero_length_requests_in_batch():
    wl = W.extend_small(prefix_lens=(10, 0, 50, 3), extend_lens=(0, 33, 0, 5))
    d = DeviceExtend(wl)
    d.run()
    exp, _ = oracle_extend(wl)
    tol_check(from_dev(d.out), exp, W.BF16, "extend with empty chunks")
    assert _err(d.err) == 0


def test_extend_ragged_batch_of_40():
    """40 requests with chunks of 1..299 tokens after prefixes of 0..899: short
    last query blocks (whose second Q tile holds no token and is skipped),
    diagonal steps at every offset, every row compared."""
    rng = np.random.default_rng(77)
    ext = rng.integers(1, 300, size=40)
    pre = rng.integers(0, 900, size=40)
    wl = W.extend_small(prefix_lens=tuple(int(x) for x in pre), extend_lens=tuple(int(x) for x in ext),
                        num_q_heads=32, num_kv_heads=8, num_slots=int((pre + ext).sum()) + 64, seed=1500)
    d = DeviceExtend(wl)
    d.run()
    exp, _ = oracle_extend(wl)
    tol_check(from_dev(d.out), exp, W.BF16, "extend, 40 ragged requests")
    assert _err(d.err) == 0


def _chunk_rows(prefix: int, e: int, hq: int, hkv: int, seed: int):
    """Rows to compare in a chunk: the first and last token of every 128-row
    query tile (128 / G tokens), the tokens whose visible keys end on a
    64-key step boundary or just past one (the diagonal steps), and seeded
    others."""
    tq = 128 // (hq // hkv)
    rows = set()
    for t0 in range(0, e, tq):
        rows.update([t0, min(e, t0 + tq) - 1])
    for i in range(e):
        if (prefix + i + 1) % 64 in (0, 1):
            rows.add(i)
    rows.update(np.random.default_rng(seed).choice(e, 32, replace=False).tolist())
    return sorted(rows)


@pytest.mark.parametrize("step", [0, 1, 2, 3])
def test_extend_chunked_prefill_step(step):
    """Chunk `step` (prefix 2048 * step) of an 8192-token prompt in 2048-token
    chunks, at full size: the rows of _chunk_rows compared; then the step's
    128-request decode batch on the same pool, every output compared."""
    mix = W.chunked_prefill_step(step=step)
    wl = mix.extend
    d = DeviceExtend(wl)
    d.run()
    rows = _chunk_rows(int(wl.prefix_lens[0]), int(wl.extend_lens[0]), wl.num_q_heads,
                       wl.pool.num_kv_heads, 9 + step)
    exp, planes = oracle_extend(wl, rows=rows)
    tol_check(from_dev(d.out)[rows], exp[rows], W.BF16, f"chunked prefill extend c{step}")
    dd = DeviceDecode(mix.decode, pool=d.pool, table=d.table)
    dd.run()
    expd, _ = oracle_decode(mix.decode, planes=planes)
    tol_check(from_dev(dd.out), expd, W.BF16, f"chunked prefill decode c{step}")
    assert _err(d.err) == 0 and _err(dd.err) == 0


def test_radix_shared_prefix_extend_then_decode():
    """Shared 4096-token prefix, 256 suffixes extended in one call, then 64 decode steps;
    34 sampled requests (the shortest and longest suffixes included) checked
    after the extend and after decode steps 1 and 64."""
    rs = W.radix_shared_prefix()
    wl = rs.extend
    d = DeviceExtend(wl)
    d.run()
    rng = np.random.default_rng(11)
    el = wl.extend_lens
    req = sorted(set([int(np.argmin(el)), int(np.argmax(el))] +
                     rng.choice(wl.batch, 32, replace=False).tolist()))
    assert len(req) >= 32
    rows = np.concatenate([np.arange(wl.q_offsets[r], wl.q_offsets[r + 1]) for r in req])
    exp, planes = oracle_extend(wl, rows=rows)
    tol_check(from_dev(d.out)[rows], exp[rows], W.BF16, "radix extend")
    for t in range(1, rs.decode_steps + 1):
        dwl = rs.decode_step(t)
        dd = DeviceDecode(dwl, pool=d.pool, table=d.table)
        dd.run()
        want = req if t in (1, rs.decode_steps) else []
        expd, planes = oracle_decode(dwl, requests=want, planes=planes)
        if want:
            tol_check(from_dev(dd.out)[want], expd[want], W.BF16, f"radix decode t={t}")
        assert _err(dd.err) == 0


def test_decode_equals_extend_with_one_row():
    wl = W.decode_paged_small()
    d = DeviceDecode(wl)
    d.run()
    B = wl.batch
    out = torch.empty_like(d.out)
    api.extend_attn(d.pool, 0, d.q, d.table, d.table_idx, d.seq_lens - 1,
                    torch.ones(B, dtype=torch.int32, device="cuda"),
                    torch.arange(B + 1, dtype=torch.int32, device="cuda"), 1, out,
                    scale=wl.scale, dev_err=d.err)
    torch.cuda.synchronize()
    a, b = from_dev(d.out), from_dev(out)
    assert np.max(np.abs(a - b)) <= 2e-2
