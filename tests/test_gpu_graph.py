"""store_kv + decode_attn captured in CUDA graphs with fixed buffers (needs a B200).

The serving engine on the pages replays decode from CUDA graphs captured for a
ladder of batch sizes; a real batch is padded up to the captured size with
dummy requests whose table row points at a dummy slot and whose context
length is 1 ("Mini-SGLang 完整剖析", §4.6.6 and §5.3).  Every per-step value the
kernels read (lengths, table rows, slots, queries) lives in device buffers, so
one captured graph serves any batch up to its size.  Here each graph is
replayed twice with different real batches and the real rows are compared
with the float64 oracle.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle

from gpu_helpers import device_pool, from_dev, i32, oracle_decode, to_dev, tol_check
from paged_kv_gqa_scatter_b200 import api
from paged_kv_gqa_scatter_b200 import workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

MAX_BS = 256
LADDER = [1, 8, 64, 256]


def test_decode_graph_ladder_with_dummy_padding():
    rng = np.random.default_rng(77)
    R = 300
    lens = rng.integers(1, 700, size=R).astype(np.int32)
    total = int(lens.sum())
    # One spare slot beyond the requests' slots becomes the dummy slot.
    wl = W.decode_small(seq_lens=lens, num_slots=total + 1, num_q_heads=32, num_kv_heads=8, seed=1500)
    used = set(np.concatenate([wl.page_table[wl.table_idx[r], :lens[r]] for r in range(R)]).tolist())
    dummy_slot = int(next(s for s in range(wl.pool.num_slots) if s not in used))
    dummy_row = wl.page_table.shape[0] - 1          # the table's spare last row
    assert dummy_row not in set(wl.table_idx.tolist())
    table_np = wl.page_table.copy()
    table_np[dummy_row, :] = dummy_slot
    expected, _ = oracle_decode(wl)                 # every request's output after its store

    pool = device_pool(wl.pool, wl.k_planes, wl.v_planes, layers=[0])
    table = api.PageTable(i32(table_np))
    Hq, row = wl.num_q_heads, wl.pool.row_elems
    q_all, k_all, v_all = to_dev(wl.q, W.BF16), to_dev(wl.k_new, W.BF16), to_dev(wl.v_new, W.BF16)
    loc_all, sl_all, ti_all = i32(wl.out_loc), i32(wl.seq_lens), i32(wl.table_idx)

    # Fixed buffers sized for the largest graph.
    q = torch.zeros(MAX_BS, Hq, 128, dtype=torch.bfloat16, device="cuda")
    k_new = torch.zeros(MAX_BS, row, dtype=torch.bfloat16, device="cuda")
    v_new = torch.zeros_like(k_new)
    out_loc = torch.full((MAX_BS,), dummy_slot, dtype=torch.int32, device="cuda")
    seq_lens = torch.ones(MAX_BS, dtype=torch.int32, device="cuda")
    table_idx = torch.full((MAX_BS,), dummy_row, dtype=torch.int32, device="cuda")
    out = torch.zeros(MAX_BS, Hq, 128, dtype=torch.bfloat16, device="cuda")
    ws = api.decode_workspace(MAX_BS, Hq)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(bs):
        api.store_kv(pool, 0, k_new[:bs], v_new[:bs], out_loc[:bs], err)
        api.decode_attn(pool, 0, q[:bs], table, table_idx[:bs], seq_lens[:bs], out[:bs], ws,
                        scale=wl.scale, dev_err=err)

    def load_batch(bs, idx):
        B = len(idx)
        ii = torch.as_tensor(idx, dtype=torch.long, device="cuda")
        q[:B].copy_(q_all[ii]); k_new[:B].copy_(k_all[ii]); v_new[:B].copy_(v_all[ii])
        out_loc[:B].copy_(loc_all[ii]); seq_lens[:B].copy_(sl_all[ii]); table_idx[:B].copy_(ti_all[ii])
        q[B:bs].zero_(); k_new[B:bs].zero_(); v_new[B:bs].zero_()
        out_loc[B:bs].fill_(dummy_slot); seq_lens[B:bs].fill_(1); table_idx[B:bs].fill_(dummy_row)

    # Eager warm-up (first launches happen outside capture), then capture
    # largest first sharing one memory pool, as the engine on the pages does.
    for bs in LADDER:
        load_batch(bs, list(range(min(bs, R))))
        step(bs)
    torch.cuda.synchronize()
    graphs = {}
    mempool = None
    s = torch.cuda.Stream()
    for bs in sorted(LADDER, reverse=True):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, pool=mempool, stream=s):
            step(bs)
        mempool = g.pool()
        graphs[bs] = g
    torch.cuda.synchronize()

    for bs in LADDER:
        for B in sorted({bs, max(1, bs // 2 + 1)}):
            idx = rng.choice(R, size=B, replace=False)
            load_batch(bs, idx)
            out.fill_(0)
            torch.cuda.synchronize()
            graphs[bs].replay()
            torch.cuda.synchronize()
            tol_check(from_dev(out[:B]), expected[idx], W.BF16, f"graph bs={bs} real={B}")
    assert int(err.item()) == 0


def _capture(fn):
    """Warm up eagerly once, then capture fn in a CUDA graph."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        fn()
    torch.cuda.synchronize()
    return g


def test_fused_store_then_cascade_decode_in_graph():
    """qk_norm_rope_store followed by decode_attn_cascade, captured once and
    replayed with two different qkv inputs in the same fixed buffer: each
    replay equals (bit for bit) the same two calls run eagerly, and the
    eager result matches the oracle's store and decode."""
    gd = W.grouped_decode(groups=((128, 6), (700, 10)), max_suffix=200, seed=61)
    d = gd.decode
    Hq, Hkv, B = d.num_q_heads, d.pool.num_kv_heads, d.batch
    rng = np.random.Generator(np.random.PCG64(62))
    pos_np = (d.seq_lens - 1).astype(np.int32)
    cache_np = W.rotary_table(4096)
    qw_np = W.f32_to_bf16_bits(1.0 + 0.1 * rng.standard_normal(128).astype(np.float32))
    kw_np = W.f32_to_bf16_bits(1.0 + 0.1 * rng.standard_normal(128).astype(np.float32))
    qkv_a = W.draw_values(rng, (B, (Hq + 2 * Hkv) * 128), W.BF16, 2.0)
    qkv_b = W.draw_values(rng, (B, (Hq + 2 * Hkv) * 128), W.BF16, 2.0)
    mp = int(gd.group_prefix_lens.max())
    table = api.PageTable(i32(d.page_table))
    ti, sl, loc, pos = i32(d.table_idx), i32(d.seq_lens), i32(d.out_loc), i32(pos_np)
    off, pre = i32(gd.group_offsets), i32(gd.group_prefix_lens)
    cache = torch.from_numpy(cache_np).cuda()
    qw, kw = to_dev(qw_np, W.BF16), to_dev(kw_np, W.BF16)

    def make():
        pool = device_pool(d.pool, d.k_planes, d.v_planes, layers=[0])
        qkv = torch.empty((B, (Hq + 2 * Hkv) * 128), dtype=torch.bfloat16, device="cuda")
        q_out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
        out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
        ws = api.decode_cascade_workspace(B, Hq, mp)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")

        def fn():
            api.qk_norm_rope_store(pool, 0, qkv, Hq, pos, cache, loc, q_out, qw, kw, 1e-6, err)
            api.decode_attn_cascade(pool, 0, q_out, table, ti, sl, off, pre, mp, out, ws,
                                    scale=d.scale, dev_err=err)
        return qkv, out, err, fn

    qkv_e, out_e, err_e, fn_e = make()
    qkv_g, out_g, err_g, fn_g = make()
    qkv_g.copy_(to_dev(qkv_a, W.BF16))
    g = _capture(fn_g)
    for host in (qkv_a, qkv_b):
        qkv_e.copy_(to_dev(host, W.BF16))
        fn_e()
        qkv_g.copy_(to_dev(host, W.BF16))
        out_g.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_e, out_g)
    assert int(err_e.item()) == 0 and int(err_g.item()) == 0
    # The eager result of the second input against the oracle.
    kp = {0: d.k_planes[0].copy()}
    vp = {0: d.v_planes[0].copy()}
    q = oracle.qk_norm_rope_store(qkv_b, Hq, Hkv, 128, pos_np, cache_np, qw_np, kw_np, 1e-6, kp, vp, 0,
                                  d.out_loc)
    exp = oracle.decode_attn(oracle.to_storage(q, "bf16"), kp, vp, 0, d.page_table, d.table_idx,
                             d.seq_lens, 1, d.scale)
    tol_check(from_dev(out_e), exp, W.BF16, "fused store + cascade decode")


def test_fp8_store_and_decode_in_graph():
    """store_kv + decode_attn over an FP8 pool, captured and replayed twice;
    each replay equals the eager calls bit for bit."""
    wl = W.with_fp8_pool(W.decode_small(num_q_heads=32), seed=63)

    def make():
        from gpu_helpers import DeviceDecode
        dd = DeviceDecode(wl)
        return dd, dd.run

    de, fe = make()
    dg, fg = make()
    g = _capture(fg)
    for scale in (1.0, -0.5):
        for dd in (de, dg):
            dd.q.copy_(to_dev(wl.q, W.BF16) * scale)
        fe()
        dg.out.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(de.out, dg.out)
    assert int(de.err.item()) == 0 and int(dg.err.item()) == 0


@pytest.mark.parametrize("fp8", [False, True])
def test_paged_decode_in_graph_with_new_queries(fp8):
    """Page size 16 (page-box stages, tensor maps passed as kernel parameters)
    captured once and replayed with two different query sets: each replay
    must match the oracle on the queries in the buffer at replay time."""
    base = W.decode_paged_small(page_size=16, seq_lens=(1, 15, 17, 33, 300, 1029, 47), seed=1700)
    wl = W.with_fp8_pool(base, seed=71) if fp8 else base
    pool = device_pool(wl.pool, wl.k_planes, wl.v_planes, layers=[0])
    table = api.PageTable(i32(wl.page_table))
    q = to_dev(wl.q, W.BF16)
    k_new, v_new = to_dev(wl.k_new, W.BF16), to_dev(wl.v_new, W.BF16)
    loc, sl, ti = i32(wl.out_loc), i32(wl.seq_lens), i32(wl.table_idx)
    out = torch.zeros_like(q)
    ws = api.decode_workspace(wl.batch, wl.num_q_heads)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        api.store_kv(pool, 0, k_new, v_new, loc, err)
        api.decode_attn(pool, 0, q, table, ti, sl, out, ws, scale=wl.scale, dev_err=err)

    g = _capture(step)
    rng = np.random.default_rng(17)
    for trial in range(2):
        qs = wl.q if trial == 0 else W.draw_values(rng, wl.q.shape, W.BF16)
        q.copy_(to_dev(qs, W.BF16))
        out.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        wq = dataclasses.replace(wl, q=qs)
        if fp8:
            kp = {l: a.copy() for l, a in wl.k_planes.items()}
            vp = {l: a.copy() for l, a in wl.v_planes.items()}
            oracle.store_kv_fp8(kp, vp, 0, wl.k_new, wl.v_new, wl.out_loc, wl.pool.num_kv_heads, 128,
                                wl.pool.k_scale, wl.pool.v_scale)
            exp = oracle.decode_attn(qs, oracle.dequant_planes(kp, wl.pool.k_scale, [0]),
                                     oracle.dequant_planes(vp, wl.pool.v_scale, [0]), 0, wl.page_table,
                                     wl.table_idx, wl.seq_lens, 16, wl.scale)
        else:
            exp, _ = oracle_decode(wq)
        tol_check(from_dev(out), exp, W.BF16, f"paged decode in a graph, trial {trial}, fp8={fp8}")
    assert int(err.item()) == 0
