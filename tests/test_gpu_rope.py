"""GPU parity for the fused q/k RMSNorm + RoPE + store_kv call against the oracle.

Tolerances: the kernel computes in fp32 from the stored inputs and rounds once
to the pool type; the oracle computes in float64 and rounds once.  bf16
results may differ by one rounding of the output (half an ulp each side), so
each element must satisfy |got - exact| <= 2^-8 |exact| + 2^-18 m, m being the
row's largest |value| before rotation (fp32 cancellation in the rotation);
and at least 99% of elements must equal the oracle's rounded value exactly.
The fp32 check build must be within 4e-6 (|exact| + m).  V rows are a bit copy.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import device_pool, from_dev, i32, to_dev, tol_check
from paged_kv_gqa_scatter_b200 import api
from paged_kv_gqa_scatter_b200 import workloads as W

pytestmark = pytest.mark.gpu

D = W.HEAD_DIM


def _oracle(wl: W.RopeStoreWorkload):
    """Expected q (float64, unrounded), k rows (float64, unrounded) and the
    host planes after the oracle's store."""
    kp = {l: a.copy() for l, a in wl.k_planes.items()}
    vp = {l: a.copy() for l, a in wl.v_planes.items()}
    hkv = wl.pool.num_kv_heads
    q = oracle.qk_norm_rope_store(wl.qkv, wl.num_q_heads, hkv, D, wl.positions, wl.cos_sin_cache,
                                  wl.q_norm_w, wl.k_norm_w, wl.eps, kp, vp, wl.layer, wl.out_loc,
                                  storage=wl.pool.dtype)
    x = oracle.to_f64(wl.qkv).reshape(wl.n_tokens, wl.num_q_heads + 2 * hkv, D)
    kx = x[:, wl.num_q_heads:wl.num_q_heads + hkv]
    k = oracle.rope_rotate_half(oracle.rms_norm(kx, wl.k_norm_w, wl.eps), wl.positions,
                                wl.cos_sin_cache)
    qn = oracle.rms_norm(x[:, :wl.num_q_heads], wl.q_norm_w, wl.eps)
    kn = oracle.rms_norm(kx, wl.k_norm_w, wl.eps)
    return q, k, qn, kn, kp, vp


def _check_rows(got, exact, normed, dtype, what):
    """got/exact/normed [..., D] float64."""
    m = np.abs(normed).max(axis=-1, keepdims=True)
    err = np.abs(got - exact)
    if dtype == W.BF16:
        bound = 2.0 ** -8 * np.abs(exact) + 2.0 ** -18 * m
        rounded = oracle.to_storage(exact, "bf16")
        gotbits = W.f32_to_bf16_bits(got.astype(np.float32))
        same = float(np.mean(rounded == gotbits))
        assert same >= 0.99, f"{what}: only {same:.4f} of elements equal the oracle's rounding"
    else:
        bound = 4e-6 * (np.abs(exact) + m)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} out of tolerance, max err {err.max():.3e}, "
                           f"first {np.argwhere(bad)[:3].tolist()}")


class DevRope:
    def __init__(self, wl: W.RopeStoreWorkload, pos64=False, loc64=False, cache=None):
        dt = wl.pool.dtype
        self.wl = wl
        self.pool = device_pool(wl.pool, wl.k_planes, wl.v_planes)
        self.qkv = to_dev(wl.qkv, dt)
        pos = torch.from_numpy(wl.positions.astype(np.int64))
        self.pos = (pos if pos64 else pos.to(torch.int32)).cuda()
        loc = torch.from_numpy(wl.out_loc.astype(np.int64))
        self.loc = (loc if loc64 else loc.to(torch.int32)).cuda()
        self.cache = torch.from_numpy(wl.cos_sin_cache if cache is None else cache).cuda()
        self.qw = None if wl.q_norm_w is None else to_dev(wl.q_norm_w, dt)
        self.kw = None if wl.k_norm_w is None else to_dev(wl.k_norm_w, dt)
        self.q_out = torch.empty((wl.n_tokens, wl.num_q_heads, D), dtype=self.qkv.dtype,
                                 device="cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(self):
        wl = self.wl
        api.qk_norm_rope_store(self.pool, wl.layer, self.qkv, wl.num_q_heads, self.pos, self.cache,
                               self.loc, self.q_out, self.qw, self.kw, wl.eps, self.err)
        torch.cuda.synchronize()


def _subset(wl: W.RopeStoreWorkload, keep) -> W.RopeStoreWorkload:
    keep = np.asarray(keep, dtype=np.int64)
    return dataclasses.replace(wl, qkv=wl.qkv[keep], positions=wl.positions[keep],
                               out_loc=wl.out_loc[keep])


def _plane_bits(t: torch.Tensor, dtype: str) -> np.ndarray:
    if dtype == W.BF16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def _compare(wl: W.RopeStoreWorkload, dev: DevRope, skip_tokens=(), v_copied=()):
    """q/k rows of every token not in skip_tokens against the oracle; the V
    plane bit-exact (tokens in v_copied had their v row stored although their
    q/k were rejected); every K slot the kept tokens do not own unchanged."""
    skip = set(int(t) for t in skip_tokens)
    keep = [t for t in range(wl.n_tokens) if t not in skip]
    sub = _subset(wl, keep)
    q, k, qn, kn, kp, vp = _oracle(sub)
    dt = wl.pool.dtype
    _check_rows(from_dev(dev.q_out)[keep], q, qn, dt, "q_out")
    gk = from_dev(dev.pool.k[wl.layer])[sub.out_loc]
    _check_rows(gk, k, kn, dt, "k rows")
    hq, hkv = wl.num_q_heads, wl.pool.num_kv_heads
    for t in v_copied:
        vp[wl.layer][wl.out_loc[t]] = wl.qkv[t, (hq + hkv) * D:].reshape(hkv, D)
    assert np.array_equal(_plane_bits(dev.pool.v[wl.layer], dt), vp[wl.layer]), "v rows"
    others = np.setdiff1d(np.arange(wl.pool.num_slots), wl.out_loc)
    assert np.array_equal(_plane_bits(dev.pool.k[wl.layer], dt)[others], kp[wl.layer][others])


@pytest.mark.parametrize("dtype", [W.BF16, W.F32])
@pytest.mark.parametrize("norms", [True, False])
def test_rope_store_matches_oracle(dtype, norms):
    wl = W.rope_store_step(dtype, norms=norms)
    dev = DevRope(wl)
    dev.run()
    assert int(dev.err.item()) == 0
    _compare(wl, dev)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (32, 8), (64, 8), (4, 1), (16, 2)])
def test_rope_store_head_counts(hq, hkv):
    wl = W.rope_store_step(W.BF16, num_q_heads=hq, num_kv_heads=hkv, seed=77 + hq + hkv)
    dev = DevRope(wl)
    dev.run()
    assert int(dev.err.item()) == 0
    _compare(wl, dev)


@pytest.mark.parametrize("pos64,loc64", [(True, False), (False, True), (True, True)])
def test_rope_store_index_widths(pos64, loc64):
    wl = W.rope_store_step(W.BF16, seed=91)
    dev = DevRope(wl, pos64=pos64, loc64=loc64)
    dev.run()
    assert int(dev.err.item()) == 0
    _compare(wl, dev)


def test_rope_store_position_edges():
    """Position 0 (identity rotation), the last cached position, and a ragged
    token count spanning many blocks."""
    maxp = 8192
    pos = np.concatenate([[0, maxp - 1, 1, maxp - 2], np.arange(0, maxp, 37)])
    wl = W.rope_store_step(W.BF16, positions=pos, max_position=maxp, num_slots=8192, seed=5)
    dev = DevRope(wl)
    dev.run()
    assert int(dev.err.item()) == 0
    _compare(wl, dev)


@pytest.mark.parametrize("n,hq,hkv", [(64, 16, 8), (256, 32, 8), (64, 64, 8), (1000, 32, 8)])
def test_rope_store_launch_shapes(n, hq, hkv):
    """Both launch shapes: decode-sized batches split every token's rows over
    several blocks (64 and 256 tokens, the decode steps of the Qwen3-0.6B and
    Qwen3-8B shapes), large batches walk a token's rows in one block."""
    rng = np.random.default_rng(100 + n + hq)
    pos = rng.integers(0, 8192, size=n).astype(np.int32)
    wl = W.rope_store_step(W.BF16, positions=pos, num_q_heads=hq, num_kv_heads=hkv,
                           num_slots=max(4096, 2 * n), seed=200 + n + hq)
    dev = DevRope(wl)
    dev.run()
    assert int(dev.err.item()) == 0
    _compare(wl, dev)


def test_rope_store_bad_position_zeroes_and_flags():
    maxp = 1024
    pos = np.array([3, maxp, 7, -1, 500], dtype=np.int32)
    wl = W.rope_store_step(W.BF16, positions=pos, max_position=maxp, seed=11)
    dev = DevRope(wl)
    dev.run()
    assert int(dev.err.item()) & api.DEV_ERR_POSITION
    bad = [1, 3]
    assert np.all(from_dev(dev.q_out)[bad] == 0.0)
    assert np.all(from_dev(dev.pool.k[0])[wl.out_loc[bad]] == 0.0)
    # The good tokens match; the bad tokens' v rows are still stored.
    _compare(wl, dev, skip_tokens=bad, v_copied=bad)


def test_rope_store_bad_slot_skipped_and_flagged():
    wl = W.rope_store_step(W.BF16, seed=12)
    wl.out_loc[4] = wl.pool.num_slots + 3
    dev = DevRope(wl)
    dev.run()
    assert int(dev.err.item()) & api.DEV_ERR_SLOT_RANGE
    # Nothing of token 4 reaches the pool; the rest matches.
    _compare(wl, dev, skip_tokens=[4])
    # Token 4's q is still produced: the oracle on that token alone, stored
    # to a valid slot of a scratch copy of the pool.
    alone = dataclasses.replace(_subset(wl, [4]), out_loc=np.zeros(1, dtype=np.int32))
    q, _, qn, _, _, _ = _oracle(alone)
    _check_rows(from_dev(dev.q_out)[[4]], q, qn, W.BF16, "q_out of the bad-slot token")


def test_rope_store_empty_is_noop():
    wl = W.rope_store_step(W.BF16, positions=np.zeros(0, dtype=np.int32), seed=13)
    dev = DevRope(wl)
    before = dev.pool.k[0].clone()
    dev.run()
    assert int(dev.err.item()) == 0
    assert torch.equal(before, dev.pool.k[0])


def test_rope_store_then_decode():
    """The fused step feeding decode: decode over the pool the fused call wrote,
    with its q, equals the oracle's store followed by the oracle's decode."""
    base = W.decode_small(W.BF16)
    B = base.batch
    pos = base.seq_lens.astype(np.int32) - 1
    wl = W.rope_store_step(W.BF16, positions=pos, num_slots=base.pool.num_slots, seed=14)
    wl.out_loc = base.out_loc.copy()
    wl.k_planes = {0: base.k_planes[0].copy()}
    wl.v_planes = {0: base.v_planes[0].copy()}
    dev = DevRope(wl)
    dev.run()
    table = api.PageTable(i32(base.page_table))
    out = torch.empty_like(dev.q_out)
    ws = api.decode_workspace(B, base.num_q_heads)
    api.decode_attn(dev.pool, 0, dev.q_out, table, i32(base.table_idx), i32(base.seq_lens), out, ws,
                    scale=base.scale, dev_err=dev.err)
    torch.cuda.synchronize()
    assert int(dev.err.item()) == 0
    q, k, qn, kn, kp, vp = _oracle(wl)
    q_st = oracle.to_storage(q, "bf16")
    exp = oracle.decode_attn(q_st, kp, vp, 0, base.page_table, base.table_idx, base.seq_lens,
                             1, base.scale)
    tol_check(from_dev(out), exp, W.BF16, "decode after fused store")
