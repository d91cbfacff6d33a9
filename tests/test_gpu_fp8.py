"""GPU parity for the scaled FP8 (E4M3) KV pool against the oracle.

* store_kv / gather: the stored codes are bit-exact (both sides quantise the
  float32 product x * RN32(1 / scale) with round-to-nearest-even).
* decode: attention over the dequantised pool, |err| <= 1e-2 + 1e-2 |ref|.
* extend and cascade decode: attention over the dequantised pool (the
  tensor cores take f16 operands: E4M3 widens to f16 exactly, bf16 q is
  converted to f16), same bound as decode.
* fused norm/RoPE/store: v codes bit-exact (a bf16 value times the inverse
  scale is the same float32 product on both sides); k codes come from an
  fp32 kernel value and a float64 oracle value, so they may differ by one
  code where the two straddle a rounding boundary: the dequantised k must be
  within one E4M3 step (2^-3 relative, or 2^-9 * scale near zero) and 97% of
  the codes must agree.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import DeviceDecode, device_pool, from_dev, i32, to_dev, tol_check
from paged_kv_gqa_scatter_b200 import api
from paged_kv_gqa_scatter_b200 import workloads as W

pytestmark = pytest.mark.gpu

D = W.HEAD_DIM


def scale_check(got: np.ndarray, exp: np.ndarray, what: str, frac: float = 1e-2):
    """Decode outputs over E4M3 pools average many random-sign values, so they
    are small (about 0.01-0.1) next to the 1e-2 absolute bound; also require
    the error to stay within `frac` of the largest output magnitude.  The
    kernel's own error (p rounded to f16 before PV) is far below that."""
    err = float(np.abs(got - exp).max())
    bound = frac * float(np.abs(exp).max())
    assert err <= bound, f"{what}: max error {err:.3e} above {frac} x max |ref| = {bound:.3e}"


def _codes(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def _oracle_store(wl):
    kp = {l: a.copy() for l, a in wl.k_planes.items()}
    vp = {l: a.copy() for l, a in wl.v_planes.items()}
    oracle.store_kv_fp8(kp, vp, wl.layer, wl.k_new, wl.v_new, wl.out_loc, wl.pool.num_kv_heads, D,
                        wl.pool.k_scale, wl.pool.v_scale)
    return kp, vp


def _oracle_decode(wl, kp, vp, requests=None):
    return oracle.decode_attn(wl.q, oracle.dequant_planes(kp, wl.pool.k_scale, [wl.layer]),
                              oracle.dequant_planes(vp, wl.pool.v_scale, [wl.layer]), wl.layer,
                              wl.page_table, wl.table_idx, wl.seq_lens, wl.pool.page_size, wl.scale,
                              requests=requests)


@pytest.mark.parametrize("loc64", [False, True])
def test_fp8_store_codes_bit_exact(loc64):
    wl = W.with_fp8_pool(W.decode_small())
    d = DeviceDecode(wl)
    loc = d.out_loc.long() if loc64 else d.out_loc
    api.store_kv(d.pool, 0, d.k_new, d.v_new, loc, d.err)
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    kp, vp = _oracle_store(wl)
    assert np.array_equal(_codes(d.pool.k[0]), kp[0])
    assert np.array_equal(_codes(d.pool.v[0]), vp[0])


def test_fp8_store_saturates():
    """Rows far beyond 448 * scale store the largest code, with its sign."""
    wl = W.with_fp8_pool(W.decode_small(), k_scale=0.001, v_scale=0.001)
    d = DeviceDecode(wl)
    api.store_kv(d.pool, 0, d.k_new, d.v_new, d.out_loc, d.err)
    torch.cuda.synchronize()
    kp, vp = _oracle_store(wl)
    got = _codes(d.pool.k[0])
    assert np.array_equal(got, kp[0])
    rows = got[wl.out_loc]
    assert np.any((rows & 0x7F) == 0x7E)  # some values did saturate


def test_fp8_store_inverse_scale_is_a_float32_quotient():
    """Scale 7: x = 91/1024 (bf16 0x3DB6) times the float32 1/7 lands one
    float32 step above the E4M3 tie 6.5 * 2^-9 and stores code 0x07 (0x87 for
    -x); the exact quotient would tie to the even code 0x06.  Both sides must
    take the float32 path, in every slot of the rows."""
    wl = W.with_fp8_pool(W.decode_small(), k_scale=7.0, v_scale=7.0)
    k_new = wl.k_new.copy()
    v_new = wl.v_new.copy()
    k_new[:, 0::2] = 0x3DB6
    v_new[:, 1::2] = 0xBDB6
    wl.k_new, wl.v_new = k_new, v_new
    d = DeviceDecode(wl)
    api.store_kv(d.pool, 0, d.k_new, d.v_new, d.out_loc, d.err)
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    kp, vp = _oracle_store(wl)
    got_k, got_v = _codes(d.pool.k[0]), _codes(d.pool.v[0])
    assert np.array_equal(got_k, kp[0]) and np.array_equal(got_v, vp[0])
    Hkv = wl.pool.num_kv_heads
    rows_k = got_k[wl.out_loc].reshape(wl.batch, Hkv * D)
    rows_v = got_v[wl.out_loc].reshape(wl.batch, Hkv * D)
    assert np.all(rows_k[:, 0::2] == 0x07) and np.all(rows_v[:, 1::2] == 0x87)


def test_fp8_gather_bit_exact():
    wl = W.with_fp8_pool(W.decode_paged_small(), seed=3)
    d = DeviceDecode(wl)
    B = wl.batch
    offs = np.zeros(B + 1, dtype=np.int64)
    offs[1:] = np.cumsum(wl.seq_lens)
    total = int(offs[-1])
    ko = torch.empty((total, wl.pool.num_kv_heads, D), dtype=torch.float8_e4m3fn, device="cuda")
    vo = torch.empty_like(ko)
    api.gather_kv(d.pool, 0, d.table, d.table_idx, d.seq_lens, torch.from_numpy(offs).cuda(), ko, vo, d.err)
    torch.cuda.synchronize()
    rows = oracle.gather_kv(wl.k_planes, wl.v_planes, 0, wl.page_table, wl.table_idx, wl.seq_lens,
                            wl.pool.page_size)
    assert np.array_equal(_codes(ko), np.concatenate([kr for kr, _ in rows]))
    assert np.array_equal(_codes(vo), np.concatenate([vr for _, vr in rows]))


@pytest.mark.parametrize("maker,hq", [("decode_small", 16), ("decode_small", 32), ("decode_small", 8),
                                      ("decode_small", 64), ("decode_paged_small", 32)])
def test_fp8_decode_matches_oracle(maker, hq):
    base = getattr(W, maker)(num_q_heads=hq) if maker == "decode_small" else W.decode_paged_small()
    wl = W.with_fp8_pool(base, seed=hq)
    d = DeviceDecode(wl)
    d.run()
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    kp, vp = _oracle_store(wl)
    exp = _oracle_decode(wl, kp, vp)
    tol_check(from_dev(d.out), exp, W.BF16, f"fp8 decode {maker} hq={hq}")
    scale_check(from_dev(d.out), exp, f"fp8 decode {maker} hq={hq}")


def test_fp8_decode_qwen3_06b_full():
    """The bench's decode step over an E4M3 copy of its pool (64 requests,
    141,622 context tokens, Hq 16, Hkv 8)."""
    wl = W.with_fp8_pool(W.decode_qwen3_06b(num_layers=1, layer=0))
    d = DeviceDecode(wl)
    d.run()
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    kp, vp = _oracle_store(wl)
    rng = np.random.default_rng(9)
    req = sorted(rng.choice(wl.batch, 12, replace=False).tolist())
    exp = _oracle_decode(wl, kp, vp, requests=req)
    tol_check(from_dev(d.out)[req], exp[req], W.BF16, "fp8 decode-qwen3-0.6b")
    scale_check(from_dev(d.out)[req], exp[req], "fp8 decode-qwen3-0.6b")


class _DequantPlanes:
    """Code planes (dict or tiled) read as float64 values code * scale, slot by
    slot, so a tiled pool never has to be decoded whole."""

    def __init__(self, planes, scale):
        self.planes, self.scale = planes, float(np.float32(scale))

    def __getitem__(self, layer):
        view = self.planes[layer]
        scale = self.scale

        class _Layer:
            def __getitem__(self, slots):
                return oracle.e4m3_decode(view[slots]) * scale

        return _Layer()


def test_fp8_decode_qwen3_8b_sampled():
    """The headline batch (256 requests, 1k-32k, page size 16, so decode loads
    page boxes) over an E4M3 copy of one layer of its pool: 16 sampled
    requests, the longest and shortest included."""
    from gpu_helpers import host_planes_copy
    wl = W.with_fp8_pool(W.decode_qwen3_8b(num_layers=1))
    d = DeviceDecode(wl)
    d.run()
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    kp, vp = host_planes_copy(wl.k_planes), host_planes_copy(wl.v_planes)
    oracle.store_kv_fp8(kp, vp, wl.layer, wl.k_new, wl.v_new, wl.out_loc, wl.pool.num_kv_heads, D,
                        wl.pool.k_scale, wl.pool.v_scale)
    lens = wl.seq_lens
    req = sorted(set([int(np.argmax(lens)), int(np.argmin(lens))] +
                     np.random.default_rng(5).choice(wl.batch, 14, replace=False).tolist()))
    exp = oracle.decode_attn(wl.q, _DequantPlanes(kp, wl.pool.k_scale), _DequantPlanes(vp, wl.pool.v_scale),
                             wl.layer, wl.page_table, wl.table_idx, wl.seq_lens, wl.pool.page_size, wl.scale,
                             requests=req)
    tol_check(from_dev(d.out)[req], exp[req], W.BF16, "fp8 decode-qwen3-8b")
    scale_check(from_dev(d.out)[req], exp[req], "fp8 decode-qwen3-8b")


def test_fp8_decode_nan_codes_in_unreferenced_slots():
    """Every slot no context reads holds the E4M3 NaN code 0x7F; page boxes load
    the tails of last pages and the rows before a CTA's first token, which must
    be masked out (p = 0 does not clear NaN)."""
    from gpu_helpers import poison_unreferenced, referenced_slots
    wl = W.with_fp8_pool(W.decode_paged_small(page_size=16, seq_lens=(1, 15, 17, 33, 300, 1029, 47),
                                              seed=1600), seed=7)
    keep = referenced_slots(wl)
    for planes in (wl.k_planes, wl.v_planes):
        poison_unreferenced(planes, 0, keep, np.uint8(0x7F))
    d = DeviceDecode(wl)
    d.run()
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    assert torch.isfinite(d.out.float()).all(), "a masked NaN row reached the output"
    kp, vp = _oracle_store(wl)
    exp = _oracle_decode(wl, kp, vp)
    tol_check(from_dev(d.out), exp, W.BF16, "fp8 decode, NaN codes in unreferenced slots")
    scale_check(from_dev(d.out), exp, "fp8 decode, NaN codes in unreferenced slots")


@pytest.mark.parametrize("page_size", [1, 16])
def test_fp8_decode_group_16(page_size):
    """E4M3 pool, 128 query heads over 8 KV heads (G = 16)."""
    wl = W.with_fp8_pool(W.decode_paged_small(page_size=page_size, num_q_heads=128, num_kv_heads=8,
                                              seed=1900 + page_size), seed=19)
    d = DeviceDecode(wl)
    d.run()
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    kp, vp = _oracle_store(wl)
    exp = _oracle_decode(wl, kp, vp)
    tol_check(from_dev(d.out), exp, W.BF16, f"fp8 decode G=16 P={page_size}")
    scale_check(from_dev(d.out), exp, f"fp8 decode G=16 P={page_size}")


def test_fp8_rope_store():
    wl = W.rope_store_step(W.BF16, seed=31)
    hq, hkv = wl.num_q_heads, wl.pool.num_kv_heads
    ks, vs = float(np.float32(0.02)), float(np.float32(0.03))
    spec = W.PoolSpec(1, wl.pool.num_slots, hkv, D, 1, W.F8, ks, vs)
    rng = np.random.Generator(np.random.PCG64(77))
    kp0 = {0: W.draw_e4m3_codes(rng, (spec.num_slots, hkv, D))}
    vp0 = {0: W.draw_e4m3_codes(rng, (spec.num_slots, hkv, D))}
    pool = device_pool(spec, kp0, vp0)
    qkv = to_dev(wl.qkv, W.BF16)
    q_out = torch.empty((wl.n_tokens, hq, D), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.qk_norm_rope_store(pool, 0, qkv, hq, i32(wl.positions), torch.from_numpy(wl.cos_sin_cache).cuda(),
                           i32(wl.out_loc), q_out, to_dev(wl.q_norm_w, W.BF16), to_dev(wl.k_norm_w, W.BF16),
                           wl.eps, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # Oracle: q and k in float64 (bf16 planes as scratch), v codes by quantize.
    kb = {0: np.zeros((spec.num_slots, hkv, D), dtype=np.uint16)}
    vb = {0: np.zeros((spec.num_slots, hkv, D), dtype=np.uint16)}
    q = oracle.qk_norm_rope_store(wl.qkv, hq, hkv, D, wl.positions, wl.cos_sin_cache, wl.q_norm_w,
                                  wl.k_norm_w, wl.eps, kb, vb, 0, wl.out_loc, storage="bf16")
    x = oracle.to_f64(wl.qkv).reshape(wl.n_tokens, hq + 2 * hkv, D)
    k = oracle.rope_rotate_half(oracle.rms_norm(x[:, hq:hq + hkv], wl.k_norm_w, wl.eps), wl.positions,
                                wl.cos_sin_cache)
    v_codes = oracle.quantize(wl.qkv[:, (hq + hkv) * D:], vs).reshape(wl.n_tokens, hkv, D)
    # q_out as in the bf16 path.
    got_q = from_dev(q_out)
    assert np.all(np.abs(got_q - q) <= 2.0 ** -8 * np.abs(q) + 2.0 ** -18 * np.abs(q).max(axis=-1, keepdims=True))
    gk = _codes(pool.k[0])[wl.out_loc]
    gv = _codes(pool.v[0])[wl.out_loc]
    assert np.array_equal(gv, v_codes)
    kdeq = oracle.e4m3_decode(gk) * ks
    bound = 2.0 ** -3 * np.abs(k) + 2.0 ** -9 * ks
    assert np.all(np.abs(kdeq - k) <= bound)
    same = np.mean(gk == oracle.quantize(k.astype(np.float32), ks).reshape(gk.shape))
    assert same >= 0.97, same
    # Every other slot is untouched.
    others = np.setdiff1d(np.arange(spec.num_slots), wl.out_loc)
    assert np.array_equal(_codes(pool.k[0])[others], kp0[0][others])
    assert np.array_equal(_codes(pool.v[0])[others], vp0[0][others])


def _oracle_extend(wl, rows=None):
    kp = {l: a.copy() for l, a in wl.k_planes.items()}
    vp = {l: a.copy() for l, a in wl.v_planes.items()}
    oracle.store_kv_fp8(kp, vp, wl.layer, wl.k_new, wl.v_new, wl.out_loc, wl.pool.num_kv_heads, D,
                        wl.pool.k_scale, wl.pool.v_scale)
    return oracle.extend_attn(wl.q, oracle.dequant_planes(kp, wl.pool.k_scale, [wl.layer]),
                              oracle.dequant_planes(vp, wl.pool.v_scale, [wl.layer]), wl.layer,
                              wl.page_table, wl.table_idx, wl.prefix_lens, wl.extend_lens,
                              wl.q_offsets, wl.pool.page_size, wl.scale, rows=rows)


@pytest.mark.parametrize("hq,hkv,page_size", [(16, 8, 1), (32, 8, 1), (8, 8, 1), (64, 8, 1), (16, 8, 64)])
def test_fp8_extend_matches_oracle(hq, hkv, page_size):
    """Extend over an E4M3 pool: ragged prefixes 0 / 37 / 130 with chunks of
    45 / 1 / 200 tokens; the chunk's own rows are quantised by store_kv."""
    wl = W.with_fp8_pool(W.extend_small(num_q_heads=hq, num_kv_heads=hkv, page_size=page_size), seed=hq)
    from gpu_helpers import DeviceExtend
    d = DeviceExtend(wl)
    d.run()
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    tol_check(from_dev(d.out), _oracle_extend(wl), W.BF16, f"fp8 extend hq={hq} P={page_size}")


def test_fp8_extend_chunked_prefill_sampled():
    """The 2048-token chunk at prefix 6144 (Hq 32, Hkv 8) over an E4M3 pool;
    64 sampled rows against the oracle."""
    wl = W.with_fp8_pool(W.chunked_prefill_step(step=3).extend)
    from gpu_helpers import DeviceExtend
    d = DeviceExtend(wl)
    d.run()
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    rows = np.sort(np.random.default_rng(4).choice(wl.total_q, 64, replace=False))
    exp = _oracle_extend(wl, rows=rows)
    tol_check(from_dev(d.out)[rows], exp[rows], W.BF16, "fp8 extend chunk c3")


def test_fp8_cascade_decode():
    gd = W.grouped_decode(groups=((64, 3), (1000, 20), (0, 2)), max_suffix=150, seed=71)
    wl = W.with_fp8_pool(gd.decode, seed=72)
    d = DeviceDecode(wl)
    api.store_kv(d.pool, 0, d.k_new, d.v_new, d.out_loc, d.err)
    mp = int(gd.group_prefix_lens.max())
    ws = api.decode_cascade_workspace(wl.batch, wl.num_q_heads, mp)
    out = torch.empty_like(d.q)
    api.decode_attn_cascade(d.pool, 0, d.q, d.table, d.table_idx, d.seq_lens, i32(gd.group_offsets),
                            i32(gd.group_prefix_lens), mp, out, ws, scale=wl.scale, dev_err=d.err)
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    kp, vp = _oracle_store(wl)
    tol_check(from_dev(out), _oracle_decode(wl, kp, vp), W.BF16, "fp8 cascade decode")


def test_fp32_cascade_unsupported():
    gd = W.grouped_decode(W.F32, groups=((64, 2),), seed=73)
    d = DeviceDecode(gd.decode)
    ws = api.decode_cascade_workspace(gd.decode.batch, gd.decode.num_q_heads, 64)
    with pytest.raises(RuntimeError, match="unsupported"):
        api.decode_attn_cascade(d.pool, 0, d.q, d.table, d.table_idx, d.seq_lens, i32(gd.group_offsets),
                                i32(gd.group_prefix_lens), 64, torch.empty_like(d.q), ws,
                                scale=gd.decode.scale)
