"""Structure of the seeded synthetic workloads (CPU only)."""
import numpy as np
import pytest

from paged_kv_gqa_scatter_b200 import workloads as W


def _check_decode(wl, check_pages=True):
    B = wl.batch
    assert wl.q.shape == (B, wl.num_q_heads, W.HEAD_DIM)
    assert wl.k_new.shape == (B, wl.pool.row_elems)
    assert np.all(wl.seq_lens >= 1)
    assert wl.table_idx.shape == (B,) and len(set(wl.table_idx.tolist())) == B
    assert np.unique(wl.out_loc).shape[0] == B  # distinct slots per call
    P = wl.pool.page_size
    for r in range(B):
        row = wl.page_table[wl.table_idx[r]]
        n = int(wl.seq_lens[r])
        assert wl.out_loc[r] == row[n - 1]
        assert row[:n].max() < wl.pool.num_slots
        if check_pages and P > 1:
            first = row[0:n:P]
            assert np.all(first % P == 0)
            for j in range(0, n, P):
                m = min(P, n - j)
                assert np.array_equal(row[j:j + m], row[j] + np.arange(m))


def test_decode_small_shapes():
    wl = W.decode_small()
    assert wl.seq_lens.tolist() == [17, 33, 50, 64]
    _check_decode(wl)
    # Every request's slots are distinct across requests (one permutation).
    used = np.concatenate([wl.page_table[wl.table_idx[r], :wl.seq_lens[r]] for r in range(4)])
    assert np.unique(used).shape[0] == used.shape[0]


def test_decode_small_is_seeded():
    a, b = W.decode_small(), W.decode_small()
    assert np.array_equal(a.q, b.q) and np.array_equal(a.k_planes[0], b.k_planes[0])


def test_decode_paged_small():
    _check_decode(W.decode_paged_small())


def test_decode_qwen3_8b_structure():
    wl = W.decode_qwen3_8b(num_pages=20000, batch=32)
    _check_decode(wl)
    assert wl.seq_lens.min() >= 1024 and wl.seq_lens.max() <= 32768
    assert wl.alias_factor > 0


def test_extend_small():
    wl = W.extend_small(page_size=4)
    assert wl.total_q == int(wl.extend_lens.sum())
    assert np.unique(wl.out_loc).shape[0] == wl.total_q


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 65504.0], dtype=np.float32)
    bits = W.f32_to_bf16_bits(x)
    back = W.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1.0); 1 + 3*2^-8 -> 1 + 2^-6.
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 65536.0]


def test_grouped_decode_structure():
    """Members of a group share the prefix slots; suffix slots are private and
    distinct; every context covers its group's prefix plus the stored token."""
    for P in (1, 16, 64):
        gd = W.grouped_decode(page_size=P)
        d = gd.decode
        off, plen = gd.group_offsets, gd.group_prefix_lens
        assert off[0] == 0 and off[-1] == d.batch and np.all(np.diff(off) >= 1)
        seen = []
        for g in range(len(plen)):
            rows = [d.table_idx[r] for r in range(off[g], off[g + 1])]
            p = int(plen[g])
            for r, row in zip(range(off[g], off[g + 1]), rows):
                assert np.array_equal(d.page_table[row, :p], d.page_table[rows[0], :p])
                assert d.seq_lens[r] >= p + 1
                seen.append(d.page_table[row, p:d.seq_lens[r]])
            seen.append(d.page_table[rows[0], :p])
        allslots = np.concatenate(seen)
        assert len(np.unique(allslots)) == len(allslots)
        assert np.all(allslots < d.pool.num_slots)
        if P > 1:
            assert np.all(plen % P == 0)


def test_fp8_pool_variant():
    base = W.decode_small()
    wl = W.with_fp8_pool(base)
    assert wl.pool.dtype == W.F8 and wl.pool.io_dtype == W.BF16
    assert wl.k_planes[0].dtype == np.uint8 and wl.k_planes[0].shape == base.k_planes[0].shape
    codes = wl.k_planes[0]
    assert not np.any((codes & 0x7F) == 0x7F)                 # no NaN codes
    ex = (codes >> 3) & 0xF
    assert ex.min() >= 4 and ex.max() <= 9
    assert np.array_equal(wl.q, base.q) and np.array_equal(wl.k_new, base.k_new)
    assert wl.pool.k_scale == float(np.float32(0.05))


def test_rope_store_step_inputs():
    wl = W.rope_store_step()
    assert wl.qkv.shape == (wl.n_tokens, (wl.num_q_heads + 2 * wl.pool.num_kv_heads) * W.HEAD_DIM)
    assert np.all((wl.positions >= 0) & (wl.positions < wl.cos_sin_cache.shape[0]))
    assert len(np.unique(wl.out_loc)) == wl.n_tokens
    cs = wl.cos_sin_cache.astype(np.float64)
    # cos^2 + sin^2 = 1 for every stored angle (float32 table).
    assert np.allclose(cs[:, :64] ** 2 + cs[:, 64:] ** 2, 1.0, atol=1e-6)
    assert np.array_equal(cs[0, :64], np.ones(64)) and np.array_equal(cs[0, 64:], np.zeros(64))


def test_fp8_pool_variant_of_the_tiled_qwen3_8b_pool():
    """The E4M3 copy of the Qwen3-8B batch keeps the tiled pool: a code block
    of the same shape, tiled over the same slots; table and lengths unchanged;
    no NaN code."""
    base = W.decode_qwen3_8b(num_layers=2)
    wl = W.with_fp8_pool(base)
    assert isinstance(wl.k_planes, W.TiledPlane) and isinstance(wl.v_planes, W.TiledPlane)
    for plane, src in ((wl.k_planes, base.k_planes), (wl.v_planes, base.v_planes)):
        assert plane.block.dtype == np.uint8 and plane.block.shape == src.block.shape
        assert plane.num_slots == src.num_slots and plane.num_layers == src.num_layers
        assert not np.any((plane.block & 0x7F) == 0x7F)
    assert wl.pool.dtype == W.F8 and wl.pool.page_size == 16
    assert np.array_equal(wl.page_table, base.page_table) and np.array_equal(wl.seq_lens, base.seq_lens)
    # A slot of layer 1 reads the block row (num_slots + slot) mod block rows.
    nb = wl.k_planes.block.shape[0]
    assert np.array_equal(wl.k_planes[1][np.array([5])][0], wl.k_planes.block[(wl.pool.num_slots + 5) % nb])
