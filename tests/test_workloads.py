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
