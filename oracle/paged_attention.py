"""Plain float64 CPU oracle for attention over a paged KV pool.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports, links or calls
this module; only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA path.

It states what the hot path computes, step by step, as the pages define it,
with no blocking, splitting or fusion:

* ``store_kv``  -- "Mini-SGLang 完整剖析" (blog.rzhang-lab.cn/post/3) §4.4.3
  (the pool is one tensor ``(2, layers, pages, page_size, kv_heads, head_dim)``
  flattened to ``(pages*page_size, kv_heads, head_dim)``; new rows are
  scattered into it at ``out_loc``) and §4.6.7 (the backend stores the step's
  K/V before calling the attention kernel).
* ``slots_of``  -- same page, §4.6.4: the page table is kept token-granular;
  backends with larger pages slice every ``page_size``-th column and divide by
  ``page_size`` to get page ids.  "mini-sglang 深度分析报告" (nightvoyager.top)
  states the same page_size-1 table design.
* attention     -- §1.2 (decode: one new query per request over its whole
  history) and "深入解析 mini-sglang" (yunpan.plus), chunked prefill (a chunk
  reuses the cached KV of the chunks before it).  The formula itself,
  ``softmax(q k^T / sqrt(d)) v`` with a causal mask and grouped KV heads, is
  the textbook definition; the pages do not print it.

Readings where the pages are silent (each is also listed in the design notes):
  * the context of a decode request includes the token ``store_kv`` just
    wrote (``cache_seqlens`` is the total KV length, §4.6.4);
  * query head ``h`` reads KV head ``h // (Hq // Hkv)`` (KV heads are the
    sharding unit, §4.5.3);
  * causal alignment is bottom-right: query ``i`` of a chunk sits at absolute
    position ``prefix_len + i`` and sees keys ``0 .. prefix_len + i``;
  * an empty context yields a zero output row.

Element storage: bf16 values are uint16 bit patterns and widen to float64
exactly; fp32 values widen exactly too.  All arithmetic is float64.
"""
from __future__ import annotations

import numpy as np


def to_f64(x) -> np.ndarray:
    """Exact widening of stored elements (bf16 bit patterns or float32) to float64."""
    a = np.asarray(x)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if a.dtype in (np.float32, np.float64):
        return a.astype(np.float64)
    raise TypeError(f"unsupported element storage {a.dtype}")


# ---------------------------------------------------------------------------
# store_kv: scatter rows into the pool (bit copy).
# ---------------------------------------------------------------------------
def store_kv(k_planes, v_planes, layer: int, k_rows, v_rows, out_loc, num_kv_heads: int,
             head_dim: int) -> None:
    """Write ``k_rows[i]`` / ``v_rows[i]`` (each ``num_kv_heads*head_dim``
    elements) into slot ``out_loc[i]`` of ``layer``, in place, as a bit copy.
    ``k_planes[layer]`` is indexable by slot.  Slots within one call are
    assumed distinct (the pages hand each new token its own slot)."""
    out_loc = np.asarray(out_loc, dtype=np.int64)
    n = out_loc.shape[0]
    if n == 0:
        return
    kr = np.asarray(k_rows).reshape(n, num_kv_heads, head_dim)
    vr = np.asarray(v_rows).reshape(n, num_kv_heads, head_dim)
    kl = k_planes[layer]
    vl = v_planes[layer]
    for i in range(n):
        kl[out_loc[i]] = kr[i]
        vl[out_loc[i]] = vr[i]


# ---------------------------------------------------------------------------
# Page-table translation and gather.
# ---------------------------------------------------------------------------
def slots_of(page_table, row: int, n: int, page_size: int) -> np.ndarray:
    """Pool slots of tokens ``0..n-1`` of the request in table row ``row``.

    page_size 1: the entry itself.  page_size P > 1: take the entry at the
    first column of the token's page (every P-th column), divide by P to get
    the page id, and address offset ``j mod P`` inside that page.
    """
    table = np.asarray(page_table)
    j = np.arange(n, dtype=np.int64)
    if page_size == 1:
        return table[row, :n].astype(np.int64)
    first_col = page_size * (j // page_size)
    page = table[row, first_col].astype(np.int64) // page_size
    return page * page_size + (j % page_size)


def gather_kv(k_planes, v_planes, layer: int, page_table, table_idx, seq_lens, page_size: int):
    """Per request, its K and V rows in token order, as stored (no conversion)."""
    out = []
    for r in range(len(seq_lens)):
        s = slots_of(page_table, int(table_idx[r]), int(seq_lens[r]), page_size)
        out.append((np.asarray(k_planes[layer][s]), np.asarray(v_planes[layer][s])))
    return out


# ---------------------------------------------------------------------------
# Attention.
# ---------------------------------------------------------------------------
def attend(q, K, V, key_limit, scale: float) -> np.ndarray:
    """Grouped-query attention of query rows against one request's keys.

    q: [nq][Hq][d]; K, V: [n][Hkv][d]; key_limit[i]: query row i sees keys
    ``0 .. key_limit[i]-1``.  Returns float64 [nq][Hq][d].
    """
    q = to_f64(q)
    K = to_f64(K)
    V = to_f64(V)
    nq, Hq, d = q.shape
    n, Hkv, _ = K.shape
    G = Hq // Hkv
    out = np.zeros((nq, Hq, d), dtype=np.float64)
    lim = np.asarray(key_limit, dtype=np.int64)
    if n == 0 or nq == 0:
        return out
    allowed = np.arange(n)[None, :] < lim[:, None]              # [nq][n]
    for h in range(Hq):
        g = h // G
        s = (q[:, h, :] @ K[:, g, :].T) * scale                 # [nq][n]
        s = np.where(allowed, s, -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        p = np.where(allowed, np.exp(s - m), 0.0)
        den = p.sum(axis=1, keepdims=True)
        o = p @ V[:, g, :]
        out[:, h, :] = np.where(den > 0, o / np.where(den > 0, den, 1.0), 0.0)
    return out


def decode_attn(q, k_planes, v_planes, layer: int, page_table, table_idx, seq_lens,
                page_size: int, scale: float, requests=None) -> np.ndarray:
    """One query token per request against its whole context (``seq_lens[r]``
    tokens, the just-stored one included).  Returns float64 [B][Hq][d]; rows of
    requests not in ``requests`` (when given) are left zero."""
    q = np.asarray(q)
    B = len(seq_lens)
    out = np.zeros(q.shape, dtype=np.float64)
    reqs = range(B) if requests is None else requests
    for r in reqs:
        n = int(seq_lens[r])
        s = slots_of(page_table, int(table_idx[r]), n, page_size)
        K = k_planes[layer][s]
        V = v_planes[layer][s]
        out[r:r + 1] = attend(q[r:r + 1], K, V, [n], scale)
    return out


def extend_attn(q, k_planes, v_planes, layer: int, page_table, table_idx, prefix_lens,
                extend_lens, q_offsets, page_size: int, scale: float, rows=None) -> np.ndarray:
    """Causal attention of each request's chunk over its cached prefix plus the
    chunk itself.  Query row ``q_offsets[r] + i`` is at absolute position
    ``prefix_lens[r] + i`` and sees keys ``0 .. prefix_lens[r] + i``.  Returns
    float64 [total_q][Hq][d]; with ``rows`` given, only those query rows are
    computed (others stay zero)."""
    q = np.asarray(q)
    out = np.zeros(q.shape, dtype=np.float64)
    want = None if rows is None else set(int(x) for x in rows)
    for r in range(len(extend_lens)):
        p = int(prefix_lens[r])
        e = int(extend_lens[r])
        if e == 0:
            continue
        base = int(q_offsets[r])
        idx = np.arange(e)
        if want is not None:
            idx = np.array([i for i in idx if base + i in want], dtype=np.int64)
            if idx.size == 0:
                continue
        n = p + e
        s = slots_of(page_table, int(table_idx[r]), n, page_size)
        K = k_planes[layer][s]
        V = v_planes[layer][s]
        out[base + idx] = attend(q[base + idx], K, V, p + idx + 1, scale)
    return out


# ---------------------------------------------------------------------------
# Split-KV bookkeeping (the combine step, stated on its own).
# ---------------------------------------------------------------------------
def partial_state(q_row, K, V, scale: float):
    """Softmax state of one query row over a key subset: per head the running
    max ``m`` (natural-log domain), the sum ``l`` of exp(s - m), and the
    un-normalised output ``o = sum exp(s - m) v``."""
    q_row = to_f64(q_row)
    K = to_f64(K)
    V = to_f64(V)
    Hq, d = q_row.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    m = np.full(Hq, -np.inf)
    l = np.zeros(Hq)
    o = np.zeros((Hq, d))
    if K.shape[0] == 0:
        return m, l, o
    for h in range(Hq):
        g = h // G
        s = (K[:, g, :] @ q_row[h]) * scale
        m[h] = s.max()
        p = np.exp(s - m[h])
        l[h] = p.sum()
        o[h] = p @ V[:, g, :]
    return m, l, o


def combine_states(states):
    """Merge softmax states of disjoint key subsets: rescale each by
    exp(m_s - M) with M the largest max, sum, and normalise."""
    ms = np.stack([s[0] for s in states])          # [S][Hq]
    ls = np.stack([s[1] for s in states])
    os_ = np.stack([s[2] for s in states])         # [S][Hq][d]
    M = ms.max(axis=0)
    Ms = np.where(np.isfinite(M), M, 0.0)
    w = np.where(np.isfinite(ms), np.exp(ms - Ms[None, :]), 0.0)
    num = (w[:, :, None] * os_).sum(axis=0)
    den = (w * ls).sum(axis=0)
    return np.where(den[:, None] > 0, num / np.where(den > 0, den, 1.0)[:, None], 0.0)
