"""Pins for the float64 oracle: checks against things other than the oracle.

Every ``pin_*`` takes an oracle namespace (the real ``oracle`` package, or a
copy with a planted mistake) and raises AssertionError when the oracle
disagrees with a closed form, a brute-force computation written here
independently (pure Python loops over dense, contiguous K/V with ``math.exp``),
or an invariant that the mathematics fixes.  ``ALL_PINS`` lists them; the
mutation test checks that each planted mistake trips at least one.
"""
from __future__ import annotations

import math
import os

import numpy as np

D = 128
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# Independent helpers (no oracle code).
# ---------------------------------------------------------------------------
def _bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float values to bf16-representable float64 values (RNE)."""
    f = np.asarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def _bits(x: np.ndarray) -> np.ndarray:
    """bf16-representable float64 values -> uint16 bit patterns."""
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def brute_attention(q_rows, keys, vals, limits, scale, Hkv):
    """Dense attention with explicit loops.  q_rows: list of [Hq][d] (float),
    keys/vals: [n][Hkv][d] dense in token order, limits: keys visible per row."""
    out = []
    Hq = len(q_rows[0])
    G = Hq // Hkv
    for qi, qr in enumerate(q_rows):
        lim = limits[qi]
        row = []
        for h in range(Hq):
            g = h // G
            if lim == 0:
                row.append([0.0] * D)
                continue
            sc = []
            for j in range(lim):
                acc = 0.0
                for c in range(D):
                    acc += float(qr[h][c]) * float(keys[j][g][c])
                sc.append(acc * scale)
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            tot = math.fsum(w)
            o = []
            for c in range(D):
                o.append(math.fsum(w[j] * float(vals[j][g][c]) for j in range(lim)) / tot)
            row.append(o)
        out.append(row)
    return np.array(out, dtype=np.float64)


class PagedCase:
    """Dense per-request sequences scattered into a single-layer pool through a
    seeded slot permutation, with a token-granular table (page_size 1 or P)."""

    def __init__(self, rng, Hq, Hkv, lens, page_size=1, num_slots=None, value_scale=1.0):
        self.Hq, self.Hkv, self.P = Hq, Hkv, page_size
        self.lens = [int(x) for x in lens]
        P = page_size
        pages = [(n + P - 1) // P for n in self.lens]
        total_pages = sum(pages) + 3
        self.num_slots = num_slots or total_pages * P
        self.keys = [_bf16_round(rng.standard_normal((n, Hkv, D)) * value_scale) for n in self.lens]
        self.vals = [_bf16_round(rng.standard_normal((n, Hkv, D))) for n in self.lens]
        perm = rng.permutation(self.num_slots // P)
        self.table = np.zeros((len(lens) + 1, max(1, max(pages) * P)), dtype=np.int32)
        self.table_idx = rng.permutation(len(lens)).astype(np.int32)
        kp = np.zeros((self.num_slots, Hkv, D), dtype=np.uint16)
        vp = np.zeros((self.num_slots, Hkv, D), dtype=np.uint16)
        k = 0
        for r, n in enumerate(self.lens):
            ph = perm[k:k + pages[r]]
            k += pages[r]
            ent = (ph[:, None] * P + np.arange(P)[None, :]).reshape(-1)
            self.table[self.table_idx[r], :pages[r] * P] = ent
            kp[ent[:n]] = _bits(self.keys[r])
            vp[ent[:n]] = _bits(self.vals[r])
        self.kp = {0: kp}
        self.vp = {0: vp}

    def q(self, rng, rows):
        return _bf16_round(rng.standard_normal((rows, self.Hq, D)))


def _close(a, b, tol=1e-12):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol * (1.0 + np.max(np.abs(b)) if b.size else 1.0), f"max err {err}"


# ---------------------------------------------------------------------------
# Pins.
# ---------------------------------------------------------------------------
def pin_store_bit_copy(orc):
    """store_kv is a bit copy into the named slots; every other slot keeps its bits."""
    rng = np.random.default_rng(7)
    S, Hkv = 64, 2
    kp = {0: rng.integers(0, 1 << 16, (S, Hkv, D), dtype=np.uint16)}
    vp = {0: rng.integers(0, 1 << 16, (S, Hkv, D), dtype=np.uint16)}
    k0, v0 = kp[0].copy(), vp[0].copy()
    loc = np.array([5, 63, 0, 17], dtype=np.int64)
    kr = rng.integers(0, 1 << 16, (4, Hkv * D), dtype=np.uint16)
    vr = rng.integers(0, 1 << 16, (4, Hkv * D), dtype=np.uint16)
    orc.store_kv(kp, vp, 0, kr, vr, loc, Hkv, D)
    for i, s in enumerate(loc):
        assert np.array_equal(kp[0][s].reshape(-1), kr[i])
        assert np.array_equal(vp[0][s].reshape(-1), vr[i])
    rest = np.setdiff1d(np.arange(S), loc)
    assert np.array_equal(kp[0][rest], k0[rest]) and np.array_equal(vp[0][rest], v0[rest])


def pin_page_translation_golden(orc):
    """Hand-derived translation of a page_size-4 token table (tests/golden)."""
    vals = {}
    with open(os.path.join(GOLDEN, "page_translation.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, *rest = line.split()
            vals[key] = [int(x) for x in rest]
    P = vals["page_size"][0]
    table = np.array([vals["row"]], dtype=np.int32)
    got = orc.slots_of(table, 0, vals["n"][0], P)
    assert list(got) == vals["slots"], (list(got), vals["slots"])
    # The first column of each page divided by P gives the listed page ids.
    assert [int(table[0, c]) // P for c in range(0, vals["n"][0], P)] == vals["pages"]


def pin_gather_matches_dense(orc):
    """Gathering through the table returns each request's tokens in order."""
    rng = np.random.default_rng(11)
    for P in (1, 4):
        c = PagedCase(rng, 4, 2, [1, 9, 23], page_size=P)
        got = orc.gather_kv(c.kp, c.vp, 0, c.table, c.table_idx, c.lens, P)
        for r in range(len(c.lens)):
            assert np.array_equal(got[r][0], _bits(c.keys[r]))
            assert np.array_equal(got[r][1], _bits(c.vals[r]))


def pin_two_key_closed_form(orc):
    """Two keys with scores 0 and s give the logistic weights (tests/golden)."""
    cases = []
    with open(os.path.join(GOLDEN, "two_key_softmax.txt")) as f:
        for line in f:
            if line.startswith("case"):
                _, a, b = line.split()
                cases.append((float(a), float(b)))
    for a, b in cases:
        q = np.zeros((1, 1, D)); q[0, 0, 0] = a
        K = np.zeros((2, 1, D)); K[1, 0, 0] = b
        V = np.zeros((2, 1, D)); V[0, 0, 1] = 1.0; V[1, 0, 2] = 1.0
        s = a * b / math.sqrt(D)
        out = orc.attend(q.astype(np.float32), K.astype(np.float32), V.astype(np.float32), [2],
                         1.0 / math.sqrt(D))
        w1 = math.exp(s) / (1.0 + math.exp(s))
        exp = np.zeros(D); exp[1] = 1.0 - w1; exp[2] = w1
        _close(out[0, 0], exp, 1e-14)


def pin_decode_brute_force(orc):
    """Paged decode equals dense brute-force attention (tiny, G = 2)."""
    rng = np.random.default_rng(13)
    for P in (1, 4):
        c = PagedCase(rng, 4, 2, [1, 7, 33], page_size=P)
        q = c.q(rng, 3)
        got = orc.decode_attn(_bits(q), c.kp, c.vp, 0, c.table, c.table_idx, c.lens, P,
                              1.0 / math.sqrt(D))
        for r in range(3):
            exp = brute_attention([q[r]], c.keys[r], c.vals[r], [c.lens[r]],
                                  1.0 / math.sqrt(D), 2)
            _close(got[r:r + 1], exp)


def pin_extend_brute_force(orc):
    """Paged causal extend equals dense brute-force attention (tiny, G = 4)."""
    rng = np.random.default_rng(17)
    prefix = [0, 5, 12]
    ext = [6, 1, 9]
    lens = [p + e for p, e in zip(prefix, ext)]
    for P in (1, 4):
        c = PagedCase(rng, 8, 2, lens, page_size=P)
        q = c.q(rng, sum(ext))
        off = np.concatenate([[0], np.cumsum(ext)]).astype(np.int32)
        got = orc.extend_attn(_bits(q), c.kp, c.vp, 0, c.table, c.table_idx, prefix, ext, off, P,
                              1.0 / math.sqrt(D))
        for r in range(3):
            rows = [q[off[r] + i] for i in range(ext[r])]
            lim = [prefix[r] + i + 1 for i in range(ext[r])]
            exp = brute_attention(rows, c.keys[r], c.vals[r], lim, 1.0 / math.sqrt(D), 2)
            _close(got[off[r]:off[r + 1]], exp)


def pin_slot_permutation(orc):
    """Relabelling physical slots (pool and table together) changes nothing."""
    rng = np.random.default_rng(19)
    c = PagedCase(rng, 8, 4, [3, 40, 17])
    q = _bits(c.q(rng, 3))
    a = orc.decode_attn(q, c.kp, c.vp, 0, c.table, c.table_idx, c.lens, 1, 0.1)
    pi = rng.permutation(c.num_slots)
    kp = {0: np.empty_like(c.kp[0])}
    vp = {0: np.empty_like(c.vp[0])}
    kp[0][pi] = c.kp[0]
    vp[0][pi] = c.vp[0]
    t2 = pi[c.table].astype(np.int32)
    b = orc.decode_attn(q, kp, vp, 0, t2, c.table_idx, c.lens, 1, 0.1)
    assert np.array_equal(a, b)


def pin_chunked_equals_unchunked(orc):
    """A prefill split into chunks (each chunk over the earlier ones) equals one pass."""
    rng = np.random.default_rng(23)
    N = 30
    c = PagedCase(rng, 4, 2, [N])
    q = _bits(c.q(rng, N))
    sc = 1.0 / math.sqrt(D)
    one = orc.extend_attn(q, c.kp, c.vp, 0, c.table, c.table_idx, [0], [N], [0, N], 1, sc)
    parts = []
    for p, e in ((0, 8), (8, 13), (21, 9)):
        parts.append(orc.extend_attn(q[p:p + e], c.kp, c.vp, 0, c.table, c.table_idx, [p], [e],
                                     [0, e], 1, sc))
    _close(np.concatenate(parts), one)


def pin_shared_prefix_equals_private(orc):
    """Requests reading a prefix from shared slots match requests with private copies."""
    rng = np.random.default_rng(29)
    Hq, Hkv, L, S = 8, 2, 12, 128
    pre_k = _bits(_bf16_round(rng.standard_normal((L, Hkv, D))))
    pre_v = _bits(_bf16_round(rng.standard_normal((L, Hkv, D))))
    suf = [5, 9]
    kp = {0: np.zeros((S, Hkv, D), np.uint16)}
    vp = {0: np.zeros((S, Hkv, D), np.uint16)}
    kp2 = {0: np.zeros((S, Hkv, D), np.uint16)}
    vp2 = {0: np.zeros((S, Hkv, D), np.uint16)}
    shared = np.arange(L)
    t_sh = np.zeros((3, 40), np.int32)
    t_pr = np.zeros((3, 40), np.int32)
    kp[0][shared] = pre_k; vp[0][shared] = pre_v
    nxt = L
    sk = [_bits(_bf16_round(rng.standard_normal((s, Hkv, D)))) for s in suf]
    sv = [_bits(_bf16_round(rng.standard_normal((s, Hkv, D)))) for s in suf]
    for r, s in enumerate(suf):
        own = np.arange(nxt, nxt + s); nxt += s
        t_sh[r, :L] = shared; t_sh[r, L:L + s] = own
        kp[0][own] = sk[r]; vp[0][own] = sv[r]
        priv = np.arange(nxt, nxt + L + s); nxt += L + s
        t_pr[r, :L + s] = priv
        kp2[0][priv[:L]] = pre_k; vp2[0][priv[:L]] = pre_v
        kp2[0][priv[L:]] = sk[r]; vp2[0][priv[L:]] = sv[r]
    q = _bits(_bf16_round(rng.standard_normal((sum(suf), Hq, D))))
    off = [0, suf[0], sum(suf)]
    a = orc.extend_attn(q, kp, vp, 0, t_sh, [0, 1], [L, L], suf, off, 1, 0.09)
    b = orc.extend_attn(q, kp2, vp2, 0, t_pr, [0, 1], [L, L], suf, off, 1, 0.09)
    assert np.array_equal(a, b)


def pin_one_token_returns_v(orc):
    """A one-token context returns that token's V exactly."""
    rng = np.random.default_rng(31)
    c = PagedCase(rng, 8, 4, [1, 1])
    q = _bits(c.q(rng, 2))
    out = orc.decode_attn(q, c.kp, c.vp, 0, c.table, c.table_idx, c.lens, 1, 0.3)
    for r in range(2):
        for h in range(8):
            assert np.array_equal(out[r, h], c.vals[r][0, h // 2])


def pin_constant_k_mean_v(orc):
    """Identical keys give uniform weights: the output is the mean of V."""
    rng = np.random.default_rng(37)
    n, Hkv = 21, 2
    k_row = _bf16_round(rng.standard_normal((Hkv, D)))
    K = np.repeat(k_row[None], n, axis=0)
    V = _bf16_round(rng.standard_normal((n, Hkv, D)))
    q = _bf16_round(rng.standard_normal((1, 4, D)))
    out = orc.attend(_bits(q), _bits(K), _bits(V), [n], 0.5)
    for h in range(4):
        _close(out[0, h], V[:, h // 2].mean(axis=0), 1e-14)


def pin_constant_k_mean_v_group_16(orc):
    """The same closed form at a GQA group of 16 (32 query heads over 2 KV
    heads): query head h averages KV head h // 16's values."""
    rng = np.random.default_rng(38)
    n, Hkv, Hq = 13, 2, 32
    k_row = _bf16_round(rng.standard_normal((Hkv, D)))
    K = np.repeat(k_row[None], n, axis=0)
    V = _bf16_round(rng.standard_normal((n, Hkv, D)))
    q = _bf16_round(rng.standard_normal((1, Hq, D)))
    out = orc.attend(_bits(q), _bits(K), _bits(V), [n], 0.5)
    for h in range(Hq):
        _close(out[0, h], V[:, h // 16].mean(axis=0), 1e-14)


def pin_decode_equals_extend_one_row(orc):
    """decode over n tokens equals extend with prefix n-1 and one new row."""
    rng = np.random.default_rng(41)
    c = PagedCase(rng, 8, 2, [19, 4])
    q = _bits(c.q(rng, 2))
    d = orc.decode_attn(q, c.kp, c.vp, 0, c.table, c.table_idx, c.lens, 1, 0.2)
    e = orc.extend_attn(q, c.kp, c.vp, 0, c.table, c.table_idx, [18, 3], [1, 1], [0, 1, 2], 1, 0.2)
    assert np.array_equal(d, e)


def pin_scale_invariance(orc):
    """Multiplying q by 2 and k by 1/2 (exact in bf16) leaves outputs unchanged."""
    rng = np.random.default_rng(43)
    K = _bf16_round(rng.standard_normal((15, 2, D)))
    V = _bf16_round(rng.standard_normal((15, 2, D)))
    q = _bf16_round(rng.standard_normal((3, 4, D)))
    a = orc.attend(_bits(q), _bits(K), _bits(V), [15, 7, 1], 0.11)
    b = orc.attend(_bits(q * 2), _bits(K * 0.5), _bits(V), [15, 7, 1], 0.11)
    _close(a, b, 1e-15)


def pin_identical_heads(orc):
    """Query heads of one group with identical q give identical outputs; other
    groups read their own KV head."""
    rng = np.random.default_rng(47)
    K = _bf16_round(rng.standard_normal((9, 2, D)))
    V = _bf16_round(rng.standard_normal((9, 2, D)))
    qh = _bf16_round(rng.standard_normal(D))
    q = np.repeat(np.repeat(qh[None, None], 4, axis=1), 1, axis=0)
    out = orc.attend(_bits(q), _bits(K), _bits(V), [9], 0.1)
    assert np.array_equal(out[0, 0], out[0, 1]) and np.array_equal(out[0, 2], out[0, 3])
    assert not np.allclose(out[0, 0], out[0, 2])
    exp0 = brute_attention([q[0]], K, V, [9], 0.1, 2)
    _close(out, exp0)


def pin_split_combine(orc):
    """Softmax states of disjoint key chunks merge to the unsplit result."""
    rng = np.random.default_rng(53)
    K = _bf16_round(rng.standard_normal((50, 2, D)) * 2)
    V = _bf16_round(rng.standard_normal((50, 2, D)))
    q = _bf16_round(rng.standard_normal((4, D)))
    full = orc.attend(_bits(q[None]), _bits(K), _bits(V), [50], 0.2)[0]
    for cuts in ((0, 50), (0, 13, 50), (0, 1, 2, 30, 50)):
        st = [orc.partial_state(_bits(q), _bits(K[a:b]), _bits(V[a:b]), 0.2)
              for a, b in zip(cuts[:-1], cuts[1:])]
        _close(orc.combine_states(st), full)


def pin_empty_context_zero(orc):
    """A request with no visible keys gets a zero row (reading c6)."""
    q = np.ones((1, 2, D), np.float32)
    out = orc.attend(q, np.zeros((0, 1, D), np.float32), np.zeros((0, 1, D), np.float32), [0], 1.0)
    assert np.array_equal(out, np.zeros((1, 2, D)))


ALL_PINS = [pin_store_bit_copy, pin_page_translation_golden, pin_gather_matches_dense,
            pin_two_key_closed_form, pin_decode_brute_force, pin_extend_brute_force,
            pin_slot_permutation, pin_chunked_equals_unchunked, pin_shared_prefix_equals_private,
            pin_one_token_returns_v, pin_constant_k_mean_v, pin_constant_k_mean_v_group_16,
            pin_decode_equals_extend_one_row,
            pin_scale_invariance, pin_identical_heads, pin_split_combine, pin_empty_context_zero]


# ---------------------------------------------------------------------------
# q/k RMSNorm + RoPE + store pins.
# ---------------------------------------------------------------------------
def rope_cache(max_pos, d, base=10000.0, dtype=np.float32):
    """cos | sin halves per position, built here from the angle definition."""
    half = d // 2
    inv = base ** (-2.0 * np.arange(half) / d)
    ang = np.arange(max_pos)[:, None] * inv[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(dtype)


def pin_bf16_rounding(orc):
    """Nearest-even rounding to bf16 on hand-picked values and ties."""
    vals = [1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -40, -2.5, 0.0,
            3.0 * 2 ** -7, 65280.0, 2.0 ** -100]
    want = [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC020, 0x0000, 0x3CC0, 0x477F, 0x0D80]
    got = orc.to_storage(np.array(vals), "bf16")
    assert [int(x) for x in got] == want, [hex(int(x)) for x in got]


def pin_rms_norm_closed_form(orc):
    """A constant vector c has RMS |c|; a 3-4-0 vector has RMS 5/sqrt(d)."""
    d = D
    w = np.linspace(0.5, 1.5, d)
    y = orc.rms_norm(np.full((1, d), -3.0), w, 0.0)
    _close(y[0], -w, 1e-15)
    x = np.zeros((1, d)); x[0, 0] = 3.0; x[0, 1] = 4.0
    y = orc.rms_norm(x, np.ones(d), 0.0)
    r = 5.0 / math.sqrt(d)
    _close(y[0, :2], [3.0 / r, 4.0 / r], 1e-15)
    # eps enters under the root: mean(x^2) = 1, eps = 3 -> scale 1/2.
    y = orc.rms_norm(np.ones((1, d)), np.ones(d), 3.0)
    _close(y[0], np.full(d, 0.5), 1e-15)


def pin_rope_closed_form(orc):
    """Position 0 is the identity; a unit vector in dim i turns by angle
    p * base^(-2i/d) into dim i + d/2."""
    cache = rope_cache(64, D)
    rng = np.random.default_rng(61)
    x = rng.standard_normal((1, 3, D))
    _close(orc.rope_rotate_half(x, [0], cache), x, 1e-15)
    for i, p in ((0, 5), (17, 63), (63, 1)):
        e = np.zeros((1, 1, D)); e[0, 0, i] = 1.0
        y = orc.rope_rotate_half(e, [p], cache)[0, 0]
        th = p * 10000.0 ** (-2.0 * i / D)
        exp = np.zeros(D); exp[i] = math.cos(th); exp[i + D // 2] = math.sin(th)
        _close(y, exp, 1e-6)   # the cache holds float32 cos/sin


def pin_rope_relative_position(orc):
    """Rotated dot products depend only on the position difference, and the
    rotation keeps each vector's norm."""
    cache = rope_cache(256, D, dtype=np.float64)
    rng = np.random.default_rng(67)
    q = rng.standard_normal((1, 1, D))
    k = rng.standard_normal((1, 1, D))
    ref = None
    for shift in (0, 7, 100):
        a = orc.rope_rotate_half(q, [40 + shift], cache)
        b = orc.rope_rotate_half(k, [13 + shift], cache)
        dot = float((a * b).sum())
        ref = dot if ref is None else ref
        assert abs(dot - ref) < 1e-9 * (1 + abs(ref)), (dot, ref)
        assert abs(np.linalg.norm(a) - np.linalg.norm(q)) < 1e-9


def pin_fused_store(orc):
    """The fused step returns normed, rotated q; writes rotated k and the
    untouched v (bit copy) at out_loc; other slots keep their bits."""
    rng = np.random.default_rng(71)
    Hq, Hkv, N, S = 4, 2, 3, 16
    qkv = _bits(_bf16_round(rng.standard_normal((N, (Hq + 2 * Hkv) * D))))
    pos = np.array([0, 9, 31])
    cache = rope_cache(32, D)
    wq = _bf16_round(rng.uniform(0.5, 1.5, D))
    wk = _bf16_round(rng.uniform(0.5, 1.5, D))
    kp = {0: rng.integers(0, 1 << 16, (S, Hkv, D), dtype=np.uint16)}
    vp = {0: rng.integers(0, 1 << 16, (S, Hkv, D), dtype=np.uint16)}
    k0, v0 = kp[0].copy(), vp[0].copy()
    loc = np.array([4, 11, 0])
    q = orc.qk_norm_rope_store(qkv, Hq, Hkv, D, pos, cache, _bits(wq), _bits(wk), 1e-6, kp, vp, 0, loc)
    x = orc.to_f64(qkv)
    # position 0 leaves the normed q unrotated
    q0 = x[0, :Hq * D].reshape(Hq, D)
    _close(q[0], q0 / np.sqrt((q0 ** 2).mean(axis=1, keepdims=True) + 1e-6) * wq, 1e-12)
    v_in = qkv[:, (Hq + Hkv) * D:].reshape(N, Hkv, D)
    for i, sl in enumerate(loc):
        assert np.array_equal(vp[0][sl], v_in[i])
    k_first = x[0, Hq * D:(Hq + Hkv) * D].reshape(Hkv, D)
    kn = k_first / np.sqrt((k_first ** 2).mean(axis=1, keepdims=True) + 1e-6) * wk
    assert np.array_equal(kp[0][4], _bits(_bf16_round(kn)))
    rest = np.setdiff1d(np.arange(S), loc)
    assert np.array_equal(kp[0][rest], k0[rest]) and np.array_equal(vp[0][rest], v0[rest])


ALL_PINS += [pin_bf16_rounding, pin_rms_norm_closed_form, pin_rope_closed_form,
             pin_rope_relative_position, pin_fused_store]


# ---------------------------------------------------------------------------
# FP8 (E4M3) pool pins.
# ---------------------------------------------------------------------------
# Hand-derived codes: value -> code (sign | exponent field << 3 | mantissa),
# exponent bias 7, subnormal quantum 2^-9, largest finite 448 = 0x7E.
E4M3_CASES = [
    (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (500.0, 0x7E), (-1000.0, 0xFE),
    (464.0, 0x7E),                 # halfway 448 / 480: ties to even, 448
    (240.0, 0x77),                 # 1.875 * 2^7
    (2.0 ** -6, 0x08),             # smallest normal
    (2.0 ** -9, 0x01),             # smallest subnormal
    (2.0 ** -10, 0x00),            # halfway 0 / 2^-9: ties to even, 0
    (3 * 2.0 ** -10, 0x02),        # halfway 2^-9 / 2^-8: ties to even, 2^-8
    (1.4 * 2.0 ** -9, 0x01), (1.6 * 2.0 ** -9, 0x02),
    (1.0625, 0x38),                # halfway 1 / 1.125: even mantissa 0
    (1.1875, 0x3A),                # halfway 1.125 / 1.25: even mantissa 2
    (1.9375, 0x40),                # rounds up into the next binade: 2.0
    (0.0, 0x00), (-0.0, 0x80), (-3.5, 0xC6),
]


def pin_e4m3_codes(orc):
    got = orc.e4m3_encode(np.array([v for v, _ in E4M3_CASES]))
    want = [c for _, c in E4M3_CASES]
    assert [int(x) for x in got] == want, [(v, hex(int(g))) for (v, _), g in zip(E4M3_CASES, got)]


def pin_e4m3_decode_table(orc):
    """All 256 codes: the value of each, built here from the format's fields,
    and encode(decode(c)) == c for every finite code."""
    codes = np.arange(256, dtype=np.uint8)
    dec = orc.e4m3_decode(codes)
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            assert math.isnan(dec[c])
            continue
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        assert dec[c] == (-v if s else v), (c, dec[c], v)
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(orc.e4m3_encode(orc.e4m3_decode(finite)), finite)


def pin_fp8_quantize_scale(orc):
    """The stored code is that of x * (1/s) in float32: with s = 2, 2.125 ->
    1.0625 -> 1.0 (tie to even), 3.0 -> 1.5, -896 -> -448 (saturated)."""
    got = orc.quantize(np.array([2.125, 3.0, -896.0], dtype=np.float32), 2.0)
    assert [int(x) for x in got] == [0x38, 0x3C, 0xFE]
    bf = _bits(np.array([2.125, 3.0]))
    assert [int(x) for x in orc.quantize(bf, 2.0)] == [0x38, 0x3C]


def pin_fp8_one_token_returns_dequantised_v(orc):
    """Store through the FP8 pool, then a one-token decode returns the token's
    dequantised V: code(v / s) * s, here exactly v for values that are E4M3
    numbers times s."""
    rng = np.random.default_rng(53)
    Hkv, Hq, S = 2, 4, 16
    ks, vs = 0.75, 1.5
    grid = np.array([(1 + m / 8.0) * 2.0 ** e for e in range(-3, 3) for m in range(8)])
    v_vals = rng.choice(grid, size=(1, Hkv * D)) * rng.choice([-1.0, 1.0], size=(1, Hkv * D)) * vs
    k_vals = rng.standard_normal((1, Hkv * D)).astype(np.float32)
    kp = {0: np.zeros((S, Hkv, D), dtype=np.uint8)}
    vp = {0: np.zeros((S, Hkv, D), dtype=np.uint8)}
    orc.store_kv_fp8(kp, vp, 0, k_vals, v_vals.astype(np.float32), [5], Hkv, D, ks, vs)
    assert np.count_nonzero(vp[0][np.arange(S) != 5]) == 0
    table = np.array([[5]], dtype=np.int32)
    q = _bits(rng.standard_normal((1, Hq, D)))
    out = orc.decode_attn(q, orc.dequant_planes(kp, ks), orc.dequant_planes(vp, vs), 0, table,
                          [0], [1], 1, 0.1)
    for h in range(Hq):
        assert np.array_equal(out[0, h], v_vals[0].reshape(Hkv, D)[h // 2])


def pin_fp8_quantize_inverse_in_float32(orc):
    """The inverse scale is a float32 quotient, worked by hand for s = 7 and
    x = 91/1024 (bf16 0x3DB6):

    * 2^26 / 7 = 9586980.57..., so RN32(1/7) = 9586981 * 2^-26, and
      7 * 9586981 = 2^26 + 3: RN32(1/7) = (1 + 3 * 2^-26) / 7.
    * x * RN32(1/7) = 13 * 2^-10 + 39 * 2^-36.  On [2^-7, 2^-6) a float32 step
      is 2^-30 and 39 * 2^-36 is 0.61 of it, so the float32 product is
      t = 13 * 2^-10 + 2^-30.
    * E4M3's subnormal quantum is 2^-9: 13 * 2^-10 is 6.5 quanta, a tie, and t
      lies above it, so t rounds to 7 quanta: code 0x07 (0x87 for -x).  With
      the exact 1/7 the product would be the tie itself, which goes to the even
      code 0x06."""
    x = np.array([0x3DB6, 0xBDB6], dtype=np.uint16)
    assert float(orc.to_f64(x[:1])[0]) == 91 / 1024
    assert [int(c) for c in orc.quantize(x, 7.0)] == [0x07, 0x87]
    assert [int(c) for c in orc.quantize(np.array([91 / 1024], dtype=np.float32), 7.0)] == [0x07]


ALL_PINS += [pin_e4m3_codes, pin_e4m3_decode_table, pin_fp8_quantize_scale,
             pin_fp8_one_token_returns_dequantised_v, pin_fp8_quantize_inverse_in_float32]
