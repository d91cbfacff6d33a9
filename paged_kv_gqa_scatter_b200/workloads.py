"""Seeded synthetic inputs for the paged KV pool path.

This module only draws inputs: pool contents, page tables, sequence lengths,
queries, the new K/V rows of a step and the slots they go to.  It holds none
of the attention, gather or scatter arithmetic, so both the CUDA library and
the CPU oracle can be fed from it without sharing any of the method.

Workload shapes follow the serving engine described on the pages
"Mini-SGLang 完整剖析" (blog.rzhang-lab.cn/post/3, §1.3 KV cache sizing, §1.4
paged pool, §4.4.3 pool tensor, §4.6.4 token-granular page table) and
"深入解析 mini-sglang" (yunpan.plus, chunked prefill).  Every generator uses
numpy's PCG64 seeded with 1000 + the workload number.

Storage conventions shared by every workload:

* A pool plane (K or V) is ``[num_layers][num_slots][num_kv_heads][head_dim]``.
  On the host a plane is a dict ``layer -> array[num_slots][Hkv][d]`` that
  holds only the layers a workload touches; bf16 values are kept as their
  uint16 bit patterns, fp32 values as float32.
* ``page_table`` is int32 ``[rows][cols]`` in token granularity: entry
  ``[row][j]`` is the pool slot of token ``j``.  With ``page_size > 1`` the
  entries of one page are consecutive slots starting at a multiple of
  ``page_size``.
* Decode ``seq_lens`` count the token stored by this step's ``store_kv``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

HEAD_DIM = 128
BF16 = "bf16"
F32 = "f32"
F8 = "fp8"  # scaled E4M3 pool: uint8 codes on the host; q / k / v rows stay bf16


def seed_for(workload_number: int) -> int:
    return 1000 + int(workload_number)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); return the bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def draw_values(rng: np.random.Generator, shape, dtype: str, scale: float = 1.0) -> np.ndarray:
    """iid N(0, 1) values times ``scale``: float32 draws, rounded to bf16 for bf16."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    if dtype == BF16:
        return f32_to_bf16_bits(x)
    if dtype == F32:
        return x
    raise ValueError(f"unknown dtype {dtype}")


def storage_dtype(dtype: str):
    return {BF16: np.uint16, F32: np.float32, F8: np.uint8}[dtype]


def draw_e4m3_codes(rng: np.random.Generator, shape, min_exp: int = 4, max_exp: int = 9) -> np.ndarray:
    """Random E4M3 codes: sign and mantissa uniform, exponent field uniform in
    [min_exp, max_exp] (values of magnitude 2^(min_exp-7) .. < 2^(max_exp-6));
    never a NaN code.  Drawn directly as codes, so no rounding is involved."""
    sign = rng.integers(0, 2, size=shape, dtype=np.uint8) << np.uint8(7)
    ex = rng.integers(min_exp, max_exp, size=shape, dtype=np.uint8, endpoint=True) << np.uint8(3)
    man = rng.integers(0, 8, size=shape, dtype=np.uint8)
    return sign | ex | man


class TiledPlane:
    """A pool plane too large for host memory, filled by repeating one block.

    Flat slot ``i = layer * num_slots + slot`` holds ``block[i % len(block)]``.
    Writes (a step's stored tokens) are kept as per-slot overrides.  Indexing
    ``plane[layer]`` returns a view object that supports ``view[slots]`` and
    ``view[slots] = rows`` with slot arrays, like a numpy layer array.
    """

    def __init__(self, block: np.ndarray, num_layers: int, num_slots: int):
        self.block = block
        self.num_layers = int(num_layers)
        self.num_slots = int(num_slots)
        self.overrides: Dict[int, Dict[int, np.ndarray]] = {}

    def __getitem__(self, layer: int) -> "_TiledLayer":
        return _TiledLayer(self, int(layer))

    def __contains__(self, layer) -> bool:
        return 0 <= int(layer) < self.num_layers


class _TiledLayer:
    def __init__(self, plane: TiledPlane, layer: int):
        self.plane = plane
        self.layer = layer

    @property
    def dtype(self):
        return self.plane.block.dtype

    def __getitem__(self, slots):
        slots = np.asarray(slots, dtype=np.int64)
        nb = self.plane.block.shape[0]
        rows = self.plane.block[(self.layer * self.plane.num_slots + slots) % nb].copy()
        ov = self.plane.overrides.get(self.layer)
        if ov:
            flat = slots.reshape(-1)
            out = rows.reshape((-1,) + self.plane.block.shape[1:])
            for i, s in enumerate(flat):
                r = ov.get(int(s))
                if r is not None:
                    out[i] = r
            rows = out.reshape(rows.shape)
        return rows

    def __setitem__(self, slots, rows):
        slots = np.asarray(slots, dtype=np.int64).reshape(-1)
        rows = np.asarray(rows).reshape((slots.shape[0],) + self.plane.block.shape[1:])
        ov = self.plane.overrides.setdefault(self.layer, {})
        for s, r in zip(slots, rows):
            ov[int(s)] = r.copy()


@dataclasses.dataclass
class PoolSpec:
    num_layers: int
    num_slots: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    dtype: str
    k_scale: float = 1.0  # F8 pools: dequantisation scales
    v_scale: float = 1.0

    @property
    def io_dtype(self) -> str:
        """Element type of q, out and the rows written into the pool."""
        return BF16 if self.dtype == F8 else self.dtype

    @property
    def row_elems(self) -> int:
        return self.num_kv_heads * self.head_dim


@dataclasses.dataclass
class DecodeWorkload:
    """One decode step: store one new token per request, then attend."""
    name: str
    pool: PoolSpec
    num_q_heads: int
    layer: int
    k_planes: object          # dict layer -> [S][Hkv][d]  or TiledPlane
    v_planes: object
    page_table: np.ndarray    # int32 [rows][cols]
    table_idx: np.ndarray     # int32 [B]
    seq_lens: np.ndarray      # int32 [B], includes the new token
    q: np.ndarray             # [B][Hq][d]
    k_new: np.ndarray         # [B][Hkv*d]
    v_new: np.ndarray         # [B][Hkv*d]
    out_loc: np.ndarray       # int32 [B]
    scale: float

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    def kv_tokens(self) -> int:
        return int(self.seq_lens.astype(np.int64).sum())


@dataclasses.dataclass
class ExtendWorkload:
    """One extend (prefill chunk) call: store the chunk, then attend causally."""
    name: str
    pool: PoolSpec
    num_q_heads: int
    layer: int
    k_planes: object
    v_planes: object
    page_table: np.ndarray
    table_idx: np.ndarray     # int32 [B]
    prefix_lens: np.ndarray   # int32 [B]
    extend_lens: np.ndarray   # int32 [B]
    q_offsets: np.ndarray     # int32 [B+1], exclusive cumsum of extend_lens
    q: np.ndarray             # [total_q][Hq][d]
    k_new: np.ndarray         # [total_q][Hkv*d]
    v_new: np.ndarray
    out_loc: np.ndarray       # int32 [total_q]
    scale: float

    @property
    def batch(self) -> int:
        return int(self.extend_lens.shape[0])

    @property
    def total_q(self) -> int:
        return int(self.q_offsets[-1])

    def causal_pairs(self) -> int:
        """Unmasked (query, key) pairs per query head."""
        p = self.prefix_lens.astype(np.int64)
        e = self.extend_lens.astype(np.int64)
        return int((e * p + e * (e + 1) // 2).sum())


def _new_plane_dict(spec: PoolSpec, layers) -> Dict[int, np.ndarray]:
    st = storage_dtype(spec.dtype)
    return {int(l): np.zeros((spec.num_slots, spec.num_kv_heads, spec.head_dim), dtype=st)
            for l in layers}


def _fill_slots(rng, plane: np.ndarray, slots: np.ndarray, dtype: str, scale: float = 1.0):
    vals = draw_values(rng, (slots.shape[0],) + plane.shape[1:], dtype, scale)
    plane[slots] = vals


def _token_table(rows: int, cols: int, fill: int = 0) -> np.ndarray:
    return np.full((rows, cols), fill, dtype=np.int32)


# ---------------------------------------------------------------------------
# Workload 1: small single-layer decode, the oracle-sized case.
# ---------------------------------------------------------------------------
def decode_small(dtype: str = BF16, seq_lens=(17, 33, 50, 64), num_q_heads: int = 16,
                 num_kv_heads: int = 8, num_slots: int = 512, seed: Optional[int] = None,
                 k_scale: float = 1.0) -> DecodeWorkload:
    """4 requests with contexts {17, 33, 50, 64} (new token included), Hq 16, Hkv 8,
    a 512-slot single-layer pool; one seeded slot permutation handed out to the
    requests in order; ``out_loc`` is each request's last slot."""
    rng = np.random.Generator(np.random.PCG64(seed_for(1) if seed is None else seed))
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B = seq_lens.shape[0]
    total = int(seq_lens.sum())
    if total > num_slots:
        raise ValueError("pool too small for the requested contexts")
    spec = PoolSpec(1, num_slots, num_kv_heads, HEAD_DIM, 1, dtype)
    perm = rng.permutation(num_slots).astype(np.int32)
    cols = int(seq_lens.max())
    table = _token_table(B + 1, cols)
    table_idx = rng.permutation(B).astype(np.int32)
    pos = 0
    for r in range(B):
        n = int(seq_lens[r])
        table[table_idx[r], :n] = perm[pos:pos + n]
        pos += n
    kp = _new_plane_dict(spec, [0])
    vp = _new_plane_dict(spec, [0])
    all_slots = np.arange(num_slots)
    _fill_slots(rng, kp[0], all_slots, dtype, k_scale)
    _fill_slots(rng, vp[0], all_slots, dtype)
    q = draw_values(rng, (B, num_q_heads, HEAD_DIM), dtype)
    k_new = draw_values(rng, (B, spec.row_elems), dtype, k_scale)
    v_new = draw_values(rng, (B, spec.row_elems), dtype)
    out_loc = np.array([table[table_idx[r], seq_lens[r] - 1] for r in range(B)], dtype=np.int32)
    return DecodeWorkload("decode-small", spec, num_q_heads, 0, kp, vp, table, table_idx,
                          seq_lens, q, k_new, v_new, out_loc, 1.0 / math.sqrt(HEAD_DIM))


# ---------------------------------------------------------------------------
# Workload 2: Qwen3-0.6B-shaped decode step (the headline benchmark case).
# ---------------------------------------------------------------------------
def decode_qwen3_06b(dtype: str = BF16, batch: int = 64, min_len: int = 512, max_len: int = 4096,
                     num_slots: int = 300_000, num_layers: int = 28, layer: int = 13,
                     num_q_heads: int = 16, num_kv_heads: int = 8,
                     seed: Optional[int] = None) -> DecodeWorkload:
    """64 requests, contexts uniform in [512, 4096]; Hq 16, Hkv 8; K scaled by 0.5;
    page_size 1; slots drawn without replacement from a 300k-slot, 28-layer pool;
    layer 13 is the one attended.  Only the referenced slots get values."""
    rng = np.random.Generator(np.random.PCG64(seed_for(2) if seed is None else seed))
    seq_lens = rng.integers(min_len, max_len, size=batch, endpoint=True).astype(np.int32)
    total = int(seq_lens.astype(np.int64).sum())
    if total > num_slots:
        raise ValueError("pool too small")
    spec = PoolSpec(num_layers, num_slots, num_kv_heads, HEAD_DIM, 1, dtype)
    slots = rng.choice(num_slots, size=total, replace=False).astype(np.int32)
    cols = int(max_len)
    table = _token_table(batch + 1, cols)
    table_idx = rng.permutation(batch).astype(np.int32)
    pos = 0
    for r in range(batch):
        n = int(seq_lens[r])
        table[table_idx[r], :n] = slots[pos:pos + n]
        pos += n
    kp = _new_plane_dict(spec, [layer])
    vp = _new_plane_dict(spec, [layer])
    _fill_slots(rng, kp[layer], slots, dtype, 0.5)
    _fill_slots(rng, vp[layer], slots, dtype)
    q = draw_values(rng, (batch, num_q_heads, HEAD_DIM), dtype)
    k_new = draw_values(rng, (batch, spec.row_elems), dtype, 0.5)
    v_new = draw_values(rng, (batch, spec.row_elems), dtype)
    out_loc = np.array([table[table_idx[r], seq_lens[r] - 1] for r in range(batch)], dtype=np.int32)
    return DecodeWorkload("decode-qwen3-0.6b", spec, num_q_heads, layer, kp, vp, table, table_idx,
                          seq_lens, q, k_new, v_new, out_loc, 1.0 / math.sqrt(HEAD_DIM))


# ---------------------------------------------------------------------------
# Workload 3: Qwen3-8B-shaped large decode batch over a 36-layer pool.
# ---------------------------------------------------------------------------
# Physical 16-token pages of the Qwen3-8B decode pool: 36 layers x 45,056
# pages x 16 slots x 4 KB = 106 GB, about 0.55 of a B200's memory.  Fixed (not
# sized from free memory) so that every run builds the same page aliasing.
QWEN3_8B_POOL_PAGES = 45_056


def decode_qwen3_8b(num_pages: int = QWEN3_8B_POOL_PAGES, dtype: str = BF16, batch: int = 256, min_len: int = 1024,
                    max_len: int = 32768, num_layers: int = 36, page_size: int = 16,
                    num_q_heads: int = 32, num_kv_heads: int = 8, block_slots: int = 1 << 16,
                    seed: Optional[int] = None) -> DecodeWorkload:
    """256 requests, contexts log-uniform in [1k, 32k]; Hq 32, Hkv 8; page_size 16.

    The stated workload (about 2.35M context tokens x 36 layers x 4 KB) is larger
    than one GPU's memory, so the pool holds ``num_pages`` physical pages: every
    request's last page is private (it receives the step's new token), and the
    other logical pages map onto the remaining physical pages through one seeded
    permutation taken cyclically, so some history pages are shared between
    requests.  Pool contents repeat a seeded block of ``block_slots`` slots
    (see ``TiledPlane``).  ``layer`` is 0; callers loop over all layers.
    """
    rng = np.random.Generator(np.random.PCG64(seed_for(3) if seed is None else seed))
    lo, hi = math.log(min_len), math.log(max_len)
    seq_lens = np.floor(np.exp(rng.uniform(lo, hi, size=batch))).astype(np.int64)
    seq_lens = np.clip(seq_lens, min_len, max_len).astype(np.int32)
    P = page_size
    pages_per_req = (seq_lens.astype(np.int64) + P - 1) // P
    hist_pages = num_pages - batch
    if hist_pages < 1:
        raise ValueError("num_pages must exceed the batch size")
    perm = rng.permutation(hist_pages).astype(np.int64)
    cols = int(((max_len + P - 1) // P) * P)
    table = _token_table(batch + 1, cols)
    table_idx = rng.permutation(batch).astype(np.int32)
    k = 0
    offs = np.arange(P, dtype=np.int64)
    for r in range(batch):
        npg = int(pages_per_req[r])
        phys = np.empty(npg, dtype=np.int64)
        phys[:npg - 1] = perm[(k + np.arange(npg - 1)) % hist_pages]
        k += npg - 1
        phys[npg - 1] = hist_pages + r
        ent = (phys[:, None] * P + offs[None, :]).reshape(-1)
        table[table_idx[r], :npg * P] = ent.astype(np.int32)
    num_slots = num_pages * P
    spec = PoolSpec(num_layers, num_slots, num_kv_heads, HEAD_DIM, P, dtype)
    kb = draw_values(rng, (block_slots, num_kv_heads, HEAD_DIM), dtype)
    vb = draw_values(rng, (block_slots, num_kv_heads, HEAD_DIM), dtype)
    kp = TiledPlane(kb, num_layers, num_slots)
    vp = TiledPlane(vb, num_layers, num_slots)
    q = draw_values(rng, (batch, num_q_heads, HEAD_DIM), dtype)
    k_new = draw_values(rng, (batch, spec.row_elems), dtype)
    v_new = draw_values(rng, (batch, spec.row_elems), dtype)
    out_loc = np.array([table[table_idx[r], seq_lens[r] - 1] for r in range(batch)], dtype=np.int32)
    wl = DecodeWorkload("decode-qwen3-8b", spec, num_q_heads, 0, kp, vp, table, table_idx,
                        seq_lens, q, k_new, v_new, out_loc, 1.0 / math.sqrt(HEAD_DIM))
    wl.alias_factor = float((pages_per_req - 1).sum()) / float(hist_pages)
    return wl


# ---------------------------------------------------------------------------
# Workload 4: chunked prefill mixed step.
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class MixedStep:
    extend: ExtendWorkload
    decode: DecodeWorkload


def chunked_prefill_step(step: int = 3, dtype: str = BF16, num_prompts: int = 8,
                         prompt_len: int = 8192, chunk: int = 2048, decode_batch: int = 128,
                         decode_len: int = 2048, num_q_heads: int = 32, num_kv_heads: int = 8,
                         seed: Optional[int] = None) -> MixedStep:
    """8 prompts of 8192 tokens prefilled in 2048-token chunks, one chunk per
    step (step s runs prompt s // 4, chunk s % 4, so its prefix is 2048 * (s % 4)),
    plus 128 running decode requests at context 2048 (new token included).
    Both calls share one single-layer pool and one page table; all slots come
    from one seeded permutation.  The pool holds every prompt's tokens before
    this chunk and every decode request's history; the chunk's own rows and the
    decode requests' new rows arrive through ``store_kv``."""
    rng = np.random.Generator(np.random.PCG64(seed_for(4) if seed is None else seed))
    chunks_per_prompt = prompt_len // chunk
    pr, c = divmod(int(step), chunks_per_prompt)
    if pr >= num_prompts:
        raise ValueError("step out of range")
    num_slots = num_prompts * prompt_len + decode_batch * decode_len
    spec = PoolSpec(1, num_slots, num_kv_heads, HEAD_DIM, 1, dtype)
    perm = rng.permutation(num_slots).astype(np.int32)
    rows = num_prompts + decode_batch + 1
    cols = max(prompt_len, decode_len)
    table = _token_table(rows, cols)
    row_of = rng.permutation(num_prompts + decode_batch).astype(np.int32)
    pos = 0
    for i in range(num_prompts):
        table[row_of[i], :prompt_len] = perm[pos:pos + prompt_len]
        pos += prompt_len
    for i in range(decode_batch):
        table[row_of[num_prompts + i], :decode_len] = perm[pos:pos + decode_len]
        pos += decode_len
    kp = _new_plane_dict(spec, [0])
    vp = _new_plane_dict(spec, [0])
    # Full sequences of every prompt; the current chunk's rows are held back.
    prompt_k = draw_values(rng, (num_prompts, prompt_len, spec.row_elems), dtype)
    prompt_v = draw_values(rng, (num_prompts, prompt_len, spec.row_elems), dtype)
    p0 = c * chunk
    for i in range(num_prompts):
        sl = table[row_of[i], :prompt_len]
        keep = np.ones(prompt_len, dtype=bool)
        if i == pr:
            keep[p0:] = False  # this chunk and later ones are not in the pool yet
        kp[0][sl[keep]] = prompt_k[i][keep].reshape(-1, num_kv_heads, HEAD_DIM)
        vp[0][sl[keep]] = prompt_v[i][keep].reshape(-1, num_kv_heads, HEAD_DIM)
    dec_rows = row_of[num_prompts:]
    hist = table[dec_rows, :decode_len - 1].reshape(-1)
    _fill_slots(rng, kp[0], hist, dtype)
    _fill_slots(rng, vp[0], hist, dtype)
    scale = 1.0 / math.sqrt(HEAD_DIM)
    # Extend call: one request (the chunk).
    e_q = draw_values(rng, (chunk, num_q_heads, HEAD_DIM), dtype)
    ext = ExtendWorkload(
        f"chunked-prefill-extend-c{c}", spec, num_q_heads, 0, kp, vp, table,
        np.array([row_of[pr]], dtype=np.int32), np.array([p0], dtype=np.int32),
        np.array([chunk], dtype=np.int32), np.array([0, chunk], dtype=np.int32), e_q,
        np.ascontiguousarray(prompt_k[pr, p0:p0 + chunk]),
        np.ascontiguousarray(prompt_v[pr, p0:p0 + chunk]),
        table[row_of[pr], p0:p0 + chunk].astype(np.int32).copy(), scale)
    d_q = draw_values(rng, (decode_batch, num_q_heads, HEAD_DIM), dtype)
    d_k = draw_values(rng, (decode_batch, spec.row_elems), dtype)
    d_v = draw_values(rng, (decode_batch, spec.row_elems), dtype)
    seq = np.full(decode_batch, decode_len, dtype=np.int32)
    dec = DecodeWorkload("chunked-prefill-decode", spec, num_q_heads, 0, kp, vp, table,
                         dec_rows.astype(np.int32).copy(), seq, d_q, d_k, d_v,
                         table[dec_rows, decode_len - 1].astype(np.int32).copy(), scale)
    return MixedStep(ext, dec)


# ---------------------------------------------------------------------------
# Workload 5: radix shared-prefix serving.
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class RadixServe:
    """Shared 4096-token prefix, per-request suffix extend, then decode steps.

    ``extend`` covers all requests' suffixes in one call (layer 0 inputs; the
    same per-layer inputs are reused on every layer).  ``decode_step(t)`` builds
    decode step t (1-based) after the extend and t - 1 earlier decode steps.
    """
    extend: ExtendWorkload
    decode_q: np.ndarray      # [steps][B][Hq][d]
    decode_k: np.ndarray      # [steps][B][Hkv*d]
    decode_v: np.ndarray
    decode_steps: int

    def decode_step(self, t: int) -> DecodeWorkload:
        e = self.extend
        B = e.batch
        seq = (e.prefix_lens + e.extend_lens + t).astype(np.int32)
        out_loc = np.array([e.page_table[e.table_idx[r], seq[r] - 1] for r in range(B)],
                           dtype=np.int32)
        return DecodeWorkload(f"radix-decode-t{t}", e.pool, e.num_q_heads, e.layer, e.k_planes,
                              e.v_planes, e.page_table, e.table_idx, seq,
                              self.decode_q[t - 1], self.decode_k[t - 1], self.decode_v[t - 1],
                              out_loc, e.scale)


def radix_shared_prefix(dtype: str = BF16, batch: int = 256, prefix_len: int = 4096,
                        min_suffix: int = 64, max_suffix: int = 512, decode_steps: int = 64,
                        num_layers: int = 32, num_q_heads: int = 32, num_kv_heads: int = 8,
                        seed: Optional[int] = None, layer: int = 0) -> RadixServe:
    """256 requests share one 4096-token prefix on the same physical slots; each
    has a unique suffix of U{64..512} tokens, extended in one call, then 64
    decode steps.  32-layer pool, Hkv 8 (128 KB of KV per token), Hq 32."""
    rng = np.random.Generator(np.random.PCG64(seed_for(5) if seed is None else seed))
    suffix = rng.integers(min_suffix, max_suffix, size=batch, endpoint=True).astype(np.int32)
    per_req = suffix.astype(np.int64) + decode_steps
    num_slots = int(prefix_len + per_req.sum())
    spec = PoolSpec(num_layers, num_slots, num_kv_heads, HEAD_DIM, 1, dtype)
    perm = rng.permutation(num_slots).astype(np.int32)
    prefix_slots = perm[:prefix_len]
    cols = int(prefix_len + max_suffix + decode_steps)
    table = _token_table(batch + 1, cols)
    table_idx = rng.permutation(batch).astype(np.int32)
    pos = prefix_len
    for r in range(batch):
        row = table_idx[r]
        table[row, :prefix_len] = prefix_slots
        m = int(per_req[r])
        table[row, prefix_len:prefix_len + m] = perm[pos:pos + m]
        pos += m
    kp = _new_plane_dict(spec, [layer])
    vp = _new_plane_dict(spec, [layer])
    _fill_slots(rng, kp[layer], prefix_slots, dtype)
    _fill_slots(rng, vp[layer], prefix_slots, dtype)
    total_q = int(suffix.sum())
    q_off = np.zeros(batch + 1, dtype=np.int32)
    q_off[1:] = np.cumsum(suffix)
    q = draw_values(rng, (total_q, num_q_heads, HEAD_DIM), dtype)
    k_new = draw_values(rng, (total_q, spec.row_elems), dtype)
    v_new = draw_values(rng, (total_q, spec.row_elems), dtype)
    out_loc = np.concatenate([table[table_idx[r], prefix_len:prefix_len + suffix[r]]
                              for r in range(batch)]).astype(np.int32)
    ext = ExtendWorkload("radix-extend", spec, num_q_heads, layer, kp, vp, table, table_idx,
                         np.full(batch, prefix_len, dtype=np.int32), suffix, q_off, q, k_new,
                         v_new, out_loc, 1.0 / math.sqrt(HEAD_DIM))
    dq = draw_values(rng, (decode_steps, batch, num_q_heads, HEAD_DIM), dtype)
    dk = draw_values(rng, (decode_steps, batch, spec.row_elems), dtype)
    dv = draw_values(rng, (decode_steps, batch, spec.row_elems), dtype)
    return RadixServe(ext, dq, dk, dv, decode_steps)


# ---------------------------------------------------------------------------
# Small extend cases for parity tests.
# ---------------------------------------------------------------------------
def extend_small(dtype: str = BF16, prefix_lens=(0, 37, 130), extend_lens=(45, 1, 200),
                 num_q_heads: int = 16, num_kv_heads: int = 8, num_slots: int = 1024,
                 page_size: int = 1, seed: int = 1100, stored_prefix: bool = True) -> ExtendWorkload:
    """A ragged extend batch sized for the oracle: prefixes already in the pool,
    the chunks' own rows stored by ``store_kv``."""
    rng = np.random.Generator(np.random.PCG64(seed))
    p = np.asarray(prefix_lens, dtype=np.int32)
    e = np.asarray(extend_lens, dtype=np.int32)
    B = p.shape[0]
    n = p.astype(np.int64) + e
    P = page_size
    pages = (n + P - 1) // P
    num_pages = num_slots // P
    if pages.sum() > num_pages:
        raise ValueError("pool too small")
    perm = rng.permutation(num_pages).astype(np.int64)
    cols = int(max(1, ((n.max() + P - 1) // P) * P))
    table = _token_table(B + 1, cols)
    table_idx = rng.permutation(B).astype(np.int32)
    k = 0
    for r in range(B):
        phys = perm[k:k + pages[r]]
        k += int(pages[r])
        ent = (phys[:, None] * P + np.arange(P)[None, :]).reshape(-1)
        table[table_idx[r], :pages[r] * P] = ent.astype(np.int32)
    spec = PoolSpec(1, num_slots, num_kv_heads, HEAD_DIM, P, dtype)
    kp = _new_plane_dict(spec, [0])
    vp = _new_plane_dict(spec, [0])
    _fill_slots(rng, kp[0], np.arange(num_slots), dtype)
    _fill_slots(rng, vp[0], np.arange(num_slots), dtype)
    total_q = int(e.sum())
    q_off = np.zeros(B + 1, dtype=np.int32)
    q_off[1:] = np.cumsum(e)
    q = draw_values(rng, (total_q, num_q_heads, HEAD_DIM), dtype)
    k_new = draw_values(rng, (total_q, spec.row_elems), dtype)
    v_new = draw_values(rng, (total_q, spec.row_elems), dtype)
    out_loc = np.concatenate([table[table_idx[r], p[r]:p[r] + e[r]] for r in range(B)]
                             ).astype(np.int32) if total_q else np.zeros(0, np.int32)
    return ExtendWorkload("extend-small", spec, num_q_heads, 0, kp, vp, table, table_idx, p, e,
                          q_off, q, k_new, v_new, out_loc, 1.0 / math.sqrt(HEAD_DIM))


def decode_paged_small(dtype: str = BF16, seq_lens=(1, 16, 17, 300, 1029), page_size: int = 16,
                       num_q_heads: int = 32, num_kv_heads: int = 8, num_slots: int = 4096,
                       seed: int = 1101, k_scale: float = 1.0) -> DecodeWorkload:
    """Small decode batch with page_size > 1 (permuted pages), ragged lengths."""
    rng = np.random.Generator(np.random.PCG64(seed))
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B = seq_lens.shape[0]
    P = page_size
    pages = (seq_lens.astype(np.int64) + P - 1) // P
    num_pages = num_slots // P
    if pages.sum() > num_pages:
        raise ValueError("pool too small")
    perm = rng.permutation(num_pages).astype(np.int64)
    cols = int(((seq_lens.max() + P - 1) // P) * P)
    table = _token_table(B + 1, cols)
    table_idx = rng.permutation(B).astype(np.int32)
    k = 0
    for r in range(B):
        phys = perm[k:k + pages[r]]
        k += int(pages[r])
        ent = (phys[:, None] * P + np.arange(P)[None, :]).reshape(-1)
        table[table_idx[r], :pages[r] * P] = ent.astype(np.int32)
    spec = PoolSpec(1, num_slots, num_kv_heads, HEAD_DIM, P, dtype)
    kp = _new_plane_dict(spec, [0])
    vp = _new_plane_dict(spec, [0])
    _fill_slots(rng, kp[0], np.arange(num_slots), dtype, k_scale)
    _fill_slots(rng, vp[0], np.arange(num_slots), dtype)
    q = draw_values(rng, (B, num_q_heads, HEAD_DIM), dtype)
    k_new = draw_values(rng, (B, spec.row_elems), dtype, k_scale)
    v_new = draw_values(rng, (B, spec.row_elems), dtype)
    out_loc = np.array([table[table_idx[r], seq_lens[r] - 1] for r in range(B)], dtype=np.int32)
    return DecodeWorkload("decode-paged-small", spec, num_q_heads, 0, kp, vp, table, table_idx,
                          seq_lens, q, k_new, v_new, out_loc, 1.0 / math.sqrt(HEAD_DIM))


# ---------------------------------------------------------------------------
# The step ahead of attention: q/k norm + RoPE + store, on a fused qkv output.
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class RopeStoreWorkload:
    """One layer's qkv rows for N tokens, their positions and slots."""
    name: str
    pool: PoolSpec
    num_q_heads: int
    layer: int
    k_planes: Dict[int, np.ndarray]
    v_planes: Dict[int, np.ndarray]
    qkv: np.ndarray            # [N][(Hq + 2 Hkv) * d]
    positions: np.ndarray      # int32 [N]
    cos_sin_cache: np.ndarray  # float32 [max_position][d]: cos halves, then sin halves
    q_norm_w: Optional[np.ndarray]  # [d] or None
    k_norm_w: Optional[np.ndarray]
    eps: float
    out_loc: np.ndarray        # int32 [N]

    @property
    def n_tokens(self) -> int:
        return int(self.qkv.shape[0])


def rotary_table(max_position: int, head_dim: int = HEAD_DIM, base: float = 1e6) -> np.ndarray:
    """The RotaryEmbedding input table: row p holds cos(p * base^(-2i/d)) for
    i < d/2, then the sines of the same angles, as float32.  It is a model
    constant handed to both sides, like a weight."""
    half = head_dim // 2
    inv = base ** (-(2.0 * np.arange(half, dtype=np.float64)) / head_dim)
    ang = np.arange(max_position, dtype=np.float64)[:, None] * inv[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)


def rope_store_step(dtype: str = BF16, positions=None, num_q_heads: int = 16,
                    num_kv_heads: int = 8, num_slots: int = 4096, max_position: int = 8192,
                    norms: bool = True, seed: Optional[int] = None, x_scale: float = 2.0,
                    name: str = "rope-store") -> RopeStoreWorkload:
    """N tokens of a Qwen3-style layer: qkv rows N(0, x_scale^2), norm weights
    1 + N(0, 0.1^2) (learned scales near one), positions as given (default 45
    tokens spread over [0, max_position)), distinct random slots of a
    single-layer pool whose other slots hold random rows."""
    rng = np.random.Generator(np.random.PCG64(seed_for(6) if seed is None else seed))
    if positions is None:
        positions = rng.integers(0, max_position, size=45)
    positions = np.asarray(positions, dtype=np.int32)
    n = positions.shape[0]
    spec = PoolSpec(1, num_slots, num_kv_heads, HEAD_DIM, 1, dtype)
    kp = _new_plane_dict(spec, [0])
    vp = _new_plane_dict(spec, [0])
    all_slots = np.arange(num_slots)
    _fill_slots(rng, kp[0], all_slots, dtype)
    _fill_slots(rng, vp[0], all_slots, dtype)
    row = (num_q_heads + 2 * num_kv_heads) * HEAD_DIM
    qkv = draw_values(rng, (n, row), dtype, x_scale)
    qw = kw = None
    if norms:
        w = 1.0 + 0.1 * rng.standard_normal(size=(2, HEAD_DIM)).astype(np.float32)
        qw = f32_to_bf16_bits(w[0]) if dtype == BF16 else w[0].copy()
        kw = f32_to_bf16_bits(w[1]) if dtype == BF16 else w[1].copy()
    out_loc = rng.choice(num_slots, size=n, replace=False).astype(np.int32)
    return RopeStoreWorkload(name, spec, num_q_heads, 0, kp, vp, qkv, positions,
                             rotary_table(max_position), qw, kw, 1e-6, out_loc)


# ---------------------------------------------------------------------------
# Decode batches whose requests share prefixes, in groups.
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class GroupedDecode:
    """A decode step plus its grouping: requests group_offsets[g] ..
    group_offsets[g+1] - 1 share their first group_prefix_lens[g] slots."""
    decode: DecodeWorkload
    group_offsets: np.ndarray      # int32 [groups + 1]
    group_prefix_lens: np.ndarray  # int32 [groups]


def grouped_decode(dtype: str = BF16, groups=((0, 3), (1, 1), (63, 2), (64, 5), (65, 1),
                                              (1000, 70), (2500, 4)),
                   min_suffix: int = 0, max_suffix: int = 300, num_q_heads: int = 16,
                   num_kv_heads: int = 8, page_size: int = 1, seed: Optional[int] = None,
                   name: str = "grouped-decode") -> GroupedDecode:
    """Groups given as (prefix_len, members).  Each group's prefix occupies its
    own slots (pages), shared by every member's table row; each member then has
    a private suffix of U{min..max} tokens plus the token this step stores
    (so a member's context is prefix + suffix + 1).  With page_size > 1 the
    prefix lengths are rounded up to whole pages."""
    rng = np.random.Generator(np.random.PCG64(seed_for(7) if seed is None else seed))
    P = page_size
    plens = [int(-(-p // P) * P) for p, _ in groups]
    members = [int(m) for _, m in groups]
    B = int(sum(members))
    suffix = rng.integers(min_suffix, max_suffix, size=B, endpoint=True).astype(np.int64) + 1
    pages_needed = sum(p // P for p in plens) + int(sum(-(-s // P) for s in suffix))
    num_pages = pages_needed + 8
    num_slots = num_pages * P
    page_perm = rng.permutation(num_pages).astype(np.int64)
    nxt = 0

    def take(n_tokens):
        nonlocal nxt
        k = -(-n_tokens // P)
        ph = page_perm[nxt:nxt + k]
        nxt += k
        return (ph[:, None] * P + np.arange(P)[None, :]).reshape(-1)[:n_tokens]

    seq = np.zeros(B, dtype=np.int32)
    cols = int(max(plens) + suffix.max())
    cols = -(-cols // P) * P
    table = _token_table(B + 1, cols)
    table_idx = rng.permutation(B).astype(np.int32)
    off = np.zeros(len(groups) + 1, dtype=np.int32)
    r = 0
    for gi, (p, m) in enumerate(zip(plens, members)):
        shared = take(p) if p else np.zeros(0, dtype=np.int64)
        for _ in range(m):
            row = table_idx[r]
            table[row, :p] = shared
            own = take(int(suffix[r]))
            table[row, p:p + own.shape[0]] = own
            seq[r] = p + own.shape[0]
            r += 1
        off[gi + 1] = r
    spec = PoolSpec(1, num_slots, num_kv_heads, HEAD_DIM, P, dtype)
    kp = _new_plane_dict(spec, [0])
    vp = _new_plane_dict(spec, [0])
    _fill_slots(rng, kp[0], np.arange(num_slots), dtype)
    _fill_slots(rng, vp[0], np.arange(num_slots), dtype)
    q = draw_values(rng, (B, num_q_heads, HEAD_DIM), dtype)
    k_new = draw_values(rng, (B, spec.row_elems), dtype)
    v_new = draw_values(rng, (B, spec.row_elems), dtype)
    out_loc = np.array([table[table_idx[i], seq[i] - 1] for i in range(B)], dtype=np.int32)
    dec = DecodeWorkload(name, spec, num_q_heads, 0, kp, vp, table, table_idx, seq, q, k_new,
                         v_new, out_loc, 1.0 / math.sqrt(HEAD_DIM))
    return GroupedDecode(dec, off, np.asarray(plens, dtype=np.int32))


# ---------------------------------------------------------------------------
# FP8 (scaled E4M3) pools.
# ---------------------------------------------------------------------------
def with_fp8_pool(wl, k_scale: float = 0.05, v_scale: float = 0.09, seed: Optional[int] = None):
    """The same decode step or extend call over an E4M3 pool: every slot of the
    touched layers holds random codes (see draw_e4m3_codes); q and the new K/V
    rows stay the bf16 values of ``wl``; the scales are not powers of two, so
    the stored codes of the new rows depend on float32 rounding of
    x * (1 / scale)."""
    rng = np.random.Generator(np.random.PCG64(seed_for(8) if seed is None else seed))
    if wl.pool.dtype != BF16:
        raise ValueError("needs a bf16 workload")
    spec = dataclasses.replace(wl.pool, dtype=F8, k_scale=float(np.float32(k_scale)),
                               v_scale=float(np.float32(v_scale)))
    if isinstance(wl.k_planes, TiledPlane):
        # Tiled pools (decode-qwen3-8b): a code block of the same size, tiled the same way.
        kp = TiledPlane(draw_e4m3_codes(rng, wl.k_planes.block.shape), spec.num_layers, spec.num_slots)
        vp = TiledPlane(draw_e4m3_codes(rng, wl.v_planes.block.shape), spec.num_layers, spec.num_slots)
    else:
        shape = (spec.num_slots, spec.num_kv_heads, spec.head_dim)
        kp = {l: draw_e4m3_codes(rng, shape) for l in wl.k_planes}
        vp = {l: draw_e4m3_codes(rng, shape) for l in wl.v_planes}
    return dataclasses.replace(wl, name=wl.name + "-fp8", pool=spec, k_planes=kp, v_planes=vp)
