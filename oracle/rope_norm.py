"""Float64 oracle for the step ahead of attention: q/k RMSNorm, RoPE, store_kv.

TEST INFRASTRUCTURE ONLY (see the package header): used by tests and the CPU
baseline, never by the library.

What the pages state ("Mini-SGLang 完整剖析", blog.rzhang-lab.cn/post/3):
  * §4.6.7 -- the attention layer splits the fused qkv output into q, k, v;
    models with q/k norms (Qwen3) normalise q and k per head in place; RoPE is
    applied in place to q and k at the batch's positions; then the backend
    stores k and v into the pool at out_loc and runs attention.
  * §4.5.6 -- one RotaryEmbedding(head_dim, rotary_dim, max_position, base,
    scaling) is shared by all layers and holds a cos_sin_cache of shape
    (max_position, rotary_dim).
Readings where they are silent (also listed in the design notes):
  * RMSNorm: y = x / sqrt(mean(x^2) + eps) * w over head_dim, w per dim.
  * RoPE: rotate-half ("NeoX") pairing, dims i and i + rotary_dim/2 rotate by
    the angle of frequency i; rotary_dim = head_dim.  The cache row for
    position p holds cos of the rotary_dim/2 angles, then their sins.
All arithmetic here is float64 on the exact input values.
"""
from __future__ import annotations

import numpy as np

from .paged_attention import to_f64


def rms_norm(x, w, eps: float):
    """x [..., d]; w [d] (or None for no norm).  Returns float64."""
    x = to_f64(x)
    if w is None:
        return x
    w = to_f64(w)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * w


def rope_rotate_half(x, pos, cos_sin_cache):
    """x [n, heads, d] float64; pos [n] ints; cache [max_pos, d] (cos | sin halves)."""
    x = np.asarray(x, dtype=np.float64)
    cache = to_f64(cos_sin_cache)
    d = x.shape[-1]
    half = d // 2
    cs = cache[np.asarray(pos, dtype=np.int64)]          # [n, d]
    cos = cs[:, None, :half]
    sin = cs[:, None, half:]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def to_storage(x, storage: str):
    """Round float64 values to the pool's element type, nearest-even, directly
    from float64: bf16 keeps 8 significant bits (returned as uint16 bit
    patterns), fp32 keeps 24."""
    x = np.asarray(x, dtype=np.float64)
    if storage == "f32":
        return x.astype(np.float32)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    y = np.ldexp(np.rint(m * 256.0), e - 8)  # rint rounds half to even
    return (y.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def qk_norm_rope_store(qkv, num_q_heads: int, num_kv_heads: int, head_dim: int, positions,
                       cos_sin_cache, q_norm_w, k_norm_w, eps: float, k_planes, v_planes,
                       layer: int, out_loc, storage: str = "bf16"):
    """The fused step on N tokens.

    qkv: [N][(Hq + 2 Hkv) * d] (q | k | v per token).  Returns q_out float64
    [N][Hq][d] and writes k (normed, rotated) and v into the pool planes at
    out_loc, rounded to the pool's storage."""
    qkv = to_f64(qkv)
    N = qkv.shape[0]
    Hq, Hkv, d = num_q_heads, num_kv_heads, head_dim
    q = qkv[:, :Hq * d].reshape(N, Hq, d)
    k = qkv[:, Hq * d:(Hq + Hkv) * d].reshape(N, Hkv, d)
    v = qkv[:, (Hq + Hkv) * d:].reshape(N, Hkv, d)
    q = rope_rotate_half(rms_norm(q, q_norm_w, eps), positions, cos_sin_cache)
    k = rope_rotate_half(rms_norm(k, k_norm_w, eps), positions, cos_sin_cache)
    loc = np.asarray(out_loc, dtype=np.int64)
    kl = k_planes[layer]
    vl = v_planes[layer]
    for i in range(N):
        kl[loc[i]] = to_storage(k[i], storage)
        vl[loc[i]] = to_storage(v[i], storage)
    return q
