"""Float64 oracle for a KV pool stored as scaled FP8 E4M3.

TEST INFRASTRUCTURE ONLY (see the package header): used by tests and the CPU
baseline, never by the library.  It shares no code with the CUDA path.

The pages keep K/V in the model's dtype; an FP8 pool is not on them.  The
reading taken here is the common per-tensor scaled form: each pool plane has
one float32 dequantisation scale s (one for K, one for V); a stored code c
stands for decode(c) * s; a row x (bf16 or fp32) is stored as the code of
t = RN32(x * RN32(1 / s)), rounded to E4M3 to nearest even and saturated to
+-448.  Both the scale inversion and the product are float32 operations with
round-to-nearest so that the quantisation decision is taken in the same
precision as in a float32 kernel; the rounding of t to E4M3 is then exact.

E4M3 (the OCP FP8 "E4M3" format): 1 sign bit, 4 exponent bits (bias 7), 3
mantissa bits; exponent field 0 is subnormal (value m/8 * 2^-6); there are no
infinities; 0x7F / 0xFF are NaN; the largest finite magnitude is 1.75 * 2^8 =
448 and the smallest subnormal 2^-9.

Attention over such a pool is attention over the dequantised values:
``dequant_planes`` turns the code planes into float64 value planes that the
attention oracle (``decode_attn`` / ``extend_attn``) takes unchanged.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """uint8 E4M3 codes -> float64 values (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, e - 7)
    sub = np.ldexp(m / 8.0, -6)
    v = np.where(e == 0, sub, normal)
    v = np.where((c & 0x7F) == 0x7F, np.nan, v)
    return sign * v


def e4m3_encode(t) -> np.ndarray:
    """Float values -> E4M3 codes: round to nearest, ties to even, magnitudes
    beyond 448 saturate to 448 (NaN inputs are not expected)."""
    t = np.asarray(t, dtype=np.float64)
    a = np.abs(t)
    # Quantum of the binade holding |t|: 2^(e-3) for normal values (e >= -6),
    # 2^-9 for subnormals.
    _, ex = np.frexp(a)                      # a = f * 2^ex, 0.5 <= f < 1
    e = np.maximum(ex - 1, -6)
    q = np.ldexp(1.0, e - 3)
    r = np.rint(a / q) * q                   # rint: half to even (a/q exact)
    r = np.minimum(r, E4M3_MAX)
    # Encode the rounded magnitude.
    _, ex2 = np.frexp(np.where(r > 0, r, 1.0))
    e2 = ex2 - 1
    is_sub = (r < 2.0 ** -6)
    mant_sub = np.rint(r / 2.0 ** -9).astype(np.int64)            # 0..8 (8 = min normal)
    exp_field = np.where(is_sub, 0, e2 + 7).astype(np.int64)
    mant_norm = np.rint((r / np.ldexp(1.0, e2) - 1.0) * 8.0).astype(np.int64)
    code = np.where(is_sub, mant_sub, (exp_field << 3) | mant_norm)
    code = np.where(is_sub & (mant_sub == 8), 0x08, code)         # rounded up to 2^-6
    code = code | np.where(np.signbit(t), 0x80, 0)
    return code.astype(np.uint8)


def quantize(x, scale: float) -> np.ndarray:
    """Stored codes of values ``x`` (bf16 bit patterns, float32 or float64 that
    are float32-representable) for a plane with dequantisation scale ``scale``."""
    a = np.asarray(x)
    if a.dtype == np.uint16:
        xf = (a.astype(np.uint32) << 16).view(np.float32)
    else:
        xf = a.astype(np.float32)
    inv = np.float32(1.0) / np.float32(scale)                    # float32, round to nearest
    t = (xf * inv).astype(np.float32)                             # float32 product
    return e4m3_encode(t)


def store_kv_fp8(k_planes, v_planes, layer: int, k_rows, v_rows, out_loc, num_kv_heads: int,
                 head_dim: int, k_scale: float, v_scale: float) -> None:
    """store_kv into an FP8 pool: slot out_loc[i] of ``layer`` receives the
    codes of k_rows[i] (scale k_scale) and v_rows[i] (scale v_scale)."""
    out_loc = np.asarray(out_loc, dtype=np.int64)
    n = out_loc.shape[0]
    if n == 0:
        return
    kr = quantize(np.asarray(k_rows), k_scale).reshape(n, num_kv_heads, head_dim)
    vr = quantize(np.asarray(v_rows), v_scale).reshape(n, num_kv_heads, head_dim)
    kl = k_planes[layer]
    vl = v_planes[layer]
    for i in range(n):
        kl[out_loc[i]] = kr[i]
        vl[out_loc[i]] = vr[i]


def dequant_planes(planes, scale: float, layers=None):
    """Code planes (dict layer -> uint8 [S][Hkv][d]) -> float64 value planes."""
    keys = list(planes.keys()) if layers is None else list(layers)
    return {l: e4m3_decode(planes[l]) * float(np.float32(scale)) for l in keys}
