"""The float64 oracle against closed forms, brute force and invariants (CPU)."""
import importlib.util
import os
import sys
import types

import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle)


# Planted mistakes: each replaces one fragment of the oracle's source with a
# plausible error.  Every mutant must fail at least one pin.
MUTATIONS = {
    "gqa_mapping_modulo": ("g = h // G\n        s = (q[:, h, :]", "g = h % Hkv\n        s = (q[:, h, :]"),
    "scale_dropped": ("* scale                 # [nq][n]", "                 # [nq][n]"),
    "causal_off_by_one": ("p + idx + 1, scale)", "p + idx, scale)"),
    "page_column_wrong": ("first_col = page_size * (j // page_size)", "first_col = j // page_size"),
    "page_offset_dropped": ("page * page_size + (j % page_size)", "page * page_size"),
    "pv_uses_keys": ("o = p @ V[:, g, :]\n        out[:, h, :]", "o = p @ K[:, g, :]\n        out[:, h, :]"),
    "softmax_sign": ("p = np.where(allowed, np.exp(s - m), 0.0)", "p = np.where(allowed, np.exp(m - s), 0.0)"),
    "store_v_from_k": ("vl[out_loc[i]] = vr[i]", "vl[out_loc[i]] = kr[i]"),
    "combine_weight_sign": ("np.exp(ms - Ms[None, :])", "np.exp(Ms[None, :] - ms)"),
    "decode_drops_new_token": ("attend(q[r:r + 1], K, V, [n], scale)", "attend(q[r:r + 1], K, V, [n - 1], scale)"),
    "combine_forgets_l": ("den = (w * ls).sum(axis=0)", "den = w.sum(axis=0)"),
    "partial_max_wrong": ("p = np.exp(s - m[h])", "p = np.exp(s)"),
    "decode_ignores_table_idx": (
        "s = slots_of(page_table, int(table_idx[r]), n, page_size)\n        K = k_planes[layer][s]\n"
        "        V = v_planes[layer][s]\n        out[r:r + 1]",
        "s = slots_of(page_table, r, n, page_size)\n        K = k_planes[layer][s]\n"
        "        V = v_planes[layer][s]\n        out[r:r + 1]"),
    "extend_ignores_table_idx": (
        "s = slots_of(page_table, int(table_idx[r]), n, page_size)\n        K = k_planes[layer][s]\n"
        "        V = v_planes[layer][s]\n        out[base + idx]",
        "s = slots_of(page_table, r, n, page_size)\n        K = k_planes[layer][s]\n"
        "        V = v_planes[layer][s]\n        out[base + idx]"),
    "extend_ignores_q_offsets": ("base = int(q_offsets[r])", "base = 0"),
    "extend_drops_prefix": ("n = p + e\n", "n = e\n"),
    "mask_includes_limit": ("allowed = np.arange(n)[None, :] < lim[:, None]",
                            "allowed = np.arange(n)[None, :] <= lim[:, None]"),
    "gather_returns_k_for_v": ("np.asarray(v_planes[layer][s])))", "np.asarray(k_planes[layer][s])))"),
    "gather_ignores_table_idx": ("s = slots_of(page_table, int(table_idx[r]), int(seq_lens[r]), page_size)",
                                 "s = slots_of(page_table, r, int(seq_lens[r]), page_size)"),
}

# The same for the q/k norm + RoPE oracle.
ROPE_MUTATIONS = {
    "rope_sin_sign": ("x2 * cos + x1 * sin", "x2 * cos - x1 * sin"),
    "rope_interleaved_pairs": ("x1 = x[..., :half]\n    x2 = x[..., half:]", "x1 = x[..., 0::2]\n    x2 = x[..., 1::2]"),
    "rms_sum_not_mean": ("ms = np.mean(x * x, axis=-1, keepdims=True)", "ms = np.sum(x * x, axis=-1, keepdims=True)"),
    "rms_eps_outside": ("return x / np.sqrt(ms + eps) * w", "return x / (np.sqrt(ms) + eps) * w"),
    "bf16_truncates": ("y = np.ldexp(np.rint(m * 256.0), e - 8)", "y = np.ldexp(np.trunc(m * 256.0), e - 8)"),
    "v_gets_rotated": ("vl[loc[i]] = to_storage(v[i], storage)", "vl[loc[i]] = to_storage(k[i], storage)"),
    "k_not_normed": ("k = rope_rotate_half(rms_norm(k, k_norm_w, eps), positions, cos_sin_cache)",
                     "k = rope_rotate_half(k, positions, cos_sin_cache)"),
    "q_not_normed": ("q = rope_rotate_half(rms_norm(q, q_norm_w, eps), positions, cos_sin_cache)",
                     "q = rope_rotate_half(q, positions, cos_sin_cache)"),
    "rope_cos_sin_swapped": ("cos = cs[:, None, :half]\n    sin = cs[:, None, half:]",
                             "cos = cs[:, None, half:]\n    sin = cs[:, None, :half]"),
    "rope_first_half_sign": ("x1 * cos - x2 * sin", "x1 * cos + x2 * sin"),
    "norm_weight_dropped": ("return x / np.sqrt(ms + eps) * w", "return x / np.sqrt(ms + eps)"),
    "k_v_slices_swapped": ("k = qkv[:, Hq * d:(Hq + Hkv) * d].reshape(N, Hkv, d)\n"
                           "    v = qkv[:, (Hq + Hkv) * d:].reshape(N, Hkv, d)",
                           "v = qkv[:, Hq * d:(Hq + Hkv) * d].reshape(N, Hkv, d)\n"
                           "    k = qkv[:, (Hq + Hkv) * d:].reshape(N, Hkv, d)"),
    "bf16_keeps_7_bits": ("y = np.ldexp(np.rint(m * 256.0), e - 8)", "y = np.ldexp(np.rint(m * 128.0), e - 7)"),
}


# The same for the FP8 pool oracle.
FP8_MUTATIONS = {
    "e4m3_bias_off": ("normal = np.ldexp(1.0 + m / 8.0, e - 7)", "normal = np.ldexp(1.0 + m / 8.0, e - 8)"),
    "e4m3_truncates": ("r = np.rint(a / q) * q", "r = np.floor(a / q) * q"),
    "e4m3_no_saturation": ("r = np.minimum(r, E4M3_MAX)", "r = r"),
    "e4m3_subnormal_quantum": ("e = np.maximum(ex - 1, -6)", "e = np.maximum(ex - 1, -7)"),
    "quantize_divides": ("t = (xf * inv).astype(np.float32)", "t = (xf / inv).astype(np.float32)"),
    "dequant_forgets_scale": ("e4m3_decode(planes[l]) * float(np.float32(scale))", "e4m3_decode(planes[l])"),
    "e4m3_sign_dropped": ("code = code | np.where(np.signbit(t), 0x80, 0)", "code = code"),
    "e4m3_nan_codes_finite": ("v = np.where((c & 0x7F) == 0x7F, np.nan, v)", "v = v"),
    "e4m3_subnormals_as_normals": ("v = np.where(e == 0, sub, normal)", "v = normal"),
    "quantize_inverse_in_float64": ("inv = np.float32(1.0) / np.float32(scale)",
                                    "inv = np.float64(1.0) / np.float64(scale)"),
    "fp8_store_v_with_k_scale": ("vr = quantize(np.asarray(v_rows), v_scale)",
                                 "vr = quantize(np.asarray(v_rows), k_scale)"),
}


def _mutant(name):
    """The oracle package with one planted mistake (in any one module)."""
    base = os.path.dirname(oracle.__file__)
    src = {m: open(os.path.join(base, m + ".py")).read()
           for m in ("paged_attention", "rope_norm", "fp8_pool")}
    for mod, table in (("paged_attention", MUTATIONS), ("rope_norm", ROPE_MUTATIONS),
                       ("fp8_pool", FP8_MUTATIONS)):
        if name in table:
            old, new = table[name]
            assert src[mod].count(old) == 1, f"mutation {name} does not match the oracle source once"
            src[mod] = src[mod].replace(old, new)
    m1 = types.ModuleType(f"oracle_pa_{name}")
    exec(compile(src["paged_attention"], f"<mutant {name} paged_attention>", "exec"), m1.__dict__)
    m2 = types.ModuleType(f"oracle_rn_{name}")
    m2.__dict__["to_f64"] = m1.to_f64
    rn = src["rope_norm"].replace("from .paged_attention import to_f64\n", "")
    exec(compile(rn, f"<mutant {name} rope_norm>", "exec"), m2.__dict__)
    m3 = types.ModuleType(f"oracle_fp8_{name}")
    exec(compile(src["fp8_pool"], f"<mutant {name} fp8_pool>", "exec"), m3.__dict__)
    mod = types.ModuleType(f"oracle_mutant_{name}")
    for k in oracle.__all__:
        for m in (m1, m2, m3):
            if hasattr(m, k):
                mod.__dict__[k] = getattr(m, k)
                break
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS) + sorted(ROPE_MUTATIONS) + sorted(FP8_MUTATIONS))
def test_planted_mistake_is_caught(name):
    mod = _mutant(name)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mod)
        except AssertionError:
            failed.append(pin.__name__)
        except Exception as e:  # a crash also counts as caught
            failed.append(f"{pin.__name__}:{type(e).__name__}")
    assert failed, f"planted mistake {name} passed every pin"
