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
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src_path = os.path.join(os.path.dirname(oracle.__file__), "paged_attention.py")
    src = open(src_path).read()
    assert src.count(old) == 1, f"mutation {name} does not match the oracle source once"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
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
