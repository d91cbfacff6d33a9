"""CPU float64 oracle for the paged KV pool hot path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.  It shares no
code with the CUDA path.

Parity status per function (what pins it, in ``tests/test_oracle_pins.py``):
  store_kv, slots_of, gather_kv -- closed forms (bit copy; hand-derived page
      translation fixture in tests/golden) and brute force;
  attend, decode_attn, extend_attn -- brute-force dense attention on tiny
      inputs, a two-key closed form, and the invariants (slot permutation,
      chunked == unchunked, shared prefix == private copy, one-token context
      returns V, constant K returns mean V, decode == extend with one row,
      q*c with k/c, identical query heads);
  partial_state, combine_states -- merging split states equals the unsplit
      result;
  rms_norm, rope_rotate_half, qk_norm_rope_store, to_storage -- closed forms
      (unit-RMS vectors, identity at position 0, a single-pair rotation by a
      known angle), norm preservation, the relative-position property of
      rotated dot products, exact bf16 rounding of hand-picked ties;
  e4m3_encode, e4m3_decode, quantize, store_kv_fp8, dequant_planes -- a
      hand-derived code table (ties, subnormals, saturation), the value of
      all 256 codes built from the format's fields, the float32 scaling
      decision, and a one-token decode returning the dequantised V.
The pages print no worked numerical example for any of these, so no stored
value comes from them.
"""
from .paged_attention import (attend, combine_states, decode_attn, extend_attn, gather_kv,
                              partial_state, slots_of, store_kv, to_f64)
from .rope_norm import qk_norm_rope_store, rms_norm, rope_rotate_half, to_storage
from .fp8_pool import dequant_planes, e4m3_decode, e4m3_encode, quantize, store_kv_fp8

__all__ = ["attend", "combine_states", "decode_attn", "dequant_planes", "e4m3_decode",
           "e4m3_encode", "extend_attn", "gather_kv", "partial_state", "qk_norm_rope_store",
           "quantize", "rms_norm", "rope_rotate_half", "slots_of", "store_kv", "store_kv_fp8",
           "to_f64", "to_storage"]
