"""Paged KV pool attention for B200 (sm_100a): store_kv, decode_attn, extend_attn.

The compute path is the C-ABI CUDA library ``libpkv.so`` (include/pkv.h);
``api`` is its torch-facing binding and ``workloads`` draws seeded synthetic
inputs.  Importing the package loads nothing; the library is built and loaded
on first use of ``api``.
"""
__all__ = ["api", "workloads", "build"]
