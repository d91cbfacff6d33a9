"""Torch-facing binding of the pkv C ABI: same call names, marshalling only.

PyTorch provides device memory and streams; every step of the path runs in
the CUDA kernels of ``libpkv.so``.  Each call passes ``tensor.data_ptr()``
values and the current CUDA stream to the C entry point and raises
``PkvError`` on a non-zero status.  There is no CPU path.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from . import _lib

DTYPE_CODES = {torch.bfloat16: 0, torch.float32: 1, torch.float8_e4m3fn: 2}
HEAD_DIM = 128

# pkv_device_error bits OR-ed into a call's dev_err word.
DEV_ERR_SLOT_RANGE = 1
DEV_ERR_TABLE_RANGE = 2
DEV_ERR_EMPTY_CONTEXT = 4
DEV_ERR_BAD_LENGTH = 8
DEV_ERR_PAGE_ALIGN = 16
DEV_ERR_TIMEOUT = 32
DEV_ERR_POSITION = 64


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


class Workspace:
    """A library-owned workspace (pkv_workspace_create): a scratch buffer for
    decode / cascade decode and a device error word.  Pass it as `workspace`
    and as `dev_err`; read_device_error() waits for the stream and returns and
    clears the error bits."""

    def __init__(self, max_batch: int, max_q_heads: int, max_prefix_len: int = 0):
        lib = _lib.load()
        h = ctypes.c_void_p()
        _lib.check(lib.pkv_workspace_create(max_batch, max_q_heads, max_prefix_len, ctypes.byref(h)),
                   "workspace_create")
        self._h = h

    def buffer(self):
        n = ctypes.c_size_t()
        p = _lib.load().pkv_workspace_buffer(self._h, ctypes.byref(n))
        return int(p), int(n.value)

    def error_word(self) -> int:
        return int(_lib.load().pkv_workspace_error_word(self._h))

    def read_device_error(self, stream=None) -> int:
        code = ctypes.c_int32()
        _lib.check(_lib.load().pkv_read_device_error(self._h, _stream_ptr(stream), ctypes.byref(code)),
                   "read_device_error")
        return int(code.value)

    def close(self) -> None:
        if self._h is not None and self._h.value:
            _lib.load().pkv_workspace_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, Workspace):
        return t.error_word()
    return int(t.data_ptr())


def _ws(w):
    """(pointer, bytes) of a workspace tensor or Workspace object."""
    if isinstance(w, Workspace):
        return w.buffer()
    return int(w.data_ptr()), w.numel() * w.element_size()


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not isinstance(t, Workspace) and not t.is_cuda:
            raise ValueError("pkv calls take CUDA tensors")


class KVPool:
    """K and V planes ``[num_layers][num_slots][num_kv_heads][128]`` (caller memory).

    ``k`` and ``v`` may be views with any layer/slot strides as long as each
    slot's heads and dims are contiguous (the pool layout of include/pkv.h).
    """

    def __init__(self, k: torch.Tensor, v: torch.Tensor, page_size: int = 1,
                 k_scale: float = 1.0, v_scale: float = 1.0):
        if k.shape != v.shape or k.dtype != v.dtype or k.dim() != 4:
            raise ValueError("k and v must be matching 4-D tensors")
        if k.stride(3) != 1 or k.stride(2) != k.shape[3] or v.stride() != k.stride():
            raise ValueError("heads and dims of a slot must be contiguous, same strides for k and v")
        if k.dtype not in DTYPE_CODES:
            raise ValueError(f"unsupported pool dtype {k.dtype}")
        _require_cuda(k, v)
        self.k, self.v = k, v
        self.page_size = int(page_size)
        self.c = _lib.PkvPool(
            k=k.data_ptr(), v=v.data_ptr(), num_layers=k.shape[0], num_slots=k.shape[1],
            layer_stride=k.stride(0), slot_stride=k.stride(1), num_kv_heads=k.shape[2],
            head_dim=k.shape[3], page_size=self.page_size, dtype=DTYPE_CODES[k.dtype],
            k_scale=float(k_scale), v_scale=float(v_scale))
        self.k_scale, self.v_scale = float(k_scale), float(v_scale)

    @classmethod
    def empty(cls, num_layers, num_slots, num_kv_heads, dtype=torch.bfloat16, page_size=1,
              device="cuda", zero=True, k_scale=1.0, v_scale=1.0):
        mk = torch.zeros if zero else torch.empty
        k = mk((num_layers, num_slots, num_kv_heads, HEAD_DIM), dtype=dtype, device=device)
        v = mk((num_layers, num_slots, num_kv_heads, HEAD_DIM), dtype=dtype, device=device)
        return cls(k, v, page_size, k_scale, v_scale)

    @property
    def io_dtype(self):
        """dtype of the rows a call writes into the pool, and of q / out."""
        return torch.bfloat16 if self.k.dtype == torch.float8_e4m3fn else self.k.dtype

    @property
    def num_kv_heads(self) -> int:
        return self.k.shape[2]

    @property
    def dtype(self):
        return self.k.dtype


class PageTable:
    """int32 ``[rows][cols]`` token-granular page table (a CUDA tensor view)."""

    def __init__(self, entries: torch.Tensor):
        if entries.dtype != torch.int32 or entries.dim() != 2 or entries.stride(1) != 1:
            raise ValueError("page table must be a 2-D int32 tensor with contiguous rows")
        _require_cuda(entries)
        self.entries = entries
        self.c = _lib.PkvPageTable(entries=entries.data_ptr(), rows=entries.shape[0],
                                   cols=entries.shape[1], row_stride=entries.stride(0))


def store_kv(pool: KVPool, layer: int, k: torch.Tensor, v: torch.Tensor, out_loc: torch.Tensor,
             dev_err: Optional[torch.Tensor] = None, stream=None) -> None:
    """pkv_store_kv: scatter rows of k/v ([N][Hkv*128], row-strided) to out_loc."""
    _require_cuda(k, v, out_loc, dev_err)
    if k.dim() == 3:
        k = k.reshape(k.shape[0], -1)
    if v.dim() == 3:
        v = v.reshape(v.shape[0], -1)
    if k.stride(1) != 1 or v.stride(1) != 1 or k.dtype != pool.io_dtype or v.dtype != pool.io_dtype:
        raise ValueError("k/v rows must be contiguous and of the pool's row dtype")
    if out_loc.dtype not in (torch.int32, torch.int64) or not out_loc.is_contiguous():
        raise ValueError("out_loc must be contiguous int32 or int64")
    lib = _lib.load()
    _lib.check(lib.pkv_store_kv(ctypes.byref(pool.c), layer, k.data_ptr(), k.stride(0),
                                v.data_ptr(), v.stride(0), out_loc.data_ptr(),
                                1 if out_loc.dtype == torch.int64 else 0, out_loc.shape[0],
                                _ptr(dev_err), _stream_ptr(stream)), "store_kv")


def qk_norm_rope_store(pool: KVPool, layer: int, qkv: torch.Tensor, num_q_heads: int,
                       positions: torch.Tensor, cos_sin_cache: torch.Tensor, out_loc: torch.Tensor,
                       q_out: torch.Tensor, q_norm_weight: Optional[torch.Tensor] = None,
                       k_norm_weight: Optional[torch.Tensor] = None, eps: float = 1e-6,
                       dev_err: Optional[torch.Tensor] = None, stream=None) -> None:
    """pkv_qk_norm_rope_store: q/k RMSNorm + RoPE, then k/v into the pool, q into q_out."""
    _require_cuda(qkv, positions, cos_sin_cache, out_loc, q_out, q_norm_weight, k_norm_weight, dev_err)
    if qkv.dim() != 2 or qkv.dtype != pool.io_dtype or (qkv.shape[0] > 0 and qkv.stride(1) != 1):
        raise ValueError("qkv must be [tokens][(Hq + 2 Hkv) * 128] rows of the pool's row dtype")
    if cos_sin_cache.dtype != torch.float32 or not cos_sin_cache.is_contiguous():
        raise ValueError("cos_sin_cache must be contiguous float32 [max_position][128]")
    for t, name in ((positions, "positions"), (out_loc, "out_loc")):
        if t.dtype not in (torch.int32, torch.int64) or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous int32 or int64")
    lib = _lib.load()
    _lib.check(lib.pkv_qk_norm_rope_store(
        ctypes.byref(pool.c), layer, qkv.data_ptr(), qkv.stride(0), num_q_heads,
        positions.data_ptr(), 1 if positions.dtype == torch.int64 else 0, cos_sin_cache.data_ptr(),
        cos_sin_cache.shape[0], _ptr(q_norm_weight), _ptr(k_norm_weight), float(eps),
        out_loc.data_ptr(), 1 if out_loc.dtype == torch.int64 else 0, qkv.shape[0],
        q_out.data_ptr(), _ptr(dev_err), _stream_ptr(stream)), "qk_norm_rope_store")


def selftest_wait_timeout(dev_err: torch.Tensor, stream=None) -> None:
    """pkv_selftest_wait_timeout: a kernel whose barrier wait must give up
    after about one second and set DEV_ERR_TIMEOUT in dev_err."""
    _require_cuda(dev_err)
    _lib.check(_lib.load().pkv_selftest_wait_timeout(dev_err.data_ptr(), _stream_ptr(stream)),
               "selftest_wait_timeout")


def gather_kv(pool: KVPool, layer: int, table: PageTable, table_idx: torch.Tensor,
              seq_lens: torch.Tensor, row_offsets: torch.Tensor, k_out: torch.Tensor,
              v_out: torch.Tensor, dev_err: Optional[torch.Tensor] = None, stream=None) -> None:
    """pkv_gather_kv: copy each request's rows through the table into k_out/v_out."""
    _require_cuda(table_idx, seq_lens, row_offsets, k_out, v_out, dev_err)
    lib = _lib.load()
    _lib.check(lib.pkv_gather_kv(ctypes.byref(pool.c), layer, ctypes.byref(table.c),
                                 table_idx.data_ptr(), seq_lens.data_ptr(), row_offsets.data_ptr(),
                                 seq_lens.shape[0], k_out.data_ptr(), v_out.data_ptr(),
                                 _ptr(dev_err), _stream_ptr(stream)), "gather_kv")


def decode_workspace_bytes(batch: int, num_q_heads: int) -> int:
    return int(_lib.load().pkv_decode_workspace_bytes(batch, num_q_heads))


def decode_workspace(batch: int, num_q_heads: int, device="cuda") -> torch.Tensor:
    n = decode_workspace_bytes(batch, num_q_heads)
    return torch.empty(max(16, n), dtype=torch.uint8, device=device)


def decode_attn(pool: KVPool, layer: int, q: torch.Tensor, table: PageTable,
                table_idx: torch.Tensor, seq_lens: torch.Tensor, out: torch.Tensor,
                workspace: torch.Tensor, scale: Optional[float] = None,
                dev_err: Optional[torch.Tensor] = None, stream=None) -> None:
    """pkv_decode_attn: q [B][Hq][128] -> out [B][Hq][128] over each request's context."""
    _require_cuda(q, table_idx, seq_lens, out, workspace, dev_err)
    if not (q.is_contiguous() and out.is_contiguous()):
        raise ValueError("q and out must be contiguous")
    if q.dtype != pool.io_dtype or out.dtype != pool.io_dtype:
        raise ValueError("q/out dtype must match the pool")
    B, Hq, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    lib = _lib.load()
    _lib.check(lib.pkv_decode_attn(ctypes.byref(pool.c), layer, q.data_ptr(), Hq,
                                   ctypes.byref(table.c), table_idx.data_ptr(), seq_lens.data_ptr(),
                                   B, scale, out.data_ptr(), *_ws(workspace), _ptr(dev_err),
                                   _stream_ptr(stream)), "decode_attn")


def decode_attn_noalloc(pool: KVPool, layer: int, q: torch.Tensor, table: PageTable,
                        table_idx: torch.Tensor, seq_lens: torch.Tensor, out: torch.Tensor,
                        scale: Optional[float] = None, dev_err: Optional[torch.Tensor] = None,
                        stream=None) -> None:
    """pkv_decode_attn_noalloc: decode_attn without a workspace, for callers that
    cannot allocate device memory.  Its scratch is a fixed array inside the
    library shared by every call on the device, so calls that may overlap on
    the GPU must not be issued; the first call on a device should happen
    outside stream capture."""
    _require_cuda(q, table_idx, seq_lens, out, dev_err)
    if not (q.is_contiguous() and out.is_contiguous()):
        raise ValueError("q and out must be contiguous")
    if q.dtype != pool.io_dtype or out.dtype != pool.io_dtype:
        raise ValueError("q/out dtype must match the pool")
    B, Hq, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    lib = _lib.load()
    _lib.check(lib.pkv_decode_attn_noalloc(ctypes.byref(pool.c), layer, q.data_ptr(), Hq,
                                           ctypes.byref(table.c), table_idx.data_ptr(),
                                           seq_lens.data_ptr(), B, scale, out.data_ptr(),
                                           _ptr(dev_err), _stream_ptr(stream)), "decode_attn_noalloc")


def decode_cascade_workspace_bytes(batch: int, num_q_heads: int, max_prefix_len: int) -> int:
    return int(_lib.load().pkv_decode_cascade_workspace_bytes(batch, num_q_heads, max_prefix_len))


def decode_cascade_workspace(batch: int, num_q_heads: int, max_prefix_len: int,
                             device="cuda") -> torch.Tensor:
    n = decode_cascade_workspace_bytes(batch, num_q_heads, max_prefix_len)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def decode_attn_cascade(pool: KVPool, layer: int, q: torch.Tensor, table: PageTable,
                        table_idx: torch.Tensor, seq_lens: torch.Tensor,
                        group_offsets: torch.Tensor, group_prefix_lens: torch.Tensor,
                        max_prefix_len: int, out: torch.Tensor, workspace: torch.Tensor,
                        scale: Optional[float] = None, dev_err: Optional[torch.Tensor] = None,
                        stream=None) -> None:
    """pkv_decode_attn_cascade: decode_attn with each group's shared prefix
    attended once per group (tensor cores) and merged with the suffixes."""
    _require_cuda(q, table_idx, seq_lens, group_offsets, group_prefix_lens, out, workspace, dev_err)
    if not (q.is_contiguous() and out.is_contiguous()):
        raise ValueError("q and out must be contiguous")
    if q.dtype != pool.io_dtype or out.dtype != pool.io_dtype:
        raise ValueError("q/out dtype must match the pool")
    for t, name in ((group_offsets, "group_offsets"), (group_prefix_lens, "group_prefix_lens")):
        if t.dtype != torch.int32 or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous int32")
    B, Hq, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    lib = _lib.load()
    _lib.check(lib.pkv_decode_attn_cascade(
        ctypes.byref(pool.c), layer, q.data_ptr(), Hq, ctypes.byref(table.c), table_idx.data_ptr(),
        seq_lens.data_ptr(), B, group_offsets.data_ptr(), group_prefix_lens.data_ptr(),
        group_prefix_lens.numel(), int(max_prefix_len), scale, out.data_ptr(), *_ws(workspace),
        _ptr(dev_err), _stream_ptr(stream)),
        "decode_attn_cascade")


def extend_workspace_bytes(batch: int, num_q_heads: int, total_q: int) -> int:
    return int(_lib.load().pkv_extend_workspace_bytes(batch, num_q_heads, total_q))


def extend_attn(pool: KVPool, layer: int, q: torch.Tensor, table: PageTable,
                table_idx: torch.Tensor, prefix_lens: torch.Tensor, extend_lens: torch.Tensor,
                q_offsets: torch.Tensor, max_extend_len: int, out: torch.Tensor,
                scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
                dev_err: Optional[torch.Tensor] = None, stream=None) -> None:
    """pkv_extend_attn: causal attention of each request's chunk over prefix + chunk."""
    _require_cuda(q, table_idx, prefix_lens, extend_lens, q_offsets, out, workspace, dev_err)
    if not (q.is_contiguous() and out.is_contiguous()):
        raise ValueError("q and out must be contiguous")
    if q.dtype != pool.io_dtype or out.dtype != pool.io_dtype:
        raise ValueError("q/out dtype must match the pool")
    T, Hq, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws_ptr = _ptr(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    lib = _lib.load()
    _lib.check(lib.pkv_extend_attn(ctypes.byref(pool.c), layer, q.data_ptr(), Hq,
                                   ctypes.byref(table.c), table_idx.data_ptr(),
                                   prefix_lens.data_ptr(), extend_lens.data_ptr(),
                                   q_offsets.data_ptr(), extend_lens.shape[0], T,
                                   int(max_extend_len), scale, out.data_ptr(), ws_ptr, ws_bytes,
                                   _ptr(dev_err), _stream_ptr(stream)), "extend_attn")
