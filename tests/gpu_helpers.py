"""Move seeded workloads onto the GPU and compute oracle expectations.

Inputs come from ``paged_kv_gqa_scatter_b200.workloads``; expectations come
only from ``oracle`` applied to those same host inputs.  Nothing here reads
back a device result to feed the oracle.
"""
from __future__ import annotations

import copy

import numpy as np
import torch

import oracle
from paged_kv_gqa_scatter_b200 import api
from paged_kv_gqa_scatter_b200 import workloads as W

TORCH_DTYPE = {W.BF16: torch.bfloat16, W.F32: torch.float32, W.F8: torch.float8_e4m3fn}


def to_dev(arr: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Host element array (bf16 bits, float32, or E4M3 codes) -> device tensor of the element type."""
    if dtype == W.BF16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).to(device)
    if dtype == W.F8:
        return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.uint8)).to(device).view(torch.float8_e4m3fn)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


def i32(arr, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.int32)).to(device)


def from_dev(t: torch.Tensor) -> np.ndarray:
    """Device result -> float64 host array (exact widening)."""
    return t.float().cpu().numpy().astype(np.float64)


def device_pool(spec: W.PoolSpec, k_planes, v_planes, layers=None) -> api.KVPool:
    """Allocate the full layer-stacked pool and copy in the host contents of
    ``layers`` (default: every layer the host planes hold)."""
    dt = TORCH_DTYPE[spec.dtype]
    pool = api.KVPool.empty(spec.num_layers, spec.num_slots, spec.num_kv_heads, dtype=dt,
                            page_size=spec.page_size, zero=True, k_scale=spec.k_scale,
                            v_scale=spec.v_scale)
    if isinstance(k_planes, W.TiledPlane):
        lay = range(spec.num_layers) if layers is None else layers
        for plane, dst in ((k_planes, pool.k), (v_planes, pool.v)):
            blk = to_dev(plane.block, spec.dtype)
            nb = blk.shape[0]
            for l in lay:
                flat0 = l * spec.num_slots
                s = 0
                while s < spec.num_slots:
                    off = (flat0 + s) % nb
                    m = min(nb - off, spec.num_slots - s)
                    dst[l, s:s + m].copy_(blk[off:off + m])
                    s += m
    else:
        lay = list(k_planes.keys()) if layers is None else layers
        for l in lay:
            pool.k[l].copy_(to_dev(k_planes[l], spec.dtype))
            pool.v[l].copy_(to_dev(v_planes[l], spec.dtype))
    torch.cuda.synchronize()
    return pool


def host_planes_copy(planes):
    if isinstance(planes, W.TiledPlane):
        c = W.TiledPlane(planes.block, planes.num_layers, planes.num_slots)
        c.overrides = {l: dict(d) for l, d in planes.overrides.items()}
        return c
    return {l: a.copy() for l, a in planes.items()}


def tol_check(got: np.ndarray, exp: np.ndarray, dtype: str, what: str = ""):
    """bf16: |got - exp| <= 1e-2 + 1e-2 |exp|; fp32 check build: |got - exp| <= 1e-4."""
    err = np.abs(got - exp)
    if dtype == W.BF16:
        bound = 1e-2 + 1e-2 * np.abs(exp)
    else:
        bound = np.full_like(exp, 1e-4)
    bad = err > bound
    if np.any(bad):
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; max err "
                             f"{err.max():.3e}; first bad indices {idx.tolist()}")
    return float(err.max()) if err.size else 0.0


class DeviceDecode:
    """A DecodeWorkload on the device: pool, table, inputs, outputs, workspace."""

    def __init__(self, wl: W.DecodeWorkload, pool: api.KVPool = None, table=None):
        self.wl = wl
        dt = wl.pool.io_dtype
        self.pool = pool if pool is not None else device_pool(wl.pool, wl.k_planes, wl.v_planes,
                                                              layers=[wl.layer])
        self.table = table if table is not None else api.PageTable(i32(wl.page_table))
        self.table_idx = i32(wl.table_idx)
        self.seq_lens = i32(wl.seq_lens)
        self.q = to_dev(wl.q, dt)
        self.k_new = to_dev(wl.k_new, dt)
        self.v_new = to_dev(wl.v_new, dt)
        self.out_loc = i32(wl.out_loc)
        self.out = torch.empty_like(self.q)
        self.ws = api.decode_workspace(wl.batch, wl.num_q_heads)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(self, store=True):
        wl = self.wl
        if store:
            api.store_kv(self.pool, wl.layer, self.k_new, self.v_new, self.out_loc, self.err)
        api.decode_attn(self.pool, wl.layer, self.q, self.table, self.table_idx, self.seq_lens,
                        self.out, self.ws, scale=wl.scale, dev_err=self.err)


def oracle_decode(wl: W.DecodeWorkload, requests=None, planes=None):
    """Expected decode output: oracle store_kv on a copy of the host pool, then
    oracle decode_attn.  Returns (out float64 [B][Hq][d], planes after store)."""
    if planes is None:
        kp, vp = host_planes_copy(wl.k_planes), host_planes_copy(wl.v_planes)
    else:
        kp, vp = planes
    oracle.store_kv(kp, vp, wl.layer, wl.k_new, wl.v_new, wl.out_loc, wl.pool.num_kv_heads,
                    wl.pool.head_dim)
    out = oracle.decode_attn(wl.q, kp, vp, wl.layer, wl.page_table, wl.table_idx, wl.seq_lens,
                             wl.pool.page_size, wl.scale, requests=requests)
    return out, (kp, vp)


class DeviceExtend:
    def __init__(self, wl: W.ExtendWorkload, pool: api.KVPool = None, table=None):
        self.wl = wl
        dt = wl.pool.io_dtype
        self.pool = pool if pool is not None else device_pool(wl.pool, wl.k_planes, wl.v_planes,
                                                              layers=[wl.layer])
        self.table = table if table is not None else api.PageTable(i32(wl.page_table))
        self.table_idx = i32(wl.table_idx)
        self.prefix = i32(wl.prefix_lens)
        self.ext = i32(wl.extend_lens)
        self.qoff = i32(wl.q_offsets)
        self.q = to_dev(wl.q, dt)
        self.k_new = to_dev(wl.k_new, dt)
        self.v_new = to_dev(wl.v_new, dt)
        self.out_loc = i32(wl.out_loc)
        self.out = torch.empty_like(self.q)
        self.max_ext = int(wl.extend_lens.max()) if wl.batch else 0
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(self, store=True, layer=None):
        wl = self.wl
        layer = wl.layer if layer is None else layer
        if store:
            api.store_kv(self.pool, layer, self.k_new, self.v_new, self.out_loc, self.err)
        api.extend_attn(self.pool, layer, self.q, self.table, self.table_idx, self.prefix,
                        self.ext, self.qoff, self.max_ext, self.out, scale=wl.scale,
                        dev_err=self.err)


def oracle_extend(wl: W.ExtendWorkload, rows=None, planes=None):
    if planes is None:
        kp, vp = host_planes_copy(wl.k_planes), host_planes_copy(wl.v_planes)
    else:
        kp, vp = planes
    oracle.store_kv(kp, vp, wl.layer, wl.k_new, wl.v_new, wl.out_loc, wl.pool.num_kv_heads,
                    wl.pool.head_dim)
    out = oracle.extend_attn(wl.q, kp, vp, wl.layer, wl.page_table, wl.table_idx, wl.prefix_lens,
                             wl.extend_lens, wl.q_offsets, wl.pool.page_size, wl.scale, rows=rows)
    return out, (kp, vp)


def referenced_slots(wl) -> np.ndarray:
    """Pool slots that some request's context reads (the stored token included)."""
    used = [oracle.slots_of(wl.page_table, int(wl.table_idx[r]), int(wl.seq_lens[r]), wl.pool.page_size)
            for r in range(wl.batch)]
    return np.unique(np.concatenate(used))


def poison_unreferenced(planes, layer, keep, value):
    """Set every slot of `layer` outside `keep` to `value` (a NaN pattern)."""
    a = planes[layer]
    mask = np.ones(a.shape[0], dtype=bool)
    mask[keep] = False
    a[mask] = value
