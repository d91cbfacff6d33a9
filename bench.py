"""Benchmark of the paged KV pool hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode-qwen3-0.6b|decode-qwen3-8b|chunked-prefill|radix-prefix]

Default workload (one "step"): the Qwen3-0.6B-shaped decode step -- 64
requests with contexts uniform in [512, 4096], Hq 16, Hkv 8, d 128, bf16,
page_size 1 over a 300k-slot, 28-layer pool (layer 13): store_kv of the 64
new tokens, then decode_attn (split-KV partials + combine).  The metric is
decode KV GB/s: K/V bytes of every context token (all KV heads, both planes)
plus page-table, query and output bytes, divided by device time.  Inputs are
larger than L2 (~0.6 GB of KV per step), so no L2 flush is needed.

Under torchrun each rank runs an independent replica on its own GPU (the
path needs no collective); value = total bytes of all ranks / max-over-ranks
time, "scaling": "weak".

``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, BF16_FALLBACK_TFLOPS, 1400.0, "fallback"


def source_hash(*names):
    """Hash of the code (comments and blank lines removed) of the named
    sources: a recorded ncu figure stays valid across comment-only edits and
    becomes stale when the code changes."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "paged_kv_gqa_scatter_b200", "csrc", n)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
        h.update("\n".join(lines).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, src_hash: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or None
    when the kernel's source has changed since the counters were taken or the
    capture was of another workload."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(kernel)
        if e and e.get("source_hash") == src_hash and e.get("workload") == workload:
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value of x over the ranks (device time is taken as the slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, steps: int, ms_max: float, world: int) -> float:
    """Whole-job rate: the units every rank processed over the slowest rank's time (units/s)."""
    return world * units_per_rank_step * steps / (ms_max / 1e3)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ---------------------------------------------------------------------------
# decode workload (the headline)
# ---------------------------------------------------------------------------
def decode_bytes(wl) -> int:
    """Algorithmic bytes of one decode_attn call: every context token's K and V
    rows (all KV heads), its page-table entry (one per token at page_size 1, one
    per page otherwise), the queries and the outputs."""
    B, Hq = wl.batch, wl.num_q_heads
    esz = ESIZE[wl.pool.dtype]
    io = ESIZE[wl.pool.io_dtype]
    n = wl.seq_lens.astype(np.int64)
    row = wl.pool.num_kv_heads * 128 * esz
    P = wl.pool.page_size
    table = int(n.sum()) * 4 if P == 1 else int(((n + P - 1) // P).sum()) * 4
    return int(n.sum()) * 2 * row + table + 2 * B * Hq * 128 * io + 8 * B


ESIZE = {"bf16": 2, "f32": 4, "fp8": 1}


def store_bytes(wl) -> int:
    """Read each new K and V row (row dtype), write it to the pool (pool dtype)."""
    row_in = wl.pool.num_kv_heads * 128 * ESIZE[wl.pool.io_dtype]
    row_out = wl.pool.num_kv_heads * 128 * ESIZE[wl.pool.dtype]
    return wl.batch * (2 * (row_in + row_out) + 4)


def cpu_decode_sample(wl, budget_s: float = 12.0):
    """Time the oracle on the first requests of the workload until ~budget_s of
    CPU work; return (GB/s in the metric's bytes, sample description)."""
    import oracle
    from paged_kv_gqa_scatter_b200 import workloads as W
    kp = {l: a for l, a in wl.k_planes.items()} if isinstance(wl.k_planes, dict) else wl.k_planes
    vp = {l: a for l, a in wl.v_planes.items()} if isinstance(wl.v_planes, dict) else wl.v_planes
    done, nbytes = 0, 0
    esz = 2 if wl.pool.dtype == "bf16" else 4
    row = wl.pool.num_kv_heads * 128 * esz
    t0 = time.perf_counter()
    for r in range(wl.batch):
        oracle.decode_attn(wl.q, kp, vp, wl.layer, wl.page_table, wl.table_idx, wl.seq_lens,
                           wl.pool.page_size, wl.scale, requests=[r])
        n = int(wl.seq_lens[r])
        nbytes += n * (2 * row + 4) + 2 * wl.num_q_heads * 128 * esz + 8
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return nbytes / dt / 1e9, f"oracle decode_attn on the first {done} of {wl.batch} requests " \
                              f"({nbytes / 1e6:.1f} MB of KV), float64 numpy", dt


def run_decode(args, world, rank, local):
    import torch
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from paged_kv_gqa_scatter_b200 import api, _lib
    from paged_kv_gqa_scatter_b200 import workloads as W

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.workload == "decode-qwen3-8b":
        free, _ = torch.cuda.mem_get_info()
        P = args.page_size or 16
        bytes_per_page = 36 * P * 8 * 128 * 2 * 2
        num_pages = int(0.6 * free // bytes_per_page)
        wl = W.decode_qwen3_8b(num_pages=num_pages, page_size=P)
        if P != 16:
            wl.name = f"decode-qwen3-8b-p{P}"
        layers = list(range(wl.pool.num_layers))
    else:
        nl = 28 if args.pool_layers is None else args.pool_layers
        wl = W.decode_qwen3_06b(num_layers=nl, layer=min(13, nl - 1))
        if args.kv_dtype == "fp8":
            wl = W.with_fp8_pool(wl)
        layers = [wl.layer]
    lib = _lib.load()

    # ---- device residency (inputs resident in HBM before the timed region) ----
    def tdev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    spec = wl.pool
    fp8 = spec.dtype == "fp8"

    def tpool(a):  # host plane contents -> device tensor of the pool's type
        if fp8:
            return torch.from_numpy(np.ascontiguousarray(a)).to(dev).view(torch.float8_e4m3fn)
        return tdev(a)

    pool = api.KVPool.empty(spec.num_layers, spec.num_slots, spec.num_kv_heads, page_size=spec.page_size,
                            device=dev, zero=not isinstance(wl.k_planes, W.TiledPlane),
                            dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16,
                            k_scale=spec.k_scale, v_scale=spec.v_scale)
    if isinstance(wl.k_planes, W.TiledPlane):
        for plane, dst in ((wl.k_planes, pool.k), (wl.v_planes, pool.v)):
            blk = tdev(plane.block)
            flat = dst.view(-1, spec.num_kv_heads, 128)
            nb = blk.shape[0]
            for s in range(0, flat.shape[0], nb):
                m = min(nb, flat.shape[0] - s)
                flat[s:s + m].copy_(blk[:m])
    else:
        for l in layers:
            pool.k[l].copy_(tpool(wl.k_planes[l]))
            pool.v[l].copy_(tpool(wl.v_planes[l]))
    table = api.PageTable(torch.from_numpy(wl.page_table).to(dev))
    table_idx = torch.from_numpy(wl.table_idx).to(dev)
    seq_lens = torch.from_numpy(wl.seq_lens).to(dev)
    q = tdev(wl.q)
    k_new = tdev(wl.k_new)
    v_new = tdev(wl.v_new)
    out_loc = torch.from_numpy(wl.out_loc).to(dev)
    out = torch.empty_like(q)
    ws = api.decode_workspace(wl.batch, wl.num_q_heads, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        for l in layers:
            api.store_kv(pool, l, k_new, v_new, out_loc, err)
            api.decode_attn(pool, l, q, table, table_idx, seq_lens, out, ws, scale=wl.scale, dev_err=err)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- the step as the serving engine runs decode: captured once in a CUDA
    # graph (fixed buffers) and replayed; eager launches if capture fails ------
    nL = len(layers)
    graph, launch_mode = None, "cuda graph replay of one step"
    try:
        gs = torch.cuda.Stream(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            step()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
    except Exception as exc:  # reported in the output, not hidden
        graph, launch_mode = None, f"eager (graph capture failed: {type(exc).__name__})"

    # ---- timed region: exactly K steps ----------------------------------------
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    start.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step()
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_total = start.elapsed_time(stop)
    ms_total = max_over_ranks(ms_total, world)

    # ---- the same K steps launched eagerly, back to back (reported) -----------
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(args.steps):
        step()
    eb.record(stream)
    torch.cuda.synchronize()
    eager_us = round(ea.elapsed_time(eb) / args.steps * 1e3, 2)

    # ---- per-call durations for the roofline: K more steps, events around
    # each call on the launching stream (the events cost the calls their
    # launch overlap, so this loop is not the one `value` comes from) -------
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps * nL)]
    i = 0
    for _ in range(args.steps):
        for l in layers:
            ev[i][0].record(stream)
            api.store_kv(pool, l, k_new, v_new, out_loc, err)
            ev[i][1].record(stream)
            api.decode_attn(pool, l, q, table, table_idx, seq_lens, out, ws, scale=wl.scale, dev_err=err)
            ev[i][2].record(stream)
            i += 1
    torch.cuda.synchronize()
    dec_ms = [e[1].elapsed_time(e[2]) for e in ev]
    st_ms = [e[0].elapsed_time(e[1]) for e in ev]
    errv = int(err.item())

    per_call = decode_bytes(wl)
    step_bytes = nL * (per_call + store_bytes(wl))
    value = job_throughput(step_bytes, args.steps, ms_total, world) / 1e9
    hbm, bf16, bf16s, peak_src = measured_peaks()
    dec_avg_ms = sum(dec_ms) / len(dec_ms)
    achieved = per_call / (dec_avg_ms / 1e3) / 1e9
    traffic = recorded_traffic("decode_split_kernel", source_hash("decode.cu", "common.cuh"), wl.name)

    # ---- e2e through the C ABI with host buffers -------------------------------
    import torch as _t
    h_q = _t.from_numpy(np.ascontiguousarray(wl.q).view(np.int16)).pin_memory()
    h_k = _t.from_numpy(np.ascontiguousarray(wl.k_new).view(np.int16)).pin_memory()
    h_v = _t.from_numpy(np.ascontiguousarray(wl.v_new).view(np.int16)).pin_memory()
    h_loc = _t.from_numpy(wl.out_loc).pin_memory()
    h_sl = _t.from_numpy(wl.seq_lens).pin_memory()
    h_ti = _t.from_numpy(wl.table_idx).pin_memory()
    h_pt = _t.from_numpy(wl.page_table).pin_memory()
    h_out = _t.empty(out.shape, dtype=_t.int16).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (h_q, h_k, h_v, h_loc, h_sl, h_ti, h_pt))
    d2h = h_out.numel() * h_out.element_size()

    # Two sets of device buffers: the host->device copies of step k+1 run on
    # an upload stream while step k computes, and step k's output is read
    # back on a download stream.  Every step's inputs are copied and its
    # output read inside the timed region.
    # The step's inputs travel as one packed buffer (one copy per step): q,
    # k_new, v_new, out_loc, seq_lens, table_idx and the page table, each at
    # a 256-byte aligned offset; the device side takes typed views of it.
    parts = [("q", h_q, q), ("k", h_k, k_new), ("v", h_v, v_new), ("loc", h_loc, out_loc),
             ("sl", h_sl, seq_lens), ("ti", h_ti, table_idx), ("pt", h_pt, table.entries)]
    offs, total_b = {}, 0
    for name, h, _ in parts:
        offs[name] = total_b
        total_b += (h.numel() * h.element_size() + 255) // 256 * 256
    h_pack = _t.empty(total_b, dtype=_t.uint8).pin_memory()
    for name, h, _ in parts:
        nb = h.numel() * h.element_size()
        h_pack[offs[name]:offs[name] + nb].copy_(h.reshape(-1).view(_t.uint8))

    h2d = total_b  # the bytes actually copied per step (with alignment padding)

    def dev_set():
        buf = torch.empty(total_b, dtype=torch.uint8, device=dev)
        d = {"buf": buf, "out": torch.empty_like(out)}
        for name, h, like in parts:
            nb = h.numel() * h.element_size()
            d[name] = buf[offs[name]:offs[name] + nb].view(like.dtype).view(like.shape)
        d["table"] = api.PageTable(d["pt"])
        return d

    sets = [dev_set(), dev_set()]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    up_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]

    def upload(bi):
        d = sets[bi]
        up.wait_event(comp_done[bi])  # the set's previous step has finished with it
        with torch.cuda.stream(up):
            d["buf"].copy_(h_pack, non_blocking=True)
        up_done[bi].record(up)

    def e2e_run(nsteps):
        up.wait_stream(stream)
        upload(0)
        for k in range(nsteps):
            bi = k & 1
            d = sets[bi]
            if k + 1 < nsteps:
                upload(1 - bi)
            stream.wait_event(up_done[bi])
            stream.wait_event(down_done[bi])  # the previous read-back of this set's out
            for l in layers:
                api.store_kv(pool, l, d["k"], d["v"], d["loc"], err)
                api.decode_attn(pool, l, d["q"], d["table"], d["ti"], d["sl"], d["out"], ws,
                                scale=wl.scale, dev_err=err)
            comp_done[bi].record(stream)
            down.wait_event(comp_done[bi])
            with torch.cuda.stream(down):
                h_out.copy_(d["out"].view(_t.int16), non_blocking=True)
            down_done[bi].record(down)
        stream.wait_stream(up)
        stream.wait_stream(down)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_val = job_throughput(step_bytes, args.steps, e2e_ms, world) / 1e9

    result = {
        "metric": "paged decode-attn KV GB/s",
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_total / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8-e4m3 pool, bf16 q/out" if fp8 else "bf16",
        "data": ("synthetic (seeded random E4M3 codes in the pool, scales 0.05 / 0.09; bf16 q and new rows)"
                 if fp8 else
                 "synthetic (seeded PCG64 N(0,1) values rounded to bf16; K x0.5)" if wl.name.endswith("0.6b")
                 else "synthetic (seeded PCG64 N(0,1) block tiled over the pool)"),
        "config": {
            "workload": wl.name,
            "batch": wl.batch,
            "context_tokens": int(wl.seq_lens.sum()),
            "num_q_heads": wl.num_q_heads, "num_kv_heads": spec.num_kv_heads, "head_dim": 128,
            "page_size": spec.page_size, "pool_slots": spec.num_slots, "pool_layers": spec.num_layers,
            "layers_per_step": nL,
            "step": "store_kv + decode_attn (split partials + combine) per layer",
            "launch": launch_mode,
            "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"replicas x{world}",
        },
        "decode_tok_per_s_per_layer": round(world * wl.batch * args.steps * nL / (ms_total / 1e3), 1),
        "decode_call_us": round(dec_avg_ms * 1e3, 2),
        "store_kv_call_us": round(sum(st_ms) / len(st_ms) * 1e3, 2),
        "step_us": round(ms_total / args.steps * 1e3, 2),
        "eager_step_us": eager_us,
        "roofline": {
            "kernel": "decode_attn (decode_split_kernel + decode_combine_kernel, timed together)",
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": hbm,
            "peak_source": peak_src,
            "unit": "GB/s",
            "frac": round(achieved / hbm, 4),
            "traffic": traffic,
            "algorithmic_bytes_per_launch": per_call,
        },
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "pipeline": "one packed host->device copy per step; step k+1's copy overlaps step k; read-back on its own stream",
                "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * args.steps * nL,
        "device_error_word": errv,
        "clocks": clk,
    }
    if args.workload == "decode-qwen3-8b":
        result["config"]["alias_factor"] = round(getattr(wl, "alias_factor", 0.0), 3)

    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fp8:
        gbs, sample, _ = cpu_decode_sample(wl)
        result["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": blas_threads(),
                                  "kind": "oracle", "sample": sample}
    if not args.no_extend and args.workload == "decode-qwen3-0.6b":
        result["extend"] = run_extend_measure(dev, warmup=3, iters=max(5, args.steps), fp8=fp8)
        if not fp8:
            result["qk_norm_rope_store"] = run_rope_measure(dev, iters=max(5, args.steps))
    return result


def rope_bytes(n: int, hq: int, hkv: int, esize: int = 2) -> int:
    """Algorithmic bytes of one fused q/k norm + RoPE + store call: each token's
    qkv row read, its q row and its k and v rows written, its position, slot
    and cos/sin row read (the norm weights are negligible)."""
    row = (hq + 2 * hkv) * 128 * esize
    return n * (2 * row + 4 + 4 + 128 * 4)


def run_rope_measure(dev, iters=10, warmup=3):
    """The fused q/k norm + RoPE + store call on three shapes: this decode
    step's 64 tokens (Hq 16, Hkv 8), and 2048- and 16384-token prefill batches
    of the Qwen3-8B shape (Hq 32, Hkv 8).  L2 is flushed before every timed call."""
    import torch
    from paged_kv_gqa_scatter_b200 import api
    from paged_kv_gqa_scatter_b200 import workloads as W
    hbm, _, _, src = measured_peaks()
    # L2 flush by reading a 256 MB buffer: it leaves clean lines, so the timed
    # call does not pay for writing back a flush buffer's dirty ones.
    flush = torch.ones(64 << 20, dtype=torch.int32, device=dev)
    cache = torch.from_numpy(W.rotary_table(40960)).to(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(6)
    out = {}
    for name, n, hq, hkv in (("decode batch 64, Hq 16 Hkv 8", 64, 16, 8),
                             ("prefill chunk 2048, Hq 32 Hkv 8", 2048, 32, 8),
                             ("prefill batch 16384, Hq 32 Hkv 8", 16384, 32, 8)):
        row = (hq + 2 * hkv) * 128
        qkv = torch.randn(n, row, device=dev, generator=g).to(torch.bfloat16)
        slots = 4 * n
        pool = api.KVPool.empty(1, slots, hkv, device=dev)
        pos = torch.randint(0, 40960, (n,), device=dev, dtype=torch.int32, generator=g)
        loc = torch.randperm(slots, device=dev, generator=g)[:n].to(torch.int32)
        w = (1.0 + 0.1 * torch.randn(2, 128, device=dev, generator=g)).to(torch.bfloat16)
        q_out = torch.empty(n, hq, 128, device=dev, dtype=torch.bfloat16)
        err = torch.zeros(1, dtype=torch.int32, device=dev)

        def call():
            api.qk_norm_rope_store(pool, 0, qkv, hq, pos, cache, loc, q_out, w[0], w[1], 1e-6, err)
        for _ in range(warmup):
            call()
        s = torch.cuda.current_stream(dev)
        ts = []
        for _ in range(iters):
            flush.sum()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            call()
            b.record(s)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ts.sort()
        us = ts[len(ts) // 2] * 1e3
        nbytes = rope_bytes(n, hq, hkv)
        gbs = nbytes / us / 1e3
        out[name] = {"us": round(us, 3), "bytes": nbytes, "GB/s": round(gbs, 1),
                     "frac": round(gbs / hbm, 4), "peak": hbm, "peak_source": src,
                     "device_error_word": int(err.item())}
        if n == 16384:
            out[name]["traffic"] = recorded_traffic("qk_norm_rope_store_kernel",
                                                    source_hash("rope_store.cu", "common.cuh"),
                                                    "rope prefill 16384")
    return out


def run_extend_measure(dev, warmup=3, iters=10, fp8=False):
    """Extend TFLOP/s on the chunked-prefill step (2048-token chunk at prefix 6144,
    Hq 32, Hkv 8): causal FLOPs = 4 d Hq (e p + e (e+1) / 2).  fp8: the same
    chunk over an E4M3 copy of the pool."""
    import torch
    from paged_kv_gqa_scatter_b200 import api
    from paged_kv_gqa_scatter_b200 import workloads as W
    mix = W.chunked_prefill_step(step=3)
    wl = W.with_fp8_pool(mix.extend) if fp8 else mix.extend

    def tdev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    def tpool(a):
        if fp8:
            return torch.from_numpy(np.ascontiguousarray(a)).to(dev).view(torch.float8_e4m3fn)
        return tdev(a)

    spec = wl.pool
    pool = api.KVPool.empty(spec.num_layers, spec.num_slots, spec.num_kv_heads, device=dev,
                            dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16,
                            k_scale=spec.k_scale, v_scale=spec.v_scale)
    pool.k[0].copy_(tpool(wl.k_planes[0]))
    pool.v[0].copy_(tpool(wl.v_planes[0]))
    table = api.PageTable(torch.from_numpy(wl.page_table).to(dev))
    ti = torch.from_numpy(wl.table_idx).to(dev)
    pl = torch.from_numpy(wl.prefix_lens).to(dev)
    el = torch.from_numpy(wl.extend_lens).to(dev)
    qo = torch.from_numpy(wl.q_offsets).to(dev)
    q = tdev(wl.q)
    out = torch.empty_like(q)
    api.store_kv(pool, 0, tdev(wl.k_new), tdev(wl.v_new), torch.from_numpy(wl.out_loc).to(dev))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    mx = int(wl.extend_lens.max())
    for _ in range(warmup):
        api.extend_attn(pool, 0, q, table, ti, pl, el, qo, mx, out, scale=wl.scale, dev_err=err)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for a, b in evs:
        a.record(s)
        api.extend_attn(pool, 0, q, table, ti, pl, el, qo, mx, out, scale=wl.scale, dev_err=err)
        b.record(s)
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in evs)
    med = ms[len(ms) // 2]
    flops = 4 * 128 * wl.num_q_heads * wl.causal_pairs()
    _, bf16, _, src = measured_peaks()
    tf = flops / (med / 1e3) / 1e12
    return {"workload": "chunked-prefill extend, 2048-token chunk at prefix 6144, Hq 32 Hkv 8"
                        + (", E4M3 pool" if fp8 else ""),
            "tflops": round(tf, 2), "ms": round(med, 4), "flops": flops,
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": bf16,
                         "peak_source": src, "unit": "TFLOP/s", "frac": round(tf / bf16, 4),
                         "traffic": None if fp8 else recorded_traffic("extend_tc_kernel",
                                                                      source_hash("extend_tc.cu", "common.cuh"),
                                                                      "chunked-prefill extend c3")},
            "device_error_word": int(err.item())}


def _dev_pool(W, api, torch, wl, dev, layers):
    """Device pool for a workload: host plane contents copied to `layers`."""
    spec = wl.pool
    pool = api.KVPool.empty(spec.num_layers, spec.num_slots, spec.num_kv_heads,
                            page_size=spec.page_size, device=dev)
    src_layer = next(iter(wl.k_planes.keys()))
    hk = torch.from_numpy(np.ascontiguousarray(wl.k_planes[src_layer]).view(np.int16)).view(torch.bfloat16).to(dev)
    hv = torch.from_numpy(np.ascontiguousarray(wl.v_planes[src_layer]).view(np.int16)).view(torch.bfloat16).to(dev)
    for l in layers:
        pool.k[l].copy_(hk)
        pool.v[l].copy_(hv)
    return pool


def _flops_extend(wl):
    return 4 * 128 * wl.num_q_heads * wl.causal_pairs()


def run_chunked_prefill(args, world, rank, local):
    """One step = the four 2048-token chunks of one 8192-token prompt (prefix
    0, 2048, 4096, 6144), each with its store_kv and the 128-request decode
    batch at context 2048 (two calls per chunk on one stream)."""
    import torch
    from paged_kv_gqa_scatter_b200 import api
    from paged_kv_gqa_scatter_b200 import workloads as W
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    mix = W.chunked_prefill_step(step=3)
    ext, dec = mix.extend, mix.decode

    def tdev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    pool = _dev_pool(W, api, torch, ext, dev, [0])
    table = api.PageTable(torch.from_numpy(ext.page_table).to(dev))
    e_q, e_k, e_v = tdev(ext.q), tdev(ext.k_new), tdev(ext.v_new)
    e_ti = torch.from_numpy(ext.table_idx).to(dev)
    e_el = torch.from_numpy(ext.extend_lens).to(dev)
    e_qo = torch.from_numpy(ext.q_offsets).to(dev)
    row = ext.page_table[ext.table_idx[0]]
    chunk = int(ext.extend_lens[0])
    e_loc = [torch.from_numpy(row[c * chunk:(c + 1) * chunk].astype(np.int32)).to(dev) for c in range(4)]
    e_pl = [torch.tensor([c * chunk], dtype=torch.int32, device=dev) for c in range(4)]
    e_out = torch.empty_like(e_q)
    d_q, d_k, d_v = tdev(dec.q), tdev(dec.k_new), tdev(dec.v_new)
    d_ti = torch.from_numpy(dec.table_idx).to(dev)
    d_sl = torch.from_numpy(dec.seq_lens).to(dev)
    d_loc = torch.from_numpy(dec.out_loc).to(dev)
    d_out = torch.empty_like(d_q)
    ws = api.decode_workspace(dec.batch, dec.num_q_heads, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream(dev)
    evs = []

    def step(record):
        for c in range(4):
            es = [torch.cuda.Event(enable_timing=True) for _ in range(3)] if record else None
            api.store_kv(pool, 0, e_k, e_v, e_loc[c], err)
            api.store_kv(pool, 0, d_k, d_v, d_loc, err)
            if record: es[0].record(s)
            api.extend_attn(pool, 0, e_q, table, e_ti, e_pl[c], e_el, e_qo, chunk, e_out,
                            scale=ext.scale, dev_err=err)
            if record: es[1].record(s)
            api.decode_attn(pool, 0, d_q, table, d_ti, d_sl, d_out, ws, scale=dec.scale, dev_err=err)
            if record:
                es[2].record(s)
                evs.append(es)

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    start.record(s)
    for _ in range(args.steps):
        step(True)
    stop.record(s)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(start.elapsed_time(stop), world)
    ext_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    pairs = sum(chunk * (c * chunk) + chunk * (chunk + 1) // 2 for c in range(4))
    ext_flops = 4 * 128 * ext.num_q_heads * pairs * args.steps
    dec_bytes = decode_bytes(dec) * 4 * args.steps
    _, bf16, _, src = measured_peaks()
    hbm, _, _, hsrc = measured_peaks()
    tf = ext_flops / (ext_ms / 1e3) / 1e12
    gbs = dec_bytes / (dec_ms / 1e3) / 1e9
    return {
        "metric": "chunked-prefill step: extend-attn TFLOP/s",
        "value": round(world * tf, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded PCG64 N(0,1) values rounded to bf16)",
        "config": {"workload": "chunked-prefill", "prompt": 8192, "chunk": chunk,
                   "decode_batch": dec.batch, "decode_context": int(dec.seq_lens[0]),
                   "num_q_heads": ext.num_q_heads, "num_kv_heads": ext.pool.num_kv_heads,
                   "step": "4 chunks x (store_kv chunk + decode rows, extend_attn, decode_attn)",
                   "parallelism": f"replicas x{world}"},
        "extend": {"tflops": round(tf, 2), "ms_per_step": round(ext_ms / args.steps, 4),
                   "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": bf16,
                                "peak_source": src, "unit": "TFLOP/s", "frac": round(tf / bf16, 4)}},
        "decode": {"gbs": round(gbs, 1), "ms_per_step": round(dec_ms / args.steps, 4),
                   "tok_per_s_per_layer": round(dec.batch * 4 * args.steps / (dec_ms / 1e3), 1),
                   "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm,
                                "peak_source": hsrc, "unit": "GB/s", "frac": round(gbs / hbm, 4)}},
        "gpu_launches": args.steps * 4 * 5,
        "device_error_word": int(err.item()),
        "clocks": clk,
    }


def radix_unique_bytes(dec) -> int:
    """Bytes a decode step must read at least once: the shared prefix's K/V
    once, every request's own tokens, its table entries, q and out."""
    row = dec.pool.num_kv_heads * 128 * 2 * 2
    own = int((dec.seq_lens.astype(np.int64) - 4096).sum())
    return (4096 + own) * row + int(dec.seq_lens.astype(np.int64).sum()) * 4 + 2 * dec.q.size * 2


def run_radix(args, world, rank, local):
    """Radix shared-prefix serving on a 32-layer pool: one step = the extend of
    all 256 suffixes on every layer (store_kv + extend_attn per layer), then
    decode step 1 on every layer (store_kv + decode, per layer).  The decode
    is the cascade call (the shared prefix attended once for the whole batch)
    unless --radix-decode plain; the other form is timed beside the step on
    two layers for comparison."""
    import torch
    from paged_kv_gqa_scatter_b200 import api
    from paged_kv_gqa_scatter_b200 import workloads as W
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    # --pool-layers below 32 shrinks the pool (and the layers stepped) for
    # profiling; the per-layer work is unchanged.
    rs = W.radix_shared_prefix(num_layers=32 if args.pool_layers is None else min(32, args.pool_layers))
    ext = rs.extend
    dec = rs.decode_step(1)
    L = ext.pool.num_layers

    def tdev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    pool = _dev_pool(W, api, torch, ext, dev, range(L))
    table = api.PageTable(torch.from_numpy(ext.page_table).to(dev))
    e_q, e_k, e_v = tdev(ext.q), tdev(ext.k_new), tdev(ext.v_new)
    e_ti = torch.from_numpy(ext.table_idx).to(dev)
    e_pl = torch.from_numpy(ext.prefix_lens).to(dev)
    e_el = torch.from_numpy(ext.extend_lens).to(dev)
    e_qo = torch.from_numpy(ext.q_offsets).to(dev)
    e_loc = torch.from_numpy(ext.out_loc).to(dev)
    e_out = torch.empty_like(e_q)
    mx = int(ext.extend_lens.max())
    d_q, d_k, d_v = tdev(dec.q), tdev(dec.k_new), tdev(dec.v_new)
    d_ti = torch.from_numpy(dec.table_idx).to(dev)
    d_sl = torch.from_numpy(dec.seq_lens).to(dev)
    d_loc = torch.from_numpy(dec.out_loc).to(dev)
    d_out = torch.empty_like(d_q)
    ws = api.decode_workspace(dec.batch, dec.num_q_heads, device=dev)
    g_off = torch.tensor([0, dec.batch], dtype=torch.int32, device=dev)
    g_pre = torch.tensor([4096], dtype=torch.int32, device=dev)
    cws = api.decode_cascade_workspace(dec.batch, dec.num_q_heads, 4096, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream(dev)
    ext_ev, dec_ev = [], []
    cascade = args.radix_decode == "cascade"

    def decode(l, use_cascade):
        if use_cascade:
            api.decode_attn_cascade(pool, l, d_q, table, d_ti, d_sl, g_off, g_pre, 4096, d_out, cws,
                                    scale=dec.scale, dev_err=err)
        else:
            api.decode_attn(pool, l, d_q, table, d_ti, d_sl, d_out, ws, scale=dec.scale, dev_err=err)

    def step(record):
        for l in range(L):
            api.store_kv(pool, l, e_k, e_v, e_loc, err)
            a = torch.cuda.Event(enable_timing=True) if record else None
            b = torch.cuda.Event(enable_timing=True) if record else None
            if record: a.record(s)
            api.extend_attn(pool, l, e_q, table, e_ti, e_pl, e_el, e_qo, mx, e_out, scale=ext.scale, dev_err=err)
            if record:
                b.record(s)
                ext_ev.append((a, b))
        for l in range(L):
            api.store_kv(pool, l, d_k, d_v, d_loc, err)
            a = torch.cuda.Event(enable_timing=True) if record else None
            b = torch.cuda.Event(enable_timing=True) if record else None
            if record: a.record(s)
            decode(l, cascade)
            if record:
                b.record(s)
                dec_ev.append((a, b))

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    start.record(s)
    for _ in range(args.steps):
        step(True)
    stop.record(s)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(start.elapsed_time(stop), world)
    ext_ms = sum(a.elapsed_time(b) for a, b in ext_ev)
    dec_ms = sum(a.elapsed_time(b) for a, b in dec_ev)
    # The other decode form on layers 0 and L-1, outside the timed step.
    other = []
    for l in (0, L - 1):
        for rep_i in range(4):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            decode(l, not cascade)
            b.record(s)
            if rep_i > 0:
                other.append((a, b))
    torch.cuda.synchronize()
    other_ms = sorted(a.elapsed_time(b) for a, b in other)[len(other) // 2]
    ext_flops = _flops_extend(ext) * L * args.steps
    logical = decode_bytes(dec) * L * args.steps
    _, bf16, _, src = measured_peaks()
    hbm, _, _, hsrc = measured_peaks()
    tf = ext_flops / (ext_ms / 1e3) / 1e12
    return {
        "metric": "radix shared-prefix: extend-attn TFLOP/s",
        "value": round(world * tf, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded PCG64 N(0,1) values rounded to bf16; per-layer inputs reused)",
        "config": {"workload": "radix-prefix", "layers": L, "batch": ext.batch, "prefix": 4096,
                   "suffix_tokens": ext.total_q, "num_q_heads": ext.num_q_heads,
                   "num_kv_heads": ext.pool.num_kv_heads,
                   "step": ("per layer store_kv + extend_attn, then per layer store_kv + "
                            + ("decode_attn_cascade" if cascade else "decode_attn") + " (decode step 1)"),
                   "parallelism": f"replicas x{world}"},
        "extend": {"tflops": round(tf, 2), "ms_per_layer": round(ext_ms / (L * args.steps), 4),
                   "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": bf16,
                                "peak_source": src, "unit": "TFLOP/s", "frac": round(tf / bf16, 4)}},
        "decode": {"call": "decode_attn_cascade" if cascade else "decode_attn",
                   "ms_per_layer": round(dec_ms / (L * args.steps), 4),
                   "tok_per_s_per_layer": round(dec.batch * L * args.steps / (dec_ms / 1e3), 1),
                   "logical_gbs": round(logical / (dec_ms / 1e3) / 1e9, 1),
                   "unique_bytes_per_layer": radix_unique_bytes(dec),
                   "prefix_flops_per_layer": 4 * 128 * dec.num_q_heads * dec.batch * 4096,
                   "other_call": "decode_attn" if cascade else "decode_attn_cascade",
                   "other_ms_per_layer": round(other_ms, 4),
                   "note": "logical bytes count the shared 4096-token prefix once per request"},
        "gpu_launches": args.steps * L * (2 + (5 if cascade else 3)),
        "device_error_word": int(err.item()),
        "clocks": clk,
    }


# ---------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, world, rank):
    from paged_kv_gqa_scatter_b200 import workloads as W
    if rank != 0:
        return None
    wl = W.decode_qwen3_06b()
    budget = float(os.environ.get("PKV_REF_STEP_SECONDS", "4"))
    for _ in range(args.warmup):
        cpu_decode_sample(wl, budget_s=0.5)
    vals, secs, sample = [], 0.0, ""
    for _ in range(args.steps):
        v, sample, dt = cpu_decode_sample(wl, budget_s=budget)
        vals.append(v)
        secs += dt
    value = statistics.median(vals)
    cores = blas_threads()
    return {
        "impl": "reference",
        "metric": "paged decode-attn KV GB/s",
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded PCG64 N(0,1) values rounded to bf16; K x0.5)",
        "config": {"workload": wl.name, "batch": wl.batch, "num_q_heads": wl.num_q_heads,
                   "num_kv_heads": wl.pool.num_kv_heads, "head_dim": 128, "page_size": 1,
                   "pool_slots": wl.pool.num_slots, "pool_layers": wl.pool.num_layers},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample + f"; {budget:.0f} s per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode-qwen3-0.6b",
                    choices=["decode-qwen3-0.6b", "decode-qwen3-8b", "chunked-prefill", "radix-prefix"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pool-layers", type=int, default=None,
                    help="pool layers of decode-qwen3-0.6b (28) or radix-prefix (32); fewer only for profiling")
    ap.add_argument("--no-extend", action="store_true")
    ap.add_argument("--page-size", type=int, default=None,
                    help="page size of decode-qwen3-8b (16 as stated; 64 is TRT-LLM's size)")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="pool element type of decode-qwen3-0.6b (fp8: scaled E4M3 codes, bf16 q/out)")
    ap.add_argument("--radix-decode", choices=["cascade", "plain"], default="cascade",
                    help="decode call of the radix-prefix workload's step")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    world, rank, local = dist_setup()
    if args.workload == "chunked-prefill":
        res = run_chunked_prefill(args, world, rank, local)
    elif args.workload == "radix-prefix":
        res = run_radix(args, world, rank, local)
    else:
        res = run_decode(args, world, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
