"""Benchmark of the paged KV pool hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload all|decode-qwen3-8b|decode-qwen3-0.6b|chunked-prefill|radix-prefix]

Default (``--workload all``) prints ONE JSON line.  Its headline is the
largest single-GPU decode workload, the Qwen3-8B-shaped batch: 256 requests
with contexts log-uniform in [1k, 32k], Hq 32, Hkv 8, d 128, bf16, page_size
16, over a 36-layer pool.  One step is store_kv of the 256 new tokens plus
decode_attn (split-KV partials + combine) on every one of the 36 layers.  The
metric is decode KV GB/s: the K/V bytes of every context token (all KV
heads, both planes) plus page-table, query and output bytes, over device
time.  Every layer reads about 9 GB, far more than L2, so there is no flush.

The other workloads ride along in the same line, under "workloads", each
with its own roofline and float64-oracle CPU baseline:
  * decode-qwen3-0.6b: 64 requests, contexts U[512, 4096], Hq 16, one layer of
    a 28-layer, 300k-slot pool (page_size 1);
  * chunked-prefill: the four 2048-token chunks of an 8192-token prompt (Hq 32,
    Hkv 8), each with its store_kv, plus the 128-request decode batch at 2k;
  * radix-prefix: 256 requests sharing a 4096-token prefix on a 32-layer pool;
    the extend of every suffix on every layer, then decode step 1 (cascade).
``--workload X`` prints workload X alone as its own line (for profiling).

Under torchrun each rank runs an independent replica on its own GPU (the
path needs no collective); value = total bytes of all ranks / max-over-ranks
time, "scaling": "weak".

``--impl reference`` times the float64 CPU oracle on bounded samples of the
headline workload and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
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
NOMINAL_HBM_GBS = 8000.0  # B200 nominal HBM3e bandwidth; decode is also reported against it


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
    """Per-launch DRAM bytes of `kernel` on `workload` from the committed ncu
    summaries, or None when the kernel's source has changed since the counters
    were taken or no capture of that workload exists."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        for key in (f"{kernel}@{workload}", kernel):
            e = d.get(key)
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
# algorithmic work per call
# ---------------------------------------------------------------------------
ESIZE = {"bf16": 2, "f32": 4, "fp8": 1}


def decode_bytes(wl) -> int:
    """Algorithmic bytes of one decode_attn call: every context token's K and V
    rows (all KV heads), its page-table entry (one per token at page_size 1, one
    per page otherwise), the queries and the outputs, and the lengths and
    table-row indices."""
    B, Hq = wl.batch, wl.num_q_heads
    esz = ESIZE[wl.pool.dtype]
    io = ESIZE[wl.pool.io_dtype]
    n = wl.seq_lens.astype(np.int64)
    row = wl.pool.num_kv_heads * 128 * esz
    P = wl.pool.page_size
    table = int(n.sum()) * 4 if P == 1 else int(((n + P - 1) // P).sum()) * 4
    return int(n.sum()) * 2 * row + table + 2 * B * Hq * 128 * io + 8 * B


def store_bytes(n_tokens: int, spec) -> int:
    """Read each new K and V row (row dtype), write it to the pool (pool
    dtype), read its slot index."""
    row_in = spec.num_kv_heads * 128 * ESIZE[spec.io_dtype]
    row_out = spec.num_kv_heads * 128 * ESIZE[spec.dtype]
    return n_tokens * (2 * (row_in + row_out) + 4)


def extend_flops(num_q_heads: int, pairs: int) -> int:
    """Causal extend FLOPs: QK^T and PV over the unmasked (query, key) pairs,
    2 FLOPs per multiply-add, head_dim 128."""
    return 4 * 128 * num_q_heads * int(pairs)


def rope_bytes(n: int, hq: int, hkv: int, esize: int = 2) -> int:
    """Algorithmic bytes of one fused q/k norm + RoPE + store call: each token's
    qkv row read, its q row and its k and v rows written, its position, slot
    and cos/sin row read (the norm weights are negligible)."""
    row = (hq + 2 * hkv) * 128 * esize
    return n * (2 * row + 4 + 4 + 128 * 4)


# ---------------------------------------------------------------------------
# CPU baselines: the float64 oracle on the host cores, on bounded samples
# ---------------------------------------------------------------------------
def cpu_decode_sample(wl, requests, layers, budget_s: float):
    """Time oracle decode_attn request by request on `layers` until the
    requests are done or `budget_s` has passed; return (GB/s over the sample's
    metric bytes, sample description, seconds, bytes, requests done)."""
    import oracle
    esz = ESIZE[wl.pool.dtype]
    row = wl.pool.num_kv_heads * 128 * esz
    P = wl.pool.page_size
    done, nbytes, ntok = 0, 0, 0
    t0 = time.perf_counter()
    stop = False
    for layer in layers:
        for r in requests:
            oracle.decode_attn(wl.q, wl.k_planes, wl.v_planes, layer, wl.page_table, wl.table_idx,
                               wl.seq_lens, P, wl.scale, requests=[r])
            n = int(wl.seq_lens[r])
            table = n * 4 if P == 1 else (n + P - 1) // P * 4
            nbytes += n * 2 * row + table + 2 * wl.num_q_heads * 128 * 2 + 8
            ntok += n
            done += 1
            if time.perf_counter() - t0 > budget_s:
                stop = True
                break
        if stop:
            break
    dt = time.perf_counter() - t0
    desc = (f"oracle decode_attn (float64 numpy) on {done} (request, layer) pairs of "
            f"{wl.batch} requests x layers {list(layers)}: {ntok} KV tokens, {nbytes / 1e6:.1f} MB")
    return nbytes / dt / 1e9, desc, dt, nbytes, done


def cpu_extend_sample(wl, chunks, rows_per_chunk: int, budget_s: float, seed: int):
    """Time oracle extend_attn on sampled query rows.  `chunks` lists
    (prefix_len, extend_len, q_offset, table_row) of the chunks to sample;
    returns (TFLOP/s over the sampled rows' causal FLOPs, description, s)."""
    import oracle
    rng = np.random.default_rng(seed)
    flops, nrows = 0, 0
    t0 = time.perf_counter()
    for (p, e, qo, trow) in chunks:
        i = np.sort(rng.choice(e, size=min(rows_per_chunk, e), replace=False))
        oracle.extend_attn(wl.q[qo:qo + e], wl.k_planes, wl.v_planes, wl.layer, wl.page_table,
                           np.array([trow], np.int32), np.array([p], np.int32),
                           np.array([e], np.int32), np.array([0, e], np.int32),
                           wl.pool.page_size, wl.scale, rows=i)
        flops += extend_flops(wl.num_q_heads, int((p + i + 1).sum()))
        nrows += len(i)
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    desc = (f"oracle extend_attn (float64 numpy) on {nrows} sampled query rows of "
            f"{len(chunks)} chunk(s); TFLOP/s over those rows' causal FLOPs")
    return flops / dt / 1e12, desc, dt


def cpu_baseline_obj(value, unit, sample, extrapolated=None):
    d = {"value": round(value, 6), "unit": unit, "cores": blas_threads(), "kind": "oracle",
         "sample": sample}
    if extrapolated:
        d["extrapolated"] = extrapolated
    return d


# ---------------------------------------------------------------------------
# device set-up helpers
# ---------------------------------------------------------------------------
def tdev(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)


def device_pool(api, torch, wl, dev, layers):
    """Device pool of a workload's shape with the host contents of `layers`
    (TiledPlane pools: every layer, from the repeated block)."""
    from paged_kv_gqa_scatter_b200 import workloads as W
    spec = wl.pool
    fp8 = spec.dtype == "fp8"
    tiled = isinstance(wl.k_planes, W.TiledPlane)
    pool = api.KVPool.empty(spec.num_layers, spec.num_slots, spec.num_kv_heads, page_size=spec.page_size,
                            device=dev, zero=not tiled,
                            dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16,
                            k_scale=spec.k_scale, v_scale=spec.v_scale)

    def tpool(a):
        if fp8:
            return torch.from_numpy(np.ascontiguousarray(a)).to(dev).view(torch.float8_e4m3fn)
        return tdev(a, dev)

    if tiled:
        for plane, dst in ((wl.k_planes, pool.k), (wl.v_planes, pool.v)):
            blk = tpool(plane.block)
            flat = dst.view(-1, spec.num_kv_heads, 128)
            nb = blk.shape[0]
            for s in range(0, flat.shape[0], nb):
                m = min(nb, flat.shape[0] - s)
                flat[s:s + m].copy_(blk[:m])
    else:
        src = list(wl.k_planes.keys())
        for l in layers:
            sl = l if l in wl.k_planes else src[0]
            pool.k[l].copy_(tpool(wl.k_planes[sl]))
            pool.v[l].copy_(tpool(wl.v_planes[sl]))
    torch.cuda.synchronize()
    return pool


def capture(torch, dev, fn, warm: int):
    """Capture fn() once in a CUDA graph on a side stream and replay it `warm`
    times; None if capture is not possible."""
    try:
        gs = torch.cuda.Stream(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gs):
            fn()
        for _ in range(warm):
            g.replay()
        torch.cuda.synchronize()
        return g
    except Exception:
        return None


def time_replays(torch, stream, g, fn, n: int) -> float:
    """Device ms of n back-to-back replays of graph g (or n eager calls of fn
    when g is None), events on the launching stream."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        if g is not None:
            g.replay()
        else:
            fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def free_device(torch):
    import gc
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# decode workloads (the headline and the Qwen3-0.6B step)
# ---------------------------------------------------------------------------
def qwen3_8b_workload(args, free_bytes):
    """The Qwen3-8B decode batch at its fixed pool size (0.6 x free memory if
    that does not fit); returns (workload, pool note)."""
    from paged_kv_gqa_scatter_b200 import workloads as W
    P = args.page_size or 16
    nl = 36 if args.pool_layers is None else max(1, min(36, args.pool_layers))
    pages = W.QWEN3_8B_POOL_PAGES * 16 // P
    note = f"fixed {pages} pages of {P} slots"
    if nl * pages * P * 4096 > 0.9 * free_bytes:
        pages = int(0.6 * free_bytes // (nl * P * 4096))
        note = f"{pages} pages of {P} slots (0.6 x free memory; the fixed size did not fit)"
    wl = W.decode_qwen3_8b(num_pages=pages, page_size=P, num_layers=nl)
    if P != 16:
        wl.name = f"decode-qwen3-8b-p{P}"
    return wl, note


def run_decode(args, world, rank, local, name):
    import torch
    from paged_kv_gqa_scatter_b200 import api
    from paged_kv_gqa_scatter_b200 import workloads as W

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if name == "decode-qwen3-8b":
        free, _ = torch.cuda.mem_get_info()
        wl, pool_note = qwen3_8b_workload(args, free)
        if args.kv_dtype == "fp8":
            wl = W.with_fp8_pool(wl)
        layers = list(range(wl.pool.num_layers))
    else:
        nl = 28 if args.pool_layers is None else args.pool_layers
        wl = W.decode_qwen3_06b(num_layers=nl, layer=min(13, nl - 1))
        pool_note = "fixed 300,000 slots"
        if args.kv_dtype == "fp8":
            wl = W.with_fp8_pool(wl)
        layers = [wl.layer]
    spec = wl.pool
    fp8 = spec.dtype == "fp8"
    nL = len(layers)
    pool = device_pool(api, torch, wl, dev, layers)
    table = api.PageTable(torch.from_numpy(wl.page_table).to(dev))
    table_idx = torch.from_numpy(wl.table_idx).to(dev)
    seq_lens = torch.from_numpy(wl.seq_lens).to(dev)
    q, k_new, v_new = tdev(wl.q, dev), tdev(wl.k_new, dev), tdev(wl.v_new, dev)
    out_loc = torch.from_numpy(wl.out_loc).to(dev)
    out = torch.empty_like(q)
    ws = api.decode_workspace(wl.batch, wl.num_q_heads, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def store_all():
        for l in layers:
            api.store_kv(pool, l, k_new, v_new, out_loc, err)

    def decode_all():
        for l in layers:
            api.decode_attn(pool, l, q, table, table_idx, seq_lens, out, ws, scale=wl.scale, dev_err=err)

    def step():
        for l in layers:
            api.store_kv(pool, l, k_new, v_new, out_loc, err)
            api.decode_attn(pool, l, q, table, table_idx, seq_lens, out, ws, scale=wl.scale, dev_err=err)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # The step as the serving engine runs decode: captured once in a CUDA graph
    # (fixed buffers) and replayed.  Decode-only and store-only graphs give the
    # per-call kernel times for the roofline without events between the calls.
    g_step = capture(torch, dev, step, args.warmup)
    g_dec = capture(torch, dev, decode_all, 2)
    g_store = capture(torch, dev, store_all, 2)
    launch_mode = "cuda graph replay of one step" if g_step is not None else "eager (graph capture failed)"

    # ---- timed region: exactly K steps ----------------------------------------
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    ms_total = time_replays(torch, stream, g_step, step, args.steps)
    barrier(world)
    clk = clocks.stop()
    ms_total = max_over_ranks(ms_total, world)

    # ---- kernel times for the roofline: decode-only and store-only replays ----
    dec_ms = time_replays(torch, stream, g_dec, decode_all, args.steps) / (args.steps * nL)
    st_ms = time_replays(torch, stream, g_store, store_all, args.steps) / (args.steps * nL)
    eager_us = time_replays(torch, stream, None, step, args.steps) / args.steps * 1e3
    errv = int(err.item())

    per_call = decode_bytes(wl)
    st_b = store_bytes(wl.batch, spec)
    step_bytes = nL * (per_call + st_b)
    value = job_throughput(step_bytes, args.steps, ms_total, world) / 1e9
    hbm, _, _, peak_src = measured_peaks()
    achieved = per_call / (dec_ms / 1e3) / 1e9
    traffic = recorded_traffic("decode_split_kernel", source_hash("decode.cu", "common.cuh"), wl.name)

    # ---- e2e through the C ABI with host buffers -------------------------------
    e2e = run_decode_e2e(args, world, dev, stream, wl, pool, layers, ws, err, q, k_new, v_new,
                         out_loc, seq_lens, table_idx, table, out, step_bytes)

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
                 else "synthetic (seeded PCG64 N(0,1) block of 65,536 slots tiled over the pool)"),
        "config": {
            "workload": wl.name,
            "batch": wl.batch,
            "context_tokens": int(wl.seq_lens.sum()),
            "num_q_heads": wl.num_q_heads, "num_kv_heads": spec.num_kv_heads, "head_dim": 128,
            "page_size": spec.page_size, "pool_slots": spec.num_slots, "pool_layers": spec.num_layers,
            "pool": pool_note,
            "layers_per_step": nL,
            "step": "store_kv + decode_attn (split partials + combine) per layer",
            "launch": launch_mode,
            "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"replicas x{world}",
        },
        "decode_tok_per_s_per_layer": round(world * wl.batch * args.steps * nL / (ms_total / 1e3), 1),
        "decode_call_us": round(dec_ms * 1e3, 2),
        "store_kv_call_us": round(st_ms * 1e3, 2),
        "store_kv_gbs": round(st_b / (st_ms / 1e3) / 1e9, 1),
        "step_us": round(ms_total / args.steps * 1e3, 2),
        "eager_step_us": round(eager_us, 2),
        "roofline": {
            "kernel": "decode_attn (decode_split_kernel + decode_combine_kernel), timed from "
                      "back-to-back replays of a graph of the step's decode calls",
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": hbm,
            "peak_source": peak_src,
            "unit": "GB/s",
            "frac": round(achieved / hbm, 4),
            "frac_of_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
            "traffic": traffic,
            "algorithmic_bytes_per_launch": per_call,
        },
        "e2e": e2e,
        "gpu_launches": 3 * args.steps * nL,
        "device_error_word": errv,
        "clocks": clk,
    }
    if name == "decode-qwen3-8b":
        result["config"]["alias_factor"] = round(getattr(wl, "alias_factor", 0.0), 3)

    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fp8:
        if name == "decode-qwen3-8b":
            # 16 requests (the longest included, the rest seeded), the first
            # and last layers; the rate is per KV byte, so the whole step's
            # oracle time extrapolates linearly in KV tokens.
            rng = np.random.default_rng(8)
            longest = int(np.argmax(wl.seq_lens))
            others = [int(x) for x in rng.choice(wl.batch, 15, replace=False) if int(x) != longest][:15]
            sample = [longest] + others
            gbs, desc, dt, nb, _ = cpu_decode_sample(wl, sample, [layers[0], layers[-1]], budget_s=20.0)
            step_s = step_bytes / (gbs * 1e9)
            result["cpu_baseline"] = cpu_baseline_obj(
                gbs, "GB/s", desc,
                extrapolated=f"per KV byte to the whole {nL}-layer step: {step_s:.0f} s per step")
        else:
            gbs, desc, dt, nb, _ = cpu_decode_sample(wl, range(wl.batch), layers, budget_s=8.0)
            result["cpu_baseline"] = cpu_baseline_obj(gbs, "GB/s", desc)
    del pool, g_step, g_dec, g_store
    free_device(torch)
    return result


def run_decode_e2e(args, world, dev, stream, wl, pool, layers, ws, err, q, k_new, v_new, out_loc,
                   seq_lens, table_idx, table, out, step_bytes):
    """The decode step through the public API with host buffers: every step
    copies its inputs (q, the new K/V rows, out_loc, seq_lens, table_idx and
    the page table) from pinned host memory and reads the step's output back,
    inside the timed region.  The copies are pipelined as an engine would:
    one packed pinned buffer per step, two device buffer sets, step k+1's
    upload on its own stream while step k computes, the read-back on a third
    stream."""
    import torch
    from paged_kv_gqa_scatter_b200 import api
    h_q = torch.from_numpy(np.ascontiguousarray(wl.q).view(np.int16)).pin_memory()
    h_k = torch.from_numpy(np.ascontiguousarray(wl.k_new).view(np.int16)).pin_memory()
    h_v = torch.from_numpy(np.ascontiguousarray(wl.v_new).view(np.int16)).pin_memory()
    h_loc = torch.from_numpy(wl.out_loc).pin_memory()
    h_sl = torch.from_numpy(wl.seq_lens).pin_memory()
    h_ti = torch.from_numpy(wl.table_idx).pin_memory()
    h_pt = torch.from_numpy(wl.page_table).pin_memory()
    h_out = torch.empty(out.shape, dtype=torch.int16).pin_memory()
    d2h = h_out.numel() * h_out.element_size()
    parts = [("q", h_q, q), ("k", h_k, k_new), ("v", h_v, v_new), ("loc", h_loc, out_loc),
             ("sl", h_sl, seq_lens), ("ti", h_ti, table_idx), ("pt", h_pt, table.entries)]
    offs, total_b = {}, 0
    for nm, h, _ in parts:
        offs[nm] = total_b
        total_b += (h.numel() * h.element_size() + 255) // 256 * 256
    h_pack = torch.empty(total_b, dtype=torch.uint8).pin_memory()
    for nm, h, _ in parts:
        nb = h.numel() * h.element_size()
        h_pack[offs[nm]:offs[nm] + nb].copy_(h.reshape(-1).view(torch.uint8))

    def dev_set():
        buf = torch.empty(total_b, dtype=torch.uint8, device=dev)
        d = {"buf": buf, "out": torch.empty_like(out)}
        for nm, h, like in parts:
            nb = h.numel() * h.element_size()
            d[nm] = buf[offs[nm]:offs[nm] + nb].view(like.dtype).view(like.shape)
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
                h_out.copy_(d["out"].view(torch.int16), non_blocking=True)
            down_done[bi].record(down)
        stream.wait_stream(up)
        stream.wait_stream(down)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_val = job_throughput(step_bytes, args.steps, e2e_ms, world) / 1e9
    return {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": total_b,
            "d2h_bytes_per_step": d2h,
            "pipeline": "one packed host->device copy per step (q, new K/V rows, out_loc, seq_lens, "
                        "table_idx, page table); step k+1's copy overlaps step k; the step's output "
                        "(last layer) read back on its own stream"}


# ---------------------------------------------------------------------------
# chunked prefill (extend) and radix shared-prefix serving
# ---------------------------------------------------------------------------
def run_chunked_prefill(args, world, rank, local):
    """One step = the four 2048-token chunks of one 8192-token prompt (prefix
    0, 2048, 4096, 6144), each with its store_kv, then the 128-request decode
    batch at context 2048 (store_kv of its new rows, decode_attn): two
    attention calls per chunk on one stream."""
    import torch
    from paged_kv_gqa_scatter_b200 import api
    from paged_kv_gqa_scatter_b200 import workloads as W
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    mix = W.chunked_prefill_step(step=3)
    ext, dec = mix.extend, mix.decode
    pool = device_pool(api, torch, ext, dev, [0])
    table = api.PageTable(torch.from_numpy(ext.page_table).to(dev))
    e_q, e_k, e_v = tdev(ext.q, dev), tdev(ext.k_new, dev), tdev(ext.v_new, dev)
    e_ti = torch.from_numpy(ext.table_idx).to(dev)
    e_el = torch.from_numpy(ext.extend_lens).to(dev)
    e_qo = torch.from_numpy(ext.q_offsets).to(dev)
    row = ext.page_table[ext.table_idx[0]]
    chunk = int(ext.extend_lens[0])
    e_loc = [torch.from_numpy(row[c * chunk:(c + 1) * chunk].astype(np.int32)).to(dev) for c in range(4)]
    e_pl = [torch.tensor([c * chunk], dtype=torch.int32, device=dev) for c in range(4)]
    e_out = torch.empty_like(e_q)
    d_q, d_k, d_v = tdev(dec.q, dev), tdev(dec.k_new, dev), tdev(dec.v_new, dev)
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
            es = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if record else None
            if record: es[0].record(s)
            api.store_kv(pool, 0, e_k, e_v, e_loc[c], err)
            if record: es[1].record(s)
            api.extend_attn(pool, 0, e_q, table, e_ti, e_pl[c], e_el, e_qo, chunk, e_out,
                            scale=ext.scale, dev_err=err)
            if record: es[2].record(s)
            api.store_kv(pool, 0, d_k, d_v, d_loc, err)
            api.decode_attn(pool, 0, d_q, table, d_ti, d_sl, d_out, ws, scale=dec.scale, dev_err=err)
            if record:
                es[3].record(s)
                evs.append((c, es))

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
    st_ms = sum(e[0].elapsed_time(e[1]) for _, e in evs)
    per_chunk_ms = [0.0] * 4
    for c, e in evs:
        per_chunk_ms[c] += e[1].elapsed_time(e[2])
    ext_ms = sum(per_chunk_ms)
    dec_ms = sum(e[2].elapsed_time(e[3]) for _, e in evs)
    pairs = [chunk * (c * chunk) + chunk * (chunk + 1) // 2 for c in range(4)]
    ext_flops = extend_flops(ext.num_q_heads, sum(pairs)) * args.steps
    dec_bytes = (decode_bytes(dec) + store_bytes(dec.batch, dec.pool)) * 4 * args.steps
    hbm, bf16, _, src = measured_peaks()
    tf = ext_flops / (ext_ms / 1e3) / 1e12
    gbs = dec_bytes / (dec_ms / 1e3) / 1e9
    st_gbs = store_bytes(chunk, ext.pool) * 4 * args.steps / (st_ms / 1e3) / 1e9
    chunks = {}
    for c in range(4):
        t = per_chunk_ms[c] / args.steps
        f = extend_flops(ext.num_q_heads, pairs[c])
        chunks[f"c{c} (prefix {c * chunk})"] = {"ms": round(t, 4), "tflops": round(f / (t / 1e3) / 1e12, 1)}
    res = {
        "metric": "chunked-prefill step: extend-attn TFLOP/s",
        "value": round(world * tf, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "dtype": "bf16",
        "data": "synthetic (seeded PCG64 N(0,1) values rounded to bf16)",
        "config": {"workload": "chunked-prefill", "prompt": 8192, "chunk": chunk,
                   "decode_batch": dec.batch, "decode_context": int(dec.seq_lens[0]),
                   "num_q_heads": ext.num_q_heads, "num_kv_heads": ext.pool.num_kv_heads,
                   "step": "4 chunks x (store_kv chunk, extend_attn, store_kv decode rows + decode_attn)",
                   "l2": "chunk K/V re-read from L2 by design; decode batch 1.07 GB > L2",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "extend_tc_kernel (all four chunks)", "bound": "tensor",
                     "achieved": round(tf, 2), "peak": bf16, "peak_source": src, "unit": "TFLOP/s",
                     "frac": round(tf / bf16, 4),
                     "traffic": recorded_traffic("extend_tc_kernel", source_hash("extend_tc.cu", "common.cuh"),
                                                 "chunked-prefill extend c3"),
                     "traffic_note": "per launch of chunk c3 (prefix 6144)",
                     "algorithmic_flops_per_step": extend_flops(ext.num_q_heads, sum(pairs))},
        "chunks": chunks,
        "decode": {"gbs": round(gbs, 1), "ms_per_step": round(dec_ms / args.steps, 4),
                   "tok_per_s_per_layer": round(dec.batch * 4 * args.steps / (dec_ms / 1e3), 1),
                   "roofline": {"kernel": "store_kv + decode_attn (128 requests at 2048)", "bound": "hbm",
                                "achieved": round(gbs, 1), "peak": hbm, "peak_source": src,
                                "unit": "GB/s", "frac": round(gbs / hbm, 4)}},
        "store_kv": {"tokens": chunk, "bytes_per_call": store_bytes(chunk, ext.pool),
                     "us_per_call": round(st_ms / (4 * args.steps) * 1e3, 2), "gbs": round(st_gbs, 1),
                     "frac": round(st_gbs / hbm, 4)},
        "gpu_launches": args.steps * 4 * 5,
        "device_error_word": int(err.item()),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.store_kv(ext.k_planes, ext.v_planes, 0, ext.k_new, ext.v_new, ext.out_loc,
                        ext.pool.num_kv_heads, 128)
        trow = int(ext.table_idx[0])
        tfc, desc, _ = cpu_extend_sample(ext, [(c * chunk, chunk, 0, trow) for c in range(4)],
                                         rows_per_chunk=12, budget_s=12.0, seed=41)
        res["cpu_baseline"] = cpu_baseline_obj(
            tfc, "TFLOP/s", desc + " (12 rows per chunk, all four chunks)",
            extrapolated="per causal FLOP to the whole step")
        gbc, descd, _, _, _ = cpu_decode_sample(dec, range(dec.batch), [0], budget_s=4.0)
        res["decode"]["cpu_baseline"] = cpu_baseline_obj(gbc, "GB/s", descd)
    del pool
    free_device(torch)
    return res


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
    pool = device_pool(api, torch, ext, dev, range(L))
    table = api.PageTable(torch.from_numpy(ext.page_table).to(dev))
    e_q, e_k, e_v = tdev(ext.q, dev), tdev(ext.k_new, dev), tdev(ext.v_new, dev)
    e_ti = torch.from_numpy(ext.table_idx).to(dev)
    e_pl = torch.from_numpy(ext.prefix_lens).to(dev)
    e_el = torch.from_numpy(ext.extend_lens).to(dev)
    e_qo = torch.from_numpy(ext.q_offsets).to(dev)
    e_loc = torch.from_numpy(ext.out_loc).to(dev)
    e_out = torch.empty_like(e_q)
    mx = int(ext.extend_lens.max())
    d_q, d_k, d_v = tdev(dec.q, dev), tdev(dec.k_new, dev), tdev(dec.v_new, dev)
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
    ext_ev, dec_ev, st_ev = [], [], []
    cascade = args.radix_decode == "cascade"

    def decode(l, use_cascade):
        if use_cascade:
            api.decode_attn_cascade(pool, l, d_q, table, d_ti, d_sl, g_off, g_pre, 4096, d_out, cws,
                                    scale=dec.scale, dev_err=err)
        else:
            api.decode_attn(pool, l, d_q, table, d_ti, d_sl, d_out, ws, scale=dec.scale, dev_err=err)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def step(record):
        for l in range(L):
            e0, e1, e2 = (ev(), ev(), ev()) if record else (None, None, None)
            if record: e0.record(s)
            api.store_kv(pool, l, e_k, e_v, e_loc, err)
            if record: e1.record(s)
            api.extend_attn(pool, l, e_q, table, e_ti, e_pl, e_el, e_qo, mx, e_out, scale=ext.scale, dev_err=err)
            if record:
                e2.record(s)
                st_ev.append((e0, e1))
                ext_ev.append((e1, e2))
        for l in range(L):
            api.store_kv(pool, l, d_k, d_v, d_loc, err)
            a, b = (ev(), ev()) if record else (None, None)
            if record: a.record(s)
            decode(l, cascade)
            if record:
                b.record(s)
                dec_ev.append((a, b))

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    start, stop = ev(), ev()
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
    st_ms = sum(a.elapsed_time(b) for a, b in st_ev)
    # The other decode form on layers 0 and L-1, outside the timed step.
    other = []
    for l in (0, L - 1):
        for rep_i in range(4):
            a, b = ev(), ev()
            a.record(s)
            decode(l, not cascade)
            b.record(s)
            if rep_i > 0:
                other.append((a, b))
    torch.cuda.synchronize()
    other_ms = sorted(a.elapsed_time(b) for a, b in other)[len(other) // 2]

    # Both decode forms as the decode workloads time their roofline: the L
    # decode calls captured once in a graph and replayed back to back, so no
    # events sit between the calls (outside the timed step).
    def decode_all(use_cascade):
        for l in range(L):
            decode(l, use_cascade)

    reps = max(3, args.steps)
    graph_ms = {}
    for form in (True, False):
        g = capture(torch, dev, lambda: decode_all(form), 2)
        t = time_replays(torch, s, g, lambda: decode_all(form), reps) / (reps * L)
        graph_ms[form] = (t, g is not None)
        del g
    flops_layer = extend_flops(ext.num_q_heads, ext.causal_pairs())
    ext_flops = flops_layer * L * args.steps
    logical = decode_bytes(dec) * L * args.steps
    hbm, bf16, _, src = measured_peaks()
    tf = ext_flops / (ext_ms / 1e3) / 1e12
    st_call = store_bytes(ext.total_q, ext.pool)
    st_gbs = st_call * L * args.steps / (st_ms / 1e3) / 1e9
    res = {
        "metric": "radix shared-prefix: extend-attn TFLOP/s",
        "value": round(world * tf, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "dtype": "bf16",
        "data": "synthetic (seeded PCG64 N(0,1) values rounded to bf16; per-layer inputs reused)",
        "config": {"workload": "radix-prefix", "layers": L, "batch": ext.batch, "prefix": 4096,
                   "suffix_tokens": ext.total_q, "num_q_heads": ext.num_q_heads,
                   "num_kv_heads": ext.pool.num_kv_heads,
                   "step": ("per layer store_kv + extend_attn, then per layer store_kv + "
                            + ("decode_attn_cascade" if cascade else "decode_attn") + " (decode step 1)"),
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "extend_tc_kernel (256 suffixes, one launch per layer)", "bound": "tensor",
                     "achieved": round(tf, 2), "peak": bf16, "peak_source": src, "unit": "TFLOP/s",
                     "frac": round(tf / bf16, 4), "ms_per_layer": round(ext_ms / (L * args.steps), 4),
                     "traffic": recorded_traffic("extend_tc_kernel", source_hash("extend_tc.cu", "common.cuh"),
                                                 "radix-prefix extend"),
                     "algorithmic_flops_per_launch": flops_layer},
        "decode": {"call": "decode_attn_cascade" if cascade else "decode_attn",
                   "ms_per_layer": round(dec_ms / (L * args.steps), 4),
                   "tok_per_s_per_layer": round(dec.batch * L * args.steps / (dec_ms / 1e3), 1),
                   "logical_gbs": round(logical / (dec_ms / 1e3) / 1e9, 1),
                   "unique_bytes_per_layer": radix_unique_bytes(dec),
                   "prefix_flops_per_layer": 4 * 128 * dec.num_q_heads * dec.batch * 4096,
                   "other_call": "decode_attn" if cascade else "decode_attn_cascade",
                   "other_ms_per_layer": round(other_ms, 4),
                   "graph_ms_per_layer": round(graph_ms[cascade][0], 4),
                   "other_graph_ms_per_layer": round(graph_ms[not cascade][0], 4),
                   "timing": ("ms_per_layer: events around each call inside the timed step; "
                              "other_ms_per_layer: the median of 6 such calls after it; *graph_ms_per_layer: "
                              f"{reps} back-to-back replays of a graph of the {L} decode calls"
                              + ("" if graph_ms[True][1] and graph_ms[False][1] else
                                 " (capture failed: eager calls)")),
                   "note": "logical bytes count the shared 4096-token prefix once per request"},
        "store_kv": {"tokens": ext.total_q, "bytes_per_call": st_call,
                     "us_per_call": round(st_ms / (L * args.steps) * 1e3, 2), "gbs": round(st_gbs, 1),
                     "frac": round(st_gbs / hbm, 4),
                     "traffic": recorded_traffic("store_kv_kernel", source_hash("store.cu", "common.cuh"),
                                                 "radix-prefix suffix store")},
        "gpu_launches": args.steps * L * (2 + (5 if cascade else 3)),
        "device_error_word": int(err.item()),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.store_kv(ext.k_planes, ext.v_planes, ext.layer, ext.k_new, ext.v_new, ext.out_loc,
                        ext.pool.num_kv_heads, 128)
        el = ext.extend_lens
        pick = [int(np.argmax(el)), int(np.argmin(el))] + \
            [int(x) for x in np.random.default_rng(51).choice(ext.batch, 4, replace=False)]
        chunks = [(int(ext.prefix_lens[r]), int(el[r]), int(ext.q_offsets[r]), int(ext.table_idx[r]))
                  for r in pick]
        tfc, desc, _ = cpu_extend_sample(ext, chunks, rows_per_chunk=24, budget_s=10.0, seed=52)
        res["cpu_baseline"] = cpu_baseline_obj(
            tfc, "TFLOP/s", desc + " (the longest and shortest suffixes and 4 seeded ones)",
            extrapolated="per causal FLOP to the whole step")
        gbc, descd, _, _, _ = cpu_decode_sample(dec, range(dec.batch), [ext.layer], budget_s=4.0)
        res["decode"]["cpu_baseline"] = cpu_baseline_obj(gbc, "GB/s", descd + " (logical bytes)")
    del pool
    free_device(torch)
    return res


def run_rope_measure(dev, iters=10, warmup=3):
    """The fused q/k norm + RoPE + store call on three shapes: a 64-token decode
    step (Hq 16, Hkv 8), and 2048- and 16384-token prefill batches of the
    Qwen3-8B shape (Hq 32, Hkv 8).  L2 is flushed before every timed call."""
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
        # Back-to-back calls replayed from a CUDA graph: no launch latency, and
        # the inputs stay in L2, as they do in a decode step right after the
        # QKV projection that writes them.
        reps, per_graph = 5, 20
        gs = torch.cuda.Stream(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            for _ in range(per_graph):
                call()
        graph.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(reps):
            graph.replay()
        b.record(s)
        torch.cuda.synchronize()
        us_graph = a.elapsed_time(b) * 1e3 / (reps * per_graph)
        del graph
        nbytes = rope_bytes(n, hq, hkv)
        gbs = nbytes / us / 1e3
        out[name] = {"us": round(us, 3), "bytes": nbytes, "GB/s": round(gbs, 1),
                     "frac": round(gbs / hbm, 4), "peak": hbm, "peak_source": src,
                     "us_graph_l2_warm": round(us_graph, 3),
                     "timing": "us: one launch after an L2 flush (CUDA events); us_graph_l2_warm: "
                               f"per call in {per_graph}-call graph replays",
                     "device_error_word": int(err.item())}
        if n == 16384:
            out[name]["traffic"] = recorded_traffic("qk_norm_rope_store_kernel",
                                                    source_hash("rope_store.cu", "common.cuh"),
                                                    "rope prefill 16384")
    del flush
    free_device(torch)
    return out


# ---------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, world, rank):
    """The oracle on the headline workload: each step is a bounded sample
    (requests taken longest-first from a seeded order, on the first layer at
    even steps and the last layer at odd ones, until the step's time budget),
    timed in KV GB/s of the sampled requests."""
    from paged_kv_gqa_scatter_b200 import workloads as W
    if rank != 0:
        return None
    wl = W.decode_qwen3_8b()
    budget = float(os.environ.get("PKV_REF_STEP_SECONDS", "4"))
    order = [int(np.argmax(wl.seq_lens))] + [int(x) for x in np.random.default_rng(9).permutation(wl.batch)
                                              if int(x) != int(np.argmax(wl.seq_lens))]
    for w in range(args.warmup):
        cpu_decode_sample(wl, order[w:w + 1], [0], budget_s=0.5)
    vals, secs, done_total = [], 0.0, 0
    pos = 0
    for s in range(args.steps):
        layer = 0 if s % 2 == 0 else wl.pool.num_layers - 1
        reqs = [order[(pos + i) % wl.batch] for i in range(wl.batch)]
        v, _, dt, _, done = cpu_decode_sample(wl, reqs, [layer], budget_s=budget)
        pos += done
        done_total += done
        vals.append(v)
        secs += dt
    value = statistics.median(vals)
    cores = blas_threads()
    sample = (f"oracle decode_attn (float64 numpy), {budget:.0f} s per step: {done_total} (request, layer) "
              f"pairs over {args.steps} steps, layers 0 and 35 alternating, longest request first")
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
        "data": "synthetic (seeded PCG64 N(0,1) block of 65,536 slots tiled over the pool)",
        "config": {"workload": wl.name, "batch": wl.batch, "num_q_heads": wl.num_q_heads,
                   "num_kv_heads": wl.pool.num_kv_heads, "head_dim": 128, "page_size": wl.pool.page_size,
                   "pool_slots": wl.pool.num_slots, "pool_layers": wl.pool.num_layers},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="all",
                    choices=["all", "decode-qwen3-8b", "decode-qwen3-0.6b", "chunked-prefill", "radix-prefix",
                             "rope-store"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pool-layers", type=int, default=None,
                    help="pool layers of decode-qwen3-8b (36), decode-qwen3-0.6b (28) or radix-prefix (32); "
                         "fewer only for profiling")
    ap.add_argument("--page-size", type=int, default=None,
                    help="page size of decode-qwen3-8b (16 as stated; 64 is TRT-LLM's size)")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="pool element type of the decode workloads (fp8: scaled E4M3 codes, bf16 q/out)")
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
    elif args.workload == "rope-store":
        import torch
        res = {"qk_norm_rope_store": run_rope_measure(torch.device("cuda", local), iters=max(5, args.steps))}
    elif args.workload in ("decode-qwen3-8b", "decode-qwen3-0.6b"):
        res = run_decode(args, world, rank, local, args.workload)
    else:
        import torch
        res = run_decode(args, world, rank, local, "decode-qwen3-8b")
        subs = {}
        subs["decode-qwen3-0.6b"] = run_decode(args, world, rank, local, "decode-qwen3-0.6b")
        subs["chunked-prefill"] = run_chunked_prefill(args, world, rank, local)
        subs["radix-prefix"] = run_radix(args, world, rank, local)
        res["workloads"] = subs
        res["qk_norm_rope_store"] = run_rope_measure(torch.device("cuda", local), iters=max(5, args.steps))
        res["gpu_launches_all_workloads"] = res["gpu_launches"] + sum(v["gpu_launches"] for v in subs.values())
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
