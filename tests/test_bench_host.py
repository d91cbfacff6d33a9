"""Host logic of bench.py on CPU: the algorithmic work counts that the
roofline figures divide by, and the reference arm's JSON line.

The work counts are checked against counts taken element by element (every
context token's rows, every distinct page a request touches, every (query,
key) pair the causal mask leaves), not against the closed forms they use.
"""
import json
import os
import subprocess
import sys
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from paged_kv_gqa_scatter_b200 import workloads as W  # noqa: E402

ESZ = {"bf16": 2, "f32": 4, "fp8": 1}


def _fake_decode(seq_lens, page_size, dtype="bf16", io_dtype="bf16", hkv=8, hq=32):
    pool = types.SimpleNamespace(dtype=dtype, io_dtype=io_dtype, num_kv_heads=hkv, page_size=page_size)
    return types.SimpleNamespace(batch=len(seq_lens), num_q_heads=hq, pool=pool,
                                 seq_lens=np.asarray(seq_lens, np.int32))


def _count_decode_bytes(wl):
    """Walk every context token: its K and V rows, and a table entry for each
    page it is the first token of; then each request's q and out rows, its
    length and its table-row index."""
    P = wl.pool.page_size
    row = wl.pool.num_kv_heads * 128 * ESZ[wl.pool.dtype]
    total = 0
    for n in wl.seq_lens.tolist():
        pages = set()
        for t in range(n):
            total += 2 * row
            pages.add(t // P)
        total += 4 * len(pages)
        total += 2 * wl.num_q_heads * 128 * ESZ[wl.pool.io_dtype]
        total += 4 + 4
    return total


@pytest.mark.parametrize("page_size", [1, 3, 16, 64])
@pytest.mark.parametrize("dtype,io", [("bf16", "bf16"), ("f32", "f32"), ("fp8", "bf16")])
def test_decode_bytes_by_token_walk(page_size, dtype, io):
    rng = np.random.default_rng(page_size)
    lens = [1, 15, 16, 17, 63, 64, 65, 200] + rng.integers(1, 700, size=6).tolist()
    wl = _fake_decode(lens, page_size, dtype, io, hkv=4 if dtype == "f32" else 8, hq=16)
    assert bench.decode_bytes(wl) == _count_decode_bytes(wl)


def test_store_bytes_by_row_walk():
    spec = types.SimpleNamespace(num_kv_heads=8, dtype="fp8", io_dtype="bf16")
    n = 37
    walk = 0
    for _ in range(n):
        for _plane in ("k", "v"):
            walk += 8 * 128 * 2  # new row read (bf16)
            walk += 8 * 128 * 1  # pool row written (E4M3)
        walk += 4  # its slot index
    assert bench.store_bytes(n, spec) == walk


def test_causal_pairs_by_mask_count():
    """Query i of a chunk (absolute position prefix + i) sees keys 0..prefix+i."""
    prefix = np.array([0, 1, 37, 128, 0, 500], np.int32)
    extend = np.array([1, 45, 200, 128, 0, 3], np.int32)
    wl = types.SimpleNamespace(prefix_lens=prefix, extend_lens=extend)
    count = 0
    for p, e in zip(prefix.tolist(), extend.tolist()):
        q = p + np.arange(e)[:, None]
        k = np.arange(p + e)[None, :]
        count += int((k <= q).sum())
    assert W.ExtendWorkload.causal_pairs(wl) == count
    assert bench.extend_flops(32, count) == 2 * 2 * 128 * 32 * count


def _run_reference(env_extra, steps=2):
    env = dict(os.environ)
    env.update(PKV_REF_STEP_SECONDS="0.5", OMP_NUM_THREADS="2", OPENBLAS_NUM_THREADS="2", MKL_NUM_THREADS="2")
    env.update(env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", str(steps), "--warmup", "3"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_json_line():
    """One JSON line with the headline's metric, unit and workload, the
    oracle described as its own cpu_baseline and an e2e with no copies."""
    r = _run_reference({"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == "paged decode-attn KV GB/s" and d["unit"] == "GB/s"
    assert d["higher_is_better"] is True and d["steps"] == 2 and d["warmup"] == 3
    assert d["config"]["workload"] == "decode-qwen3-8b"
    assert d["config"]["batch"] == 256 and d["config"]["page_size"] == 16
    assert d["value"] > 0 and d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "layers 0 and 35" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["dtype"] == "f64" and d["vs_baseline"] is None


def test_reference_arm_other_ranks_print_nothing():
    r = _run_reference({"RANK": "1", "WORLD_SIZE": "2"}, steps=1)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
