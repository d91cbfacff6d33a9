"""Failure detection on the GPU without a fault: a wait that nothing satisfies
gives up after about one second, reports PKV_DEV_ERR_TIMEOUT through the
device error word, and leaves the context usable for the next call."""
import time

import pytest
import torch

from gpu_helpers import DeviceDecode, from_dev, oracle_decode, tol_check
from paged_kv_gqa_scatter_b200 import api
from paged_kv_gqa_scatter_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    api.selftest_wait_timeout(err)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(err.item()) == api.DEV_ERR_TIMEOUT
    assert 0.9 <= dt < 10.0, dt
    # The next real call on the same context works and is correct.
    wl = W.decode_small()
    d = DeviceDecode(wl)
    d.run()
    torch.cuda.synchronize()
    assert int(d.err.item()) == 0
    exp, _ = oracle_decode(wl)
    tol_check(from_dev(d.out), exp, W.BF16, "decode after a timed-out wait")


def test_selftest_needs_an_error_word():
    with pytest.raises(RuntimeError, match="invalid"):
        _ = api._lib.check(api._lib.load().pkv_selftest_wait_timeout(None, None), "selftest")
