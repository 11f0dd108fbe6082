"""Failure detection without a GPU fault: a device wait that nothing satisfies gives up
after its limit, the host reads FA_ERR_TIMEOUT from the status word, and the context is
still usable for normal work afterwards."""
import time

import pytest
import torch

from exact_io_aware_60_b200 import fa
from exact_io_aware_60_b200 import workloads as W
from parity import compare_forward, oracle_full, run_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    torch.cuda.init()
    assert fa.fa_get_device_status() == fa.FA_OK
    t0 = time.time()
    fa.fa_selftest_wait_timeout(20000)   # 20 ms
    assert fa.fa_get_device_status() == fa.FA_ERR_TIMEOUT
    assert time.time() - t0 < 10.0
    assert fa.fa_get_device_status() == fa.FA_OK   # read-and-clear
    w = W.custom(B=1, H=2, N=130, d=64, dtype=torch.bfloat16, causal=True)
    inp = W.make_inputs(w, seed=9)
    gpu = run_gpu(inp, w.scale, True, backward=False)
    err = compare_forward(gpu, oracle_full(inp, w.scale, True, backward=False))
    assert err["o_max_abs"] <= 1e-2


def test_selftest_rejects_bad_limits():
    with pytest.raises(fa.FAError):
        fa.fa_selftest_wait_timeout(0)
    with pytest.raises(fa.FAError):
        fa.fa_selftest_wait_timeout(10 ** 7)
