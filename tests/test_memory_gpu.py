"""Peak device memory of a forward + backward pass is linear in N (P3 Theorem 1: O(N)
extra memory; the N x N score matrix never exists on the device)."""
import pytest
import torch

from exact_io_aware_60_b200 import fa
from exact_io_aware_60_b200 import workloads as W

pytestmark = pytest.mark.gpu


def peak_bytes(N):
    dev = torch.device("cuda", 0)
    w = W.custom(B=1, H=8, N=N, d=64, dtype=torch.bfloat16)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    free0 = torch.cuda.mem_get_info(dev)[0]
    g = torch.Generator(device=dev).manual_seed(0)
    q, k, v, do = (torch.randn(w.B, w.H, N, w.d, device=dev, generator=g).to(w.dtype)
                   for _ in range(4))
    o, lse = fa.forward(q, k, v, scale=w.scale)
    dq, dk, dv = fa.backward(q, k, v, o, do, lse, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    peak = torch.cuda.max_memory_allocated(dev) - base
    reserved = torch.cuda.memory_reserved(dev)
    free1 = torch.cuda.mem_get_info(dev)[0]
    del q, k, v, do, o, lse, dq, dk, dv
    return peak, free0 - free1, reserved


def test_peak_memory_linear_in_n():
    sizes = [1024, 2048, 4096, 8192, 16384]
    peak_bytes(256)  # one-time costs (module load, context growth) happen here
    peaks = []
    for N in sizes:
        peak, drop, reserved = peak_bytes(N)
        # the library allocates nothing: the device's free memory drops by no more than
        # what torch itself reserved
        assert drop <= reserved + (64 << 20)
        peaks.append(peak)
    for a, b in zip(peaks, peaks[1:]):
        assert 1.8 <= b / a <= 2.2, peaks
    # at N = 16384 one fp32 score matrix per head would be 8 x 1 GiB; the whole pass
    # uses a few tens of MB
    assert peaks[-1] < 256 << 20
