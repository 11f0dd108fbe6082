"""FP8 (E4M3) forward against the fp64 oracle.

The oracle is the same standard attention, evaluated on the values the E4M3 inputs
represent (byte value times its tensor's scale factor, exact in fp64), so input
quantisation is not an error source; the kernel's only extra rounding is P to E4M3 before
the P V product.  Tolerances follow from that: LSE uses the unrounded fp32 sum (1e-3 as
for 16-bit inputs); each weight P_ij / l_i moves by at most 2^-4 relative (E4M3 keeps 3
mantissa bits), so |O - O_ref| <= 2^-3 max |v| element-wise (worst case).  Typically the
rounding error of a weight is spread over +-2^-4 with a standard deviation of at most
2^-4 / sqrt(3) ~ 0.036, and O - O_ref is a weighted sum of such errors times
(v_j - O), so the whole-tensor relative L2 error of O stays below sqrt(2) * 0.036 ~ 5e-2."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_60_b200 import fa
from parity import LSE_ATOL, lse_err, rel_l2, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)
E4M3_MAX = 448.0


def quantise(x: torch.Tensor):
    """Per-tensor E4M3 quantisation: returns the bytes and the scale factor."""
    s = float(x.abs().max()) / E4M3_MAX
    return (x / s).to(torch.float8_e4m3fn), s


def make(B, H, N, seed, kv_range=None):
    g = torch.Generator("cpu").manual_seed(seed)
    q, k, v = (torch.randn((B, H, N, 128), generator=g) for _ in range(3))
    kv = None
    if kv_range is not None:
        kv = torch.randint(kv_range[0], kv_range[1] + 1, (B,), generator=g, dtype=torch.int32)
    return q, k, v, kv


def run_fp8(q, k, v, kv, causal):
    (q8, qs), (k8, ks), (v8, vs) = quantise(q), quantise(k), quantise(v)
    B, H, N, d = q.shape
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=DEV)
    fa.fa_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), o, lse, scale=d ** -0.5, q_scale=qs,
                  k_scale=ks, v_scale=vs, causal=causal,
                  kv_len=None if kv is None else kv.to(DEV))
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    deq = [to_f64(x8.float()) * s for x8, s in ((q8, qs), (k8, ks), (v8, vs))]
    ref = oracle.attention(*deq, scale=d ** -0.5, causal=causal,
                           kv_len=None if kv is None else kv.numpy())
    return o.cpu(), lse.cpu(), ref, deq[2]


CASES = [
    (1, 2, 128, False, None, 1),
    (2, 2, 300, True, None, 2),
    (1, 4, 1024, False, (300, 1024), 3),
    (2, 3, 517, True, (1, 517), 4),
    (1, 2, 2048, True, None, 5),
]


@pytest.mark.parametrize("B,H,N,causal,kvr,seed", CASES)
def test_fp8_forward_matches_oracle(B, H, N, causal, kvr, seed):
    q, k, v, kv = make(B, H, N, seed, kvr)
    o, lse, ref, vdeq = run_fp8(q, k, v, kv, causal)
    go = to_f64(o)
    err = np.abs(go - ref["o"])
    worst = 2.0 ** -3 * np.abs(vdeq).max() + 2.0 ** -8 * np.abs(ref["o"]).max()
    rl2 = rel_l2(go, ref["o"])
    le = lse_err(to_f64(lse), ref["lse"])
    print(f"fp8 parity: O max-abs {err.max():.3e} (bound {worst:.3e}), O rel-L2 {rl2:.3e}, "
          f"LSE {le:.3e}")
    assert err.max() <= worst
    assert rl2 <= 5e-2
    assert le <= LSE_ATOL
