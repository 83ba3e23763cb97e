"""GPU parity of w4a16_gemv_s, the decode GEMV with the AWQ activation scaling fused in ("AWQ and GPTQ
algorithms" (jsqmd.com) section 2.1 (3): the activations carry 1/s at inference; "LLM quantization speed-up"
(bjdmk.com.cn), "fused modules"): raw x and s go in, x' = fp16(x / s) is formed inside the kernel.  It must be
bit-identical to the two-pass path awq_apply_inv_scale -> w4a16_gemv (same x', same arithmetic), and within
the layer tolerance of the oracle composition inv_scale -> linear."""
import numpy as np
import pytest
import torch

from helpers import OracleCase, assert_within_tolerance, sample_pairs
from oracle import oracle as O
import weight_only_int4_05_b200 as W4

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.float16)


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (1, 1024, 4096), (1, 14336, 4096), (1, 4096, 14336),
                                   (3, 4864, 4096), (8, 1024, 4096), (12, 264, 1152), (1, 8192, 28672)])
def test_fused_inv_scale_bit_identical_to_two_pass(M, N, K):
    case = OracleCase(9, 0, M, N % 7, M, N, K)
    x = dev(case.x)
    s = W4.awq_act_scale(dev(case.xcal))
    pw = W4.awq_pack(dev(case.W), s)
    y_fused = W4.w4a16_gemv_s(x, s, pw)
    y_two = W4.w4a16_gemv(W4.awq_apply_inv_scale(x, s), pw)
    torch.cuda.synchronize()
    assert torch.equal(y_fused, y_two)
    ms, ns = sample_pairs(M, N, 800, seed=M + N)
    assert_within_tolerance(y_fused.float().cpu().numpy()[ms, ns], case.y_pairs(ms, ns), f"gemv_s M={M} N={N} K={K}")
    assert W4.awq_last_device_status() == 0


def test_fused_inv_scale_on_exact_ties():
    """x and s built so that many x / s are exact fp16 rounding midpoints (subnormal results, odd scales):
    the in-kernel fp32 division must round them to even like the oracle's fp64 division."""
    K, N = 1024, 256
    rng = np.random.default_rng(3)
    s = np.empty(K, np.float16)
    x = np.empty((1, K), np.float16)
    odd = np.array([3, 5, 7, 11, 13, 99, 1023, 2047])
    for k in range(K):
        kk, e = int(odd[k % len(odd)]), int(1 + (k // len(odd)) % 4)
        s[k] = np.float16(kk * 2.0 ** e)
        m = int(rng.integers(0, 2048 // kk)) | 1
        v = kk * 2.0 ** e * m * 2.0 ** -25
        x[0, k] = np.float16(v) if float(np.float16(v)) == v else np.float16(rng.standard_normal())
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    xd, sd = dev(x.view(np.uint16)), dev(s.view(np.uint16))
    pw = W4.awq_pack(dev(W.view(np.uint16)), sd)
    xp_ref = O.inv_scale(x.view(np.uint16), s.view(np.uint16))
    assert np.array_equal(W4.awq_apply_inv_scale(xd, sd).cpu().view(torch.int16).numpy().view(np.uint16), xp_ref)
    y_fused = W4.w4a16_gemv_s(xd, sd, pw)
    y_two = W4.w4a16_gemv(dev(xp_ref), pw)
    torch.cuda.synchronize()
    assert torch.equal(y_fused, y_two)
