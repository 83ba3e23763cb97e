"""GPU parity at group sizes 64 and 256 (the pages' --q_group_size parameter; 128 is covered everywhere
else) and on the 3-bit grid (codes 0..7 in the 4-bit layout): pack bit-exact against the oracle, GEMV (plain
and with the 1/s fused), GEMM and the mode choice within the linear layer's tolerance, every output at small
sizes and sampled outputs at a full decode shape."""
import numpy as np
import pytest
import torch

from helpers import OracleCase, assert_within_tolerance, sample_pairs
import weight_only_int4_05_b200 as W4

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.float16)


def host_u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host_u32(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def prep(case):
    s = W4.awq_act_scale(dev(case.xcal))
    xp = W4.awq_apply_inv_scale(dev(case.x), s)
    pw = W4.awq_pack(dev(case.W), s, g=case.g, w_bit=case.w_bit)
    torch.cuda.synchronize()
    qw, sc, qz = case.packed
    assert np.array_equal(host_u32(pw.qweight), qw), "qweight"
    assert np.array_equal(host_u16(pw.scales), sc), "scales"
    assert np.array_equal(host_u32(pw.qzeros), qz), "qzeros"
    return s, xp, pw


# (N, K, M): ragged N, one group per row, several tiles and passes, a split plan (152 row blocks)
SHAPES = [(40, 256, 1), (264, 1024, 3), (256, 512, 16), (1024, 2048, 9), (4864, 1024, 1), (96, 1536, 33)]


@pytest.mark.parametrize("g", [64, 256])
@pytest.mark.parametrize("N,K,M", SHAPES)
def test_group_size_pack_and_linears(g, N, K, M):
    case = OracleCase(4, 1, g, N % 5, M, N, K, g=g)
    s, xp, pw = prep(case)
    y_ref = case.y_rows()
    for name, fn in (("gemv", W4.w4a16_gemv), ("gemm", W4.w4a16_gemm), ("linear", W4.w4a16_linear)):
        y = fn(xp, pw)
        torch.cuda.synchronize()
        assert_within_tolerance(y.float().cpu().numpy(), y_ref, f"{name} g={g} N={N} K={K} M={M}")
    y_s = W4.w4a16_gemv_s(dev(case.x), s, pw)
    assert torch.equal(y_s, W4.w4a16_gemv(xp, pw)), "fused 1/s differs from the two-pass GEMV"
    assert W4.awq_last_device_status() == 0


@pytest.mark.parametrize("g", [64, 256])
def test_group_size_full_decode_shape_sampled(g):
    """Gate/up decode shape 4096 -> 14336 at M = 1 (whole row blocks per CTA) and the down shape
    14336 -> 4096, sampled outputs against the oracle, pack bit-exact."""
    for N, K in ((14336, 4096), (4096, 14336)):
        case = OracleCase(5, 1, g, 0, 1, N, K, g=g)
        _, xp, pw = prep(case)
        ms, ns = sample_pairs(1, N, 3000, seed=g)
        y = W4.w4a16_linear(xp, pw)
        torch.cuda.synchronize()
        assert_within_tolerance(y.float().cpu().numpy()[ms, ns], case.y_pairs(ms, ns), f"g={g} {K}->{N}")
    assert W4.awq_last_device_status() == 0


def test_group_size_is_checked():
    case = OracleCase(6, 1, 0, 0, 1, 64, 512, g=64)
    _, xp, pw = prep(case)
    with pytest.raises(ValueError):
        W4.w4a16_gemv(xp, pw, g=128)  # the weight was packed with g = 64
    with pytest.raises(W4.AwqError):
        W4.awq_pack(dev(case.W), None, g=32)


@pytest.mark.parametrize("g", [64, 128, 256])
@pytest.mark.parametrize("N,K,M", [(264, 1024, 1), (256, 512, 40), (4096, 4096, 1)])
def test_3bit_grid_pack_and_linears(g, N, K, M):
    """awq_pack_bits with w_bit = 3: bit-exact codes 0..7, and both linear modes on them."""
    case = OracleCase(7, 1, g, 3, M, N, K, g=g, w_bit=3)
    s, xp, pw = prep(case)
    assert case.q.max() <= 7
    ms, ns = sample_pairs(M, N, 2000, seed=g + M)
    y_ref = case.y_pairs(ms, ns)
    for name, fn in (("gemv", W4.w4a16_gemv), ("gemm", W4.w4a16_gemm)):
        y = fn(xp, pw)
        torch.cuda.synchronize()
        assert_within_tolerance(y.float().cpu().numpy()[ms, ns], y_ref, f"3-bit {name} g={g} N={N} K={K} M={M}")
    assert W4.awq_last_device_status() == 0
