"""GPU parity of the packed 3-bit layout: awq_pack3 bit-exact against the oracle's 3-bit grid and layout, and
w3a16_gemv within the linear layer's tolerance of the oracle's fp64 product of the same 3-bit codes, at every
group size, at ragged N, over several passes of M, and at the full decode shapes (sampled)."""
import numpy as np
import pytest
import torch

from helpers import OracleCase, assert_within_tolerance, sample_pairs
from oracle import oracle as O
import weight_only_int4_05_b200 as W4

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.float16)


def host_u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def prep3(case):
    s = W4.awq_act_scale(dev(case.xcal))
    xp = W4.awq_apply_inv_scale(dev(case.x), s)
    pw = W4.awq_pack3(dev(case.W), s, g=case.g)
    torch.cuda.synchronize()
    qw, sc, qz = O.pack3(case.q, case.sc, case.z, case.g)
    assert np.array_equal(pw.qweight.cpu().numpy().view(np.uint32), qw), "qweight"
    assert np.array_equal(host_u16(pw.scales), sc), "scales"
    assert np.array_equal(pw.qzeros.cpu().numpy().view(np.uint32), qz), "qzeros"
    return xp, pw


@pytest.mark.parametrize("g", [64, 128, 256])
@pytest.mark.parametrize("N,K,M", [(40, 256, 1), (264, 1024, 3), (256, 512, 16), (1024, 2048, 40), (4864, 1024, 1)])
def test_w3_pack_and_gemv(g, N, K, M):
    case = OracleCase(8, 1, g, N % 3, M, N, K, g=g, w_bit=3)
    xp, pw = prep3(case)
    y = W4.w3a16_gemv(xp, pw)
    torch.cuda.synchronize()
    assert_within_tolerance(y.float().cpu().numpy(), case.y_rows(), f"w3 g={g} N={N} K={K} M={M}")
    assert W4.awq_last_device_status() == 0


def test_w3_full_decode_shapes_sampled():
    for N, K in ((14336, 4096), (4096, 14336), (1024, 4096)):
        case = OracleCase(9, 1, 0, 0, 1, N, K, w_bit=3)
        xp, pw = prep3(case)
        ms, ns = sample_pairs(1, N, 3000, seed=N)
        y = W4.w3a16_gemv(xp, pw)
        torch.cuda.synchronize()
        assert_within_tolerance(y.float().cpu().numpy()[ms, ns], case.y_pairs(ms, ns), f"w3 {K}->{N}")
    assert W4.awq_last_device_status() == 0


def test_w3_matches_the_3bit_grid_in_the_4bit_layout():
    """The same 3-bit codes through both layouts: w3a16_gemv on awq_pack3 and w4a16_gemv on awq_pack_bits(3)
    read identical codes, scales and zeros, and their outputs agree within the summation-order difference."""
    case = OracleCase(10, 1, 0, 0, 2, 1024, 2048, w_bit=3)
    xp, pw3 = prep3(case)
    pw4 = W4.awq_pack(dev(case.W), W4.awq_act_scale(dev(case.xcal)), w_bit=3)
    y3 = W4.w3a16_gemv(xp, pw3)
    y4 = W4.w4a16_gemv(xp, pw4)
    torch.cuda.synchronize()
    assert torch.equal(pw3.scales, pw4.scales) and torch.equal(pw3.qzeros, pw4.qzeros)
    assert torch.equal(y3, y4)  # the same kernel plan and summation order; only the code unpacking differs


def test_w3_layout_is_checked():
    case = OracleCase(11, 1, 0, 0, 1, 64, 256, w_bit=3)
    xp, pw3 = prep3(case)
    with pytest.raises(ValueError):
        W4.w4a16_gemv(xp, pw3)
    with pytest.raises(ValueError):
        W4.w3a16_gemv(xp, W4.awq_pack(dev(case.W), None))
