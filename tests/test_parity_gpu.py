"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Bit-exact: the AWQ scale, the scaled activations and the three packed arrays.  Within tolerance
(max |y - y_ref| <= 1e-2 rms(y_ref), relative L2 <= 2e-3): GEMV and GEMM outputs."""
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


def run_prep_and_pack(case):
    """CUDA side of steps a1, a7 and a2-a6 from the raw synthetic inputs."""
    s = W4.awq_act_scale(dev(case.xcal))
    xp = W4.awq_apply_inv_scale(dev(case.x), s)
    pw = W4.awq_pack(dev(case.W), s)
    torch.cuda.synchronize()
    return s, xp, pw


def assert_pack_bitexact(case, pw):
    qw, sc, qz = case.packed
    assert np.array_equal(host_u32(pw.qweight), qw)
    assert np.array_equal(host_u16(pw.scales), sc)
    assert np.array_equal(host_u32(pw.qzeros), qz)


SMALL_SHAPES = [(256, 512), (40, 384), (8, 128), (264, 1152), (1024, 1024), (96, 256)]


@pytest.mark.parametrize("N,K", SMALL_SHAPES)
def test_prep_and_pack_bitexact_small(N, K):
    case = OracleCase(0, 0, 0, N % 7, 3, N, K)
    s, xp, pw = run_prep_and_pack(case)
    assert np.array_equal(host_u16(s), case.s)
    assert np.array_equal(host_u16(xp), case.xp)
    assert_pack_bitexact(case, pw)


def test_pack_without_scale_is_plain_rtn():
    from oracle import oracle as O
    case = OracleCase(1, 0, 1, 0, 1, 264, 512)
    pw = W4.awq_pack(dev(case.W), None)
    qw, sc, qz = O.awq_pack(case.W, None)
    assert np.array_equal(host_u32(pw.qweight), qw)
    assert np.array_equal(host_u16(pw.scales), sc)
    assert np.array_equal(host_u32(pw.qzeros), qz)


def test_act_scale_non_power_of_two_rows():
    from oracle import oracle as O
    rng = np.random.default_rng(3)
    xcal = (rng.standard_normal((3, 4096)) * 3).astype(np.float16).view(np.uint16)
    s = W4.awq_act_scale(dev(xcal))
    assert np.array_equal(host_u16(s), O.act_scale(xcal))


def test_config0_tiny_full_path():
    """Tiny linear, seed 0: M=1, K=512, N=256 through both modes, every output checked."""
    case = OracleCase(0, 0, 0, 0, 1, 256, 512)
    s, xp, pw = run_prep_and_pack(case)
    assert_pack_bitexact(case, pw)
    y_ref = case.y_rows()
    for fn in (W4.w4a16_gemv, W4.w4a16_gemm, W4.w4a16_linear):
        y = fn(xp, pw)
        assert_within_tolerance(y.float().cpu().numpy(), y_ref, fn.__name__)


@pytest.mark.parametrize("N,K", [(256, 512), (40, 384), (264, 1152), (8, 128), (1024, 1024)])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 17])
def test_gemv_shapes(M, N, K):
    case = OracleCase(2, 0, M, N % 5, M, N, K)
    s, xp, pw = run_prep_and_pack(case)
    y = W4.w4a16_gemv(xp, pw)
    assert_within_tolerance(y.float().cpu().numpy(), case.y_rows(), f"gemv M={M} N={N} K={K}")


@pytest.mark.parametrize("N,K", [(256, 512), (40, 384), (264, 1152), (8, 128), (1024, 1024)])
@pytest.mark.parametrize("M", [1, 7, 16, 17, 63, 64, 65, 255, 256, 257, 300])
def test_gemm_shapes(M, N, K):
    case = OracleCase(3, 0, M % 16, N % 5, M, N, K)
    s, xp, pw = run_prep_and_pack(case)
    y = W4.w4a16_gemm(xp, pw)
    assert_within_tolerance(y.float().cpu().numpy(), case.y_rows(), f"gemm M={M} N={N} K={K}")


def test_outputs_deterministic_and_workspace_reused():
    """Two shapes alternate on one shared workspace; every repeat is bit-identical."""
    a = OracleCase(4, 0, 0, 0, 1, 1024, 4096)
    b = OracleCase(4, 0, 0, 1, 4, 264, 1152)
    _, xa, pa = run_prep_and_pack(a)
    _, xb, pb = run_prep_and_pack(b)
    outs = []
    for _ in range(3):
        outs.append((W4.w4a16_gemv(xa, pa).clone(), W4.w4a16_gemv(xb, pb).clone(), W4.w4a16_gemm(xb, pb).clone()))
    torch.cuda.synchronize()
    for o in outs[1:]:
        for u, v in zip(o, outs[0]):
            assert torch.equal(u, v)
    assert_within_tolerance(outs[0][0].float().cpu().numpy(), a.y_rows(), "gemv a")
    assert_within_tolerance(outs[0][1].float().cpu().numpy(), b.y_rows(), "gemv b")


def test_linear_dispatch_matches_selected_mode():
    for M in (1, 8, 9, 64):
        case = OracleCase(5, 0, M, 0, M, 256, 512)
        _, xp, pw = run_prep_and_pack(case)
        y = W4.w4a16_linear(xp, pw)
        ref = (W4.w4a16_gemv if M <= W4.w4a16_gemv_max_m(256, 512) else W4.w4a16_gemm)(xp, pw)
        assert torch.equal(y, ref)


def test_device_status_clean_after_runs():
    assert W4.awq_last_device_status() == 0


@pytest.mark.parametrize("N", [4864, 4800])
@pytest.mark.parametrize("M", [1, 3, 8, 12])
def test_gemv_split_row_blocks_between_ctas(M, N):
    """A few row blocks more than SMs (150, 152): the units are spread evenly over the CTAs and the row blocks
    cut by CTA boundaries are summed in the workspace (deterministic slot order)."""
    assert W4.w4a16_workspace_bytes(W4.MODE_GEMV, M, N, 4096) > 0
    case = OracleCase(6, 0, M, N % 7, M, N, 4096)
    _, xp, pw = run_prep_and_pack(case)
    y = W4.w4a16_gemv(xp, pw)
    y2 = W4.w4a16_gemv(xp, pw)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    ms, ns = sample_pairs(M, N, 1500, seed=N + M)
    assert_within_tolerance(y.float().cpu().numpy()[ms, ns], case.y_pairs(ms, ns), f"gemv split M={M} N={N}")
    assert W4.awq_last_device_status() == 0
