"""GPU parity at the workloads' full sizes, in the launch configurations the benchmark times.

  * decode GEMV sweep, M=1, Llama-3-8B shapes: packed arrays bit-exact, every output within tolerance;
  * decode stack: two layers of the 7-linear stack (also with the prefetch hint) and one layer of the
    fused 4-linear stack, run as one CUDA graph with programmatic dependent launch and a shared workspace
    (the benchmark's launch paths), every output checked;
  * prefill GEMM, M=2048: packed arrays bit-exact, sampled outputs (corners + random) within tolerance;
  * crossover sweep, 70B-class shapes: both modes at M = 1 .. 256 on sampled outputs.
Inputs come from the host generator so that the oracle sees the same values."""
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


def prep(case, xrows=None):
    s = W4.awq_act_scale(dev(case.xcal))
    xp = W4.awq_apply_inv_scale(dev(case.x if xrows is None else case.x[:xrows]), s)
    pw = W4.awq_pack(dev(case.W), s)
    torch.cuda.synchronize()
    qw, sc, qz = case.packed
    assert np.array_equal(host_u16(s), case.s)
    assert np.array_equal(host_u32(pw.qweight), qw)
    assert np.array_equal(host_u16(pw.scales), sc)
    assert np.array_equal(host_u32(pw.qzeros), qz)
    return xp, pw


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)])
def test_decode_gemv_sweep_full_size(K, N):
    case = OracleCase(0, 1, 0, [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)].index((K, N)), 1, N, K)
    xp, pw = prep(case)
    assert np.array_equal(host_u16(xp), case.xp)
    y_ref = case.y_rows()
    y = W4.w4a16_linear(xp, pw)  # the heuristic picks GEMV at M=1
    assert_within_tolerance(y.float().cpu().numpy(), y_ref, f"gemv K={K} N={N}")


@pytest.mark.parametrize("prefetch,fused", [(False, False), (True, False), (False, True)])
def test_decode_stack_launch_configuration(prefetch, fused):
    import bench

    layers = 1 if fused else 2
    shapes = bench.FUSED_SHAPES if fused else bench.DECODE_SHAPES
    cases = {}

    def inputs_fn(li, j, M, N, K):
        c = OracleCase(0, 6 if fused else 2, li, j, M, N, K)
        cases[(li, j)] = c
        return dev(c.W), dev(c.xcal), dev(c.x)

    stack = bench.DecodeStack(torch.device("cuda", 0), layers=layers, inputs_fn=inputs_fn, prefetch=prefetch,
                              fused=fused)
    stack.capture()
    for _ in range(3):  # replays reuse the workspace; outputs must stay correct
        stack.step()
    torch.cuda.synchronize()
    assert W4.awq_last_device_status() == 0
    for i, (pw, xv, yv, K, N) in enumerate(stack.entries):
        c = cases[(i // len(shapes), i % len(shapes))]
        assert np.array_equal(host_u16(xv), c.xp)
        assert_within_tolerance(yv.float().cpu().numpy(), c.y_rows(), f"stack linear {i} K={K} N={N}")


@pytest.mark.parametrize("K,N", [(4096, 14336), (14336, 4096), (4096, 4096)])
def test_prefill_gemm_m2048_full_size(K, N):
    M = 2048
    case = OracleCase(0, 3, 0, [(4096, 14336), (14336, 4096), (4096, 4096)].index((K, N)), M, N, K)
    xp, pw = prep(case)
    y = W4.w4a16_linear(xp, pw).float().cpu().numpy()  # GEMM mode
    ms, ns = sample_pairs(M, N, 2000, seed=K + N)
    y_ref = case.y_pairs(ms, ns)
    assert_within_tolerance(y[ms, ns], y_ref, f"gemm M=2048 K={K} N={N}")


@pytest.mark.parametrize("K,N", [(8192, 28672), (28672, 8192)])
def test_crossover_sweep_both_modes(K, N):
    case = OracleCase(0, 4, 0, [(8192, 28672), (28672, 8192)].index((K, N)), 256, N, K)
    xp_all, pw = prep(case)
    for M in (1, 2, 4, 8, 16, 32, 64, 128, 256):
        xp = xp_all[:M].contiguous()
        ms, ns = sample_pairs(M, N, 300, seed=M)
        y_ref = case.y_pairs(ms, ns)
        for fn in (W4.w4a16_gemv, W4.w4a16_gemm):
            y = fn(xp, pw).float().cpu().numpy()
            assert_within_tolerance(y[ms, ns], y_ref, f"{fn.__name__} M={M} K={K} N={N}")


def test_prefetch_hint_changes_no_output():
    case = OracleCase(0, 1, 0, 2, 1, 14336, 4096)
    xp, pw = prep(case)
    nxt = W4.awq_pack(dev(case.W), None)
    y0 = W4.w4a16_linear(xp, pw)
    y1 = W4.w4a16_linear_pf(xp, pw, nxt)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    assert W4.awq_last_device_status() == 0
