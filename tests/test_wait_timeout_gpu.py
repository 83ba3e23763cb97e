"""The timeout path of the bounded waits, made to run out on purpose with a wait that nothing completes:
the kernel returns, the device status word reports AWQ_ERR_DEVICE_TIMEOUT once, and the context stays
usable (the tiny layer still matches the oracle afterwards)."""
import numpy as np
import pytest
import torch

from helpers import OracleCase, assert_within_tolerance
import weight_only_int4_05_b200 as W4

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.float16)


@pytest.mark.parametrize("backoff", [False, True])
def test_wait_gives_up_and_reports_timeout(backoff):
    torch.cuda.set_device(0)
    assert W4.awq_last_device_status() == 0
    assert W4.awq_selftest_wait_timeout(backoff) == 1  # the wait returned without completing
    assert W4.awq_last_device_status() == 5            # AWQ_ERR_DEVICE_TIMEOUT, then cleared
    assert W4.awq_last_device_status() == 0
    case = OracleCase(0, 0, 0, 0, 1, 256, 512)
    s = W4.awq_act_scale(dev(case.xcal))
    xp = W4.awq_apply_inv_scale(dev(case.x), s)
    pw = W4.awq_pack(dev(case.W), s)
    for fn in (W4.w4a16_gemv, W4.w4a16_gemm):
        y = fn(xp, pw).float().cpu().numpy()
        assert_within_tolerance(y, case.y_rows(), fn.__name__)
    assert W4.awq_last_device_status() == 0


def test_split_shapes_after_a_timeout_use_the_cached_workspace():
    """After a wait ran out, split shapes (cross-CTA GEMV combine at 4096 -> 4864, split-K GEMM at
    14336 -> 4096) still find every counter of the shared workspace at zero and match the oracle."""
    torch.cuda.set_device(0)
    assert W4.awq_selftest_wait_timeout(False) == 1
    assert W4.awq_last_device_status() == 5
    for (N, K, M, fn, mode) in ((4864, 4096, 1, W4.w4a16_gemv, W4.MODE_GEMV),
                                (4096, 14336, 8, W4.w4a16_gemm, W4.MODE_GEMM)):
        case = OracleCase(0, 1, 0, 2 if N > K else 3, M, N, K)
        s = W4.awq_act_scale(dev(case.xcal))
        xp = W4.awq_apply_inv_scale(dev(case.x), s)
        pw = W4.awq_pack(dev(case.W), s)
        assert W4.w4a16_workspace_bytes(mode, M, N, K) > 0
        ms, ns = np.meshgrid(np.arange(M), np.arange(0, N, 37), indexing="ij")
        y_ref = case.y_pairs(ms.ravel().astype(np.int32), ns.ravel().astype(np.int32)).reshape(ms.shape)
        for _ in range(2):
            y = fn(xp, pw).float().cpu().numpy()
            assert_within_tolerance(y[ms, ns], y_ref, f"{fn.__name__} after a timeout")
    assert W4.awq_last_device_status() == 0
