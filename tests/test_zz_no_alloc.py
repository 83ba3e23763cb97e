"""w4a16_gemv_noalloc, the GEMV entry point for callers that cannot allocate device memory (a plug-in whose
host framework owns every device allocation, or a serving loop whose device memory is fixed at start-up):
its split-K scratch is a static device array owned by the library.  Called through the C ABI on two calls
in a row (the second call finds the first call's leftovers in the shared array) and checked bit for bit
against w4a16_gemv, which runs the same kernel with a caller's workspace, and against the CPU oracle.
Runs alone in a fresh process or after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

from weight_only_int4_05_b200 import _lib, build as libbuild
import weight_only_int4_05_b200 as W4
from helpers import OracleCase, assert_within_tolerance, sample_pairs

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.float16)


def _packed(N, K, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    Wt = (torch.randn((N, K), generator=g, device="cuda") * 0.02).half()
    s = (torch.rand((K,), generator=g, device="cuda") + 0.5).half()
    x = torch.randn((8, K), generator=g, device="cuda").half()
    return W4.awq_pack(Wt, s), x


def _call_noalloc(L, x, pw, y):
    M, K = x.shape
    P = ctypes.c_void_p
    stream = P(torch.cuda.current_stream().cuda_stream)
    return L.w4a16_gemv_noalloc(P(x.data_ptr()), P(pw.qweight.data_ptr()), P(pw.scales.data_ptr()),
                                P(pw.qzeros.data_ptr()), P(y.data_ptr()), M, pw.N, K, 128, stream)


def test_noalloc_matches_gemv_on_two_calls_in_a_row():
    libbuild.build()
    L = _lib.load()
    torch.cuda.set_device(0)
    # both shapes take the split path (a few row blocks more than SMs), whose partial sums live in the
    # library's static scratch
    cases = [(_packed(4864, 8192, 1), 1), (_packed(4800, 4096, 2), 3)]
    for (pw, x_all), M in cases:
        x = x_all[:M].contiguous()
        assert W4.w4a16_workspace_bytes(W4.MODE_GEMV, M, pw.N, pw.K) > 0  # split: scratch in use
        y = torch.empty((M, pw.N), dtype=torch.float16, device="cuda")
        assert _call_noalloc(L, x, pw, y) == 0
        y_ref = W4.w4a16_gemv(x, pw)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), f"noalloc N={pw.N} differs from w4a16_gemv"
    assert W4.awq_last_device_status() == 0


def test_noalloc_matches_the_oracle():
    """A split shape (4096 -> 4864: 152 row blocks), twice in a row, against the oracle."""
    libbuild.build()
    L = _lib.load()
    torch.cuda.set_device(0)
    case = OracleCase(0, 1, 0, 2, 1, 4864, 4096)
    s = W4.awq_act_scale(dev(case.xcal))
    xp = W4.awq_apply_inv_scale(dev(case.x), s)
    pw = W4.awq_pack(dev(case.W), s)
    assert W4.w4a16_workspace_bytes(W4.MODE_GEMV, 1, pw.N, pw.K) > 0
    ms, ns = sample_pairs(1, case.N, 1500, seed=11)
    y_ref = case.y_pairs(ms, ns)
    for _ in range(2):
        y = torch.empty((1, case.N), dtype=torch.float16, device="cuda")
        assert _call_noalloc(L, xp, pw, y) == 0
        torch.cuda.synchronize()
        assert_within_tolerance(y.float().cpu().numpy()[ms, ns], y_ref, "noalloc vs oracle")
    assert W4.awq_last_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    libbuild.build()
    L = _lib.load()
    N, K, M = 6304, 4096, 16  # 197 row blocks, split between CTAs, 16 rows per pass
    need = L.w4a16_workspace_bytes(1, M, N, K, 128)
    assert need > (512 << 10)
    FAKE = ctypes.c_void_p(0x10000)
    st = L.w4a16_gemv_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, M, N, K, 128, None)
    assert st == 6  # AWQ_ERR_WORKSPACE, nothing launched
