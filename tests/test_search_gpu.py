"""GPU parity of the AWQ scale search (awq_search_scale) against the oracle's search: the same loss at every
grid point, the same winning alpha, and the winner's scale bit for bit.  Both modes of the layer are reached:
R <= 32 calibration rows run the GEMV, more the GEMM.  Loss tolerance: in GEMV mode every product is exact
and summed in fp32, so the losses agree to 1e-4 relative (the layer's fp16 outputs may differ in the last
place where fp32 and fp64 sums straddle a rounding boundary; the reference product is fp32 on the GPU).  In
GEMM mode each dequantized weight (q - z) S is rounded to fp16 before the tensor-core product (about 2^-11
relative per weight, against the ~1e-2 quantization error the loss measures), which moves the loss by up to
about (2^-11 / 1e-2) ~ 5e-2 of its square root's relative size: 1e-3 relative."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
import synth
import weight_only_int4_05_b200 as W4

pytestmark = pytest.mark.gpu

LOSS_RTOL_GEMV = 1e-4
LOSS_RTOL_GEMM = 1e-3


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.float16)


def host_u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_search(W, xcal, n_grid, g=128, what=""):
    N, K = W.shape
    LOSS_RTOL = LOSS_RTOL_GEMV if xcal.shape[0] <= W4.w4a16_gemv_max_m(N, K) else LOSS_RTOL_GEMM
    res = W4.awq_search_scale(dev(W), dev(xcal), n_grid=n_grid, g=g)
    torch.cuda.synchronize()
    best, alpha, s_ref, L_ref = O.awq_search(W, xcal, n_grid, g)
    L = res.losses.cpu().numpy()
    rel = np.abs(L - L_ref) / L_ref
    assert np.all(rel <= LOSS_RTOL), f"{what}: loss rel err {rel.max():.2e} at {int(np.argmax(rel))}"
    srt = np.sort(L_ref)
    if (srt[1] - srt[0]) > 10 * LOSS_RTOL * srt[0]:
        assert res.best == best, f"{what}: GPU picked {res.best}, oracle {best}"
        assert np.array_equal(host_u16(res.s), s_ref)
    else:  # a near tie: either winner is valid, and its scale must be that alpha's
        assert L_ref[res.best] <= srt[0] * (1 + 10 * LOSS_RTOL)
        assert np.array_equal(host_u16(res.s), O.act_pow(xcal, res.best / n_grid))
    assert W4.awq_last_device_status() == 0
    return res, best, L_ref


@pytest.mark.parametrize("R", [64, 16])
def test_search_tiny_layer(R):
    """The tiny layer's shapes (K = 512, N = 256), grid of 21 points, GEMM (R = 64) and GEMV (R = 16)."""
    d = synth.linear_inputs(0, 0, 0, 0, 1, 256, 512)
    xcal = d["xcal"].view(np.uint16)[:R]
    res, best, L = check_search(d["W"].view(np.uint16), xcal, 20, what=f"tiny R={R}")
    assert 0 < best < 20  # the loss curve has an interior minimum on this data


def test_search_decode_shape():
    """A Llama-3-8B attention projection (4096 -> 4096), 16 calibration rows, grid of 5 points."""
    d = synth.linear_inputs(0, 2, 0, 0, 1, 4096, 4096)
    check_search(d["W"].view(np.uint16), d["xcal"].view(np.uint16)[:16], 4, what="4096x4096")


def test_search_salient_channel_and_group_64():
    """The oracle pin's hand-built salient channel, at group size 64: alpha > 0 must win on both sides."""
    rng = np.random.default_rng(53)
    N, K, R = 64, 256, 32
    Wd = 0.02 * rng.standard_normal((N, K))
    Wd[:, 0] = 0.0015 * rng.standard_normal(N)
    x = rng.standard_normal((R, K))
    x[:, 0] *= 40.0
    W = Wd.astype(np.float16).view(np.uint16)
    xcal = x.astype(np.float16).view(np.uint16)
    res, best, L = check_search(W, xcal, 10, g=64, what="salient g=64")
    assert res.best > 0 and L[0] > 2.0 * L[res.best]


def test_search_result_feeds_the_layer():
    """The search's scale is what awq_pack and awq_apply_inv_scale then take: packing with it is bit-exact
    against the oracle's pack with the oracle's winner."""
    d = synth.linear_inputs(1, 0, 0, 1, 1, 128, 256)
    W, xcal = d["W"].view(np.uint16), d["xcal"].view(np.uint16)
    res = W4.awq_search_scale(dev(W), dev(xcal), n_grid=8)
    pw = W4.awq_pack(dev(W), res.s)
    torch.cuda.synchronize()
    _, _, s_ref, _ = O.awq_search(W, xcal, 8)
    qw, sc, qz = O.awq_pack(W, s_ref)
    assert np.array_equal(pw.qweight.cpu().numpy().view(np.uint32), qw)
    assert np.array_equal(host_u16(pw.scales), sc)


def test_search_argument_checks():
    W = torch.zeros((64, 256), dtype=torch.float16, device="cuda")
    with pytest.raises(W4.AwqError):
        W4.awq_search_scale(W, torch.zeros((8, 256), dtype=torch.float16, device="cuda"), n_grid=0)
    with pytest.raises(ValueError):
        W4.awq_search_scale(W, torch.zeros((8, 128), dtype=torch.float16, device="cuda"))
