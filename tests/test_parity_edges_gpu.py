"""GPU parity on the method's edge cases and on the stream-ordering contract.

  * pack on constructed groups, bit-exact against the oracle: constant and all-zero groups (the 1e-5 scale
    floor), all-positive and all-negative groups (zero point clamped to 0 / 15, codes clamped), exact ties
    w'/S = k + 1/2 (round half to even), groups holding +0 and -0, fp16-subnormal weights, values far from
    the usual range, with s absent, with power-of-two s and with a generic AWQ-like s;
  * AWQ scale -> pack -> 1/s -> GEMV -> GEMM on one stream with no host synchronisation between the calls,
    at the full decode shapes, 20 times over, the packed buffers reused and the weight alternating (a linear
    that read packed weights before pack finished would see the other weight), and the same sequence
    captured in a CUDA graph;
  * activations in the thousands (fp16 partial sums of a few products would overflow there; the kernels
    accumulate in fp32);
  * the M = 2048 prefill GEMM with every 128 x 256 output tile, every 32-row quarter and every 16-column
    epilogue chunk sampled;
  * GEMM token tiles of 64 to 208 columns over 128 k-blocks, repeated in a CUDA graph: bit-identical outputs and
    no timeout (the stage ring's count is a multiple of the dequant warpgroups).
The source passages: "LLM quantization speed-up" (bjdmk.com.cn), "quantization parameters" (zero-point
quantization, group 128); "LLM-AWQ academic impact", "quantization flow" (real quantization, then inference
on the packed weights)."""
import numpy as np
import pytest
import torch

from helpers import OracleCase, assert_within_tolerance
from oracle import oracle as O
import weight_only_int4_05_b200 as W4

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.float16)


def host_u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host_u32(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


PATTERNS = ("constant", "zeros", "signed_zeros", "positive", "negative", "ties", "with_zeros", "subnormal",
            "normal", "large", "one_outlier", "two_values")


def edge_group(kind, rng):
    """128 fp16 weights of one group, constructed for one edge case of the grid."""
    if kind == "constant":
        return np.full(128, rng.normal(0, 0.05), np.float16)
    if kind == "zeros":
        return np.zeros(128, np.float16)
    if kind == "signed_zeros":
        return np.where(rng.random(128) < 0.5, np.float16(0.0), np.float16(-0.0)).astype(np.float16)
    if kind == "positive":
        return np.abs(rng.normal(0.05, 0.02, 128)).astype(np.float16) + np.float16(0.001)
    if kind == "negative":
        return -(np.abs(rng.normal(0.05, 0.02, 128)).astype(np.float16) + np.float16(0.001))
    if kind == "ties":  # min -7.5 S', max +7.5 S' with S' a power of two: every value is (k + 1/2) S'
        sp = 2.0 ** rng.integers(-9, -4)
        v = (rng.integers(-8, 7, 128) + 0.5) * sp
        v[0], v[1] = -7.5 * sp, 7.5 * sp
        return v.astype(np.float16)
    if kind == "with_zeros":
        v = rng.normal(0, 0.02, 128).astype(np.float16)
        v[rng.integers(0, 128, 16)] = np.float16(0.0)
        v[rng.integers(0, 128, 16)] = np.float16(-0.0)
        return v
    if kind == "subnormal":  # |w| below the smallest normal fp16 (6.1e-5)
        return (rng.normal(0, 2e-5, 128)).astype(np.float16)
    if kind == "large":
        return rng.normal(0, 300.0, 128).astype(np.float16)
    if kind == "one_outlier":
        v = rng.normal(0, 0.01, 128).astype(np.float16)
        v[rng.integers(0, 128)] = np.float16(rng.choice([-1.0, 1.0]) * 2.0)
        return v
    if kind == "two_values":
        a, b = rng.normal(0, 0.05, 2)
        return np.where(rng.random(128) < 0.5, a, b).astype(np.float16)
    return rng.normal(0, 0.02, 128).astype(np.float16)


def edge_weight(N, K, seed):
    rng = np.random.default_rng(seed)
    W = np.empty((N, K), np.float16)
    for n in range(N):
        for g in range(K // 128):
            W[n, g * 128:(g + 1) * 128] = edge_group(PATTERNS[(n * 7 + g) % len(PATTERNS)], rng)
    return W.view(np.uint16)


def scale_vector(kind, K, seed):
    rng = np.random.default_rng(seed)
    if kind is None:
        return None
    if kind == "pow2":
        return (2.0 ** rng.integers(-3, 4, K)).astype(np.float16).view(np.uint16)
    return np.sqrt(np.abs(rng.normal(1.0, 0.8, K)) + 0.05).astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("s_kind", [None, "pow2", "awq"])
@pytest.mark.parametrize("N,K", [(72, 1536), (40, 128)])
def test_pack_edge_groups_bitexact(N, K, s_kind):
    W = edge_weight(N, K, seed=N + K)
    s = scale_vector(s_kind, K, seed=K)
    pw = W4.awq_pack(dev(W), None if s is None else dev(s))
    torch.cuda.synchronize()
    qw, sc, qz = O.awq_pack(W, s)
    assert np.array_equal(host_u32(pw.qweight), qw)
    assert np.array_equal(host_u16(pw.scales), sc)
    assert np.array_equal(host_u32(pw.qzeros), qz)


def test_pack_edge_groups_hit_every_branch():
    """The constructed weight really reaches the clamps, the floor and the ties (checked on the oracle)."""
    W = edge_weight(72, 1536, seed=72 + 1536)
    q, sc, z = O.quantize(W, None)
    S = sc.view(np.float16).astype(np.float32)
    assert np.any(S == np.float32(np.float16(1e-5)))       # scale floor
    assert np.any(z == 0) and np.any(z == 15)               # zero point clamped at both ends
    assert np.any(q == 0) and np.any(q == 15)
    w = W.view(np.float16).astype(np.float32)
    ratio = w / np.repeat(S, 128, axis=1)
    assert np.any(np.abs(ratio - np.floor(ratio) - 0.5) == 0)  # exact ties
    assert np.any((W == 0x8000))                               # a negative zero in the input


def _chain_cases():
    a = OracleCase(0, 7, 0, 0, 16, 14336, 4096)
    b = OracleCase(0, 7, 0, 1, 16, 14336, 4096)
    c = OracleCase(0, 7, 1, 0, 16, 4096, 14336)
    d = OracleCase(0, 7, 1, 1, 16, 4096, 14336)
    return [(a, b), (c, d)]


def _outputs_ok(case, y_gemv, y_gemm):
    ms = np.array([0] * 64 + list(range(16)) * 4, np.int32)
    ns = np.random.default_rng(case.N).integers(0, case.N, len(ms)).astype(np.int32)
    y_ref = case.y_pairs(ms, ns)
    g = y_gemv.float().cpu().numpy()
    assert_within_tolerance(g[0, ns[:64]], y_ref[:64], "gemv after pack, no sync")
    m = y_gemm.float().cpu().numpy()
    assert_within_tolerance(m[ms, ns], y_ref, "gemm after pack, no sync")


@pytest.mark.parametrize("pair", [0, 1])
def test_pack_then_linear_without_sync(pair):
    """Each iteration repacks into the same buffers (alternating weights) and runs both linears right
    after, with no synchronisation; every iteration's outputs must belong to that iteration's weight."""
    ca, cb = _chain_cases()[pair]
    inputs = [(dev(c.W), dev(c.xcal), dev(c.x)) for c in (ca, cb)]
    pw = W4.awq_pack(inputs[0][0], None)
    torch.cuda.synchronize()
    outs = []
    for it in range(20):
        Wd, xcal, x = inputs[it % 2]
        s = W4.awq_act_scale(xcal)
        W4.awq_pack(Wd, s, out=pw)
        xp = W4.awq_apply_inv_scale(x, s)
        y1 = W4.w4a16_gemv(xp[:1].contiguous(), pw)
        y2 = W4.w4a16_gemm(xp, pw)
        outs.append((y1, y2))
    torch.cuda.synchronize()
    assert W4.awq_last_device_status() == 0
    for it in (0, 1, 18, 19):
        _outputs_ok((ca, cb)[it % 2], *outs[it])
    for it in range(2, 20):  # every later iteration reproduces the first two bit for bit
        assert torch.equal(outs[it][0], outs[it % 2][0]) and torch.equal(outs[it][1], outs[it % 2][1])
    qw, sc, qz = cb.packed  # the buffers hold the last weight
    assert np.array_equal(host_u32(pw.qweight), qw)


def test_pack_then_linear_in_a_cuda_graph():
    ca, cb = _chain_cases()[0]
    inputs = [(dev(c.W), dev(c.xcal), dev(c.x)) for c in (ca, cb)]
    pw = W4.awq_pack(inputs[0][0], None)
    M, K, N = 16, ca.K, ca.N
    ss = [torch.empty(K, dtype=torch.float16, device="cuda") for _ in range(2)]
    xps = [torch.empty((M, K), dtype=torch.float16, device="cuda") for _ in range(2)]
    y1 = [torch.empty((1, N), dtype=torch.float16, device="cuda") for _ in range(2)]
    y2 = [torch.empty((M, N), dtype=torch.float16, device="cuda") for _ in range(2)]
    ws = W4.reserve_workspace(max(W4.w4a16_workspace_bytes(W4.MODE_GEMV, 1, N, K),
                                  W4.w4a16_workspace_bytes(W4.MODE_GEMM, M, N, K)))

    def seq():
        for i in range(2):
            Wd, xcal, x = inputs[i]
            W4.awq_act_scale(xcal, out=ss[i])
            W4.awq_pack(Wd, ss[i], out=pw)
            W4.awq_apply_inv_scale(x, ss[i], out=xps[i])
            W4.w4a16_gemv(xps[i][:1], pw, out=y1[i], workspace=ws)
            W4.w4a16_gemm(xps[i], pw, out=y2[i], workspace=ws)

    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        seq()
    torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        seq()
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    assert W4.awq_last_device_status() == 0
    for i, c in enumerate((ca, cb)):
        _outputs_ok(c, y1[i], y2[i])


@pytest.mark.parametrize("K,N", [(4096, 1024), (14336, 512)])
def test_linear_with_activations_in_the_thousands(K, N):
    """x' of magnitude 1000-4000 (fp16 partial sums of 16 such products would overflow)."""
    rng = np.random.default_rng(K)
    case = OracleCase(1, 8, 0, 0, 1, N, K)
    xp = (rng.choice([-1.0, 1.0], (16, K)) * rng.uniform(1000, 4000, (16, K))).astype(np.float16).view(np.uint16)
    q, sc, z = case.q, case.sc, case.z
    pw = W4.awq_pack(dev(case.W), dev(case.s))
    for M in (1, 4, 16):
        ms, ns = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        y_ref = O.linear_pairs_f64(xp[:M], q, sc, z, ms.ravel(), ns.ravel()).reshape(M, N)
        for fn in (W4.w4a16_gemv, W4.w4a16_gemm):
            y = fn(dev(xp[:M]), pw).float().cpu().numpy()
            assert np.all(np.isfinite(y)), f"{fn.__name__} M={M}: non-finite output"
            assert_within_tolerance(y, y_ref, f"{fn.__name__} M={M} K={K} N={N} |x'| in the thousands")


def test_prefill_gemm_m2048_every_tile_quarter_and_chunk():
    """(K, N) = (4096, 4096) at M = 2048: one sample in every (128-row tile, 256-token tile, 32-row quarter,
    16-column epilogue chunk) -- 16,384 outputs spread over all 256 output tiles."""
    M, K, N = 2048, 4096, 4096
    case = OracleCase(0, 3, 1, 2, M, N, K)
    s = W4.awq_act_scale(dev(case.xcal))
    xp = W4.awq_apply_inv_scale(dev(case.x), s)
    pw = W4.awq_pack(dev(case.W), s)
    y = W4.w4a16_gemm(xp, pw).float().cpu().numpy()
    rng = np.random.default_rng(7)
    ms, ns = [], []
    for nt in range(N // 128):
        for tt in range(M // 256):
            for qq in range(4):
                for ch in range(16):
                    ns.append(nt * 128 + qq * 32 + int(rng.integers(0, 32)))
                    ms.append(tt * 256 + ch * 16 + int(rng.integers(0, 16)))
    ms, ns = np.array(ms, np.int32), np.array(ns, np.int32)
    assert_within_tolerance(y[ms, ns], case.y_pairs(ms, ns), "gemm M=2048 every tile")


def test_prefill_gemm_short_last_wave_split():
    """(K, N) = (4096, 14336) at M = 2048 is 896 output tiles: six whole waves on 148 SMs run as one launch and
    the last 8 tiles as a second launch with K split 8 ways (workspace partials summed in split order).  One
    sample in every (32-row quarter, 16-column chunk) of those 8 tiles and of 8 tiles of the first launch."""
    M, K, N = 2048, 4096, 14336
    case = OracleCase(0, 3, 2, 5, M, N, K)
    s = W4.awq_act_scale(dev(case.xcal))
    xp = W4.awq_apply_inv_scale(dev(case.x), s)
    pw = W4.awq_pack(dev(case.W), s)
    y = W4.w4a16_gemm(xp, pw).float().cpu().numpy()
    n_tiles = N // 128
    rng = np.random.default_rng(13)
    ms, ns = [], []
    for tile in list(range(888, 896)) + list(range(880, 888)):
        nt, tt = tile % n_tiles, tile // n_tiles
        for qq in range(4):
            for ch in range(16):
                ns.append(nt * 128 + qq * 32 + int(rng.integers(0, 32)))
                ms.append(tt * 256 + ch * 16 + int(rng.integers(0, 16)))
    ms, ns = np.array(ms, np.int32), np.array(ns, np.int32)
    assert_within_tolerance(y[ms, ns], case.y_pairs(ms, ns), "gemm M=2048 last-wave split")
    assert W4.awq_last_device_status() == 0


@pytest.mark.parametrize("M", [64, 128, 176])
def test_gemm_token_tiles_between_48_and_256_repeat_exactly(M):
    """Token tiles of 64 to 208 columns (stages of 29-53 KB) over 128 k-blocks per tile, 30 launches in one CUDA
    graph replayed twice: every output equals the first call's bit for bit, the first call is within the layer
    tolerance of the oracle, and no bounded wait runs out.  (A ring whose stage count is not a multiple of the
    dequant warpgroups lets two warpgroups share a stage, and out-of-order copies then let a parity wait match
    an old phase: wrong tiles or a timeout, rarely.)"""
    K, N = 8192, 14336
    case = OracleCase(0, 4, 3, M, M, N, K)
    s = W4.awq_act_scale(dev(case.xcal))
    xp = W4.awq_apply_inv_scale(dev(case.x), s)
    pw = W4.awq_pack(dev(case.W), s)
    y0 = W4.w4a16_gemm(xp, pw)
    torch.cuda.synchronize()
    assert W4.awq_last_device_status() == 0
    rng = np.random.default_rng(M)
    ms = np.concatenate([[0, M - 1], rng.integers(0, M, 1500)]).astype(np.int32)
    ns = np.concatenate([[0, N - 1], rng.integers(0, N, 1500)]).astype(np.int32)
    assert_within_tolerance(y0.float().cpu().numpy()[ms, ns], case.y_pairs(ms, ns), f"gemm M={M} K={K} N={N}")
    outs = [torch.empty_like(y0) for _ in range(30)]
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        W4.w4a16_gemm(xp, pw, out=outs[0])
        st.synchronize()
        with torch.cuda.graph(g, stream=st):
            for o in outs:
                W4.w4a16_gemm(xp, pw, out=o)
    for _ in range(2):
        for o in outs:
            o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert W4.awq_last_device_status() == 0
        for o in outs:
            assert torch.equal(o, y0)
