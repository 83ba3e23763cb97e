"""Pins of the CPU oracle against things other than itself (CPU only).

Each test names the oracle function it pins and what it is pinned to: numpy's IEEE conversions, a
closed form obtained by construction, an invariant of the grid, a brute-force search, or a library
routine that the special case reduces to.  A plausible slip in the oracle (a dropped term, a wrong
sign, a transposed index) fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.txt")


def f16(a):
    return np.asarray(a, np.float16).view(np.uint16)


def h2f(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


# ---------------------------------------------------------------- fp16 conversions ---------------
def test_f16_widening_matches_numpy_all_patterns():
    """oracle_f16_to_f64 vs numpy float16 -> float64 over all 65536 bit patterns."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([O.f16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def _narrowing_sample(rng):
    # every fp16 value, every midpoint between neighbours (ties), and the midpoints nudged by
    # 1 ulp of double either way, plus random doubles spanning subnormal .. overflow
    h = np.arange(0, 0x7C00, dtype=np.uint16)
    v = h.view(np.float16).astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2
    nudged = np.concatenate([np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf)])
    rnd = np.exp(rng.uniform(np.log(1e-9), np.log(7e4), 200000))
    vals = np.concatenate([v, mids, nudged, rnd, [65504.0, 65519.0, 65519.999, 65520.0, 1e9, 0.0]])
    return np.concatenate([vals, -vals])


def test_f64_to_f16_matches_numpy_single_rounding():
    """oracle_f64_to_f16 vs numpy's direct float64 -> float16 (round to nearest even)."""
    vals = _narrowing_sample(np.random.default_rng(1))
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([O.f64_to_f16(float(d)) for d in vals], np.uint16)
    assert np.array_equal(got, ref)


def test_f32_to_f16_matches_numpy():
    """oracle_f32_to_f16 vs numpy float32 -> float16 on random float32 bit patterns and ties."""
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 2**31, 300000, dtype=np.uint32)
    bits = bits[(bits & 0x7F800000) != 0x7F800000]  # drop NaN / Inf patterns
    vals = bits.view(np.float32)
    vals = np.concatenate([vals, -vals, (h2f(np.arange(1, 0x7BFF)) + h2f(np.arange(2, 0x7C00))).astype(
        np.float32) / np.float32(2)])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([O.f32_to_f16(float(f)) for f in vals], np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- a1: AWQ scale ------------------
def test_act_scale_closed_forms():
    """oracle_act_scale: s_j = fp16(sqrt(mean_r |x_rj|)).  Columns built so that the mean absolute
    value is a known perfect square: the sign pattern, the row count and the column index all matter."""
    R, K = 64, 6
    x = np.zeros((R, K), np.float64)
    x[:, 0] = 4.0                                    # mean 4 -> 2
    x[:, 1] = np.where(np.arange(R) % 2, 9.0, -9.0)  # |.| drops the sign: mean 9 -> 3
    x[:, 2] = np.where(np.arange(R) < 16, 1.0, 0.0)  # mean 16/64 = 0.25 -> 0.5
    x[:, 3] = -0.0625                                # mean 1/16 -> 0.25
    x[:32, 4] = 2.0                                  # mean 1 -> 1
    x[:, 5] = np.where(np.arange(R) % 4 == 0, -64.0, 0.0)  # mean 16 -> 4
    s = O.act_scale(f16(x))
    assert list(h2f(s)) == [2.0, 3.0, 0.5, 0.25, 1.0, 4.0]


def test_act_scale_non_power_of_two_rows_matches_exact_rational():
    """R = 3: mean = sum/3 is inexact; the result equals fp16 of the correctly rounded sqrt of the
    correctly rounded fp64 quotient, computed here with exact rationals and math.sqrt."""
    x = f16(np.array([[1.0, 0.5, 7.0], [2.0, -0.25, 1.0], [-4.0, 0.125, 0.0]]))
    s = O.act_scale(x)
    for j in range(3):
        total = sum(Fraction(abs(v)) for v in h2f(x[:, j]))   # exact
        mean = float(total / 3)                               # one rounding (Fraction -> float)
        exp = np.array([math.sqrt(mean)]).astype(np.float16).view(np.uint16)[0]
        assert s[j] == exp


# ---------------------------------------------------------------- a7: x / s ----------------------
def test_inv_scale_powers_of_two_exact():
    """oracle_inv_scale: with s_k a power of two, x / s is exact in fp16; a multiply instead of a divide,
    or indexing s by row, fails."""
    rng = np.random.default_rng(3)
    M, K = 3, 8
    x = f16(rng.standard_normal((M, K)))
    e = np.array([-2, -1, 0, 1, 2, 3, -3, 0])
    s = f16(2.0 ** e)
    xp = O.inv_scale(x, s)
    assert np.array_equal(h2f(xp), h2f(x) / 2.0 ** e[None, :])


def test_inv_scale_x_equal_s_gives_one():
    s = f16(np.array([0.3, 1.7, 12.5, 0.001]))
    x = np.stack([s, s])
    assert np.all(h2f(O.inv_scale(x, s)) == 1.0)


# ---------------------------------------------------------------- a2..a5: grid -------------------
def _grid_group(S0, z0, codes):
    return (np.asarray(codes, np.float64) - z0) * S0


@pytest.mark.parametrize("S0,z0", [(0.0078125, 5), (0.13232421875, 8), (0.000244140625, 0),
                                   (0.5, 15), (0.0029296875, 3)])
def test_quantize_reproduces_its_own_grid(S0, z0):
    """By construction: a group whose values are exactly (j - z0) * S0 for j covering 0..15 has
    range 15 * S0, so the scale is S0, the zero is z0 and every code is recovered (closed form)."""
    rng = np.random.default_rng(int(S0 * 1e6) + z0)
    codes = np.concatenate([np.arange(16), rng.integers(0, 16, 128 - 16)])
    rng.shuffle(codes)
    w = _grid_group(S0, z0, codes)
    W = f16(w[None, :])
    assert np.array_equal(h2f(W)[0], w)  # the construction is exact in fp16
    q, sc, z = O.quantize(W)
    assert h2f(sc)[0, 0] == S0 and z[0, 0] == z0
    assert np.array_equal(q[0], codes)
    assert np.array_equal(O.dequant(q, sc, z)[0].astype(np.float64), w)


def test_quantize_all_positive_group_clamps_zero_and_top():
    """All values > 0: -min/S < 0 so the zero clamps to 0, and values above 15.5 S clamp to code 15."""
    w = np.linspace(1.0, 2.0, 128)
    q, sc, z = O.quantize(f16(w[None, :]))
    S = h2f(sc)[0, 0]
    assert z[0, 0] == 0
    assert q[0].max() == 15 and np.all(q[0][h2f(f16(w)) > 15.5 * S] == 15)


def test_quantize_degenerate_group():
    """max == min: the scale takes its floor 1e-5 (fp16 of it) and no code leaves 0..15."""
    for c in (0.0, 0.37, -0.37):
        q, sc, z = O.quantize(f16(np.full((1, 128), c)))
        assert sc[0, 0] == f16(np.float32(1e-5))[()]
        assert 0 <= q.min() and q.max() <= 15 and 0 <= z[0, 0] <= 15
        if c == 0.0:
            assert np.all(q[0] == z[0, 0])  # zero maps to the zero point exactly


def _synthetic_group_rows(N=16, K=512, seed=5):
    d = synth.linear_inputs(seed, 0, 0, 0, 1, N, K)
    s = O.act_scale(d["xcal"])
    return d["W"].view(np.uint16), s


def test_quantize_roundtrip_bound():
    """Invariant: for groups with min <= 0 <= max, |w' - (q - z) S| <= S (1/2 + 16 * 2^-11) for every
    element (1/2 from rounding to the grid; the rest from rounding the scale to fp16)."""
    W, s = _synthetic_group_rows()
    q, sc, z = O.quantize(W, s)
    wp = h2f(W) * h2f(s)[None, :]           # exact fold in fp64
    deq = O.dequant(q, sc, z).astype(np.float64)
    S = np.repeat(h2f(sc), 128, axis=1)
    assert np.all(np.abs(wp - deq) <= S * (0.5 + 16 * 2.0**-11))


def test_quantize_codes_are_nearest_grid_points_brute_force():
    """Brute force: given (S, z), each code is the nearest of the 16 grid points (j - z) S to w',
    and z is the grid offset nearest to -min/S; ties within 1e-6 S are skipped."""
    W, s = _synthetic_group_rows(N=8, K=256)
    q, sc, z = O.quantize(W, s)
    wp = h2f(W) * h2f(s)[None, :]
    G = 2
    for n in range(W.shape[0]):
        for g in range(G):
            S = h2f(sc)[n, g]
            zz = int(z[n, g])
            grp = wp[n, g * 128:(g + 1) * 128]
            dz = np.abs(-grp.min() / S - np.arange(16))
            if np.sort(dz)[1] - np.sort(dz)[0] > 1e-6:
                assert zz == int(np.argmin(dz))
            for e, v in enumerate(grp):
                d = np.abs(v - (np.arange(16) - zz) * S)
                srt = np.sort(d)
                if srt[1] - srt[0] > 1e-6 * S:
                    assert q[n, g * 128 + e] == int(np.argmin(d))


def test_quantize_group_boundaries_are_per_row_and_per_group():
    """Groups of 128 along K within each row: a row whose second group is 8x larger gets an 8x scale
    there and nowhere else; a transposed or misaligned group index fails."""
    base = np.tile(np.linspace(-0.5, 0.5, 128), 2)
    W = np.stack([base, base * np.r_[np.ones(128), 8 * np.ones(128)], base * 0.25])
    q, sc, z = O.quantize(f16(W))
    S = h2f(sc)
    assert S[1, 0] == S[0, 0] and S[1, 1] == 8 * S[0, 1] and S[2, 0] == S[0, 0] / 4
    assert np.array_equal(q[0], q[1]) and np.array_equal(q[0], q[2])


def test_quantize_fold_direction_with_power_of_two_scale():
    """Fold a2: quantize(W, s) equals quantize(fp16(W * s), s = 1) when s is a power of two (the
    product is then exact in fp16); dividing by s instead fails."""
    rng = np.random.default_rng(7)
    W = f16(0.02 * rng.standard_normal((4, 256)))
    s = f16(2.0 ** rng.integers(-2, 3, 256))
    a = O.quantize(W, s)
    b = O.quantize(f16(h2f(W) * h2f(s)[None, :]))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_quantize_s_none_equals_s_one():
    """s = NULL means s = 1 (plain round-to-nearest, the baseline AWQ is compared with)."""
    W, _ = _synthetic_group_rows(N=8, K=256)
    a = O.quantize(W, None)
    b = O.quantize(W, f16(np.ones(256)))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


# ---------------------------------------------------------------- a6: packed layout --------------
def _expected_location(n, k, K):
    """Word index and bit offset of (n, k) read off the public header's prose layout description."""
    rb, r, kc = n // 32, n % 32, k // 32
    j, e = (k % 32) // 8, k % 8
    p = e // 2 if e % 2 == 0 else 4 + e // 2
    return (rb * (K // 32) + kc) * 128 + r * 4 + j, 4 * p


def test_pack_single_nibble_placement():
    """oracle_pack: a single nonzero code lands exactly at the word and nibble the header describes."""
    N, K = 40, 256
    rng = np.random.default_rng(11)
    for _ in range(60):
        n, k, c = int(rng.integers(N)), int(rng.integers(K)), int(rng.integers(1, 16))
        q = np.zeros((N, K), np.uint8)
        q[n, k] = c
        qw, _, _ = O.pack(q, np.zeros((N, 2), np.uint16), np.zeros((N, 2), np.uint8))
        word, bit = _expected_location(n, k, K)
        exp = np.zeros_like(qw)
        exp[word] = c << bit
        assert np.array_equal(qw, exp)


def test_pack_scales_and_zeros_placement_and_padding():
    N, K = 40, 384  # N_pad = 64, G = 3
    G, Np = 3, 64
    rng = np.random.default_rng(12)
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sc = f16(rng.uniform(0.001, 0.01, (N, G)))
    z = rng.integers(0, 16, (N, G)).astype(np.uint8)
    qw, scales, qz = O.pack(q, sc, z)
    assert (qw.nbytes, scales.nbytes, qz.nbytes) == O.packed_sizes(N, K)
    for n in range(Np):
        for g in range(G):
            unit = (n // 32) * G + g        # unit-major, as the header describes
            got_s = scales[unit * 32 + n % 32]
            got_z = (qz[unit * 4 + (n % 32) // 8] >> (4 * (n % 8))) & 0xF
            if n < N:
                assert got_s == sc[n, g] and got_z == z[n, g]
            else:
                assert got_s == 0 and got_z == 0
    # padding rows hold code 0: their whole 16-byte row slot in every tile is zero
    words = qw.reshape(Np // 32, K // 32, 32, 4)
    assert np.all(words[1, :, N - 32:, :] == 0)


def test_pack_mask_property_stated_in_header():
    """The header promises: word & 0x000F000F puts channels e=0,1 in the two 16-bit halves, 0x00F000F0
    e=2,3, and the word >> 8 gives e=4,5 and e=6,7 the same way."""
    N, K = 32, 32
    codes = np.random.default_rng(13).integers(0, 16, (N, K)).astype(np.uint8)
    qw, _, _ = O.pack(codes, np.zeros((N, 1), np.uint16), np.zeros((N, 1), np.uint8))
    for r in range(N):
        for j in range(4):
            w = int(qw[r * 4 + j])
            c = codes[r, 8 * j:8 * j + 8]
            lo = lambda v: (v & 0xFFFF)  # noqa: E731
            hi = lambda v: (v >> 16)     # noqa: E731
            assert (lo(w & 0x000F000F), hi(w & 0x000F000F)) == (c[0], c[1])
            assert (lo(w & 0x00F000F0) >> 4, hi(w & 0x00F000F0) >> 4) == (c[2], c[3])
            w8 = w >> 8
            assert (lo(w8 & 0x000F000F), hi(w8 & 0x000F000F)) == (c[4], c[5])
            assert (lo(w8 & 0x00F000F0) >> 4, hi(w8 & 0x00F000F0) >> 4) == (c[6], c[7])


def test_pack_unpack_roundtrip_independent_decoder():
    """oracle_unpack (walks the storage in order) inverts oracle_pack (walks the matrix in order)."""
    rng = np.random.default_rng(14)
    for N, K in [(8, 128), (40, 256), (96, 512)]:
        G = K // 128
        q = rng.integers(0, 16, (N, K)).astype(np.uint8)
        sc = rng.integers(0, 0x7BFF, (N, G)).astype(np.uint16)
        z = rng.integers(0, 16, (N, G)).astype(np.uint8)
        out = O.unpack(*O.pack(q, sc, z), N, K)
        for a, b in zip(out, (q, sc, z)):
            assert np.array_equal(a, b)


def test_packed_bytes_match_page_memory_reduction():
    """The page's "75% less memory" for W4A16 (AWQ and GPTQ algorithms, section 2.3) against the
    packed size: (0.5 + 2/128 + 0.5/128) / 2 bytes per weight = 0.2598, a 74.0% reduction."""
    figs = {}
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            kv = line.split(";")[0]
            k, v = kv.split("=")
            figs[k.strip()] = float(v)
    assert figs["q_group_size"] == O.GROUP and figs["w_bit"] == 4
    N, K = 4096, 4096
    total = sum(O.packed_sizes(N, K))
    ratio = total / (2.0 * N * K)
    assert abs(ratio - (0.5 + 2.5 / 128) / 2) < 1e-12
    assert abs((1 - ratio) * 100 - figs["memory_reduction_percent"]) < 1.5


# ---------------------------------------------------------------- dequant + matmul ---------------
def test_dequant_zero_point_is_exact_zero_and_product_exact():
    rng = np.random.default_rng(15)
    N, K = 8, 256
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    z = rng.integers(0, 16, (N, 2)).astype(np.uint8)
    q[:, :128] = z[:, :1]  # first group: every code equals the zero point
    sc = f16(rng.uniform(1e-4, 0.5, (N, 2)))
    Wq = O.dequant(q, sc, z)
    assert np.all(Wq[:, :128] == 0.0)
    exact = (q.astype(np.float64) - np.repeat(z, 128, axis=1)) * np.repeat(h2f(sc), 128, axis=1)
    assert np.array_equal(Wq.astype(np.float64), exact)


def test_linear_f64_brute_force_and_library():
    """oracle_linear_f64 vs math.fsum over explicit products (brute force) and vs torch's CPU fp64
    matmul, on non-square shapes so that a transposed operand fails."""
    import torch

    rng = np.random.default_rng(16)
    for M, N, K in [(1, 16, 128), (3, 5, 256), (4, 16, 512)]:
        xp = f16(rng.standard_normal((M, K)))
        Wq = (rng.integers(-8, 8, (N, K)) * 0.01).astype(np.float32)
        y = O.linear_f64(xp, Wq)
        X = h2f(xp)
        for m in range(M):
            for n in range(N):
                exact = math.fsum(float(X[m, k]) * float(Wq[n, k]) for k in range(K))
                assert abs(y[m, n] - exact) <= 1e-12 * max(1.0, abs(exact))
        ref = (torch.from_numpy(X) @ torch.from_numpy(Wq.astype(np.float64)).T).numpy()
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_linear_f64_integer_exact():
    """Integer-valued operands: the fp64 sum is exact, so y equals the integer matmul bit for bit."""
    rng = np.random.default_rng(17)
    M, N, K = 2, 7, 384
    xi = rng.integers(-50, 50, (M, K))
    wi = rng.integers(-15, 16, (N, K))
    y = O.linear_f64(f16(xi.astype(np.float64)), wi.astype(np.float32))
    assert np.array_equal(y, (xi @ wi.T).astype(np.float64))


def test_linear_pairs_matches_full():
    W, s = _synthetic_group_rows(N=24, K=384)
    xp = f16(np.random.default_rng(18).standard_normal((3, 384)))
    q, sc, z = O.quantize(W, s)
    full = O.linear_f64(xp, O.dequant(q, sc, z))
    ms, ns = np.meshgrid(np.arange(3), np.arange(24), indexing="ij")
    pairs = O.linear_pairs_f64(xp, q, sc, z, ms.ravel(), ns.ravel())
    assert np.array_equal(pairs, full.ravel())


# ---------------------------------------------------------------- whole path ---------------------
def test_awq_scaling_is_neutral_before_rounding():
    """AWQ and GPTQ algorithms, section 2.1 (3): scaling weight channels by s and the activations by
    1/s leaves x W^T unchanged.  With s a power of two every rounding in the oracle is exact, so the
    whole path (fold, 1/s, quantize, matmul) must equal the same path on fp16(W s) and x / s computed
    here exactly; and in fp64 with arbitrary s the identity holds to 1e-12."""
    rng = np.random.default_rng(19)
    M, N, K = 2, 16, 256
    W = f16(0.02 * rng.standard_normal((N, K)))
    x = f16(rng.standard_normal((M, K)))
    e = rng.integers(-3, 4, K)
    s = f16(2.0 ** e)
    y_awq = O.reference_linear(O.inv_scale(x, s), W, s)
    y_ref = O.reference_linear(f16(h2f(x) / 2.0 ** e), f16(h2f(W) * 2.0 ** e))
    assert np.array_equal(y_awq, y_ref)
    sa = rng.uniform(0.3, 3.0, K)
    Wd, xd = h2f(W), h2f(x)
    a = (xd / sa) @ (Wd * sa).T
    b = xd @ Wd.T
    assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))


def test_quantized_linear_within_grid_error_bound():
    """|y_q - x' (W s)^T| <= sum_k |x'_k| S_{g(k)} (1/2 + 16 * 2^-11): the layer's error is bounded by
    the per-element grid bound (a dropped zero point or scale breaks it)."""
    d = synth.linear_inputs(21, 0, 0, 0, 2, 32, 512)
    s = O.act_scale(d["xcal"])
    xp = O.inv_scale(d["x"], s)
    q, sc, z = O.quantize(d["W"], s)
    yq = O.linear_f64(xp, O.dequant(q, sc, z))
    y = h2f(xp) @ (h2f(d["W"].view(np.uint16)) * h2f(s)[None, :]).T
    S = np.repeat(h2f(sc), 128, axis=1)
    bound = np.abs(h2f(xp)) @ (S * (0.5 + 16 * 2.0**-11)).T
    assert np.all(np.abs(yq - y) <= bound)
    # a real comparison: y is the unquantized layer (not zero), and 4-bit RTN stays well inside it
    assert np.linalg.norm(yq - y) < 0.2 * np.linalg.norm(y)


# ---------------------------------------------------------------- reading used by the fused 1/s GEMV ---
def _fp16_ties_of_division():
    """Exact fp16 rounding midpoints x / s = m 2^-25 (m odd, subnormal results) with fp16 x and s."""
    xs, ss = [], []
    for k in (3, 5, 7, 11, 13, 99, 1023, 2047):
        for e in (1, 2, 3, 4):
            s_ = k * 2.0 ** e
            for m in range(1, 2048, 2):
                v = s_ * m * 2.0 ** -25
                if v < 6.1e-5 and float(np.float16(v)) == v and float(np.float16(s_)) == s_:
                    xs.append(v)
                    ss.append(s_)
    return np.array(xs, np.float16), np.array(ss, np.float16)


def test_fp32_quotient_rounds_to_fp16_like_the_oracle_inv_scale():
    """The fused 1/s GEMV divides in fp32 and rounds once to fp16; oracle_inv_scale divides in fp64.  For
    fp16 operands the two agree: away from exact midpoints the quotient lies at least 2^-23 (relative) from
    any fp16 rounding midpoint, more than fp32's half ulp, and an exact midpoint is representable in fp32.
    Checked here on 400k random operand pairs (all exponents, subnormals, both signs) and on every exact
    subnormal tie of a family of odd scales (numpy's float32 division and float16 conversion are IEEE)."""
    rng = np.random.default_rng(5)
    n = 400000
    xb = (rng.integers(0, 0x7C00, n).astype(np.uint16) | (rng.integers(0, 2, n).astype(np.uint16) << 15))
    sb = rng.integers(0x0001, 0x7C00, n).astype(np.uint16)
    with np.errstate(all="ignore"):
        q32 = (xb.view(np.float16).astype(np.float32) / sb.view(np.float16).astype(np.float32)).astype(np.float16)
    ref = O.inv_scale(xb.reshape(1, -1), sb)[0]
    assert np.array_equal(q32.view(np.uint16), ref)
    xt, st = _fp16_ties_of_division()
    assert len(xt) > 500
    q32 = (xt.astype(np.float32) / st.astype(np.float32)).astype(np.float16).view(np.uint16)
    ref = O.inv_scale(xt.view(np.uint16).reshape(1, -1), st.view(np.uint16))[0]
    assert np.array_equal(q32, ref)
    # the ties really are ties: half of them round down to an even code, half up
    assert set(np.unique(ref & 1)) == {0}


# ---------------------------------------------------------------- other group sizes ----------------
# --q_group_size is a parameter of the page's command line ("LLM-AWQ academic impact", "quantization
# flow"); the oracle's grid and layout take the group size g as an argument.  These pins run at g = 64 and
# g = 256, where a group-size slip (a hard-wired 128, a unit of the wrong length) shows.
@pytest.mark.parametrize("g", [64, 256])
def test_quantize_reproduces_its_own_grid_other_group_sizes(g):
    """Closed form by construction, as at g = 128: a group of exact grid values (j - z0) S0 covering
    codes 0..15 gives back S0, z0 and every code -- in each of the K / g groups of the row."""
    S0, z0 = 0.0078125, 6
    rng = np.random.default_rng(g)
    K = 2 * g
    codes = np.concatenate([np.concatenate([np.arange(16), rng.integers(0, 16, g - 16)]) for _ in range(2)])
    w = (codes.astype(np.float64) - z0) * S0 * np.repeat([1.0, 4.0], g)  # second group 4x wider
    q, sc, z = O.quantize(f16(w[None, :]), None, g)
    assert sc.shape == (1, 2) and h2f(sc)[0, 0] == S0 and h2f(sc)[0, 1] == 4 * S0
    assert np.all(z == z0) and np.array_equal(q[0], codes)


@pytest.mark.parametrize("g", [64, 256])
def test_group_boundaries_other_group_sizes(g):
    """Groups are runs of g channels: scaling channels [g, 2g) of a row by 8 changes that group's scale
    and no other, and leaves every code unchanged."""
    base = np.tile(np.linspace(-0.5, 0.5, g), 3)
    W = np.stack([base, base * np.r_[np.ones(g), 8 * np.ones(g), np.ones(g)]])
    q, sc, z = O.quantize(f16(W), None, g)
    S = h2f(sc)
    assert S.shape == (2, 3)
    assert S[1, 0] == S[0, 0] and S[1, 1] == 8 * S[0, 1] and S[1, 2] == S[0, 2]
    assert np.array_equal(q[0], q[1])


@pytest.mark.parametrize("g", [64, 256])
def test_pack_units_other_group_sizes(g):
    """Header layout at group size g: unit u = rb * G + gi holds 16 g contiguous code bytes (a nonzero code
    at (n, k) lands inside unit (n / 32) * G + k / g's byte range), and its 32 scales and zeros sit at
    unit-major offsets; unpack inverts pack."""
    N, K = 40, 4 * g if g == 64 else 2 * g
    G = K // g
    rng = np.random.default_rng(3 * g)
    for _ in range(40):
        n, k, c = int(rng.integers(N)), int(rng.integers(K)), int(rng.integers(1, 16))
        q = np.zeros((N, K), np.uint8)
        q[n, k] = c
        qw, _, _ = O.pack(q, np.zeros((N, G), np.uint16), np.zeros((N, G), np.uint8), g)
        word, bit = _expected_location(n, k, K)
        assert qw[word] == c << bit and np.count_nonzero(qw) == 1
        u = (n // 32) * G + k // g
        assert u * 16 * g <= 4 * word < (u + 1) * 16 * g
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sc = rng.integers(1, 0x7BFF, (N, G)).astype(np.uint16)
    z = rng.integers(0, 16, (N, G)).astype(np.uint8)
    qw, scales, qz = O.pack(q, sc, z, g)
    assert (qw.nbytes, scales.nbytes, qz.nbytes) == O.packed_sizes(N, K, g)
    for n in range(N):
        for gi in range(G):
            unit = (n // 32) * G + gi
            assert scales[unit * 32 + n % 32] == sc[n, gi]
            assert (qz[unit * 4 + (n % 32) // 8] >> (4 * (n % 8))) & 0xF == z[n, gi]
    for a, b in zip(O.unpack(qw, scales, qz, N, K, g), (q, sc, z)):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("g", [64, 256])
def test_quantized_linear_grid_bound_other_group_sizes(g):
    """The layer's error bound of the grid holds with the scales repeated over runs of g channels."""
    d = synth.linear_inputs(23, 0, 0, 0, 2, 32, 512)
    s = O.act_scale(d["xcal"])
    xp = O.inv_scale(d["x"], s)
    q, sc, z = O.quantize(d["W"], s, g)
    yq = O.linear_f64(xp, O.dequant(q, sc, z, g))
    y = h2f(xp) @ (h2f(d["W"].view(np.uint16)) * h2f(s)[None, :]).T
    S = np.repeat(h2f(sc), g, axis=1)
    bound = np.abs(h2f(xp)) @ (S * (0.5 + 16 * 2.0**-11)).T
    assert np.all(np.abs(yq - y) <= bound)
    # a real comparison: y is the unquantized layer (not zero), and 4-bit RTN stays well inside it
    assert np.linalg.norm(yq - y) < 0.2 * np.linalg.norm(y)
    ms, ns = np.meshgrid(np.arange(2), np.arange(32), indexing="ij")
    assert np.array_equal(O.linear_pairs_f64(xp, q, sc, z, ms.ravel(), ns.ravel(), g), yq.ravel())


def test_smaller_groups_quantize_more_finely():
    """Finer groups can only narrow each group's range, so on the same data the mean squared weight error
    is ordered g = 64 <= 128 <= 256 (a group-size argument ignored somewhere makes two of them equal)."""
    d = synth.linear_inputs(29, 0, 0, 0, 1, 64, 1024)
    W = d["W"]
    errs = []
    for g in (64, 128, 256):
        q, sc, z = O.quantize(W, None, g)
        errs.append(float(np.mean((O.dequant(q, sc, z, g) - h2f(W.view(np.uint16))) ** 2)))
    assert errs[0] < errs[1] < errs[2]


# ---------------------------------------------------------------- fused gate|up + SiLU --------------
def test_silu_closed_forms():
    """silu(0) = 0; silu(ln 3) = (3/4) ln 3; silu(a) - silu(-a) = a (since sigma(a) + sigma(-a) = 1); the
    minimum of silu is -W(1/e) - ... = -0.2784645427610738 at a = -1.2784645427610738 (the root of
    1 + e^a (1 + a) ... i.e. a = -1 - W(e^-1)); silu(a) -> a for large a and -> -0 for very negative a."""
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(math.log(3.0)) - 0.75 * math.log(3.0)) < 1e-15
    a = np.linspace(-30, 30, 601)
    assert np.max(np.abs(O.silu(a) - O.silu(-a) - a)) < 1e-13
    amin = -1.2784645427610738
    assert abs(float(O.silu(amin)) - (-0.2784645427610738)) < 1e-15
    grid = np.linspace(-3, 1, 40001)
    assert abs(grid[np.argmin(O.silu(grid))] - amin) < 2e-4
    assert O.silu(1000.0) == 1000.0 and O.silu(-1000.0) == 0.0


def test_interleave_gate_up_row_order():
    """Row 32j + i of the interleaved weight is gate row 16j + i (i < 16), else up row 16j + i - 16; with
    row-wise quantization, quantizing the interleaved matrix equals interleaving the two quantizations."""
    rng = np.random.default_rng(31)
    NI, K = 48, 256
    Wg = f16(0.02 * rng.standard_normal((NI, K)))
    Wu = f16(0.02 * rng.standard_normal((NI, K)))
    Wi = O.interleave_gate_up(Wg, Wu)
    for r in range(2 * NI):
        j, i = divmod(r, 32)
        src = Wg[16 * j + i] if i < 16 else Wu[16 * j + i - 16]
        assert np.array_equal(Wi[r], src)
    s = O.act_scale(f16(rng.standard_normal((8, K))))
    qi, sci, zi = O.quantize(Wi, s)
    qg, scg, zg = O.quantize(Wg, s)
    qu, scu, zu = O.quantize(Wu, s)
    for a, b, c in ((qi, qg, qu), (sci, scg, scu), (zi, zg, zu)):
        assert np.array_equal(a, O.interleave_gate_up(b, c))


def test_gate_up_silu_one_hot_closed_form():
    """With x' = e_k (one-hot) the two linears read column k: h_j = silu(Wg[j,k]) * Wu[j,k] exactly as
    the closed form; swapping gate and up (or dropping the activation) fails."""
    rng = np.random.default_rng(37)
    NI, K, k = 16, 128, 77
    Wg = rng.integers(-8, 8, (NI, K)).astype(np.float32) * 0.25
    Wu = rng.integers(-8, 8, (NI, K)).astype(np.float32) * 0.5
    xp = np.zeros((1, K), np.uint16)
    xp[0, k] = 0x3C00  # 1.0
    h = O.gate_up_silu_f64(xp, Wg, Wu)[0]
    a, b = Wg[:, k].astype(np.float64), Wu[:, k].astype(np.float64)
    exp_h = np.array([(ai / (1.0 + math.exp(-ai))) * bi for ai, bi in zip(a, b)])
    assert np.max(np.abs(h - exp_h)) < 1e-14
    assert not np.allclose(h, O.silu(b) * a)


# ---------------------------------------------------------------- AWQ scale search -----------------
def test_act_pow_closed_forms():
    """s(alpha) = fp16(mean|x|^alpha): alpha = 0 gives exactly 1 (even for a zero channel), alpha = 0.5 is
    the fixed-exponent scale (oracle_act_scale, sqrt), alpha = 1 and 2 on rows of magnitude c give fp16(c)
    and fp16(c^2)."""
    rng = np.random.default_rng(41)
    xcal = f16(rng.standard_normal((16, 256)) * 3)
    assert np.all(O.act_pow(xcal, 0.0) == 0x3C00)
    assert np.all(O.act_pow(np.zeros((4, 8), np.uint16), 0.0) == 0x3C00)
    assert np.array_equal(O.act_pow(xcal, 0.5), O.act_scale(xcal))
    c = np.array([0.375, 1.5, 3.0, 7.25])
    rows = np.stack([c, -c, c, -c])  # |x| = c in every row
    assert np.array_equal(O.act_pow(f16(rows), 1.0), f16(c))
    assert np.array_equal(O.act_pow(f16(rows), 2.0), f16(c * c))


def _rtn_loss_numpy(W, xcal):
    """Plain RTN layer error with numpy's matmul: the alpha = 0 point of the search, computed on another
    path (s = 1, so x' = xcal exactly)."""
    q, sc, z = O.quantize(W, None)
    Wq = O.dequant(q, sc, z).astype(np.float64)
    x = h2f(xcal)
    yq = (x @ Wq.T).astype(np.float16).astype(np.float64)
    y = x @ h2f(W).T
    return float(np.sum((yq - y) ** 2))


def test_search_alpha_zero_is_plain_rtn():
    """alpha = 0 reduces the search's loss to the plain round-to-nearest layer (no scaling at all)."""
    d = synth.linear_inputs(43, 0, 0, 0, 1, 64, 256)
    W, xcal = d["W"].view(np.uint16), d["xcal"].view(np.uint16)
    L = O.awq_search_losses(W, xcal, n_grid=4)
    assert len(L) == 5
    assert abs(L[0] - _rtn_loss_numpy(W, xcal)) <= 1e-9 * L[0]


def test_search_exact_grid_loss_is_output_rounding_only():
    """Weights exactly on a 4-bit grid (every code 0..15 present in each group) quantize without error at
    alpha = 0, so the loss there is only the fp16 rounding of the output: sum (fp16(y) - y)^2 (closed form);
    a loss computed against x' instead of x, or without the square, fails."""
    rng = np.random.default_rng(47)
    N, K = 8, 256
    codes = np.stack([np.concatenate([rng.permutation(np.r_[np.arange(16), rng.integers(0, 16, 112)])
                                      for _ in range(2)]) for _ in range(N)])
    S = 2.0 ** rng.integers(-9, -5, (N, 2))
    z = rng.integers(0, 16, (N, 2))
    Wd = (codes - np.repeat(z, 128, axis=1)) * np.repeat(S, 128, axis=1)
    W = f16(Wd)
    assert np.array_equal(h2f(W), Wd)
    xcal = f16(rng.standard_normal((8, K)))
    y = h2f(xcal) @ Wd.T
    expect = float(np.sum((y.astype(np.float16).astype(np.float64) - y) ** 2))
    L = O.awq_search_losses(W, xcal, n_grid=2)
    assert abs(L[0] - expect) <= 1e-12 * max(expect, 1e-30)
    assert L[1] > L[0]  # any scaling moves the weights off their grid


def test_search_protects_a_salient_channel():
    """Hand-built case in the spirit of the page's importance E[|X_j|] (section 2.1 (2)): channel 0 carries
    activations 40x larger than the rest while its weights are small, so plain RTN (alpha = 0) wipes them
    out and the error is dominated by that channel; scaling it up (alpha > 0) must win clearly."""
    rng = np.random.default_rng(53)
    N, K, R = 16, 128, 32
    Wd = 0.02 * rng.standard_normal((N, K))
    Wd[:, 0] = 0.0015 * rng.standard_normal(N)
    x = rng.standard_normal((R, K))
    x[:, 0] *= 40.0
    best, alpha, s, L = O.awq_search(f16(Wd), f16(x), n_grid=10)
    assert best > 0 and L[0] > 3.0 * L[best]
    assert best == int(np.argmin(L)) and alpha == best / 10
    assert np.array_equal(s, O.act_pow(f16(x), alpha))
    # the chosen scale is larger on the salient channel than anywhere else
    assert h2f(s)[0] > h2f(s)[1:].max()


# ---------------------------------------------------------------- GPTQ ------------------------------
def _spd(n, seed):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((2 * n, n))
    return A.T @ A + 0.1 * np.eye(n)


def test_cholesky_and_gptq_u_match_numpy():
    """The oracle's Cholesky and its U (H^-1 = U^T U, upper) against numpy's linalg routines."""
    H = _spd(48, 61)
    assert np.allclose(O.cholesky_lower(H), np.linalg.cholesky(H), rtol=0, atol=1e-12)
    U = O.gptq_u(H)
    assert np.allclose(U, np.triu(U), atol=0)
    assert np.allclose(U, np.linalg.cholesky(np.linalg.inv(H)).T, rtol=0, atol=1e-12)
    assert np.allclose(U.T @ U @ H, np.eye(48), atol=1e-10)


@pytest.mark.parametrize("g", [64, 128, 256])
def test_gptq_identity_hessian_is_rtn(g):
    """Calibration rows c e_k (R = K): H = c^2 I + 1e-6 I, so U is diagonal and no error reaches another
    column -- GPTQ must reduce to plain round-to-nearest exactly."""
    K, N = 256, 40
    W = synth.linear_inputs(67, 0, 0, 0, 1, N, K)["W"].view(np.uint16)
    xcal = f16(1.5 * np.eye(K))
    for a, b in zip(O.gptq_quantize(W, xcal, g), O.quantize(W, None, g)):
        assert np.array_equal(a, b)


def _gptq_slow(W, xcal, g):
    """GPTQ without blocks or lazy updates: after each column, every later column is corrected at once
    (numpy fp64 linear algebra; the grid in numpy float32).  Same result as the blocked algorithm up to
    fp64 rounding."""
    Wc = h2f(W).copy()
    N, K = Wc.shape
    X = h2f(xcal)
    H = X.T @ X + 1e-6 * np.eye(K)
    U = np.linalg.cholesky(np.linalg.inv(H)).T
    q = np.zeros((N, K), np.uint8)
    sc = np.zeros((N, K // g), np.uint16)
    z = np.zeros((N, K // g), np.uint8)
    S = zz = None
    for i in range(K):
        if i % g == 0:
            v = Wc[:, i:i + g].astype(np.float32)
            mn, mx = v.min(axis=1), v.max(axis=1)
            s32 = np.maximum((mx - mn) / np.float32(15), np.float32(1e-5))
            sch = s32.astype(np.float16)
            S = sch.astype(np.float32)
            zz = np.clip(np.rint(-mn / S), 0, 15).astype(np.float32)
            sc[:, i // g] = sch.view(np.uint16)
            z[:, i // g] = zz.astype(np.uint8)
        w = Wc[:, i]
        code = np.clip(np.rint(w.astype(np.float32) / S) + zz, 0, 15)
        q[:, i] = code.astype(np.uint8)
        err = (w - (code.astype(np.float64) - zz) * S.astype(np.float64)) / U[i, i]
        Wc[:, i + 1:] -= np.outer(err, U[i, i + 1:])
    return q, sc, z


@pytest.mark.parametrize("g", [64, 128, 256])
def test_gptq_blocked_lazy_equals_immediate_updates(g):
    """The blocked algorithm with lazy batch updates (section 3.1 (3)) equals the column-by-column one
    written independently above (numpy's inverse and Cholesky, immediate updates of every later column)."""
    rng = np.random.default_rng(71 + g)
    N, K, R = 16, 512, 1024
    W = f16(0.02 * rng.standard_normal((N, K)))
    mix = np.eye(K) + 0.2 * rng.standard_normal((K, K)) / np.sqrt(K)
    xcal = f16(rng.standard_normal((R, K)) @ mix)
    for u, v in zip(O.gptq_quantize(W, xcal, g), _gptq_slow(W, xcal, g)):
        assert np.array_equal(u, v)


@pytest.mark.parametrize("g", [64, 128, 256])
def test_gptq_lowers_the_layer_error_against_rtn(g):
    """The objective of section 3.1 (1): on correlated calibration activations GPTQ's output error
    ||X (W_hat - W)^T||^2 is clearly below plain round-to-nearest's."""
    rng = np.random.default_rng(79)
    N, K, R = 64, 256, 512
    W = f16(0.02 * rng.standard_normal((N, K)))
    mix = np.eye(K) + 0.3 * rng.standard_normal((K, K)) / 16
    xcal = f16(rng.standard_normal((R, K)) @ mix)
    X, Wf = h2f(xcal), h2f(W)

    def loss(q, sc, z):
        return float(np.sum((X @ (O.dequant(q, sc, z, g).astype(np.float64) - Wf).T) ** 2))

    lg = loss(*O.gptq_quantize(W, xcal, g))
    lr = loss(*O.quantize(W, None, g))
    assert lg < 0.85 * lr


# ---------------------------------------------------------------- 3-bit grid -----------------------
# "LLM-AWQ academic impact", recommendations: choose 4-bit or 3-bit quantization by the hardware; "10 INT4
# models on 20 tasks", introduction: AWQ's INT3 results.  The 3-bit grid is the same asymmetric min/max grid
# with qmax = 7 (codes 0..7), stored in the 4-bit layout.
@pytest.mark.parametrize("S0,z0", [(0.0078125, 3), (0.5, 7), (0.000244140625, 0)])
def test_quantize_3bit_reproduces_its_own_grid(S0, z0):
    rng = np.random.default_rng(int(S0 * 1e6) + z0)
    codes = np.concatenate([np.arange(8), rng.integers(0, 8, 120)])
    rng.shuffle(codes)
    w = (codes.astype(np.float64) - z0) * S0
    q, sc, z = O.quantize(f16(w[None, :]), None, 128, 3)
    assert h2f(sc)[0, 0] == S0 and z[0, 0] == z0 and np.array_equal(q[0], codes)


def test_quantize_3bit_clamps_and_bound():
    """All-positive group: z clamps to 0 and the top code to 7; codes never exceed 7; the round-trip bound
    |w' - (q - z) S| <= S (1/2 + 8 * 2^-11) where no clamp applies; the 3-bit error exceeds the 4-bit one."""
    w = np.linspace(1.0, 2.0, 128)
    q, sc, z = O.quantize(f16(w[None, :]), None, 128, 3)
    assert z[0, 0] == 0 and q.max() == 7
    W, s = _synthetic_group_rows()
    q3, sc3, z3 = O.quantize(W, s, 128, 3)
    assert q3.max() <= 7 and z3.max() <= 7
    wp = h2f(W) * h2f(s)[None, :]
    deq3 = O.dequant(q3, sc3, z3).astype(np.float64)
    S = np.repeat(h2f(sc3), 128, axis=1)
    assert np.all(np.abs(wp - deq3) <= S * (0.5 + 8 * 2.0**-11))
    deq4 = O.dequant(*O.quantize(W, s)).astype(np.float64)
    assert np.mean((deq3 - wp) ** 2) > 3.0 * np.mean((deq4 - wp) ** 2)
    for a, b in zip(O.quantize(W, s, 128, 4), O.quantize(W, s)):
        assert np.array_equal(a, b)  # w_bit = 4 is the default grid


# ---------------------------------------------------------------- packed 3-bit layout --------------
def _expected3(n, k, K):
    """(word index, bit) of the low 2 bits and of the high bit of (n, k), read off the header's prose."""
    rb, r, kc, c = n // 32, n % 32, k // 32, k % 32
    j, p, h = c // 8, (c % 8) // 2, c % 2
    base = (rb * (K // 32) + kc) * 96 + 3 * r
    return (base + j // 2, 8 * (j % 2) + 2 * p + 16 * h), (base + 2, 4 * j + p + 16 * h)


def test_pack3_single_code_placement():
    """A single nonzero 3-bit code lands at the two words and bits the header describes."""
    N, K = 40, 256
    rng = np.random.default_rng(83)
    for _ in range(80):
        n, k, c = int(rng.integers(N)), int(rng.integers(K)), int(rng.integers(1, 8))
        q = np.zeros((N, K), np.uint8)
        q[n, k] = c
        qw, _, _ = O.pack3(q, np.zeros((N, 2), np.uint16), np.zeros((N, 2), np.uint8))
        (wl, bl), (wh, bh) = _expected3(n, k, K)
        exp = np.zeros_like(qw)
        exp[wl] |= (c & 3) << bl
        exp[wh] |= (c >> 2) << bh
        assert np.array_equal(qw, exp)


def test_pack3_sizes_roundtrip_and_extraction():
    """3 words per row per 32 channels (0.375 B per weight of codes); the independent decoder inverts the
    packer; and the extraction the header promises: for lane group j and pair p, the low bits of channels
    (8j + 2p, 8j + 2p + 1) are (word_{j/2} >> (8 (j%2) + 2p)) & 0x00030003, their high bits
    (word_2 >> (4j + p)) & 0x00010001."""
    rng = np.random.default_rng(89)
    N, K = 72, 384
    q = rng.integers(0, 8, (N, K)).astype(np.uint8)
    sc = rng.integers(1, 0x7BFF, (N, 3)).astype(np.uint16)
    z = rng.integers(0, 8, (N, 3)).astype(np.uint8)
    qw, scales, qz = O.pack3(q, sc, z)
    assert (qw.nbytes, scales.nbytes, qz.nbytes) == O.packed3_sizes(N, K)
    assert qw.nbytes == 96 * (K // 32) * 12  # N_pad = 96 rows x 12 B per 32 channels
    assert np.array_equal(O.unpack3(qw, N, K), q)
    qw4, scales4, qz4 = O.pack(q, sc, z)
    assert np.array_equal(scales, scales4) and np.array_equal(qz, qz4)  # scales and zeros as the 4-bit layout
    for n in range(0, N, 7):
        rb, r = n // 32, n % 32
        for kc in range(K // 32):
            base = (rb * (K // 32) + kc) * 96 + 3 * r
            w = [int(qw[base + i]) for i in range(3)]
            for j in range(4):
                for p in range(4):
                    lo = (w[j // 2] >> (8 * (j % 2) + 2 * p)) & 0x00030003
                    hi = (w[2] >> (4 * j + p)) & 0x00010001
                    c0, c1 = q[n, kc * 32 + 8 * j + 2 * p], q[n, kc * 32 + 8 * j + 2 * p + 1]
                    assert (lo & 0xFFFF) | ((hi & 0xFFFF) << 2) == c0
                    assert (lo >> 16) | ((hi >> 16) << 2) == c1
