"""Shared helpers for the GPU parity tests: seeded inputs, the oracle's side of each case, and the
tolerance of the linear layer (max |y - y_ref| <= 1e-2 rms(y_ref) and ||y - y_ref|| / ||y_ref|| <= 2e-3).

The CUDA side of every case starts from the same synthetic W, xcal and x as the oracle and computes
the scale, the scaled activations, the packed weight and y with the library's kernels only."""
from __future__ import annotations

import numpy as np

import synth
from oracle import oracle as O

MAXABS_TOL = 1e-2   # times rms(y_ref)
RELL2_TOL = 2e-3


class OracleCase:
    """Inputs of one linear layer and everything the oracle derives from them (lazily)."""

    def __init__(self, seed, config, layer, linear, M, N, K, g=O.GROUP, w_bit=4):
        self.M, self.N, self.K, self.g, self.w_bit = M, N, K, g, w_bit
        d = synth.linear_inputs(seed, config, layer, linear, M, N, K)
        self.W = d["W"].view(np.uint16)
        self.xcal = d["xcal"].view(np.uint16)
        self.x = d["x"].view(np.uint16)
        self.s = O.act_scale(self.xcal)
        self.xp = O.inv_scale(self.x, self.s)
        self.q, self.sc, self.z = O.quantize(self.W, self.s, g, w_bit)
        self._packed = None

    @property
    def packed(self):
        if self._packed is None:
            self._packed = O.pack(self.q, self.sc, self.z, self.g)
        return self._packed

    def y_rows(self, m_rows=None):
        """fp64 oracle outputs for rows m_rows (default: all) and every n."""
        ms = list(range(self.M)) if m_rows is None else list(m_rows)
        mm, nn = np.meshgrid(np.array(ms), np.arange(self.N), indexing="ij")
        out = O.linear_pairs_f64(self.xp, self.q, self.sc, self.z, mm.ravel(), nn.ravel(), self.g)
        return out.reshape(len(ms), self.N)

    def y_pairs(self, ms, ns):
        return O.linear_pairs_f64(self.xp, self.q, self.sc, self.z, ms, ns, self.g)


def sample_pairs(M, N, count, seed=0):
    """Sampled (m, n) output positions: the four corners, the ragged edges and random interior points."""
    rng = np.random.default_rng(seed)
    ms = [0, 0, M - 1, M - 1]
    ns = [0, N - 1, 0, N - 1]
    ms += list(rng.integers(0, M, count))
    ns += list(rng.integers(0, N, count))
    return np.array(ms, np.int32), np.array(ns, np.int32)


def tolerance_report(y, y_ref):
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    err = y - y_ref
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    maxabs = float(np.max(np.abs(err)))
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-300))
    return maxabs / max(rms, 1e-300), rel


def assert_within_tolerance(y, y_ref, what=""):
    assert np.all(np.isfinite(np.asarray(y, np.float64))), f"{what}: non-finite output"
    ma, rel = tolerance_report(y, y_ref)
    assert ma <= MAXABS_TOL and rel <= RELL2_TOL, f"{what}: maxabs/rms={ma:.3e} relL2={rel:.3e}"
    return ma, rel


# The gate|up epilogue h = fp16(silu(a) b).  Its error follows from the linear layer's: a and b each carry
# up to 1e-2 rms of their own error (in GEMM mode every dequantized weight (q - z) S is rounded to fp16 before
# the tensor-core product), which |silu'| <= 1.1 carries into h as 1.1 |b| da + |silu(a)| db, and h adds one
# fp16 rounding (2^-11 relative, doubled for margin).  The product's tail is heavier than a linear output's,
# so the bound is elementwise rather than a fraction of rms(h).  Swapping gate and up, or losing the
# activation, moves h by O(|a| |b|) and fails.
def assert_epilogue_within_tolerance(h, a_ref, b_ref, what=""):
    from oracle import oracle as O

    h = np.asarray(h, np.float64)
    a_ref = np.asarray(a_ref, np.float64)
    b_ref = np.asarray(b_ref, np.float64)
    assert np.all(np.isfinite(h)), f"{what}: non-finite output"
    h_ref = O.silu(a_ref) * b_ref
    rms_a = float(np.sqrt(np.mean(a_ref ** 2)))
    rms_b = float(np.sqrt(np.mean(b_ref ** 2)))
    bound = 2.0 ** -10 * np.abs(h_ref) + MAXABS_TOL * (1.1 * np.abs(b_ref) * rms_a + np.abs(O.silu(a_ref)) * rms_b)
    worst = float(np.max(np.abs(h - h_ref) / bound))
    rel = float(np.linalg.norm(h - h_ref) / max(np.linalg.norm(h_ref), 1e-300))
    assert worst <= 1.0 and rel <= RELL2_TOL, f"{what}: max err/bound={worst:.3f} relL2={rel:.3e}"
    return worst, rel
