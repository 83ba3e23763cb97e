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

    def __init__(self, seed, config, layer, linear, M, N, K):
        self.M, self.N, self.K = M, N, K
        d = synth.linear_inputs(seed, config, layer, linear, M, N, K)
        self.W = d["W"].view(np.uint16)
        self.xcal = d["xcal"].view(np.uint16)
        self.x = d["x"].view(np.uint16)
        self.s = O.act_scale(self.xcal)
        self.xp = O.inv_scale(self.x, self.s)
        self.q, self.sc, self.z = O.quantize(self.W, self.s)
        self._packed = None

    @property
    def packed(self):
        if self._packed is None:
            self._packed = O.pack(self.q, self.sc, self.z)
        return self._packed

    def y_rows(self, m_rows=None):
        """fp64 oracle outputs for rows m_rows (default: all) and every n."""
        ms = list(range(self.M)) if m_rows is None else list(m_rows)
        mm, nn = np.meshgrid(np.array(ms), np.arange(self.N), indexing="ij")
        out = O.linear_pairs_f64(self.xp, self.q, self.sc, self.z, mm.ravel(), nn.ravel())
        return out.reshape(len(ms), self.N)

    def y_pairs(self, ms, ns):
        return O.linear_pairs_f64(self.xp, self.q, self.sc, self.z, ms, ns)


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
