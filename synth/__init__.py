"""Seeded synthetic inputs for the W4A16 AWQ linear layer.

This module is shared by the tests, the benchmark and the oracle checks.  It holds none of the method's
arithmetic (no scale statistic, no quantization, no matmul): it only draws the weights W, the
calibration activations xcal and the activations x with the distributions of the workloads.

Recipe (host generator, bit-reproducible on any machine with IEEE doubles):
  * a counter-based stream: u64_i = splitmix64(key + i), key = splitmix64((seed << 32) ^ tensor_id);
    splitmix64 is Steele, Lea and Flood's SplitMix64 finalizer (add the golden-gamma constant
    0x9E3779B97F4A7C15, then xor-shift-multiply by 0xBF58476D1CE4E5B9 and 0x94D049BB133111EB);
  * a standard normal per element from two stream values (Box-Muller, cosine branch, fp64):
    u1 = ((a >> 11) + 1) * 2^-53 in (0, 1],  u2 = (b >> 11) * 2^-53,  z = sqrt(-2 ln u1) cos(2 pi u2);
  * W = fp16(0.02 z);  xcal, x = fp16(z), and fp16(20 z) in the outlier channels;
  * outlier channels: the round(0.01 K) positions that a Fisher-Yates shuffle of 0..K-1 (drawn from
    the stream of the linear's outlier tensor id) fixes first; the same channels for xcal and x.
A device generator (``device_*``) draws the same distributions with torch's seeded CUDA generator for
benchmark-sized stacks that the host generator would take minutes to draw.
"""
from __future__ import annotations

import numpy as np

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)

W_SIGMA = 0.02
OUTLIER_FRACTION = 0.01
OUTLIER_GAIN = 20.0
CALIB_ROWS = 64

# tensor kinds inside one linear
KIND_W, KIND_XCAL, KIND_X, KIND_OUTLIER = 0, 1, 2, 3


def _splitmix64(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = x + _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _C1
        z = (z ^ (z >> np.uint64(27))) * _C2
        return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    v = np.array([((int(seed) & 0xFFFFFFFF) << 32) ^ (int(tensor_id) & 0xFFFFFFFFFFFF)], np.uint64)
    return _splitmix64(v)[0]


def stream_u64(key: np.uint64, start: int, count: int) -> np.ndarray:
    idx = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _splitmix64(idx + key)


class _NormalStream:
    """Standard normals of one stream, produced chunk by chunk in reused buffers (large fresh
    allocations are what makes naive numpy generation slow)."""

    def __init__(self, key: np.uint64, chunk: int = 1 << 20):
        self.key = key
        self.chunk = chunk
        self.ctr = np.empty(2 * chunk, np.uint64)
        self.tmp = np.empty(2 * chunk, np.uint64)
        self.u1 = np.empty(chunk, np.float64)
        self.u2 = np.empty(chunk, np.float64)
        self.base = np.arange(2 * chunk, dtype=np.uint64)

    def block(self, start: int, c: int) -> np.ndarray:
        """Normals for elements start .. start+c-1 (c <= chunk), as a view of an internal buffer."""
        ctr, tmp = self.ctr[:2 * c], self.tmp[:2 * c]
        with np.errstate(over="ignore"):
            np.add(self.base[:2 * c], self.key + np.uint64(2 * start), out=ctr)
            np.add(ctr, _GAMMA, out=ctr)                       # splitmix64, in place
            np.right_shift(ctr, np.uint64(30), out=tmp)
            np.bitwise_xor(ctr, tmp, out=ctr)
            np.multiply(ctr, _C1, out=ctr)
            np.right_shift(ctr, np.uint64(27), out=tmp)
            np.bitwise_xor(ctr, tmp, out=ctr)
            np.multiply(ctr, _C2, out=ctr)
            np.right_shift(ctr, np.uint64(31), out=tmp)
            np.bitwise_xor(ctr, tmp, out=ctr)
        u1, u2 = self.u1[:c], self.u2[:c]
        np.right_shift(ctr[0::2], np.uint64(11), out=tmp[:c])
        np.add(tmp[:c], np.uint64(1), out=tmp[:c])
        np.multiply(tmp[:c], 2.0 ** -53, out=u1)              # (0, 1]
        np.right_shift(ctr[1::2], np.uint64(11), out=tmp[:c])
        np.multiply(tmp[:c], 2.0 ** -53, out=u2)              # [0, 1)
        np.log(u1, out=u1)
        np.multiply(u1, -2.0, out=u1)
        np.sqrt(u1, out=u1)
        np.multiply(u2, 2.0 * np.pi, out=u2)
        np.cos(u2, out=u2)
        np.multiply(u1, u2, out=u1)
        return u1


def standard_normal(key: np.uint64, count: int, chunk: int = 1 << 20) -> np.ndarray:
    """count standard normals (fp64) from stream `key`; element i uses stream values 2i and 2i+1."""
    out = np.empty(count, np.float64)
    ns = _NormalStream(key, chunk)
    for s in range(0, count, chunk):
        c = min(chunk, count - s)
        out[s:s + c] = ns.block(s, c)
    return out


def _fp16_normals(key: np.uint64, rows: int, cols: int, row_gain=None, sigma: float = 1.0,
                  chunk: int = 1 << 20) -> np.ndarray:
    """fp16 [rows][cols] = fp16(sigma * z * gain[col]) with z the stream's normals in row-major order."""
    out = np.empty(rows * cols, np.float16)
    ns = _NormalStream(key, chunk)
    total = rows * cols
    gain = None
    if row_gain is not None:
        reps = (chunk + cols - 1) // cols + 1
        gain = np.tile(row_gain.astype(np.float64) * sigma, reps)
    for s in range(0, total, chunk):
        c = min(chunk, total - s)
        z = ns.block(s, c)
        if gain is not None:
            off = s % cols
            np.multiply(z, gain[off:off + c], out=z)
        elif sigma != 1.0:
            np.multiply(z, sigma, out=z)
        out[s:s + c] = z
    return out.reshape(rows, cols)


def tensor_id(config: int, layer: int, linear: int, kind: int) -> int:
    return ((int(config) * 256 + int(layer)) * 16 + int(linear)) * 8 + int(kind)


def outlier_channels(seed: int, K: int, tid: int) -> np.ndarray:
    """round(0.01 K) channel indices from a seeded Fisher-Yates shuffle (sorted)."""
    n_out = int(round(OUTLIER_FRACTION * K))
    key = stream_key(seed, tid)
    perm = np.arange(K, dtype=np.int64)
    u = stream_u64(key, 0, K)
    for i in range(K - 1, 0, -1):
        j = int(u[K - 1 - i] % np.uint64(i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    # the shuffle above fills positions from the back; take the channels that landed last
    return np.sort(perm[K - n_out:]) if n_out > 0 else np.zeros(0, np.int64)


def weights(seed: int, tid: int, N: int, K: int) -> np.ndarray:
    """fp16 W [N][K] = fp16(0.02 z)."""
    return _fp16_normals(stream_key(seed, tid), N, K, sigma=W_SIGMA)


def activations(seed: int, tid: int, rows: int, K: int, outliers: np.ndarray) -> np.ndarray:
    """fp16 [rows][K] = fp16(z), and fp16(20 z) in the outlier channels."""
    gain = np.ones(K, np.float64)
    if len(outliers):
        gain[outliers] = OUTLIER_GAIN
    return _fp16_normals(stream_key(seed, tid), rows, K, row_gain=gain)


def linear_inputs(seed: int, config: int, layer: int, linear: int, M: int, N: int, K: int) -> dict:
    """W, xcal (64 rows), x (M rows) and the outlier channel list of one synthetic linear layer."""
    outl = outlier_channels(seed, K, tensor_id(config, layer, linear, KIND_OUTLIER))
    return {
        "W": weights(seed, tensor_id(config, layer, linear, KIND_W), N, K),
        "xcal": activations(seed, tensor_id(config, layer, linear, KIND_XCAL), CALIB_ROWS, K, outl),
        "x": activations(seed, tensor_id(config, layer, linear, KIND_X), M, K, outl),
        "outliers": outl,
    }


# ---- device generator for benchmark-sized stacks (same distributions, torch's CUDA generator) ----
def device_linear_inputs(seed: int, tid: int, M: int, N: int, K: int, device, rows: int = None):
    """Same distributions as linear_inputs, drawn on `device` with torch.Generator(seed ^ tid); `rows`
    calibration rows (default CALIB_ROWS)."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed((int(seed) << 32) ^ int(tid))
    W = (torch.randn((N, K), generator=gen, device=device, dtype=torch.float32) * W_SIGMA).half()
    n_out = int(round(OUTLIER_FRACTION * K))
    perm = torch.randperm(K, generator=gen, device=device)
    gain = torch.ones(K, device=device, dtype=torch.float32)
    gain[perm[:n_out]] = OUTLIER_GAIN
    xcal = (torch.randn((CALIB_ROWS if rows is None else rows, K), generator=gen, device=device) * gain).half()
    x = (torch.randn((M, K), generator=gen, device=device) * gain).half()
    return W, xcal, x
