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


def standard_normal(key: np.uint64, count: int, chunk: int = 1 << 22) -> np.ndarray:
    """count standard normals (fp64) from stream `key`; element i uses stream values 2i and 2i+1."""
    out = np.empty(count, np.float64)
    for s in range(0, count, chunk):
        c = min(chunk, count - s)
        u = stream_u64(key, 2 * s, 2 * c)
        a, b = u[0::2], u[1::2]
        u1 = ((a >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
        u2 = (b >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
        out[s:s + c] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return out


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
    """fp16 W [N][K] ~ N(0, 0.02^2)."""
    z = standard_normal(stream_key(seed, tid), N * K)
    return (W_SIGMA * z).astype(np.float16).reshape(N, K)


def activations(seed: int, tid: int, rows: int, K: int, outliers: np.ndarray) -> np.ndarray:
    """fp16 [rows][K] ~ N(0, 1) with the outlier channels scaled by 20 before rounding."""
    z = standard_normal(stream_key(seed, tid), rows * K).reshape(rows, K)
    if len(outliers):
        z[:, outliers] *= OUTLIER_GAIN
    return z.astype(np.float16)


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
def device_linear_inputs(seed: int, tid: int, M: int, N: int, K: int, device):
    """Same distributions as linear_inputs, drawn on `device` with torch.Generator(seed ^ tid)."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed((int(seed) << 32) ^ int(tid))
    W = (torch.randn((N, K), generator=gen, device=device, dtype=torch.float32) * W_SIGMA).half()
    n_out = int(round(OUTLIER_FRACTION * K))
    perm = torch.randperm(K, generator=gen, device=device)
    gain = torch.ones(K, device=device, dtype=torch.float32)
    gain[perm[:n_out]] = OUTLIER_GAIN
    xcal = (torch.randn((CALIB_ROWS, K), generator=gen, device=device) * gain).half()
    x = (torch.randn((M, K), generator=gen, device=device) * gain).half()
    return W, xcal, x
