"""CPU oracle for the W4A16 AWQ linear layer -- TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper around ``awq_oracle.c`` (plain single-threaded C, fp32 quantizer and fp64 matmul).
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import this
module.  It shares no code with the CUDA library under ``weight_only_int4_05_b200/``.

Every function states the step of the method it follows; the pins that tie it to something other than
itself live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "awq_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

GROUP = 128


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE arithmetic: no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_f16_to_f64.restype = ctypes.c_double
            lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
            lib.oracle_f64_to_f16.restype = ctypes.c_uint16
            lib.oracle_f64_to_f16.argtypes = [ctypes.c_double]
            lib.oracle_f32_to_f16.restype = ctypes.c_uint16
            lib.oracle_f32_to_f16.argtypes = [ctypes.c_float]
            lib.oracle_act_scale.argtypes = [P, I, I, P]
            lib.oracle_act_pow.argtypes = [P, I, I, ctypes.c_double, P]
            lib.oracle_cholesky_lower.argtypes = [P, I]
            lib.oracle_cholesky_lower.restype = I
            lib.oracle_gptq_u.argtypes = [P, I, P]
            lib.oracle_gptq_u.restype = I
            lib.oracle_gptq.argtypes = [P, P, I, I, I, I, ctypes.c_double, P, P, P]
            lib.oracle_gptq.restype = I
            lib.oracle_f64_to_f16_array.argtypes = [P, ctypes.c_size_t, P]
            lib.oracle_inv_scale.argtypes = [P, P, I, I, P]
            lib.oracle_quantize.argtypes = [P, P, I, I, I, P, P, P]
            lib.oracle_quantize_bits.argtypes = [P, P, I, I, I, I, P, P, P]
            lib.oracle_pack3.argtypes = [P, P, P, I, I, I, P, P, P]
            lib.oracle_unpack3.argtypes = [P, I, I, P]
            lib.oracle_pack.argtypes = [P, P, P, I, I, I, P, P, P]
            lib.oracle_unpack.argtypes = [P, P, P, I, I, I, P, P, P]
            lib.oracle_dequant.argtypes = [P, P, P, I, I, I, P]
            lib.oracle_linear_f64.argtypes = [P, P, I, I, I, P]
            lib.oracle_linear_pairs_f64.argtypes = [P, P, P, P, I, I, I, I, P, P, I, P]
            for name in ("oracle_act_scale", "oracle_inv_scale", "oracle_quantize", "oracle_pack",
                         "oracle_unpack", "oracle_dequant", "oracle_linear_f64", "oracle_linear_pairs_f64",
                         "oracle_act_pow", "oracle_f64_to_f16_array", "oracle_quantize_bits", "oracle_pack3",
                         "oracle_unpack3"):
                getattr(lib, name).restype = None
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16
    return a


# ---- fp16 conversions (IEEE binary16 from its definition) -----------------------------------------
def f16_to_f64(h: int) -> float:
    return _load().oracle_f16_to_f64(int(h))


def f64_to_f16(d: float) -> int:
    return int(_load().oracle_f64_to_f16(float(d)))


def f64_to_f16_array(d) -> np.ndarray:
    """Elementwise single-rounding fp64 -> fp16 bits of an array (same shape)."""
    d = np.ascontiguousarray(d, dtype=np.float64)
    h = np.empty(d.shape, np.uint16)
    _load().oracle_f64_to_f16_array(_p(d), d.size, _p(h))
    return h


def f32_to_f16(f: float) -> int:
    return int(_load().oracle_f32_to_f16(float(np.float32(f))))


# ---- a1: AWQ per-channel scale --------------------------------------------------------------------
def act_scale(xcal) -> np.ndarray:
    """s_j = fp16(sqrt(mean_r |xcal_rj|)) in fp64 ("AWQ and GPTQ algorithms", section 2.1 (2))."""
    xcal = _u16(xcal)
    R, K = xcal.shape
    s = np.empty(K, np.uint16)
    _load().oracle_act_scale(_p(xcal), R, K, _p(s))
    return s


# ---- a7: x' = x / s -------------------------------------------------------------------------------
def inv_scale(x, s) -> np.ndarray:
    """x'_mk = fp16(x_mk / s_k), fp64 division ("AWQ and GPTQ algorithms", section 2.1 (3))."""
    x = _u16(x)
    s = _u16(s)
    M, K = x.shape
    xp = np.empty_like(x)
    _load().oracle_inv_scale(_p(x), _p(s), M, K, _p(xp))
    return xp


# ---- a2..a5: fold + grid + codes ------------------------------------------------------------------
def quantize(W, s=None, g: int = GROUP, w_bit: int = 4):
    """Returns (q [N][K] uint8, sc [N][G] uint16 fp16 bits, z [N][G] uint8); codes 0 .. 2^w_bit - 1."""
    W = _u16(W)
    N, K = W.shape
    G = K // g
    q = np.empty((N, K), np.uint8)
    sc = np.empty((N, G), np.uint16)
    z = np.empty((N, G), np.uint8)
    sp = None if s is None else _p(_u16(s))
    _load().oracle_quantize_bits(_p(W), sp, N, K, g, w_bit, _p(q), _p(sc), _p(z))
    return q, sc, z


def packed_sizes(N: int, K: int, g: int = GROUP):
    Np = (N + 31) // 32 * 32
    G = K // g
    return Np * K // 2, G * Np * 2, G * Np // 2


# ---- a6: packed layout ----------------------------------------------------------------------------
def pack(q, sc, z, g: int = GROUP):
    N, K = q.shape
    Np = (N + 31) // 32 * 32
    G = K // g
    qw = np.empty(Np * K // 8, np.uint32)
    scales = np.empty(G * Np, np.uint16)
    qz = np.empty(G * Np // 8, np.uint32)
    _load().oracle_pack(_p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(sc)),
                        _p(np.ascontiguousarray(z)), N, K, g, _p(qw), _p(scales), _p(qz))
    return qw, scales, qz


def unpack(qw, scales, qz, N: int, K: int, g: int = GROUP):
    G = K // g
    q = np.empty((N, K), np.uint8)
    sc = np.empty((N, G), np.uint16)
    z = np.empty((N, G), np.uint8)
    _load().oracle_unpack(_p(np.ascontiguousarray(qw)), _p(np.ascontiguousarray(scales)),
                          _p(np.ascontiguousarray(qz)), N, K, g, _p(q), _p(sc), _p(z))
    return q, sc, z


def awq_pack(W, s=None, g: int = GROUP, w_bit: int = 4):
    """Stage-2 "real quantization": fold s, quantize and pack.  Returns (qweight, scales, qzeros)."""
    return pack(*quantize(W, s, g, w_bit), g)


# ---- dequant and matmul ---------------------------------------------------------------------------
def dequant(q, sc, z, g: int = GROUP) -> np.ndarray:
    N, K = q.shape
    Wq = np.empty((N, K), np.float32)
    _load().oracle_dequant(_p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(sc)),
                           _p(np.ascontiguousarray(z)), N, K, g, _p(Wq))
    return Wq


def linear_f64(xp, Wq) -> np.ndarray:
    """y = x' . Wq^T, plain triple loop in fp64."""
    xp = _u16(xp)
    Wq = np.ascontiguousarray(Wq, dtype=np.float32)
    M, K = xp.shape
    N = Wq.shape[0]
    y = np.empty((M, N), np.float64)
    _load().oracle_linear_f64(_p(xp), _p(Wq), M, N, K, _p(y))
    return y


def linear_pairs_f64(xp, q, sc, z, ms, ns, g: int = GROUP) -> np.ndarray:
    """y[m, n] for the listed pairs only (sampled parity at full size)."""
    xp = _u16(xp)
    M, K = xp.shape
    N = q.shape[0]
    ms = np.ascontiguousarray(ms, dtype=np.int32)
    ns = np.ascontiguousarray(ns, dtype=np.int32)
    out = np.empty(len(ms), np.float64)
    _load().oracle_linear_pairs_f64(_p(xp), _p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(sc)),
                                    _p(np.ascontiguousarray(z)), M, N, K, g, _p(ms), _p(ns), len(ms),
                                    _p(out))
    return out


def reference_linear(xp, W, s=None, g: int = GROUP) -> np.ndarray:
    """Whole path from fp16 W: quantize (with s folded) then the fp64 matmul against x'."""
    q, sc, z = quantize(W, s, g)
    return linear_f64(xp, dequant(q, sc, z, g))


# ---- fused gate|up with the SiLU activation --------------------------------------------------------
# "LLM quantization speed-up" (bjdmk.com.cn), "fused modules": several steps of the layer merged into one
# operation.  Reading: the gated MLP of the Llama-shaped decode workloads, whose gate and up projections
# read the same x' and meet in silu(gate) * up before the down projection.
def silu(a) -> np.ndarray:
    """SiLU, a / (1 + e^-a), in fp64 (e^-a overflowing to inf gives -0 for very negative a)."""
    a = np.asarray(a, np.float64)
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def interleave_gate_up(Wg, Wu) -> np.ndarray:
    """The [2 NI][K] row order the public header states for awq_pack_gate_up: row 32j + i is gate row
    16j + i for i < 16 and up row 16j + i - 16 for i >= 16 (NI a multiple of 16)."""
    Wg = np.asarray(Wg)
    Wu = np.asarray(Wu)
    NI, K = Wg.shape
    assert Wu.shape == (NI, K) and NI % 16 == 0
    out = np.empty((2 * NI, K), Wg.dtype)
    blocks = out.reshape(NI // 16, 32, K)
    blocks[:, :16] = Wg.reshape(NI // 16, 16, K)
    blocks[:, 16:] = Wu.reshape(NI // 16, 16, K)
    return out


def gate_up_silu_f64(xp, Wqg, Wqu) -> np.ndarray:
    """h = silu(x' . Wqg^T) * (x' . Wqu^T): both linears in fp64, the product in fp64."""
    return silu(linear_f64(xp, Wqg)) * linear_f64(xp, Wqu)


def gate_up_silu_pairs_f64(xp, qg, scg, zg, qu, scu, zu, ms, js, g: int = GROUP) -> np.ndarray:
    """h[m, j] for the listed pairs only, from the separately quantized gate and up weights."""
    return silu(linear_pairs_f64(xp, qg, scg, zg, ms, js, g)) * linear_pairs_f64(xp, qu, scu, zu, ms, js, g)


# ---- AWQ scale search ----------------------------------------------------------------------------
# "AWQ and GPTQ algorithms" (jsqmd.com), section 2.1 (3): choose the per-channel scale s that minimises the
# layer's output error after quantization, ||Q(W diag(s)) (diag(s)^-1 X) - W X||^2 over calibration data X;
# "LLM-AWQ academic impact" (CSDN mirror), "quantization flow": stage 1 searches, stage 2 quantizes with the
# result.  Reading: s = (mean |X|)^alpha over a grid alpha = i / n_grid, i = 0 .. n_grid; the quantized layer
# is the deployed one (x' = fp16(x / s), output rounded to fp16); the error is the squared difference with
# the exact unquantized x W^T, summed over every calibration row and output.
def act_pow(xcal, alpha: float) -> np.ndarray:
    """s_j = fp16((mean_r |xcal_rj|)^alpha), fp64 mean and power; alpha = 0 gives exactly 1."""
    xcal = _u16(xcal)
    R, K = xcal.shape
    s = np.empty(K, np.uint16)
    _load().oracle_act_pow(_p(xcal), R, K, ctypes.c_double(alpha), _p(s))
    return s


def awq_search_losses(W, xcal, n_grid: int = 20, g: int = GROUP):
    """Losses L_i, i = 0 .. n_grid, of alpha_i = i / n_grid: L = sum_{r,n} (fp16(y_q) - y)^2 with y = xcal W^T
    exact and y_q the quantized layer on x' = fp16(xcal / s_i) (every product and sum in fp64)."""
    W = _u16(W)
    xcal = _u16(xcal)
    y = linear_f64(xcal, _u16(W).view(np.float16).astype(np.float32))
    losses = np.empty(n_grid + 1, np.float64)
    for i in range(n_grid + 1):
        s = act_pow(xcal, i / n_grid)
        yq = linear_f64(inv_scale(xcal, s), dequant(*quantize(W, s, g), g))
        yq16 = f64_to_f16_array(yq).view(np.float16).astype(np.float64)  # the layer's fp16 output
        losses[i] = float(np.sum((yq16 - y) ** 2))
    return losses


def awq_search(W, xcal, n_grid: int = 20, g: int = GROUP):
    """(best index, alpha, s, losses): the first grid point of least loss and its scale."""
    losses = awq_search_losses(W, xcal, n_grid, g)
    best = int(np.argmin(losses))
    return best, best / n_grid, act_pow(xcal, best / n_grid), losses



# ---- GPTQ ----------------------------------------------------------------------------------------
# "AWQ and GPTQ algorithms" (jsqmd.com), section 3.1: the Hessian H = X^T X of the calibration activations,
# columns quantized in blocks of 128 with each column's error compensated in the later columns through the
# inverse Hessian (Cholesky), lazy batch updates after each block; section 3.3: 1e-6 on the diagonal.  The
# grid is awq_pack's (s = 1), so the result packs into the same layout.
GPTQ_DAMP = 1e-6
GPTQ_BLOCK = 128


def cholesky_lower(A) -> np.ndarray:
    A = np.array(A, np.float64, order="C")
    n = A.shape[0]
    if _load().oracle_cholesky_lower(_p(A), n) != 0:
        raise ValueError("not positive definite")
    return A


def gptq_u(H) -> np.ndarray:
    """Upper triangular U with H^-1 = U^T U."""
    H = np.ascontiguousarray(H, np.float64)
    n = H.shape[0]
    U = np.empty_like(H)
    if _load().oracle_gptq_u(_p(H), n, _p(U)) != 0:
        raise ValueError("not positive definite")
    return U


def gptq_quantize(W, xcal, g: int = GROUP, damp: float = GPTQ_DAMP):
    """GPTQ of W [N][K] on xcal [R][K]: (q [N][K], sc [N][K/g] fp16 bits, z [N][K/g]) like quantize()."""
    W = _u16(W)
    xcal = _u16(xcal)
    N, K = W.shape
    R = xcal.shape[0]
    q = np.empty((N, K), np.uint8)
    sc = np.empty((N, K // g), np.uint16)
    z = np.empty((N, K // g), np.uint8)
    if _load().oracle_gptq(_p(W), _p(xcal), N, K, R, g, ctypes.c_double(damp), _p(q), _p(sc), _p(z)) != 0:
        raise ValueError("the Hessian is not positive definite")
    return q, sc, z



# ---- the packed 3-bit layout -----------------------------------------------------------------------
def packed3_sizes(N: int, K: int, g: int = GROUP):
    """Bytes of (qweight, scales, qzeros) in the 3-bit layout: 12 bytes per row per 32 channels."""
    Np = (N + 31) // 32 * 32
    G = K // g
    return Np * K // 32 * 12, G * Np * 2, G * Np // 2


def pack3(q, sc, z, g: int = GROUP):
    N, K = q.shape
    Np = (N + 31) // 32 * 32
    G = K // g
    qw = np.empty(Np * K // 32 * 3, np.uint32)
    scales = np.empty(G * Np, np.uint16)
    qz = np.empty(G * Np // 8, np.uint32)
    _load().oracle_pack3(_p(np.ascontiguousarray(q)), _p(np.ascontiguousarray(sc)), _p(np.ascontiguousarray(z)),
                         N, K, g, _p(qw), _p(scales), _p(qz))
    return qw, scales, qz


def unpack3(qw, N: int, K: int) -> np.ndarray:
    q = np.empty((N, K), np.uint8)
    _load().oracle_unpack3(_p(np.ascontiguousarray(qw)), N, K, _p(q))
    return q


def awq_pack3(W, s=None, g: int = GROUP):
    """Quantize on the 3-bit grid and pack into the 3-bit layout: (qweight, scales, qzeros)."""
    return pack3(*quantize(W, s, g, 3), g)
