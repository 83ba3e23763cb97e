"""ctypes loader for libawq_w4a16.so (the C ABI of include/awq_w4a16.h).

Loading fails loudly when the shared library has not been built: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

EXPORTS = (
    "awq_status_string", "awq_version", "awq_packed_sizes", "awq_act_scale", "awq_apply_inv_scale",
    "awq_pack", "w4a16_gemv", "w4a16_gemm", "w4a16_linear", "w4a16_gemv_max_m", "w4a16_workspace_bytes",
    "awq_last_device_status", "w4a16_gemv_noalloc", "awq_selftest_wait_timeout",
    "w4a16_linear_pf", "w4a16_gemv_s", "awq_pack_gate_up", "w4a16_gate_up_silu", "awq_search_scale",
    "awq_search_workspace_bytes", "gptq_quantize", "gptq_workspace_bytes", "awq_pack_bits", "awq_packed3_sizes",
    "awq_pack3", "w3a16_gemv",
)

STATUS_NAMES = {0: "AWQ_OK", 1: "AWQ_ERR_INVALID_ARG", 2: "AWQ_ERR_UNSUPPORTED", 3: "AWQ_ERR_MISALIGNED",
                4: "AWQ_ERR_CUDA", 5: "AWQ_ERR_DEVICE_TIMEOUT", 6: "AWQ_ERR_WORKSPACE", 7: "AWQ_ERR_NUMERIC"}
MODE_GEMV, MODE_GEMM, MODE_LINEAR = 1, 2, 3

_lock = threading.Lock()
_lib = None


class AwqError(RuntimeError):
    def __init__(self, where: str, status: int):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


def lib_path() -> str:
    return _build.LIB_PATH


def load() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = _build.LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m weight_only_int4_05_b200.build`")
        lib = ctypes.CDLL(path)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.awq_status_string.restype = ctypes.c_char_p
        lib.awq_status_string.argtypes = [I]
        lib.awq_version.restype = I
        lib.awq_version.argtypes = []
        lib.awq_packed_sizes.restype = I
        lib.awq_packed_sizes.argtypes = [I, I, I, ctypes.POINTER(Z), ctypes.POINTER(Z), ctypes.POINTER(Z)]
        lib.awq_act_scale.restype = I
        lib.awq_act_scale.argtypes = [P, I, I, P, P]
        lib.awq_apply_inv_scale.restype = I
        lib.awq_apply_inv_scale.argtypes = [P, P, I, I, P, P]
        lib.awq_pack.restype = I
        lib.awq_pack.argtypes = [P, P, I, I, I, P, P, P, P]
        lib.awq_packed3_sizes.restype = I
        lib.awq_packed3_sizes.argtypes = [I, I, I, ctypes.POINTER(Z), ctypes.POINTER(Z), ctypes.POINTER(Z)]
        lib.awq_pack3.restype = I
        lib.awq_pack3.argtypes = [P, P, I, I, I, P, P, P, P]
        lib.w3a16_gemv.restype = I
        lib.w3a16_gemv.argtypes = [P, P, P, P, P, I, I, I, I, P, Z, P]
        lib.awq_pack_bits.restype = I
        lib.awq_pack_bits.argtypes = [P, P, I, I, I, I, P, P, P, P]
        lib.gptq_quantize.restype = I
        lib.gptq_quantize.argtypes = [P, P, I, I, I, I, ctypes.c_double, P, P, P, P, Z, P]
        lib.gptq_workspace_bytes.restype = Z
        lib.gptq_workspace_bytes.argtypes = [I, I, I, I]
        lib.awq_search_scale.restype = I
        lib.awq_search_scale.argtypes = [P, P, I, I, I, I, I, P, P, P, P, Z, P]
        lib.awq_search_workspace_bytes.restype = Z
        lib.awq_search_workspace_bytes.argtypes = [I, I, I, I, I]
        lib.awq_pack_gate_up.restype = I
        lib.awq_pack_gate_up.argtypes = [P, P, P, I, I, I, P, P, P, P]
        for name in ("w4a16_gemv", "w4a16_gemm", "w4a16_linear", "w4a16_gate_up_silu"):
            fn = getattr(lib, name)
            fn.restype = I
            fn.argtypes = [P, P, P, P, P, I, I, I, I, P, Z, P]
        lib.w4a16_gemv_s.restype = I
        lib.w4a16_gemv_s.argtypes = [P, P, P, P, P, P, I, I, I, I, P, Z, P]
        lib.w4a16_gemv_noalloc.restype = I
        lib.w4a16_gemv_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, P]
        lib.w4a16_linear_pf.restype = I
        lib.w4a16_linear_pf.argtypes = [P, P, P, P, P, I, I, I, I, P, Z, P, Z, P]
        lib.awq_selftest_wait_timeout.restype = I
        lib.awq_selftest_wait_timeout.argtypes = [I, P, P]
        lib.w4a16_gemv_max_m.restype = I
        lib.w4a16_gemv_max_m.argtypes = [I, I]
        lib.w4a16_workspace_bytes.restype = Z
        lib.w4a16_workspace_bytes.argtypes = [I, I, I, I, I]
        lib.awq_last_device_status.restype = I
        lib.awq_last_device_status.argtypes = [P]
        _lib = lib
        return lib


def check(status: int, where: str) -> None:
    if status != 0:
        raise AwqError(where, status)
