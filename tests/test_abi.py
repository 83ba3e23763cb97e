"""C ABI checks that need no GPU: the library builds, loads, exports every symbol the public header
declares, and rejects bad arguments on the host (no kernel is launched on these paths)."""
import ctypes
import os
import re

import pytest

from weight_only_int4_05_b200 import _lib, build as libbuild
from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq_w4a16.h")


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if not n.startswith("defined")))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("awq_pack", "w4a16_gemv", "w4a16_gemm", "w4a16_linear", "awq_act_scale", "awq_apply_inv_scale"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) == set(_lib.EXPORTS)


def test_version_and_status_strings(L):
    assert L.awq_version() == 100
    for code, name in _lib.STATUS_NAMES.items():
        assert L.awq_status_string(code).decode() == name


@pytest.mark.parametrize("N,K", [(256, 512), (40, 384), (14336, 4096), (8, 128), (28672, 8192)])
def test_packed_sizes_match_layout(L, N, K):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    assert L.awq_packed_sizes(N, K, 128, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == 0
    assert (a.value, b.value, c.value) == O.packed_sizes(N, K)


def test_packed_sizes_rejects(L):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    ref = (ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    assert L.awq_packed_sizes(256, 512, 32, *ref) == 2      # g not 64 / 128 / 256: unsupported
    assert L.awq_packed_sizes(256, 512, 96, *ref) == 2
    assert L.awq_packed_sizes(256, 512, 64, *ref) == 0
    assert a.value == 256 * 512 // 2 and b.value == 8 * 256 * 2 and c.value == 8 * 256 // 2  # G = 8 at g = 64
    assert L.awq_packed_sizes(256, 384, 256, *ref) == 1     # K not a multiple of g
    assert L.awq_packed_sizes(0, 512, 128, *ref) == 1
    assert L.awq_packed_sizes(256, 500, 128, *ref) == 1     # K not a multiple of g
    assert L.awq_packed_sizes(256, 512, 128, None, ref[1], ref[2]) == 1


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails before any CUDA call


def _lin(L, fn, M=1, N=256, K=512, g=128, ptrs=(FAKE,) * 5, ws=None, ws_bytes=0):
    x, qw, sc, qz, y = (ctypes.c_void_p(p) for p in ptrs)
    return getattr(L, fn)(x, qw, sc, qz, y, M, N, K, g, ctypes.c_void_p(ws), ws_bytes, None)


@pytest.mark.parametrize("fn", ["w4a16_gemv", "w4a16_gemm", "w4a16_linear"])
def test_linear_argument_checks(L, fn):
    assert _lin(L, fn, g=32) == 2
    assert _lin(L, fn, g=256, K=384) == 1  # K % g != 0
    assert _lin(L, fn, M=0) == 1
    assert _lin(L, fn, N=12) == 1          # N % 8 != 0
    assert _lin(L, fn, K=192) == 1         # K % 128 != 0
    assert _lin(L, fn, K=0) == 1
    assert _lin(L, fn, ptrs=(FAKE, 0, FAKE, FAKE, FAKE)) == 1
    assert _lin(L, fn, ptrs=(FAKE + 4, FAKE, FAKE, FAKE, FAKE)) == 3
    assert _lin(L, fn, ptrs=(FAKE, FAKE, FAKE, FAKE, FAKE + 2)) == 3


def test_pack_and_prep_argument_checks(L):
    P = ctypes.c_void_p
    assert L.awq_pack(P(FAKE), None, 256, 512, 32, P(FAKE), P(FAKE), P(FAKE), None) == 2
    assert L.awq_pack(P(FAKE), None, 256, 500, 128, P(FAKE), P(FAKE), P(FAKE), None) == 1
    assert L.awq_pack(P(FAKE), None, 0, 512, 128, P(FAKE), P(FAKE), P(FAKE), None) == 1
    assert L.awq_pack(P(FAKE + 8), None, 256, 512, 128, P(FAKE), P(FAKE), P(FAKE), None) == 3
    assert L.awq_pack(P(FAKE), P(FAKE + 2), 256, 512, 128, P(FAKE), P(FAKE), P(FAKE), None) == 3
    assert L.awq_pack(P(FAKE), None, 256, 512, 128, None, P(FAKE), P(FAKE), None) == 1
    assert L.awq_act_scale(P(FAKE), 0, 512, P(FAKE), None) == 1
    assert L.awq_act_scale(P(FAKE), 9000, 512, P(FAKE), None) == 1
    assert L.awq_act_scale(None, 64, 512, P(FAKE), None) == 1
    assert L.awq_apply_inv_scale(P(FAKE), P(FAKE), 0, 512, P(FAKE), None) == 1
    assert L.awq_apply_inv_scale(P(FAKE), None, 1, 512, P(FAKE), None) == 1


def test_workspace_query_rejects_bad_sizes(L):
    assert L.w4a16_workspace_bytes(1, 1, 12, 512, 128) == 2**64 - 1
    assert L.w4a16_workspace_bytes(9, 1, 256, 512, 128) == 2**64 - 1


def test_selftest_rejects_null_output(L):
    assert L.awq_selftest_wait_timeout(0, None, None) == 1  # AWQ_ERR_INVALID_ARG, nothing launched


def test_linear_pf_hint_checks(L):
    F = ctypes.c_void_p(0x10000)
    args = (F, F, F, F, F, 1, 256, 512, 128, None, 0)
    assert L.w4a16_linear_pf(*args, ctypes.c_void_p(0x10008), 64, None) == 3  # misaligned hint
    assert L.w4a16_linear_pf(*args, F, 24, None) == 1                         # size not a multiple of 16
    assert L.w4a16_linear_pf(F, F, F, F, F, 0, 256, 512, 128, None, 0, F, 64, None) == 1  # M < 1


def test_gemv_s_argument_checks(L):
    F = ctypes.c_void_p(0x10000)
    assert L.w4a16_gemv_s(F, None, F, F, F, F, 1, 256, 512, 128, None, 0, None) == 1      # s NULL
    assert L.w4a16_gemv_s(F, ctypes.c_void_p(0x10008), F, F, F, F, 1, 256, 512, 128, None, 0, None) == 3
    assert L.w4a16_gemv_s(F, F, F, F, F, F, 1, 256, 512, 32, None, 0, None) == 2        # g unsupported
    assert L.w4a16_gemv_s(F, F, F, F, F, F, 0, 256, 512, 128, None, 0, None) == 1       # M < 1


def test_gate_up_argument_checks(L):
    P, F = ctypes.c_void_p, ctypes.c_void_p(FAKE)
    assert L.awq_pack_gate_up(F, F, None, 24, 512, 128, F, F, F, None) == 1      # NI % 16 != 0
    assert L.awq_pack_gate_up(F, None, None, 32, 512, 128, F, F, F, None) == 1   # NULL up weight
    assert L.awq_pack_gate_up(F, F, None, 32, 512, 32, F, F, F, None) == 2       # unsupported g
    assert L.awq_pack_gate_up(P(FAKE + 8), F, None, 32, 512, 128, F, F, F, None) == 3
    assert L.w4a16_gate_up_silu(F, F, F, F, F, 1, 24, 512, 128, None, 0, None) == 1  # NI % 16 != 0
    assert L.w4a16_gate_up_silu(F, F, F, F, F, 0, 32, 512, 128, None, 0, None) == 1  # M < 1
    assert L.w4a16_gate_up_silu(F, F, F, F, F, 1, 32, 512, 32, None, 0, None) == 2   # unsupported g
    assert L.w4a16_gate_up_silu(F, F, F, F, P(FAKE + 8), 1, 32, 512, 128, None, 0, None) == 3


def test_search_argument_checks(L):
    P, F = ctypes.c_void_p, ctypes.c_void_p(FAKE)
    args = lambda N=64, K=256, R=8, g=128, n=4: (F, F, N, K, R, g, n, F, F, F, F, 1 << 30, None)  # noqa: E731
    assert L.awq_search_scale(*args(n=0)) == 1
    assert L.awq_search_scale(*args(R=0)) == 1
    assert L.awq_search_scale(*args(N=12)) == 1
    assert L.awq_search_scale(*args(K=200)) == 1
    assert L.awq_search_scale(*args(g=32)) == 2
    assert L.awq_search_workspace_bytes(64, 256, 8, 128, 4) > 64 * 256 // 2
    assert L.awq_search_workspace_bytes(64, 256, 0, 128, 4) == 2**64 - 1
    bad = list(args())
    bad[0] = P(FAKE + 8)
    assert L.awq_search_scale(*bad) == 3


def test_gptq_argument_checks(L):
    P, F = ctypes.c_void_p, ctypes.c_void_p(FAKE)
    d = ctypes.c_double(1e-6)
    assert L.gptq_quantize(F, F, 64, 192, 8, 64, d, F, F, F, F, 1 << 30, None) == 1   # K % 128 != 0
    assert L.gptq_quantize(F, F, 12, 256, 8, 128, d, F, F, F, F, 1 << 30, None) == 1  # N % 8 != 0
    assert L.gptq_quantize(F, F, 64, 256, 0, 128, d, F, F, F, F, 1 << 30, None) == 1  # R < 1
    assert L.gptq_quantize(F, F, 64, 384, 8, 256, d, F, F, F, F, 1 << 30, None) == 1  # K % g != 0
    assert L.gptq_quantize(F, F, 64, 256, 8, 32, d, F, F, F, F, 1 << 30, None) == 2   # g unsupported
    assert L.gptq_quantize(F, F, 64, 256, 8, 128, ctypes.c_double(-1.0), F, F, F, F, 1 << 30, None) == 1
    assert L.gptq_quantize(P(FAKE + 8), F, 64, 256, 8, 128, d, F, F, F, F, 1 << 30, None) == 3
    assert L.gptq_workspace_bytes(64, 256, 8, 128) >= 2 * 256 * 256 * 8 + 64 * 256 * 8
    assert L.gptq_workspace_bytes(64, 192, 8, 64) == 2**64 - 1
    assert L.awq_status_string(7) == b"AWQ_ERR_NUMERIC"


def test_pack_bits_argument_checks(L):
    P, F = ctypes.c_void_p, ctypes.c_void_p(FAKE)
    assert L.awq_pack_bits(F, None, 256, 512, 128, 5, F, F, F, None) == 2   # w_bit unsupported
    assert L.awq_pack_bits(F, None, 256, 512, 128, 2, F, F, F, None) == 2
    assert L.awq_pack_bits(F, None, 256, 500, 128, 3, F, F, F, None) == 1   # K % g != 0
    assert L.awq_pack_bits(P(FAKE + 8), None, 256, 512, 128, 3, F, F, F, None) == 3


def test_three_bit_layout_sizes_and_checks(L):
    P, F = ctypes.c_void_p, ctypes.c_void_p(FAKE)
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    assert L.awq_packed3_sizes(40, 512, 128, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == 0
    assert a.value == 64 * 512 // 32 * 12 and b.value == 4 * 64 * 2 and c.value == 4 * 64 // 2
    assert L.awq_pack3(F, None, 256, 512, 32, F, F, F, None) == 2
    assert L.awq_pack3(F, None, 256, 500, 128, F, F, F, None) == 1
    assert L.awq_pack3(P(FAKE + 8), None, 256, 512, 128, F, F, F, None) == 3
    assert L.w3a16_gemv(F, F, F, F, F, 0, 256, 512, 128, None, 0, None) == 1
    assert L.w3a16_gemv(F, F, F, F, F, 1, 256, 512, 32, None, 0, None) == 2
