"""W4A16 group-quantized linear layer (AWQ) for NVIDIA B200 -- Python binding.

Argument marshalling over the C ABI of ``include/awq_w4a16.h`` (``libawq_w4a16.so``): torch supplies
device memory and the current CUDA stream; every step of the computation runs in the library's CUDA
kernels.  The functions carry the C entry points' names.

    s  = awq_act_scale(xcal)                    # per-channel AWQ scale, fp16 [K]
    pw = awq_pack(W, s)                         # packed uint4 weights, fp16 scales, uint4 zeros
    xp = awq_apply_inv_scale(x, s)              # activations divided by s
    y  = w4a16_linear(xp, pw)                   # GEMV (decode) or tcgen05 GEMM (prefill) by M
    gu = awq_pack_gate_up(Wg, Wu, s)            # gate and up projections interleaved in one packed weight
    h  = w4a16_gate_up_silu(xp, gu)             # silu(x' Wg^T) * (x' Wu^T), one fused call
"""
from __future__ import annotations

import ctypes
from typing import NamedTuple, Optional

import torch

from . import _lib
from ._lib import AwqError, MODE_GEMM, MODE_GEMV, MODE_LINEAR

GROUP = 128

__all__ = [
    "AwqError", "PackedWeight", "GROUP", "awq_packed_sizes", "awq_act_scale", "awq_apply_inv_scale", "awq_pack",
    "w4a16_gemv", "w4a16_gemm", "w4a16_linear", "w4a16_gemv_max_m", "w4a16_workspace_bytes",
    "awq_last_device_status", "reserve_workspace", "lib_path", "w4a16_gemv_noalloc",
    "awq_selftest_wait_timeout", "w4a16_linear_pf", "w4a16_gemv_s", "awq_pack_gate_up", "w4a16_gate_up_silu",
    "SearchResult", "awq_search_scale", "gptq_quantize", "awq_pack3", "w3a16_gemv",
]


class PackedWeight(NamedTuple):
    qweight: torch.Tensor  # int32 [N_pad * K / 8]
    scales: torch.Tensor   # fp16 [G * N_pad]
    qzeros: torch.Tensor   # int32 [G * N_pad / 8]
    N: int
    K: int
    g: int = GROUP          # group size the weight was packed with
    bits: int = 4           # code layout: 4 (w4a16_* calls) or 3 (awq_pack3 / w3a16_gemv)


class SearchResult(NamedTuple):
    s: torch.Tensor        # fp16 [K]: the scale of the winning alpha
    best: int              # winning grid index
    alpha: float           # best / n_grid
    losses: torch.Tensor   # float64 [n_grid + 1]


def lib_path() -> str:
    return _lib.lib_path()


def _p(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda_fp16(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda or t.dtype != torch.float16 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA float16 tensor")


def _check_out(out: torch.Tensor, shape, device, name: str = "out") -> None:
    """A caller-supplied output must be exactly what the kernel writes: a wrong size would become an
    out-of-bounds device write instead of an error."""
    _need_cuda_fp16(out, name)
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(out.shape)}, expected {tuple(shape)}")
    if out.device != torch.device(device):
        raise ValueError(f"{name} is on {out.device}, expected {device}")


def awq_packed_sizes(N: int, K: int, g: int = GROUP):
    L = _lib.load()
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _lib.check(L.awq_packed_sizes(N, K, g, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)), "awq_packed_sizes")
    return a.value, b.value, c.value


def awq_act_scale(xcal: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need_cuda_fp16(xcal, "xcal")
    R, K = xcal.shape
    if out is not None:
        _check_out(out, (K,), xcal.device)
    s = torch.empty(K, dtype=torch.float16, device=xcal.device) if out is None else out
    L = _lib.load()
    _lib.check(L.awq_act_scale(_p(xcal), R, K, _p(s), _stream(xcal.device)), "awq_act_scale")
    return s


def awq_apply_inv_scale(x: torch.Tensor, s: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need_cuda_fp16(x, "x")
    _need_cuda_fp16(s, "s")
    M, K = x.shape
    if s.shape != (K,):
        raise ValueError(f"s has shape {tuple(s.shape)}, expected ({K},)")
    if out is not None:
        _check_out(out, (M, K), x.device)
    xp = torch.empty_like(x) if out is None else out
    L = _lib.load()
    _lib.check(L.awq_apply_inv_scale(_p(x), _p(s), M, K, _p(xp), _stream(x.device)), "awq_apply_inv_scale")
    return xp


def awq_pack(W: torch.Tensor, s: Optional[torch.Tensor] = None, g: int = GROUP,
             out: Optional[PackedWeight] = None, w_bit: int = 4) -> PackedWeight:
    """Packs W (with s folded in); `out` reuses the three buffers of an earlier PackedWeight of the same shape.
    w_bit = 3 quantizes on the 3-bit grid (codes 0..7) in the same 4-bit layout."""
    _need_cuda_fp16(W, "W")
    N, K = W.shape
    if s is not None:
        _need_cuda_fp16(s, "s")
        if s.shape != (K,):
            raise ValueError(f"s has shape {tuple(s.shape)}, expected ({K},)")
    dev = W.device
    qw, sc, qz = _packed_buffers(N, K, g, dev, out)
    L = _lib.load()
    if w_bit == 4:
        _lib.check(L.awq_pack(_p(W), _p(s), N, K, g, _p(qw), _p(sc), _p(qz), _stream(dev)), "awq_pack")
    else:
        _lib.check(L.awq_pack_bits(_p(W), _p(s), N, K, g, w_bit, _p(qw), _p(sc), _p(qz), _stream(dev)),
                   "awq_pack_bits")
    return PackedWeight(qw, sc, qz, N, K, g)


def _packed_buffers(N: int, K: int, g: int, dev, out: Optional[PackedWeight]):
    qb, sb, zb = awq_packed_sizes(N, K, g)
    if out is not None:
        if (out.N, out.K, out.g) != (N, K, g) or out.qweight.numel() * 4 != qb or out.scales.numel() * 2 != sb \
                or out.qzeros.numel() * 4 != zb or any(t.device != dev for t in out[:3]):
            raise ValueError("out does not match the packed sizes of W")
        return out.qweight, out.scales, out.qzeros
    return (torch.empty(qb // 4, dtype=torch.int32, device=dev), torch.empty(sb // 2, dtype=torch.float16, device=dev),
            torch.empty(zb // 4, dtype=torch.int32, device=dev))


def awq_pack_gate_up(Wg: torch.Tensor, Wu: torch.Tensor, s: Optional[torch.Tensor] = None, g: int = GROUP,
                     out: Optional[PackedWeight] = None) -> PackedWeight:
    """Packs the gate and up projections ([NI][K] each, the same input) as one interleaved packed weight of
    2 NI rows for w4a16_gate_up_silu (row 32j + i: gate row 16j + i for i < 16, up row 16j + i - 16 after)."""
    _need_cuda_fp16(Wg, "Wg")
    _need_cuda_fp16(Wu, "Wu")
    if Wg.shape != Wu.shape or Wg.device != Wu.device:
        raise ValueError(f"Wg {tuple(Wg.shape)} and Wu {tuple(Wu.shape)} must have one shape and device")
    NI, K = Wg.shape
    if s is not None:
        _need_cuda_fp16(s, "s")
        if s.shape != (K,):
            raise ValueError(f"s has shape {tuple(s.shape)}, expected ({K},)")
    dev = Wg.device
    qw, sc, qz = _packed_buffers(2 * NI, K, g, dev, out)
    st = _lib.load().awq_pack_gate_up(_p(Wg), _p(Wu), _p(s), NI, K, g, _p(qw), _p(sc), _p(qz), _stream(dev))
    _lib.check(st, "awq_pack_gate_up")
    return PackedWeight(qw, sc, qz, 2 * NI, K, g)


# ---- workspace: one zero-initialised buffer per device, grown on demand (the kernels leave it
# ready for the next call).  Reserve the largest size before capturing CUDA graphs.
_workspaces: dict = {}


def w4a16_workspace_bytes(mode: int, M: int, N: int, K: int, g: int = GROUP) -> int:
    return int(_lib.load().w4a16_workspace_bytes(mode, M, N, K, g))


def reserve_workspace(nbytes: int, device=None) -> torch.Tensor:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=dev)
        _workspaces[key] = ws
    return ws


def _group(pw: PackedWeight, g: Optional[int], bits: int = 4) -> int:
    if pw.bits != bits:
        raise ValueError(f"the weight has the {pw.bits}-bit layout; this call reads the {bits}-bit layout")
    if g is not None and g != pw.g:
        raise ValueError(f"g={g} but the weight was packed with g={pw.g}")
    return pw.g


def _linear_call(fn_name: str, mode: int, x: torch.Tensor, pw: PackedWeight, out, workspace, g, extra=(),
                 out_cols: Optional[int] = None, n_arg: Optional[int] = None):
    _need_cuda_fp16(x, "x")
    g = _group(pw, g)
    M, K = x.shape
    if K != pw.K:
        raise ValueError(f"x has K={K}, weight has K={pw.K}")
    N = pw.N
    cols = N if out_cols is None else out_cols
    if out is not None:
        _check_out(out, (M, cols), x.device)
    y = torch.empty((M, cols), dtype=torch.float16, device=x.device) if out is None else out
    need = w4a16_workspace_bytes(mode, M, N, K, g)
    if need == 2**64 - 1:
        raise AwqError(fn_name, 1)
    ws = workspace if workspace is not None else (reserve_workspace(need, x.device) if need > 0 else None)
    L = _lib.load()
    fn = getattr(L, fn_name)
    st = fn(_p(x), _p(pw.qweight), _p(pw.scales), _p(pw.qzeros), _p(y), M, N if n_arg is None else n_arg, K, g,
            _p(ws), 0 if ws is None else ws.numel() * ws.element_size(), *extra, _stream(x.device))
    _lib.check(st, fn_name)
    return y


def w4a16_gemv(x, pw: PackedWeight, out=None, workspace=None, g: Optional[int] = None) -> torch.Tensor:
    return _linear_call("w4a16_gemv", MODE_GEMV, x, pw, out, workspace, g)


def w4a16_gemm(x, pw: PackedWeight, out=None, workspace=None, g: Optional[int] = None) -> torch.Tensor:
    return _linear_call("w4a16_gemm", MODE_GEMM, x, pw, out, workspace, g)


def w4a16_linear(x, pw: PackedWeight, out=None, workspace=None, g: Optional[int] = None) -> torch.Tensor:
    return _linear_call("w4a16_linear", MODE_LINEAR, x, pw, out, workspace, g)


def w4a16_gate_up_silu(x, pw: PackedWeight, out=None, workspace=None, g: Optional[int] = None) -> torch.Tensor:
    """h = silu(x' Wg^T) * (x' Wu^T), [M][NI], from a weight packed by awq_pack_gate_up (pw.N = 2 NI)."""
    if pw.N % 32 != 0:
        raise ValueError("not a gate|up packed weight (N must be 2 * NI with NI % 16 == 0)")
    return _linear_call("w4a16_gate_up_silu", MODE_LINEAR, x, pw, out, workspace, g, out_cols=pw.N // 2,
                        n_arg=pw.N // 2)


def w4a16_linear_pf(x, pw: PackedWeight, next_pw: Optional[PackedWeight], out=None, workspace=None,
                    g: Optional[int] = None) -> torch.Tensor:
    """w4a16_linear that also asks for next_pw's packed codes to be brought into L2 (GEMV mode only)."""
    nxt = (None, 0) if next_pw is None else (next_pw.qweight, next_pw.qweight.numel() * next_pw.qweight.element_size())
    extra = (ctypes.c_void_p(0 if nxt[0] is None else nxt[0].data_ptr()), ctypes.c_size_t(nxt[1]))
    return _linear_call("w4a16_linear_pf", MODE_LINEAR, x, pw, out, workspace, g, extra)


def w4a16_gemv_s(x, s, pw: PackedWeight, out=None, workspace=None, g: Optional[int] = None) -> torch.Tensor:
    """GEMV on the raw activations x with the AWQ scale s divided out inside the kernel (bit-identical to
    w4a16_gemv(awq_apply_inv_scale(x, s), pw))."""
    _need_cuda_fp16(x, "x")
    g = _group(pw, g)
    _need_cuda_fp16(s, "s")
    M, K = x.shape
    if K != pw.K or s.shape != (K,):
        raise ValueError(f"x has K={K}, s has shape {tuple(s.shape)}, weight has K={pw.K}")
    N = pw.N
    if out is not None:
        _check_out(out, (M, N), x.device)
    y = torch.empty((M, N), dtype=torch.float16, device=x.device) if out is None else out
    need = w4a16_workspace_bytes(MODE_GEMV, M, N, K, g)
    ws = workspace if workspace is not None else (reserve_workspace(need, x.device) if need > 0 else None)
    st = _lib.load().w4a16_gemv_s(_p(x), _p(s), _p(pw.qweight), _p(pw.scales), _p(pw.qzeros), _p(y), M, N, K, g,
                                   _p(ws), 0 if ws is None else ws.numel() * ws.element_size(), _stream(x.device))
    _lib.check(st, "w4a16_gemv_s")
    return y


def w4a16_gemv_noalloc(x, pw: PackedWeight, out=None, g: Optional[int] = None) -> torch.Tensor:
    """GEMV whose scratch is the library's static device array (no allocation by the library; for
    callers that cannot allocate device memory).  Overlapping calls on one device race."""
    _need_cuda_fp16(x, "x")
    g = _group(pw, g)
    M, K = x.shape
    if K != pw.K:
        raise ValueError(f"x has K={K}, weight has K={pw.K}")
    if out is not None:
        _check_out(out, (M, pw.N), x.device)
    y = torch.empty((M, pw.N), dtype=torch.float16, device=x.device) if out is None else out
    L = _lib.load()
    st = L.w4a16_gemv_noalloc(_p(x), _p(pw.qweight), _p(pw.scales), _p(pw.qzeros), _p(y), M, pw.N, K, g,
                              _stream(x.device))
    _lib.check(st, "w4a16_gemv_noalloc")
    return y


def w4a16_gemv_max_m(N: int, K: int) -> int:
    return int(_lib.load().w4a16_gemv_max_m(N, K))


def awq_last_device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    st = torch.cuda.current_stream() if stream is None else stream
    return int(_lib.load().awq_last_device_status(ctypes.c_void_p(st.cuda_stream)))


def awq_selftest_wait_timeout(backoff: bool = False) -> int:
    """Runs the library's bounded-wait timeout check (about 2 s) on the current device.  Returns what the
    kernel wrote: 1 when the wait gave up and returned, 2 if it completed.  The device status word is
    left set; awq_last_device_status() then reports AWQ_ERR_DEVICE_TIMEOUT and clears it."""
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = _lib.load().awq_selftest_wait_timeout(int(bool(backoff)), ctypes.c_void_p(out.data_ptr()),
                                               _stream(out.device))
    _lib.check(st, "awq_selftest_wait_timeout")
    return int(out.item())


def awq_search_scale(W: torch.Tensor, xcal: torch.Tensor, n_grid: int = 20, g: int = GROUP,
                     workspace: Optional[torch.Tensor] = None) -> SearchResult:
    """AWQ scale search over alpha = i / n_grid on the GPU (every step in the library's kernels).  Reads the
    winner back to the host (one synchronisation at the end)."""
    _need_cuda_fp16(W, "W")
    _need_cuda_fp16(xcal, "xcal")
    N, K = W.shape
    R = xcal.shape[0]
    if xcal.shape[1] != K or xcal.device != W.device:
        raise ValueError(f"xcal {tuple(xcal.shape)} does not match W {tuple(W.shape)}")
    L = _lib.load()
    need = int(L.awq_search_workspace_bytes(N, K, R, g, n_grid))
    if need == 2**64 - 1:
        raise AwqError("awq_search_scale", 1)
    dev = W.device
    ws = workspace if workspace is not None and workspace.numel() * workspace.element_size() >= need else \
        torch.empty(need, dtype=torch.uint8, device=dev)
    losses = torch.empty(n_grid + 1, dtype=torch.float64, device=dev)
    s = torch.empty(K, dtype=torch.float16, device=dev)
    best = torch.empty(4, dtype=torch.int32, device=dev)
    st = L.awq_search_scale(_p(W), _p(xcal), N, K, R, g, n_grid, _p(losses), _p(s), _p(best), _p(ws),
                            ws.numel() * ws.element_size(), _stream(dev))
    _lib.check(st, "awq_search_scale")
    b = int(best[0].item())
    return SearchResult(s, b, b / n_grid, losses)


def gptq_quantize(W: torch.Tensor, xcal: torch.Tensor, g: int = GROUP, damp: float = 1e-6,
                  out: Optional[PackedWeight] = None, workspace: Optional[torch.Tensor] = None) -> PackedWeight:
    """GPTQ of W [N][K] on calibration activations xcal [R][K] into the packed layout of awq_pack (every step in
    the library's kernels; asynchronous)."""
    _need_cuda_fp16(W, "W")
    _need_cuda_fp16(xcal, "xcal")
    N, K = W.shape
    R = xcal.shape[0]
    if xcal.shape[1] != K or xcal.device != W.device:
        raise ValueError(f"xcal {tuple(xcal.shape)} does not match W {tuple(W.shape)}")
    L = _lib.load()
    need = int(L.gptq_workspace_bytes(N, K, R, g))
    if need == 2**64 - 1:
        raise AwqError("gptq_quantize", 1)
    dev = W.device
    ws = workspace if workspace is not None and workspace.numel() * workspace.element_size() >= need else \
        torch.empty(need, dtype=torch.uint8, device=dev)
    qw, sc, qz = _packed_buffers(N, K, g, dev, out)
    st = L.gptq_quantize(_p(W), _p(xcal), N, K, R, g, ctypes.c_double(damp), _p(qw), _p(sc), _p(qz), _p(ws),
                         ws.numel() * ws.element_size(), _stream(dev))
    _lib.check(st, "gptq_quantize")
    return PackedWeight(qw, sc, qz, N, K, g)


def awq_pack3(W: torch.Tensor, s: Optional[torch.Tensor] = None, g: int = GROUP) -> PackedWeight:
    """Quantizes W (s folded in) on the 3-bit grid into the packed 3-bit layout (0.39 B per weight), for
    w3a16_gemv."""
    _need_cuda_fp16(W, "W")
    N, K = W.shape
    if s is not None:
        _need_cuda_fp16(s, "s")
        if s.shape != (K,):
            raise ValueError(f"s has shape {tuple(s.shape)}, expected ({K},)")
    L = _lib.load()
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _lib.check(L.awq_packed3_sizes(N, K, g, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)), "awq_packed3_sizes")
    dev = W.device
    qw = torch.empty(a.value // 4, dtype=torch.int32, device=dev)
    sc = torch.empty(b.value // 2, dtype=torch.float16, device=dev)
    qz = torch.empty(c.value // 4, dtype=torch.int32, device=dev)
    _lib.check(L.awq_pack3(_p(W), _p(s), N, K, g, _p(qw), _p(sc), _p(qz), _stream(dev)), "awq_pack3")
    return PackedWeight(qw, sc, qz, N, K, g, 3)


def w3a16_gemv(x, pw: PackedWeight, out=None, workspace=None) -> torch.Tensor:
    """The decode GEMV on a weight from awq_pack3 (any M, in passes of up to 16 rows)."""
    _need_cuda_fp16(x, "x")
    g = _group(pw, None, 3)
    M, K = x.shape
    if K != pw.K:
        raise ValueError(f"x has K={K}, weight has K={pw.K}")
    N = pw.N
    if out is not None:
        _check_out(out, (M, N), x.device)
    y = torch.empty((M, N), dtype=torch.float16, device=x.device) if out is None else out
    need = w4a16_workspace_bytes(MODE_GEMV, M, N, K, g)
    ws = workspace if workspace is not None else (reserve_workspace(need, x.device) if need > 0 else None)
    st = _lib.load().w3a16_gemv(_p(x), _p(pw.qweight), _p(pw.scales), _p(pw.qzeros), _p(y), M, N, K, g, _p(ws),
                                0 if ws is None else ws.numel() * ws.element_size(), _stream(x.device))
    _lib.check(st, "w3a16_gemv")
    return y
