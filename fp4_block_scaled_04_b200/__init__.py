"""fp4_block_scaled_04_b200 -- block-scaled FP4 quantization on B200 (sm_100a).

A thin ctypes binding over ``libfp4q.so`` (C ABI: ``include/fp4q.h``).  The
Python functions carry the C names and only marshal arguments: they check
tensor placement, allocate outputs with torch (device memory and streams are
torch's), and pass raw pointers plus the current CUDA stream.  Every step of
the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback -- a missing library raises ``Fp4qLibraryMissing``.

Formats and layouts (see the header for the arithmetic):
  NVFP4  E2M1 codes + E4M3 scale per 16 values + FP32 tensor scale
  MXFP4  E2M1 codes + E8M0 scale per 32 values
  2D     NVFP4 with one scale per 16x16 tile (W and W^T codes)
  RHT    random Hadamard transform along tokens + NVFP4 (SR or RNE) of dY^T
  IF4    per-block FP4 / INT4 choice, flag in bit 7 of the scale byte
  MXFP6  FP6 (E2M3 or E3M2) codes, four per three bytes + E8M0 scale per 32
  GEMM   C = s_a s_b (A B^T) from NVFP4 operands on the tensor cores
  IF6    per-block FP6 E2M3 / INT6 choice, six-bit codes, flag in bit 7 of the scale
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "ROWWISE", "COLWISE", "RNE", "SR", "SCALE_LINEAR", "SCALE_SWIZZLED",
    "E8M0_RNE", "E8M0_CEIL", "E8M0_OCP_FLOOR", "FMT_NVFP4", "FMT_MXFP4", "FMT_IF4",
    "Fp4qError", "Fp4qLibraryMissing", "lib", "library_path",
    "fp4q_status_string", "fp4q_version", "fp4q_workspace_bytes", "fp4q_scale_bytes",
    "fp4q_amax", "fp4q_quantize_nvfp4", "fp4q_quantize_mxfp4", "fp4q_quantize_2d",
    "fp4q_rht_amax", "fp4q_quantize_rht_sr", "fp4q_quantize_if4", "fp4q_dequantize",
    "fp4q_quantize_nvfp4_noalloc", "fp4q_quantize_nvint4", "fp4q_quantize_four_over_six",
    "fp4q_quantize_backward", "fp4q_quantize_mxfp6", "FMT_MXFP6_E2M3", "FMT_MXFP6_E3M2",
    "FP6_E2M3", "FP6_E3M2", "fp4q_gemm_nvfp4", "fp4q_gemm_mxfp4", "fp4q_quantize_if6", "FMT_IF6",
    "fp4q_gemm_if4_nvfp4", "fp4q_quantize_if3", "FMT_IF3",
]

ROWWISE, COLWISE = 1, 2
RNE, SR = 0, 1
SCALE_LINEAR, SCALE_SWIZZLED = 0, 1
E8M0_RNE, E8M0_CEIL, E8M0_OCP_FLOOR = 0, 1, 2
FMT_NVFP4, FMT_MXFP4, FMT_IF4, FMT_MXFP6_E2M3, FMT_MXFP6_E3M2, FMT_IF6, FMT_IF3 = (
    0, 1, 2, 3, 4, 5, 6)
FP6_E2M3, FP6_E3M2 = 0, 1
_BF16, _FP32 = 0, 1

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libfp4q.so")


class Fp4qError(RuntimeError):
    """A C-ABI call returned a non-OK status."""

    def __init__(self, name: str, status: int):
        self.status = status
        super().__init__(f"{name} failed: {fp4q_status_string(status)}")


class Fp4qLibraryMissing(RuntimeError):
    """libfp4q.so is not built or cannot be loaded (no fallback exists)."""


_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_U = ctypes.c_uint
_U64 = ctypes.c_uint64
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "fp4q_status_string": (ctypes.c_char_p, [_I]),
    "fp4q_version": (ctypes.c_char_p, []),
    "fp4q_workspace_bytes": (_SZ, [_I64, _I64]),
    "fp4q_scale_bytes": (_SZ, [_I64, _I64, _I, _I]),
    "fp4q_amax": (_I, [_P, _I, _I64, _I64, _I64, _P, _P]),
    "fp4q_quantize_nvfp4": (_I, [_P, _I, _I64, _I64, _I64, _U, _I, _U64, _P, _P, _P, _P, _P,
                                 _P, _I, _P, _SZ, _P]),
    "fp4q_quantize_mxfp4": (_I, [_P, _I, _I64, _I64, _I64, _U, _I, _P, _P, _P, _P, _I, _P]),
    "fp4q_quantize_2d": (_I, [_P, _I, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _I, _P,
                              _SZ, _P]),
    "fp4q_rht_amax": (_I, [_P, _I, _I64, _I64, _I64, _I, _U64, _P, _P]),
    "fp4q_quantize_rht_sr": (_I, [_P, _I, _I64, _I64, _I64, _I, _I, _U64, _P, _P, _P, _P, _I,
                                  _P, _P, _SZ, _P]),
    "fp4q_quantize_if4": (_I, [_P, _I, _I64, _I64, _I64, _P, _P, _P, _P, _I, _P, _SZ, _P]),
    "fp4q_dequantize": (_I, [_I, _P, _P, _I, _I, _I, _P, _I64, _I64, _P, _I, _P]),
    "fp4q_quantize_nvfp4_noalloc": (_I, [_P, _I, _I64, _I64, _I64, _U, _I, _U64, _P, _P, _P,
                                         _P, _P, _P, _I, _P]),
    "fp4q_quantize_nvint4": (_I, [_P, _I, _I64, _I64, _I64, _P, _P, _P, _P, _I, _P, _SZ, _P]),
    "fp4q_quantize_backward": (_I, [_P, _I, _I64, _I64, _I64, _I, _I, _U64, _U64, _P, _P, _P,
                                    _P, _P, _P, _P, _P, _I, _P, _SZ, _P]),
    "fp4q_quantize_four_over_six": (_I, [_P, _I, _I64, _I64, _I64, _U, _P, _P, _P, _P, _P, _P,
                                         _I, _P, _SZ, _P]),
    "fp4q_quantize_mxfp6": (_I, [_P, _I, _I64, _I64, _I64, _I, _I, _P, _P, _I, _P]),
    "fp4q_gemm_nvfp4": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I, _I64, _P, _P]),
    "fp4q_gemm_mxfp4": (_I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _I, _I64, _P, _P]),
    "fp4q_gemm_nvfp4_withhold_loads": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I,
                                            _I64, _P, _P]),
    "fp4q_gemm_if4_workspace_bytes": (_SZ, [_I64, _I64]),
    "fp4q_gemm_if4_nvfp4": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, _P, _SZ,
                                 _P, _P]),
    "fp4q_quantize_if6": (_I, [_P, _I, _I64, _I64, _I64, _P, _P, _P, _P, _I, _P, _SZ, _P]),
    "fp4q_quantize_if3": (_I, [_P, _I, _I64, _I64, _I64, _P, _P, _P, _P, _I, _P, _SZ, _P]),
}


def lib() -> ctypes.CDLL:
    """Load libfp4q.so (built in-tree by ``python -m fp4_block_scaled_04_b200.build``)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(library_path):
                    raise Fp4qLibraryMissing(
                        f"{library_path} is missing; build it with "
                        "`python -m fp4_block_scaled_04_b200.build` (there is no fallback)")
                try:
                    L = ctypes.CDLL(library_path)
                except OSError as e:
                    raise Fp4qLibraryMissing(f"cannot load {library_path}: {e}") from e
                for name, (res, args) in _SIGNATURES.items():
                    fn = getattr(L, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = L
    return _lib


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return _BF16
    if x.dtype == torch.float32:
        return _FP32
    raise TypeError(f"input must be bfloat16 or float32, got {x.dtype}")


def _matrix(x: torch.Tensor, name: str = "x"):
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library computes on the GPU only)")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with unit column stride")
    rows, cols = x.shape
    ld = x.stride(0) if rows > 1 else cols
    return rows, cols, ld


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(name: str, status: int):
    if status != 0:
        raise Fp4qError(name, status)


_ws_cache: dict = {}


def _workspace(device: torch.device) -> torch.Tensor:
    key = (device.type, device.index)
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.empty(fp4q_workspace_bytes(), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def _u8(n, device) -> torch.Tensor:
    return torch.empty(n, dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------
# C-ABI mirrors
# ---------------------------------------------------------------------------

def fp4q_status_string(status: int) -> str:
    return lib().fp4q_status_string(int(status)).decode()


def fp4q_version() -> str:
    return lib().fp4q_version().decode()


def fp4q_workspace_bytes(rows: int = 0, cols: int = 0) -> int:
    return int(lib().fp4q_workspace_bytes(int(rows), int(cols)))


def fp4q_scale_bytes(rows: int, cols: int, block: int, scale_layout: int = SCALE_LINEAR) -> int:
    return int(lib().fp4q_scale_bytes(rows, cols, block, scale_layout))


def fp4q_amax(x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    rows, cols, ld = _matrix(x)
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    _check("fp4q_amax", lib().fp4q_amax(_ptr(x), _dtype(x), rows, cols, ld, _ptr(out),
                                        _stream(x.device)))
    return out


def fp4q_quantize_nvfp4(x: torch.Tensor, layouts: int = ROWWISE, round: int = RNE,
                        seed: int = 0, amax: torch.Tensor | None = None,
                        scale_layout: int = SCALE_LINEAR, out: dict | None = None) -> dict:
    """NVFP4 1x16; returns {'s_dec', 'q_row', 'sf_row', 'q_col', 'sf_col'} (requested ones)."""
    rows, cols, ld = _matrix(x)
    dev = x.device
    if out is None:
        out = {"s_dec": torch.empty(1, dtype=torch.float32, device=dev)}
        if layouts & ROWWISE:
            out["q_row"] = _u8((rows, cols // 2), dev)
            out["sf_row"] = _u8(fp4q_scale_bytes(rows, cols, 16, scale_layout), dev)
        if layouts & COLWISE:
            out["q_col"] = _u8((cols, rows // 2), dev)
            out["sf_col"] = _u8(fp4q_scale_bytes(cols, rows, 16, scale_layout), dev)
    ws = _workspace(dev) if amax is None else None
    _check("fp4q_quantize_nvfp4", lib().fp4q_quantize_nvfp4(
        _ptr(x), _dtype(x), rows, cols, ld, layouts, round, seed, _ptr(amax),
        _ptr(out.get("s_dec")), _ptr(out.get("q_row")), _ptr(out.get("sf_row")),
        _ptr(out.get("q_col")), _ptr(out.get("sf_col")), scale_layout, _ptr(ws),
        0 if ws is None else ws.numel(), _stream(dev)))
    return out


def fp4q_quantize_nvfp4_noalloc(x: torch.Tensor, out: dict, layouts: int = ROWWISE,
                                round: int = RNE, seed: int = 0,
                                amax: torch.Tensor | None = None,
                                scale_layout: int = SCALE_LINEAR) -> dict:
    """``fp4q_quantize_nvfp4`` for callers that cannot allocate: the outputs in
    ``out`` are the caller's buffers and, when ``amax`` is None, the library's
    own 256-byte device array holds the amax instead of a workspace.  Calls
    on one device that overlap on the GPU race on that array."""
    rows, cols, ld = _matrix(x)
    _check("fp4q_quantize_nvfp4_noalloc", lib().fp4q_quantize_nvfp4_noalloc(
        _ptr(x), _dtype(x), rows, cols, ld, layouts, round, seed, _ptr(amax),
        _ptr(out.get("s_dec")), _ptr(out.get("q_row")), _ptr(out.get("sf_row")),
        _ptr(out.get("q_col")), _ptr(out.get("sf_col")), scale_layout, _stream(x.device)))
    return out


def fp4q_quantize_mxfp4(x: torch.Tensor, layouts: int = ROWWISE, e8m0_mode: int = E8M0_RNE,
                        scale_layout: int = SCALE_LINEAR, out: dict | None = None) -> dict:
    """MXFP4 1x32; returns {'q_row', 'sf_row', 'q_col', 'sf_col'} (requested ones)."""
    rows, cols, ld = _matrix(x)
    dev = x.device
    if out is None:
        out = {}
        if layouts & ROWWISE:
            out["q_row"] = _u8((rows, cols // 2), dev)
            out["sf_row"] = _u8(fp4q_scale_bytes(rows, cols, 32, scale_layout), dev)
        if layouts & COLWISE:
            out["q_col"] = _u8((cols, rows // 2), dev)
            out["sf_col"] = _u8(fp4q_scale_bytes(cols, rows, 32, scale_layout), dev)
    _check("fp4q_quantize_mxfp4", lib().fp4q_quantize_mxfp4(
        _ptr(x), _dtype(x), rows, cols, ld, layouts, e8m0_mode, _ptr(out.get("q_row")),
        _ptr(out.get("sf_row")), _ptr(out.get("q_col")), _ptr(out.get("sf_col")), scale_layout,
        _stream(dev)))
    return out


def fp4q_quantize_mxfp6(x: torch.Tensor, fp6_format: int = FP6_E2M3, e8m0_mode: int = E8M0_RNE,
                        scale_layout: int = SCALE_LINEAR, out: dict | None = None) -> dict:
    """MXFP6 1x32 row-wise; returns {'q': [rows, cols*3/4] bytes, 'sf'}."""
    rows, cols, ld = _matrix(x)
    dev = x.device
    if out is None:
        out = {"q": _u8((rows, cols * 3 // 4), dev),
               "sf": _u8(fp4q_scale_bytes(rows, cols, 32, scale_layout), dev)}
    _check("fp4q_quantize_mxfp6", lib().fp4q_quantize_mxfp6(
        _ptr(x), _dtype(x), rows, cols, ld, fp6_format, e8m0_mode, _ptr(out["q"]),
        _ptr(out["sf"]), scale_layout, _stream(dev)))
    return out


def fp4q_quantize_if6(x: torch.Tensor, amax: torch.Tensor | None = None,
                      scale_layout: int = SCALE_LINEAR, out: dict | None = None) -> dict:
    """IF6 (FP6 E2M3 or INT6 per 16-block); returns {'s_dec', 'q' [rows, cols*3/4], 'sf'}."""
    rows, cols, ld = _matrix(x)
    dev = x.device
    if out is None:
        out = {"s_dec": torch.empty(1, dtype=torch.float32, device=dev),
               "q": _u8((rows, cols * 3 // 4), dev),
               "sf": _u8(fp4q_scale_bytes(rows, cols, 16, scale_layout), dev)}
    ws = _workspace(dev) if amax is None else None
    _check("fp4q_quantize_if6", lib().fp4q_quantize_if6(
        _ptr(x), _dtype(x), rows, cols, ld, _ptr(amax), _ptr(out.get("s_dec")), _ptr(out["q"]),
        _ptr(out["sf"]), scale_layout, _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return out


def fp4q_quantize_if3(x: torch.Tensor, amax: torch.Tensor | None = None,
                      scale_layout: int = SCALE_LINEAR, out: dict | None = None) -> dict:
    """IF3 (FP3 E2M0 or INT3 per 16-block); returns {'s_dec', 'q' [rows, cols*3/8], 'sf'}."""
    rows, cols, ld = _matrix(x)
    dev = x.device
    if out is None:
        out = {"s_dec": torch.empty(1, dtype=torch.float32, device=dev),
               "q": _u8((rows, cols * 3 // 8), dev),
               "sf": _u8(fp4q_scale_bytes(rows, cols, 16, scale_layout), dev)}
    ws = _workspace(dev) if amax is None else None
    _check("fp4q_quantize_if3", lib().fp4q_quantize_if3(
        _ptr(x), _dtype(x), rows, cols, ld, _ptr(amax), _ptr(out.get("s_dec")), _ptr(out["q"]),
        _ptr(out["sf"]), scale_layout, _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return out


def fp4q_gemm_nvfp4(qa: torch.Tensor, sfa: torch.Tensor, qb: torch.Tensor, sfb: torch.Tensor,
                    K: int, tensor_scale_a: torch.Tensor | None = None,
                    tensor_scale_b: torch.Tensor | None = None,
                    out_dtype: torch.dtype = torch.float32, out: torch.Tensor | None = None,
                    status: torch.Tensor | None = None) -> torch.Tensor:
    """C [M, N] = s_a s_b (A B^T) from NVFP4 operands: codes qa [M, K/2], qb
    [N, K/2] and their swizzled 1x16 scales (as fp4q_quantize_nvfp4 writes them)."""
    if not qa.is_cuda:
        raise ValueError("qa must be a CUDA tensor")
    M, N = qa.shape[0], qb.shape[0]
    c = torch.empty((M, N), dtype=out_dtype, device=qa.device) if out is None else out
    cdt = _BF16 if c.dtype == torch.bfloat16 else _FP32
    _check("fp4q_gemm_nvfp4", lib().fp4q_gemm_nvfp4(
        _ptr(qa), _ptr(sfa), _ptr(tensor_scale_a), _ptr(qb), _ptr(sfb), _ptr(tensor_scale_b),
        M, N, K, _ptr(c), cdt, c.stride(0) if M > 1 else N, _ptr(status), _stream(qa.device)))
    return c


def fp4q_gemm_mxfp4(qa: torch.Tensor, sfa: torch.Tensor, qb: torch.Tensor, sfb: torch.Tensor,
                    K: int, out_dtype: torch.dtype = torch.float32,
                    out: torch.Tensor | None = None,
                    status: torch.Tensor | None = None) -> torch.Tensor:
    """C [M, N] = A B^T from MXFP4 operands: codes qa [M, K/2], qb [N, K/2] and
    their swizzled 1x32 E8M0 scales (as fp4q_quantize_mxfp4 writes them)."""
    if not qa.is_cuda:
        raise ValueError("qa must be a CUDA tensor")
    M, N = qa.shape[0], qb.shape[0]
    c = torch.empty((M, N), dtype=out_dtype, device=qa.device) if out is None else out
    cdt = _BF16 if c.dtype == torch.bfloat16 else _FP32
    _check("fp4q_gemm_mxfp4", lib().fp4q_gemm_mxfp4(
        _ptr(qa), _ptr(sfa), _ptr(qb), _ptr(sfb), M, N, K, _ptr(c), cdt,
        c.stride(0) if M > 1 else N, _ptr(status), _stream(qa.device)))
    return c


def fp4q_gemm_if4_nvfp4(qa: torch.Tensor, sfa: torch.Tensor, qb: torch.Tensor, sfb: torch.Tensor,
                        K: int, tensor_scale_a: torch.Tensor | None = None,
                        tensor_scale_b: torch.Tensor | None = None,
                        out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                        status: torch.Tensor | None = None) -> torch.Tensor:
    """C [M, N] FP32 = s_a s_b (A B^T) with A in IF4 (codes [M, K/2], flagged
    swizzled scales as fp4q_quantize_if4 writes them) and B in NVFP4."""
    if not qa.is_cuda:
        raise ValueError("qa must be a CUDA tensor")
    M, N = qa.shape[0], qb.shape[0]
    c = torch.empty((M, N), dtype=torch.float32, device=qa.device) if out is None else out
    need = int(lib().fp4q_gemm_if4_workspace_bytes(M, K))
    ws = _u8(max(need, 16), qa.device) if workspace is None else workspace
    _check("fp4q_gemm_if4_nvfp4", lib().fp4q_gemm_if4_nvfp4(
        _ptr(qa), _ptr(sfa), _ptr(tensor_scale_a), _ptr(qb), _ptr(sfb), _ptr(tensor_scale_b),
        M, N, K, _ptr(c), c.stride(0) if M > 1 else N, _ptr(ws), ws.numel(), _ptr(status),
        _stream(qa.device)))
    return c


def fp4q_quantize_2d(w: torch.Tensor, amax: torch.Tensor | None = None, with_1x16: bool = False,
                     scale_layout: int = SCALE_LINEAR, emit_w: bool = True,
                     emit_wt: bool = True, out: dict | None = None) -> dict:
    """NVFP4 16x16 2D; returns {'s_dec', 'q_w', 'q_wt', 'sf_tiles', ['sf_w_1x16', 'sf_wt_1x16']}."""
    rows, cols, ld = _matrix(w, "w")
    dev = w.device
    if out is None:
        out = {"s_dec": torch.empty(1, dtype=torch.float32, device=dev),
               "sf_tiles": _u8((rows // 16, cols // 16), dev)}
        if emit_w:
            out["q_w"] = _u8((rows, cols // 2), dev)
        if emit_wt:
            out["q_wt"] = _u8((cols, rows // 2), dev)
        if with_1x16:
            out["sf_w_1x16"] = _u8(fp4q_scale_bytes(rows, cols, 16, scale_layout), dev)
            out["sf_wt_1x16"] = _u8(fp4q_scale_bytes(cols, rows, 16, scale_layout), dev)
    ws = _workspace(dev) if amax is None else None
    _check("fp4q_quantize_2d", lib().fp4q_quantize_2d(
        _ptr(w), _dtype(w), rows, cols, ld, _ptr(amax), _ptr(out.get("s_dec")),
        _ptr(out.get("q_w")), _ptr(out.get("q_wt")), _ptr(out.get("sf_tiles")),
        _ptr(out.get("sf_w_1x16")), _ptr(out.get("sf_wt_1x16")), scale_layout, _ptr(ws),
        0 if ws is None else ws.numel(), _stream(dev)))
    return out


def fp4q_rht_amax(dy: torch.Tensor, hadamard_n: int, seed: int = 0,
                  out: torch.Tensor | None = None) -> torch.Tensor:
    tokens, cols, ld = _matrix(dy, "dy")
    out = torch.empty(1, dtype=torch.float32, device=dy.device) if out is None else out
    _check("fp4q_rht_amax", lib().fp4q_rht_amax(_ptr(dy), _dtype(dy), tokens, cols, ld,
                                                hadamard_n, seed, _ptr(out),
                                                _stream(dy.device)))
    return out


def fp4q_quantize_rht_sr(dy: torch.Tensor, hadamard_n: int, round: int = SR, seed: int = 0,
                         amax_rht: torch.Tensor | None = None, scale_layout: int = SCALE_LINEAR,
                         want_rht: bool = False, out: dict | None = None) -> dict:
    """RHT along tokens + column-wise NVFP4; returns {'s_dec', 'q_t', 'sf_t', ['rht']}."""
    tokens, cols, ld = _matrix(dy, "dy")
    dev = dy.device
    if out is None:
        out = {"s_dec": torch.empty(1, dtype=torch.float32, device=dev),
               "q_t": _u8((cols, tokens // 2), dev),
               "sf_t": _u8(fp4q_scale_bytes(cols, tokens, 16, scale_layout), dev)}
        if want_rht:
            out["rht"] = torch.empty((tokens, cols), dtype=torch.float32, device=dev)
    ws = _workspace(dev) if amax_rht is None else None
    _check("fp4q_quantize_rht_sr", lib().fp4q_quantize_rht_sr(
        _ptr(dy), _dtype(dy), tokens, cols, ld, hadamard_n, round, seed, _ptr(amax_rht),
        _ptr(out.get("s_dec")), _ptr(out.get("q_t")), _ptr(out.get("sf_t")), scale_layout,
        _ptr(out.get("rht")), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return out


def fp4q_quantize_if4(x: torch.Tensor, amax: torch.Tensor | None = None,
                      scale_layout: int = SCALE_LINEAR, out: dict | None = None) -> dict:
    """IF4 row-wise 1x16; returns {'s_dec', 'q', 'sf'}."""
    rows, cols, ld = _matrix(x)
    dev = x.device
    if out is None:
        out = {"s_dec": torch.empty(1, dtype=torch.float32, device=dev),
               "q": _u8((rows, cols // 2), dev),
               "sf": _u8(fp4q_scale_bytes(rows, cols, 16, scale_layout), dev)}
    ws = _workspace(dev) if amax is None else None
    _check("fp4q_quantize_if4", lib().fp4q_quantize_if4(
        _ptr(x), _dtype(x), rows, cols, ld, _ptr(amax), _ptr(out.get("s_dec")),
        _ptr(out.get("q")), _ptr(out.get("sf")), scale_layout, _ptr(ws),
        0 if ws is None else ws.numel(), _stream(dev)))
    return out


def fp4q_quantize_backward(dy: torch.Tensor, hadamard_n: int = 16, round: int = SR,
                           seed_row: int = 0, seed_col: int = 1,
                           amax_row: torch.Tensor | None = None,
                           amax_rht: torch.Tensor | None = None,
                           scale_layout: int = SCALE_LINEAR, out: dict | None = None) -> dict:
    """Both backward operands of dY from one read: {'s_dec_row', 'q_row', 'sf_row'}
    (row-wise NVFP4, the Dgrad operand) and {'s_dec_col', 'q_t', 'sf_t'} (RHT +
    column-wise NVFP4 of dY^T, the Wgrad operand)."""
    tokens, cols, ld = _matrix(dy, "dy")
    dev = dy.device
    if out is None:
        out = {"s_dec_row": torch.empty(1, dtype=torch.float32, device=dev),
               "q_row": _u8((tokens, cols // 2), dev),
               "sf_row": _u8(fp4q_scale_bytes(tokens, cols, 16, scale_layout), dev),
               "s_dec_col": torch.empty(1, dtype=torch.float32, device=dev),
               "q_t": _u8((cols, tokens // 2), dev),
               "sf_t": _u8(fp4q_scale_bytes(cols, tokens, 16, scale_layout), dev)}
    ws = _workspace(dev) if (amax_row is None or amax_rht is None) else None
    _check("fp4q_quantize_backward", lib().fp4q_quantize_backward(
        _ptr(dy), _dtype(dy), tokens, cols, ld, hadamard_n, round, seed_row, seed_col,
        _ptr(amax_row), _ptr(amax_rht), _ptr(out.get("s_dec_row")), _ptr(out.get("s_dec_col")),
        _ptr(out.get("q_row")), _ptr(out.get("sf_row")), _ptr(out.get("q_t")),
        _ptr(out.get("sf_t")), scale_layout, _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(dev)))
    return out


def fp4q_quantize_nvint4(x: torch.Tensor, amax: torch.Tensor | None = None,
                         scale_layout: int = SCALE_LINEAR, out: dict | None = None) -> dict:
    """NVINT4 row-wise 1x16 (IF4's INT4 candidate in every block, flagged);
    returns {'s_dec', 'q', 'sf'}; decode with FMT_IF4."""
    rows, cols, ld = _matrix(x)
    dev = x.device
    if out is None:
        out = {"s_dec": torch.empty(1, dtype=torch.float32, device=dev),
               "q": _u8((rows, cols // 2), dev),
               "sf": _u8(fp4q_scale_bytes(rows, cols, 16, scale_layout), dev)}
    ws = _workspace(dev) if amax is None else None
    _check("fp4q_quantize_nvint4", lib().fp4q_quantize_nvint4(
        _ptr(x), _dtype(x), rows, cols, ld, _ptr(amax), _ptr(out.get("s_dec")),
        _ptr(out.get("q")), _ptr(out.get("sf")), scale_layout, _ptr(ws),
        0 if ws is None else ws.numel(), _stream(dev)))
    return out


def fp4q_quantize_four_over_six(x: torch.Tensor, layouts: int = ROWWISE,
                                amax: torch.Tensor | None = None,
                                scale_layout: int = SCALE_LINEAR, out: dict | None = None) -> dict:
    """NVFP4 1x16 layout with every block maximum mapped to 4 (the 4/6 method);
    returns {'s_dec', 'q_row', 'sf_row', 'q_col', 'sf_col'} (requested ones);
    decode with FMT_NVFP4."""
    rows, cols, ld = _matrix(x)
    dev = x.device
    if out is None:
        out = {"s_dec": torch.empty(1, dtype=torch.float32, device=dev)}
        if layouts & ROWWISE:
            out["q_row"] = _u8((rows, cols // 2), dev)
            out["sf_row"] = _u8(fp4q_scale_bytes(rows, cols, 16, scale_layout), dev)
        if layouts & COLWISE:
            out["q_col"] = _u8((cols, rows // 2), dev)
            out["sf_col"] = _u8(fp4q_scale_bytes(cols, rows, 16, scale_layout), dev)
    ws = _workspace(dev) if amax is None else None
    _check("fp4q_quantize_four_over_six", lib().fp4q_quantize_four_over_six(
        _ptr(x), _dtype(x), rows, cols, ld, layouts, _ptr(amax), _ptr(out.get("s_dec")),
        _ptr(out.get("q_row")), _ptr(out.get("sf_row")), _ptr(out.get("q_col")),
        _ptr(out.get("sf_col")), scale_layout, _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(dev)))
    return out


def fp4q_dequantize(fmt: int, q: torch.Tensor, sf: torch.Tensor, rows: int, cols: int,
                    block_rows: int = 1, block_cols: int = 16,
                    tensor_scale: torch.Tensor | None = None, scale_layout: int = SCALE_LINEAR,
                    out_dtype: torch.dtype = torch.float32,
                    out: torch.Tensor | None = None) -> torch.Tensor:
    """Packed codes ([rows, cols/2]; [rows, cols*3/4] for MXFP6 and IF6; [rows,
    cols*3/8] for IF3) + scales -> [rows, cols] in out_dtype (fp32 or bf16)."""
    if not q.is_cuda:
        raise ValueError("q must be a CUDA tensor")
    y = torch.empty((rows, cols), dtype=out_dtype, device=q.device) if out is None else out
    ydt = _BF16 if y.dtype == torch.bfloat16 else _FP32
    _check("fp4q_dequantize", lib().fp4q_dequantize(
        fmt, _ptr(q), _ptr(sf), scale_layout, block_rows, block_cols, _ptr(tensor_scale), rows,
        cols, _ptr(y), ydt, _stream(q.device)))
    return y
