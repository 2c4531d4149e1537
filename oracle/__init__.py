"""CPU oracle for block-scaled FP4 quantization -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct definition that the CUDA
library is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it; the library
(``fp4_block_scaled_04_b200``) never does, and the two share no code.

The arithmetic lives in ``fp4q_oracle.c`` (plain C, binary32, no FMA
contraction); this module compiles it on first use (``gcc -O2
-ffp-contract=off``) and wraps it for numpy arrays.  All arrays here are host
numpy arrays; BF16 tensors are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4q_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_LIB_OMP_PATH = os.path.join(_HERE, "liboracle_omp.so")
_lock = threading.Lock()
_lib = None          # the library the wrappers below call
_libs: dict = {}     # loaded builds by path
_use_openmp = False

BF16, FP32 = 0, 1
ROWWISE, COLWISE = 1, 2
RNE, SR = 0, 1
SCALE_LINEAR, SCALE_SWIZZLED = 0, 1
E8M0_RNE, E8M0_CEIL, E8M0_OCP_FLOOR = 0, 1, 2
FMT_NVFP4, FMT_MXFP4, FMT_IF4, FMT_MXFP6_E2M3, FMT_MXFP6_E3M2, FMT_IF6, FMT_IF3 = (
    0, 1, 2, 3, 4, 5, 6)
FP6_E2M3, FP6_E3M2 = 0, 1

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile fp4q_oracle.c into liboracle.so (idempotent).  With openmp, the
    same source with -fopenmp into liboracle_omp.so: its outer loops over
    rows, columns or tile rows then run on all host cores and produce the
    same bytes (each iteration writes whole bytes of its own)."""
    path = _LIB_OMP_PATH if openmp else _LIB_PATH
    with _lock:
        stale = (not os.path.exists(path)
                 or os.path.getmtime(path) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = path + f".{os.getpid()}.tmp"
            extra = ["-fopenmp"] if openmp else []
            subprocess.check_call(["gcc", *CFLAGS, *extra, _SRC, "-o", tmp, "-lm"])
            os.replace(tmp, path)
    return path


def use_openmp(on: bool = True) -> None:
    """Route the wrappers below to the OpenMP build (all host cores, the
    thread count from OMP_NUM_THREADS or the core count) or back to the
    single-threaded build the tests use."""
    global _lib, _use_openmp
    _use_openmp = bool(on)
    _lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = build(openmp=_use_openmp)
        if path in _libs:
            _lib = _libs[path]
            return _lib
        L = ctypes.CDLL(path)
        P, I64, I, U, U64, F = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                ctypes.c_uint, ctypes.c_uint64, ctypes.c_float)
        sig = {
            "orc_bf16_to_f32": (F, [ctypes.c_uint16]),
            "orc_f32_to_bf16": (ctypes.c_uint16, [F]),
            "orc_e2m1_value": (F, [ctypes.c_uint8]),
            "orc_e2m1_rne": (ctypes.c_uint8, [F]),
            "orc_e2m1_sr": (ctypes.c_uint8, [F, ctypes.c_uint32]),
            "orc_e4m3_value": (F, [ctypes.c_uint8]),
            "orc_e4m3_rne_sat": (ctypes.c_uint8, [F]),
            "orc_e8m0_exponent": (I, [F, I]),
            "orc_philox4x32_10": (None, [P, P, P]),
            "orc_sr_bits16": (ctypes.c_uint32, [U64, U64]),
            "orc_rht_signs": (None, [U64, I, P]),
            "orc_scale_bytes": (I64, [I64, I64, I]),
            "orc_scale_offset": (I64, [I64, I64, I64, I64, I]),
            "orc_amax": (F, [P, I, I64, I64, I64]),
            "orc_tensor_scales": (None, [F, P, P]),
            "orc_quantize_nvfp4": (I, [P, I, I64, I64, I64, U, I, U64, P, P, P, P, P, P, I]),
            "orc_quantize_nvfp4_rows": (I, [P, I, I64, I64, I64, U, I, U64, P, P, P, P, P, P, I,
                                            I64]),
            "orc_quantize_mxfp4": (I, [P, I, I64, I64, I64, U, I, P, P, P, P, I]),
            "orc_quantize_mxfp6": (I, [P, I, I64, I64, I64, I, I, P, P, I]),
            "orc_fp6_value": (F, [ctypes.c_uint8, I]),
            "orc_fp6_rne": (ctypes.c_uint8, [F, I]),
            "orc_quantize_2d": (I, [P, I, I64, I64, I64, P, P, P, P, P, P, P, I]),
            "orc_rht_norm": (F, [I]),
            "orc_rht": (I, [P, I, I64, I64, I64, I, U64, P]),
            "orc_quantize_rht": (I, [P, I, I64, I64, I64, I, I, U64, P, P, P, P, I, P]),
            "orc_quantize_rht_rows": (I, [P, I, I64, I64, I64, I, I, U64, P, P, P, P, I, P, I64]),
            "orc_if4_c76": (F, []),
            "orc_if4_c67": (F, []),
            "orc_quantize_if4": (I, [P, I, I64, I64, I64, P, P, P, P, I, I]),
            "orc_if6_cu": (F, []),
            "orc_if6_cd": (F, []),
            "orc_quantize_if6": (I, [P, I, I64, I64, I64, P, P, P, P, I, I]),
            "orc_fp3_value": (F, [ctypes.c_uint8]),
            "orc_fp3_rne": (ctypes.c_uint8, [F]),
            "orc_if3_cu": (F, []),
            "orc_if3_cd": (F, []),
            "orc_quantize_if3": (I, [P, I, I64, I64, I64, P, P, P, P, I, I]),
            "orc_quantize_four_over_six": (I, [P, I, I64, I64, I64, U, P, P, P, P, P, P, I]),
            "orc_dequantize": (I, [I, P, P, I, I, I, P, I64, I64, P, I]),
            "orc_glossary_mae": (ctypes.c_double, [P, I64, I64]),
            "orc_e2m1_rne_n": (None, [P, P, I64]),
            "orc_e2m1_sr_n": (None, [P, P, P, I64]),
            "orc_e4m3_rne_sat_n": (None, [P, P, I64]),
            "orc_e8m0_exponent_n": (None, [P, I, P, I64]),
            "orc_sr_bits16_n": (None, [U64, U64, P, I64]),
            "orc_f32_to_bf16_n": (None, [P, P, I64]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _libs[path] = L
        _lib = L
    return _lib


# ---------------------------------------------------------------------------
# numpy helpers
# ---------------------------------------------------------------------------

def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return BF16
    if x.dtype == np.float32:
        return FP32
    raise TypeError("oracle inputs are BF16 bit patterns (uint16) or float32")


def _f32(v) -> ctypes.c_float:
    return ctypes.c_float(float(v))


def scale_bytes(rows: int, cols: int, layout: int) -> int:
    return int(lib().orc_scale_bytes(rows, cols, layout))


def scale_offset(r: int, c: int, rows: int, cols: int, layout: int) -> int:
    return int(lib().orc_scale_offset(r, c, rows, cols, layout))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def e2m1_rne(v: float) -> int:
    return int(lib().orc_e2m1_rne(float(np.float32(v))))


def e2m1_rne_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.zeros(v.shape, np.uint8)
    lib().orc_e2m1_rne_n(_ptr(v), _ptr(out), v.size)
    return out


def e2m1_sr_array(v: np.ndarray, u16: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    u = np.ascontiguousarray(u16, dtype=np.uint32)
    assert u.shape == v.shape
    out = np.zeros(v.shape, np.uint8)
    lib().orc_e2m1_sr_n(_ptr(v), _ptr(u), _ptr(out), v.size)
    return out


def e4m3_rne_sat_array(s: np.ndarray) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float32)
    out = np.zeros(s.shape, np.uint8)
    lib().orc_e4m3_rne_sat_n(_ptr(s), _ptr(out), s.size)
    return out


def e8m0_exponent_array(m: np.ndarray, mode: int = E8M0_RNE) -> np.ndarray:
    m = np.ascontiguousarray(m, dtype=np.float32)
    out = np.zeros(m.shape, np.int32)
    lib().orc_e8m0_exponent_n(_ptr(m), mode, _ptr(out), m.size)
    return out


def sr_bits16_array(seed: int, first_index: int, n: int) -> np.ndarray:
    out = np.zeros(n, np.uint32)
    lib().orc_sr_bits16_n(seed, first_index, _ptr(out), n)
    return out


def f32_to_bf16_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.zeros(v.shape, np.uint16)
    lib().orc_f32_to_bf16_n(_ptr(v), _ptr(out), v.size)
    return out


def e2m1_sr(v: float, u16: int) -> int:
    return int(lib().orc_e2m1_sr(float(np.float32(v)), int(u16)))


def e2m1_value(code: int) -> float:
    return float(lib().orc_e2m1_value(int(code)))


def e4m3_rne_sat(s: float) -> int:
    return int(lib().orc_e4m3_rne_sat(float(np.float32(s))))


def e4m3_value(code: int) -> float:
    return float(lib().orc_e4m3_value(int(code)))


def e8m0_exponent(block_amax: float, mode: int = E8M0_RNE) -> int:
    return int(lib().orc_e8m0_exponent(float(np.float32(block_amax)), mode))


def philox4x32_10(counter, key) -> np.ndarray:
    c = np.asarray(counter, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def sr_bits16(seed: int, index: int) -> int:
    return int(lib().orc_sr_bits16(seed, index))


def rht_signs(seed: int, n: int) -> np.ndarray:
    out = np.zeros(n, dtype=np.float32)
    lib().orc_rht_signs(seed, n, _ptr(out))
    return out


def rht_norm(n: int) -> float:
    return float(lib().orc_rht_norm(n))


def amax(x: np.ndarray) -> float:
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    return float(lib().orc_amax(_ptr(x), _dtype_code(x), rows, cols, cols))


def tensor_scales(a: float):
    e, d = ctypes.c_float(), ctypes.c_float()
    lib().orc_tensor_scales(float(np.float32(a)), ctypes.byref(e), ctypes.byref(d))
    return e.value, d.value


def _amax_arg(a):
    if a is None:
        return None, None
    buf = np.array([a], dtype=np.float32)
    return buf, _ptr(buf)


def quantize_nvfp4(x: np.ndarray, layouts: int = ROWWISE, round: int = RNE, seed: int = 0,
                   amax: float | None = None, scale_layout: int = SCALE_LINEAR,
                   row0: int = 0) -> dict:
    """NVFP4 1x16.  row0 > 0: x is rows row0.. of a larger tensor with the same
    columns (give its amax); the stochastic-rounding bits then use the whole
    tensor's flat index."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = {"s_dec": np.zeros(1, np.float32)}
    if layouts & ROWWISE:
        out["q_row"] = np.zeros((rows, cols // 2), np.uint8)
        out["sf_row"] = np.zeros(scale_bytes(rows, cols // 16, scale_layout), np.uint8)
    if layouts & COLWISE:
        out["q_col"] = np.zeros((cols, rows // 2), np.uint8)
        out["sf_col"] = np.zeros(scale_bytes(cols, rows // 16, scale_layout), np.uint8)
    keep, ap = _amax_arg(amax)
    args = (_ptr(x), _dtype_code(x), rows, cols, cols, layouts, round, seed, ap,
            _ptr(out["s_dec"]), _ptr(out.get("q_row")), _ptr(out.get("sf_row")),
            _ptr(out.get("q_col")), _ptr(out.get("sf_col")), scale_layout)
    rc = (lib().orc_quantize_nvfp4_rows(*args, row0) if row0 else
          lib().orc_quantize_nvfp4(*args))
    if rc != 0:
        raise ValueError(f"oracle rejected shape {x.shape}")
    return out


def quantize_four_over_six(x: np.ndarray, layouts: int = ROWWISE, amax: float | None = None,
                           scale_layout: int = SCALE_LINEAR) -> dict:
    """NVFP4 1x16 layout with every block maximum mapped to 4 (the 4/6 method)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = {"s_dec": np.zeros(1, np.float32)}
    if layouts & ROWWISE:
        out["q_row"] = np.zeros((rows, cols // 2), np.uint8)
        out["sf_row"] = np.zeros(scale_bytes(rows, cols // 16, scale_layout), np.uint8)
    if layouts & COLWISE:
        out["q_col"] = np.zeros((cols, rows // 2), np.uint8)
        out["sf_col"] = np.zeros(scale_bytes(cols, rows // 16, scale_layout), np.uint8)
    keep, ap = _amax_arg(amax)
    rc = lib().orc_quantize_four_over_six(_ptr(x), _dtype_code(x), rows, cols, cols, layouts,
                                          ap, _ptr(out["s_dec"]), _ptr(out.get("q_row")),
                                          _ptr(out.get("sf_row")), _ptr(out.get("q_col")),
                                          _ptr(out.get("sf_col")), scale_layout)
    if rc != 0:
        raise ValueError(f"oracle rejected shape {x.shape}")
    return out


def quantize_backward(dy: np.ndarray, n: int, round: int = SR, seed_row: int = 0,
                      seed_col: int = 1, amax_row: float | None = None,
                      amax_rht: float | None = None, scale_layout: int = SCALE_LINEAR) -> dict:
    """Both backward operands of dY: the row-wise NVFP4 of dY (Dgrad operand,
    seed_row) and the RHT + column-wise NVFP4 of dY^T (Wgrad operand,
    seed_col) -- by definition the two oracle calls, composed."""
    r = quantize_nvfp4(dy, layouts=ROWWISE, round=round, seed=seed_row, amax=amax_row,
                       scale_layout=scale_layout)
    c = quantize_rht(dy, n, round=round, seed=seed_col, amax_rht=amax_rht,
                     scale_layout=scale_layout)
    return {"s_dec_row": r["s_dec"], "q_row": r["q_row"], "sf_row": r["sf_row"],
            "s_dec_col": c["s_dec"], "q_t": c["q_t"], "sf_t": c["sf_t"]}


def fp6_value(code: int, fmt: int) -> float:
    return float(lib().orc_fp6_value(code, fmt))


def fp6_rne(v: float, fmt: int) -> int:
    return int(lib().orc_fp6_rne(float(np.float32(v)), fmt))


def quantize_mxfp6(x: np.ndarray, fmt: int = FP6_E2M3, e8m0_mode: int = E8M0_RNE,
                   scale_layout: int = SCALE_LINEAR) -> dict:
    """MXFP6 row-wise 1x32 (E2M3 or E3M2 codes packed four per three bytes)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = {"q": np.zeros((rows, cols * 3 // 4), np.uint8),
           "sf": np.zeros(scale_bytes(rows, cols // 32, scale_layout), np.uint8)}
    rc = lib().orc_quantize_mxfp6(_ptr(x), _dtype_code(x), rows, cols, cols, fmt, e8m0_mode,
                                  _ptr(out["q"]), _ptr(out["sf"]), scale_layout)
    if rc != 0:
        raise ValueError(f"oracle rejected shape {x.shape}")
    return out


def quantize_mxfp4(x: np.ndarray, layouts: int = ROWWISE, e8m0_mode: int = E8M0_RNE,
                   scale_layout: int = SCALE_LINEAR) -> dict:
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = {}
    if layouts & ROWWISE:
        out["q_row"] = np.zeros((rows, cols // 2), np.uint8)
        out["sf_row"] = np.zeros(scale_bytes(rows, cols // 32, scale_layout), np.uint8)
    if layouts & COLWISE:
        out["q_col"] = np.zeros((cols, rows // 2), np.uint8)
        out["sf_col"] = np.zeros(scale_bytes(cols, rows // 32, scale_layout), np.uint8)
    rc = lib().orc_quantize_mxfp4(_ptr(x), _dtype_code(x), rows, cols, cols, layouts,
                                  e8m0_mode, _ptr(out.get("q_row")), _ptr(out.get("sf_row")),
                                  _ptr(out.get("q_col")), _ptr(out.get("sf_col")), scale_layout)
    if rc != 0:
        raise ValueError(f"oracle rejected shape {x.shape}")
    return out


def quantize_2d(w: np.ndarray, amax: float | None = None, with_1x16: bool = False,
                scale_layout: int = SCALE_LINEAR) -> dict:
    w = np.ascontiguousarray(w)
    rows, cols = w.shape
    out = {"s_dec": np.zeros(1, np.float32),
           "q_w": np.zeros((rows, cols // 2), np.uint8),
           "q_wt": np.zeros((cols, rows // 2), np.uint8),
           "sf_tiles": np.zeros((rows // 16, cols // 16), np.uint8)}
    if with_1x16:
        out["sf_w_1x16"] = np.zeros(scale_bytes(rows, cols // 16, scale_layout), np.uint8)
        out["sf_wt_1x16"] = np.zeros(scale_bytes(cols, rows // 16, scale_layout), np.uint8)
    keep, ap = _amax_arg(amax)
    rc = lib().orc_quantize_2d(_ptr(w), _dtype_code(w), rows, cols, cols, ap,
                               _ptr(out["s_dec"]), _ptr(out["q_w"]), _ptr(out["q_wt"]),
                               _ptr(out["sf_tiles"]), _ptr(out.get("sf_w_1x16")),
                               _ptr(out.get("sf_wt_1x16")), scale_layout)
    if rc != 0:
        raise ValueError(f"oracle rejected shape {w.shape}")
    return out


def rht(dy: np.ndarray, n: int, seed: int = 0) -> np.ndarray:
    dy = np.ascontiguousarray(dy)
    tokens, cols = dy.shape
    out = np.zeros((tokens, cols), np.float32)
    rc = lib().orc_rht(_ptr(dy), _dtype_code(dy), tokens, cols, cols, n, seed, _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected RHT arguments")
    return out


def quantize_rht(dy: np.ndarray, n: int, round: int = SR, seed: int = 0,
                 amax_rht: float | None = None, scale_layout: int = SCALE_LINEAR,
                 want_rht: bool = False, token0: int = 0) -> dict:
    """RHT + column-wise NVFP4.  token0 > 0: dy is tokens token0.. (a multiple of
    n) of a larger gradient with the same columns (give the transform's amax);
    the stochastic-rounding bits then use the whole tensor's flat index."""
    dy = np.ascontiguousarray(dy)
    tokens, cols = dy.shape
    out = {"s_dec": np.zeros(1, np.float32),
           "q_t": np.zeros((cols, tokens // 2), np.uint8),
           "sf_t": np.zeros(scale_bytes(cols, tokens // 16, scale_layout), np.uint8)}
    if want_rht:
        out["rht"] = np.zeros((tokens, cols), np.float32)
    keep, ap = _amax_arg(amax_rht)
    args = (_ptr(dy), _dtype_code(dy), tokens, cols, cols, n, round, seed, ap,
            _ptr(out["s_dec"]), _ptr(out["q_t"]), _ptr(out["sf_t"]), scale_layout,
            _ptr(out.get("rht")))
    rc = (lib().orc_quantize_rht_rows(*args, token0) if token0 else
          lib().orc_quantize_rht(*args))
    if rc != 0:
        raise ValueError("oracle rejected RHT arguments")
    return out


def if4_constants():
    return float(lib().orc_if4_c76()), float(lib().orc_if4_c67())


def quantize_if4(x: np.ndarray, amax: float | None = None, scale_layout: int = SCALE_LINEAR,
                 allow_int4: bool = True, int4_only: bool = False) -> dict:
    """IF4 (default); allow_int4=False: FP4 in every block (NVFP4);
    int4_only=True: INT4 in every block (NVINT4)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = {"s_dec": np.zeros(1, np.float32),
           "q": np.zeros((rows, cols // 2), np.uint8),
           "sf": np.zeros(scale_bytes(rows, cols // 16, scale_layout), np.uint8)}
    keep, ap = _amax_arg(amax)
    rc = lib().orc_quantize_if4(_ptr(x), _dtype_code(x), rows, cols, cols, ap,
                                _ptr(out["s_dec"]), _ptr(out["q"]), _ptr(out["sf"]),
                                scale_layout, 2 if int4_only else (1 if allow_int4 else 0))
    if rc != 0:
        raise ValueError(f"oracle rejected shape {x.shape}")
    return out


def if6_constants():
    return float(lib().orc_if6_cu()), float(lib().orc_if6_cd())


def quantize_if6(x: np.ndarray, amax: float | None = None, scale_layout: int = SCALE_LINEAR,
                 mode: int = 1) -> dict:
    """IF6 (mode 1): per 16-block FP6 E2M3 or INT6 (the 6/7 method with 31 and
    7.5); mode 0 keeps FP6 everywhere, mode 2 INT6 everywhere.  Codes
    [rows, cols * 3/4] (four 6-bit codes per three bytes)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = {"s_dec": np.zeros(1, np.float32),
           "q": np.zeros((rows, cols * 3 // 4), np.uint8),
           "sf": np.zeros(scale_bytes(rows, cols // 16, scale_layout), np.uint8)}
    keep, ap = _amax_arg(amax)
    rc = lib().orc_quantize_if6(_ptr(x), _dtype_code(x), rows, cols, cols, ap,
                                _ptr(out["s_dec"]), _ptr(out["q"]), _ptr(out["sf"]),
                                scale_layout, mode)
    if rc != 0:
        raise ValueError(f"oracle rejected shape {x.shape}")
    return out


def fp3_value(code: int) -> float:
    return float(lib().orc_fp3_value(code))


def fp3_rne(v: float) -> int:
    return int(lib().orc_fp3_rne(float(np.float32(v))))


def if3_constants():
    return float(lib().orc_if3_cu()), float(lib().orc_if3_cd())


def quantize_if3(x: np.ndarray, amax: float | None = None, scale_layout: int = SCALE_LINEAR,
                 mode: int = 1) -> dict:
    """IF3 (mode 1): per 16-block FP3 E2M0 or INT3 (the 6/7 method with 3 and
    4); mode 0 keeps FP3 everywhere, mode 2 INT3 everywhere.  Codes
    [rows, cols * 3/8] (eight 3-bit codes per three bytes)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = {"s_dec": np.zeros(1, np.float32),
           "q": np.zeros((rows, cols * 3 // 8), np.uint8),
           "sf": np.zeros(scale_bytes(rows, cols // 16, scale_layout), np.uint8)}
    keep, ap = _amax_arg(amax)
    rc = lib().orc_quantize_if3(_ptr(x), _dtype_code(x), rows, cols, cols, ap,
                                _ptr(out["s_dec"]), _ptr(out["q"]), _ptr(out["sf"]),
                                scale_layout, mode)
    if rc != 0:
        raise ValueError(f"oracle rejected shape {x.shape}")
    return out


def dequantize(fmt: int, q: np.ndarray, sf: np.ndarray, rows: int, cols: int,
               block_rows: int = 1, block_cols: int = 16, s_dec: float | None = None,
               scale_layout: int = SCALE_LINEAR, out_dtype: int = FP32) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    y = np.zeros((rows, cols), np.float32 if out_dtype == FP32 else np.uint16)
    keep, sp = _amax_arg(s_dec)
    rc = lib().orc_dequantize(fmt, _ptr(q), _ptr(sf), scale_layout, block_rows, block_cols, sp,
                              rows, cols, _ptr(y), out_dtype)
    if rc != 0:
        raise ValueError("oracle rejected dequant arguments")
    return y


def glossary_mae(x: np.ndarray, block: int) -> float:
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    return float(lib().orc_glossary_mae(_ptr(x), x.size, block))


def gemm_block_scaled(qa: np.ndarray, sfa: np.ndarray, qb: np.ndarray, sfb: np.ndarray,
                      M: int, N: int, K: int, alpha: float = 1.0, fmt: int = FMT_NVFP4,
                      scale_layout: int = SCALE_SWIZZLED) -> np.ndarray:
    """The product a block-scaled FP4 GEMM computes from quantized operands.

    Qiita note on NVFP4 training: the quantized operands feed FP4 GEMMs (Fprop
    X W^T; Wgrad dY^T X from the column-wise copies), each block's codes
    multiplied by its block scale, the two tensor scales applied to the result.
    Here: A = dequantize(qa, sfa) [M, K] and B = dequantize(qb, sfb) [N, K]
    with the block scales only (tensor scale 1, which makes every element the
    exact product g * S), then C = alpha * (A B^T), the contraction and the
    final product taken in float64 (a library matmul).  alpha carries the
    product of the two tensor scales.  fmt FMT_IF4 dequantizes A as IF4 (INT4
    blocks RN(RN(k * RN(6/7)) * S)); B is always NVFP4 then.  Returns float64
    [M, N].
    """
    blk = 32 if fmt == FMT_MXFP4 else 16       # NVFP4 and IF4 use 16-value blocks
    a = dequantize(fmt, qa, sfa, M, K, 1, blk, s_dec=1.0 if fmt != FMT_MXFP4 else None,
                   scale_layout=scale_layout)
    fb = FMT_NVFP4 if fmt == FMT_IF4 else fmt
    b = dequantize(fb, qb, sfb, N, K, 1, blk, s_dec=1.0 if fb != FMT_MXFP4 else None,
                   scale_layout=scale_layout)
    return (a.astype(np.float64) @ b.astype(np.float64).T) * float(alpha)
