"""CPU oracle for the blockwise-E4M3 FP8 linear layer (test infrastructure).

Only ``tests/``, the package smoke check and the benchmark's CPU-baseline
leg may import this module.  The product path never does: it shares no code
with the CUDA library and the library does not depend on it.

The arithmetic lives in ``fp8_oracle.c`` (plain C loops, FP64 accumulation,
OpenMP over output rows; also the SwiGLU product a fused quantize-on-output
producer has to reproduce); this module builds that file with gcc when the
shared object is missing and wraps it with numpy.  See the C file's header
for the definition it follows and the passages of the Puro-2B pages it rests
on.  All bf16 inputs are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

GROUP = 128


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile fp8_oracle.c into liboracle.so (gcc -O2, OpenMP, no fast-math).
    `src` / `out` name another copy of the source and its library (the test
    that plants mistakes in copies of the oracle builds them this way)."""
    if force or not os.path.exists(out) or (
        os.path.getmtime(out) < os.path.getmtime(src)
    ):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
             "-fno-fast-math", "-o", tmp, src, "-lm"]
        )
        os.replace(tmp, out)
    return out


def _configure(lib: ctypes.CDLL) -> ctypes.CDLL:
    p = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.orc_e4m3_decode.restype = ctypes.c_double
    lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
    lib.orc_e4m3_encode_array.restype = None
    lib.orc_e4m3_encode_array.argtypes = [p, i64, p]
    lib.orc_e4m3_decode_array.restype = None
    lib.orc_e4m3_decode_array.argtypes = [p, i64, p]
    lib.orc_bf16_to_float.restype = ctypes.c_float
    lib.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
    for name in ("orc_quant_act_rowwise", "orc_quant_act_colwise", "orc_quant_weight"):
        fn = getattr(lib, name)
        fn.restype = ctypes.c_int
        fn.argtypes = [p, i64, i64, p, p]
    for name in ("orc_gemm_fprop", "orc_gemm_dgrad", "orc_gemm_wgrad"):
        fn = getattr(lib, name)
        fn.restype = ctypes.c_int
        fn.argtypes = [p, p, p, p, i64, i64, i64, p, i64, p, p]
    lib.orc_gemm_wgrad_accum.restype = ctypes.c_int
    lib.orc_gemm_wgrad_accum.argtypes = [p, p, p, p, i64, i64, i64, p, i64, p, p, p]
    lib.orc_num_threads.restype = ctypes.c_int
    lib.orc_num_threads.argtypes = []
    lib.orc_bf16_from_double.restype = ctypes.c_uint16
    lib.orc_bf16_from_double.argtypes = [ctypes.c_double]
    lib.orc_silu_bf16.restype = ctypes.c_uint16
    lib.orc_silu_bf16.argtypes = [ctypes.c_uint16]
    lib.orc_swiglu_bf16.restype = ctypes.c_int
    lib.orc_swiglu_bf16.argtypes = [p, i64, i64, p]
    lib.orc_rmsnorm_rstd.restype = ctypes.c_int
    lib.orc_rmsnorm_rstd.argtypes = [p, i64, i64, ctypes.c_float, p]
    lib.orc_rmsnorm_apply.restype = ctypes.c_int
    lib.orc_rmsnorm_apply.argtypes = [p, i64, i64, p, p, p]
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _configure(ctypes.CDLL(_LIB_PATH))
    return _lib


@contextlib.contextmanager
def library(path: str):
    """Run every wrapper below on another build of the oracle's C source
    (a copy with a planted mistake), then restore the real one."""
    global _lib
    saved = _lib
    _lib = _configure(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = saved


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _check(rc: int, what: str):
    if rc == -2:
        raise ValueError(f"{what}: non-finite input (outside the definition)")
    if rc != 0:
        raise ValueError(f"{what}: bad arguments (rc={rc})")


def num_threads() -> int:
    return int(_load().orc_num_threads())


# ------------------------------------------------------------------ codec

def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3FN code, as float64 (NaN for 0x7F / 0xFF)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, np.float64)
    _load().orc_e4m3_decode_array(_ptr(codes), codes.size, _ptr(out))
    return out


def e4m3_encode(values) -> np.ndarray:
    """E4M3FN code of each float32 value: RNE, saturating at +-448, signed."""
    values = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(values.shape, np.uint8)
    _load().orc_e4m3_encode_array(_ptr(values), values.size, _ptr(out))
    return out


def bf16_to_float(bits) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------- quantizers

def quantize_act_rowwise(x_bits: np.ndarray):
    """1x128 groups along rows.  x_bits: uint16 [rows, cols].
    Returns (codes u8 [rows, cols], scales f32 [cols/128, rows])."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((cols // GROUP, rows), np.float32)
    _check(_load().orc_quant_act_rowwise(_ptr(x), rows, cols, _ptr(q), _ptr(s)),
           "quantize_act_rowwise")
    return q, s


def quantize_act_colwise(x_bits: np.ndarray):
    """Groups of 128 rows per column, transposed output.  x_bits: uint16
    [rows, cols].  Returns (codes u8 [cols, rows], scales f32 [rows/128, cols])."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    q = np.empty((cols, rows), np.uint8)
    s = np.empty((rows // GROUP, cols), np.float32)
    _check(_load().orc_quant_act_colwise(_ptr(x), rows, cols, _ptr(q), _ptr(s)),
           "quantize_act_colwise")
    return q, s


def quantize_weight(w_bits: np.ndarray):
    """128x128 blocks.  w_bits: uint16 [n, k].
    Returns (codes u8 [n, k], scales f32 [n/128, k/128])."""
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    q = np.empty((n, k), np.uint8)
    s = np.empty((n // GROUP, k // GROUP), np.float32)
    _check(_load().orc_quant_weight(_ptr(w), n, k, _ptr(q), _ptr(s)),
           "quantize_weight")
    return q, s


# ------------------------------------------------------------------ GEMMs

def _rows_arg(rows, total):
    if rows is None:
        return None, total
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if r.size and (r.min() < 0 or r.max() >= total):
        raise IndexError("row index out of range")
    return r, r.size


def gemm_fprop(xq, sx, wq, sw, rows=None):
    """Y = X W^T from codes and scales.  xq u8 [M, K], sx f32 [K/128, M],
    wq u8 [N, K], sw f32 [N/128, K/128].  Returns (y, bound) float64
    [len(rows) or M, N]."""
    xq = _c(xq, np.uint8); sx = _c(sx, np.float32)
    wq = _c(wq, np.uint8); sw = _c(sw, np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    assert wq.shape[1] == K and sx.shape == (K // GROUP, M) and sw.shape == (N // GROUP, K // GROUP)
    r, nr = _rows_arg(rows, M)
    y = np.empty((nr, N), np.float64)
    b = np.empty((nr, N), np.float64)
    _check(_load().orc_gemm_fprop(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K,
                                  None if r is None else _ptr(r), nr, _ptr(y), _ptr(b)),
           "gemm_fprop")
    return y, b


def gemm_dgrad(dyq, sdy, wq, sw, rows=None):
    """dX = dY W from codes and scales.  dyq u8 [M, N], sdy f32 [N/128, M],
    wq u8 [N, K] (the fprop codes), sw f32 [N/128, K/128].
    Returns (dx, bound) float64 [len(rows) or M, K]."""
    dyq = _c(dyq, np.uint8); sdy = _c(sdy, np.float32)
    wq = _c(wq, np.uint8); sw = _c(sw, np.float32)
    M, N = dyq.shape
    K = wq.shape[1]
    assert wq.shape[0] == N and sdy.shape == (N // GROUP, M) and sw.shape == (N // GROUP, K // GROUP)
    r, nr = _rows_arg(rows, M)
    y = np.empty((nr, K), np.float64)
    b = np.empty((nr, K), np.float64)
    _check(_load().orc_gemm_dgrad(_ptr(dyq), _ptr(sdy), _ptr(wq), _ptr(sw), M, N, K,
                                  None if r is None else _ptr(r), nr, _ptr(y), _ptr(b)),
           "gemm_dgrad")
    return y, b


def gemm_wgrad(dyqT, sdyT, xqT, sxT, rows=None):
    """dW = dY^T X from along-token codes.  dyqT u8 [N, M], sdyT f32
    [M/128, N], xqT u8 [K, M], sxT f32 [M/128, K].
    Returns (dw, bound) float64 [len(rows) or N, K]."""
    dyqT = _c(dyqT, np.uint8); sdyT = _c(sdyT, np.float32)
    xqT = _c(xqT, np.uint8); sxT = _c(sxT, np.float32)
    N, M = dyqT.shape
    K = xqT.shape[0]
    assert xqT.shape[1] == M and sdyT.shape == (M // GROUP, N) and sxT.shape == (M // GROUP, K)
    r, nr = _rows_arg(rows, N)
    y = np.empty((nr, K), np.float64)
    b = np.empty((nr, K), np.float64)
    _check(_load().orc_gemm_wgrad(_ptr(dyqT), _ptr(sdyT), _ptr(xqT), _ptr(sxT), N, K, M,
                                  None if r is None else _ptr(r), nr, _ptr(y), _ptr(b)),
           "gemm_wgrad")
    return y, b


def gemm_wgrad_accum(dyqT, sdyT, xqT, sxT, dw_in=None, rows=None):
    """Main-gradient accumulation: dw_in + dY^T X in FP64 on the selected
    output rows.  dw_in float64 [N, K] (the running main gradient; an FP32
    array converts exactly) or None for zeros.  Returns (dw, bound) float64
    [len(rows) or N, K]; bound is this call's wgrad bound."""
    dyqT = _c(dyqT, np.uint8); sdyT = _c(sdyT, np.float32)
    xqT = _c(xqT, np.uint8); sxT = _c(sxT, np.float32)
    N, M = dyqT.shape
    K = xqT.shape[0]
    assert xqT.shape[1] == M and sdyT.shape == (M // GROUP, N) and sxT.shape == (M // GROUP, K)
    if dw_in is not None:
        dw_in = _c(dw_in, np.float64)
        assert dw_in.shape == (N, K)
    r, nr = _rows_arg(rows, N)
    y = np.empty((nr, K), np.float64)
    b = np.empty((nr, K), np.float64)
    _check(_load().orc_gemm_wgrad_accum(_ptr(dyqT), _ptr(sdyT), _ptr(xqT), _ptr(sxT), N, K, M,
                                        None if r is None else _ptr(r), nr,
                                        None if dw_in is None else _ptr(dw_in), _ptr(y), _ptr(b)),
           "gemm_wgrad_accum")
    return y, b


# ----------------------------------------------------------------- SwiGLU

def bf16_from_double(v: float) -> int:
    """Bit pattern of the bfloat16 nearest to v (ties to even)."""
    return int(_load().orc_bf16_from_double(float(v)))


def silu_bf16(g_bits) -> np.ndarray:
    """silu of bfloat16 values (uint16 bit patterns), evaluated in double and
    rounded once to bfloat16."""
    g = np.ascontiguousarray(g_bits, dtype=np.uint16)
    fn = _load().orc_silu_bf16
    return np.array([fn(int(b)) for b in g.ravel()], dtype=np.uint16).reshape(g.shape)


def swiglu_bf16(gate_up_bits: np.ndarray) -> np.ndarray:
    """H = bf16(bf16(silu(gate)) * up) for a gate_up activation
    [rows, 2 * ffn] (gate first).  Returns uint16 bits [rows, ffn]."""
    x = _c(gate_up_bits, np.uint16)
    rows, cols = x.shape
    if cols % 2:
        raise ValueError("gate_up must have an even number of columns")
    h = np.empty((rows, cols // 2), np.uint16)
    _check(_load().orc_swiglu_bf16(_ptr(x), rows, cols // 2, _ptr(h)), "swiglu_bf16")
    return h


# ---------------------------------------------------------------- RMSNorm

def rmsnorm_rstd(x_bits: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """r = fp32(1 / sqrt(mean(x^2) + eps)) per row of a bfloat16 [rows, cols]
    (uint16 bits), the sum of squares in double."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    r = np.empty(rows, np.float32)
    _check(_load().orc_rmsnorm_rstd(_ptr(x), rows, cols, float(eps), _ptr(r)), "rmsnorm_rstd")
    return r


def rmsnorm_apply(x_bits: np.ndarray, r: np.ndarray, gamma_bits: np.ndarray) -> np.ndarray:
    """y = bf16(gamma * bf16(fp32(x * r))) for x [rows, cols] (bfloat16
    bits), r [rows] (float32) and gamma [cols] (bfloat16 bits).  Returns
    uint16 bits [rows, cols]."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    r = _c(r, np.float32)
    g = _c(gamma_bits, np.uint16)
    if r.shape != (rows,) or g.shape != (cols,):
        raise ValueError("r must be [rows] and gamma [cols]")
    y = np.empty((rows, cols), np.uint16)
    _check(_load().orc_rmsnorm_apply(_ptr(x), rows, cols, _ptr(r), _ptr(g), _ptr(y)), "rmsnorm_apply")
    return y
