"""ctypes binding of the C ABI in include/fp8blk.h (argument marshalling only).

Every function here has the name of the C entry point it calls.  Tensors are
torch CUDA tensors; outputs the caller does not pass are allocated with torch
(device memory only: the library itself never allocates).  A non-zero status
raises Fp8Error.  The library must have been built (``python -m
blockwise_fp8_pretraining_b200.build``); there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

from . import build as _build

ROWWISE, COLWISE, BOTH = 1, 2, 3
MAX_CONTRACTION_FPROP = 32768
GEMM_SPLIT_MIN_WORK_DEFAULT = 160      # FP8_GEMM_SPLIT_MIN_WORK_DEFAULT

_lib = None


class Fp8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        msg = f"{where}: {status_string(status)} (status {status})"
        if status == 5:
            msg += f": {fp8_last_cuda_error()}"
        super().__init__(msg)


def lib_path() -> str:
    return _build.LIB


def header_functions() -> list[str]:
    """Names of the functions include/fp8blk.h declares."""
    with open(_build.HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fp8_\w+)\s*\(", text, flags=re.M)


def load() -> ctypes.CDLL:
    """Load libfp8blk.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise OSError(f"{path} is missing: build it with python -m blockwise_fp8_pretraining_b200.build")
    lib = ctypes.CDLL(path)
    p, i64, i32, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int
    sz = ctypes.c_size_t
    sig = {
        "fp8_quantize_act_1x128": [p, i64, i64, i32, p, p, p, p, p],
        "fp8_quantize_weight_128x128": [p, i64, i64, p, p, p, p],
        "fp8_swiglu_quantize_1x128": [p, i64, i64, i32, p, p, p, p, p],
        "fp8_rmsnorm_rstd": [p, i64, i64, ctypes.c_float, p, p],
        "fp8_rmsnorm_quantize_1x128": [p, i64, i64, p, p, i32, p, p, p, p, p],
        "fp8_selftest_silu_bf16": [p, p],
        "fp8_block_gemm_fprop": [p, p, p, p, p, i64, i64, i64, p, sz, p],
        "fp8_block_gemm_dgrad": [p, p, p, p, p, i64, i64, i64, p, sz, p],
        "fp8_block_gemm_wgrad": [p, p, p, p, p, i64, i64, i64, p, sz, p],
        "fp8_block_gemm_wgrad_accum_f32": [p, p, p, p, p, i64, i64, i64, p, sz, p],
        "fp8_block_gemm_wgrad_reduce_scatter_f32": [p, p, p, p, p, i32, i64, i64, i64, p, sz, p],
        "fp8_gemm_workspace_bytes": [p],
        "fp8_block_gemm_wgrad_static_ws": [p, p, p, p, p, i64, i64, i64, p],
        "fp8_get_error": [],
        "fp8_clear_error": [],
        "fp8_set_wait_timeout_ns": [ctypes.c_uint64],
        "fp8_set_gemm_split_min_work": [ctypes.c_int64],
        "fp8_cast_e4m3_scaled": [p, ctypes.c_float, p, i64, p],
        "fp8_selftest_wait_timeout": [p],
        "fp8_selftest_stall_next": [i32],
        "fp8_selftest_gemm_schedule": [i64, i64, i64, i32, i32, p, i64, p],
        "fp8_selftest_division": [p, p],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = st
    lib.fp8_status_string.argtypes = [st]
    lib.fp8_status_string.restype = ctypes.c_char_p
    lib.fp8_last_cuda_error.argtypes = []
    lib.fp8_last_cuda_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load().fp8_status_string(int(status)).decode()
    except OSError:
        return "library not loaded"


def _check(status: int, where: str):
    if status != 0:
        raise Fp8Error(status, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check_devices(named, current: int, stream=None) -> None:
    """The library launches on the current CUDA device, so every tensor (and
    an explicit torch stream) must live there; a pointer into another GPU's
    memory would be dereferenced by the wrong device."""
    for name, t in named:
        if t is not None and t.device.index != current:
            raise ValueError(f"{name} is on {t.device} but the current CUDA device is cuda:{current}; "
                             f"call inside torch.cuda.device({t.device.index})")
    if isinstance(stream, torch.cuda.Stream) and stream.device.index != current:
        raise ValueError(f"stream is on {stream.device} but the current CUDA device is cuda:{current}")


def _launch_checks(named, stream) -> None:
    _check_devices(named, torch.cuda.current_device(), stream)


def _record(stream, allocated) -> None:
    """Outputs allocated here belong to the current stream's pool; when the
    kernel runs on another torch stream, tie their lifetime to that stream
    too so their memory is not reused while the kernel still writes it.
    (With a raw stream handle that is the caller's job.)"""
    if isinstance(stream, torch.cuda.Stream):
        for t in allocated:
            if t is not None:
                t.record_stream(stream)


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _want(t: torch.Tensor, dtype, shape, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _out(t, dtype, shape, device, name):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    return _want(t, dtype, shape, name)


# ------------------------------------------------------------------ kernels

def fp8_quantize_act_1x128(x, mode=BOTH, q_row=None, s_row=None, q_colT=None, s_col=None,
                           stream=None):
    """Quantize a bf16 activation [rows, cols].  Returns (q_row, s_row,
    q_colT, s_col); entries of a grouping the mode leaves out are None."""
    lib = load()
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    rows, cols = x.shape
    _want(x, torch.bfloat16, (rows, cols), "x")
    dev = x.device
    given_q_row, given_s_row = q_row is not None, s_row is not None
    given_q_colT, given_s_col = q_colT is not None, s_col is not None
    if mode & ROWWISE:
        q_row = _out(q_row, torch.uint8, (rows, cols), dev, "q_row")
        s_row = _out(s_row, torch.float32, (cols // 128, rows), dev, "s_row")
    else:
        q_row = s_row = None
    if mode & COLWISE:
        q_colT = _out(q_colT, torch.uint8, (cols, rows), dev, "q_colT")
        s_col = _out(s_col, torch.float32, (rows // 128, cols), dev, "s_col")
    else:
        q_colT = s_col = None
    _launch_checks([("x", x), ("q_row", q_row), ("s_row", s_row), ("q_colT", q_colT), ("s_col", s_col)],
                   stream)
    _record(stream, [t for t, given in ((q_row, given_q_row), (s_row, given_s_row),
                                         (q_colT, given_q_colT), (s_col, given_s_col)) if not given])
    _check(lib.fp8_quantize_act_1x128(_ptr(x), rows, cols, int(mode), _ptr(q_row), _ptr(s_row),
                                      _ptr(q_colT), _ptr(s_col), _stream(stream)),
           "fp8_quantize_act_1x128")
    return q_row, s_row, q_colT, s_col


def fp8_swiglu_quantize_1x128(gate_up, mode=BOTH, q_row=None, s_row=None, q_colT=None, s_col=None,
                              stream=None):
    """Quantize H = silu(gate) * up (bf16 roundings as the unfused path) of
    a bf16 gate_up activation [rows, 2 * ffn] without forming H in memory.
    Returns (q_row, s_row, q_colT, s_col) of H [rows, ffn]; entries of a
    grouping the mode leaves out are None."""
    lib = load()
    if gate_up.dtype != torch.bfloat16 or gate_up.dim() != 2 or gate_up.shape[1] % 2:
        raise TypeError("gate_up must be a 2-D bfloat16 tensor with an even number of columns")
    rows, cols2 = gate_up.shape
    ffn = cols2 // 2
    _want(gate_up, torch.bfloat16, (rows, cols2), "gate_up")
    dev = gate_up.device
    given = [t is not None for t in (q_row, s_row, q_colT, s_col)]
    if mode & ROWWISE:
        q_row = _out(q_row, torch.uint8, (rows, ffn), dev, "q_row")
        s_row = _out(s_row, torch.float32, (ffn // 128, rows), dev, "s_row")
    else:
        q_row = s_row = None
    if mode & COLWISE:
        q_colT = _out(q_colT, torch.uint8, (ffn, rows), dev, "q_colT")
        s_col = _out(s_col, torch.float32, (rows // 128, ffn), dev, "s_col")
    else:
        q_colT = s_col = None
    outs = (q_row, s_row, q_colT, s_col)
    _launch_checks([("gate_up", gate_up), ("q_row", q_row), ("s_row", s_row), ("q_colT", q_colT),
                    ("s_col", s_col)], stream)
    _record(stream, [t for t, g in zip(outs, given) if not g])
    _check(lib.fp8_swiglu_quantize_1x128(_ptr(gate_up), rows, ffn, int(mode), _ptr(q_row), _ptr(s_row),
                                         _ptr(q_colT), _ptr(s_col), _stream(stream)),
           "fp8_swiglu_quantize_1x128")
    return outs


def fp8_rmsnorm_rstd(x, eps=1e-6, rstd=None, stream=None):
    """RMSNorm's rstd[i] = 1 / sqrt(mean(x[i]^2) + eps) (float32 [rows]) of a
    bf16 x [rows, cols]."""
    lib = load()
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    rows, cols = x.shape
    _want(x, torch.bfloat16, (rows, cols), "x")
    given = rstd is not None
    rstd = _out(rstd, torch.float32, (rows,), x.device, "rstd")
    _launch_checks([("x", x), ("rstd", rstd)], stream)
    if not given:
        _record(stream, [rstd])
    _check(lib.fp8_rmsnorm_rstd(_ptr(x), rows, cols, float(eps), _ptr(rstd), _stream(stream)), "fp8_rmsnorm_rstd")
    return rstd


def fp8_rmsnorm_quantize_1x128(x, rstd, gamma, mode=BOTH, q_row=None, s_row=None, q_colT=None, s_col=None,
                               stream=None):
    """Quantize y = bf16(gamma * bf16(x * rstd)) (RMSNorm's output; rstd
    float32 [rows], gamma bf16 [cols]) of a bf16 x [rows, cols] without
    forming y in memory.  Returns (q_row, s_row, q_colT, s_col) of y;
    entries of a grouping the mode leaves out are None."""
    lib = load()
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    rows, cols = x.shape
    _want(x, torch.bfloat16, (rows, cols), "x")
    _want(rstd, torch.float32, (rows,), "rstd")
    _want(gamma, torch.bfloat16, (cols,), "gamma")
    dev = x.device
    given = [t is not None for t in (q_row, s_row, q_colT, s_col)]
    if mode & ROWWISE:
        q_row = _out(q_row, torch.uint8, (rows, cols), dev, "q_row")
        s_row = _out(s_row, torch.float32, (cols // 128, rows), dev, "s_row")
    else:
        q_row = s_row = None
    if mode & COLWISE:
        q_colT = _out(q_colT, torch.uint8, (cols, rows), dev, "q_colT")
        s_col = _out(s_col, torch.float32, (rows // 128, cols), dev, "s_col")
    else:
        q_colT = s_col = None
    outs = (q_row, s_row, q_colT, s_col)
    _launch_checks([("x", x), ("rstd", rstd), ("gamma", gamma), ("q_row", q_row), ("s_row", s_row),
                    ("q_colT", q_colT), ("s_col", s_col)], stream)
    _record(stream, [t for t, g in zip(outs, given) if not g])
    _check(lib.fp8_rmsnorm_quantize_1x128(_ptr(x), rows, cols, _ptr(rstd), _ptr(gamma), int(mode), _ptr(q_row),
                                          _ptr(s_row), _ptr(q_colT), _ptr(s_col), _stream(stream)),
           "fp8_rmsnorm_quantize_1x128")
    return outs


def fp8_quantize_weight_128x128(w, wq=None, sw=None, wqT=None, transposed=True, stream=None):
    """Quantize a bf16 weight [n, k] in 128x128 blocks.  Returns (wq, sw, wqT);
    wqT is None when transposed is False and no buffer is passed."""
    lib = load()
    if w.dtype != torch.bfloat16 or w.dim() != 2:
        raise TypeError("w must be a 2-D bfloat16 tensor")
    n, k = w.shape
    _want(w, torch.bfloat16, (n, k), "w")
    allocated = [t is None for t in (wq, sw, wqT)]
    wq = _out(wq, torch.uint8, (n, k), w.device, "wq")
    sw = _out(sw, torch.float32, (n // 128, k // 128), w.device, "sw")
    if wqT is not None or transposed:
        wqT = _out(wqT, torch.uint8, (k, n), w.device, "wqT")
    _launch_checks([("w", w), ("wq", wq), ("sw", sw), ("wqT", wqT)], stream)
    _record(stream, [t for t, a in zip((wq, sw, wqT), allocated) if a])
    _check(lib.fp8_quantize_weight_128x128(_ptr(w), n, k, _ptr(wq), _ptr(sw), _ptr(wqT),
                                           _stream(stream)),
           "fp8_quantize_weight_128x128")
    return wq, sw, wqT


def _workspace(ws):
    """(pointer, bytes) of an optional GEMM workspace tensor (see
    fp8_gemm_workspace_bytes): contiguous, on the current device, zeroed
    before its first use."""
    if ws is None:
        return ctypes.c_void_p(0), 0
    if not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()


def fp8_gemm_workspace_bytes() -> int:
    """Bytes of the GEMM workspace on the current device."""
    n = ctypes.c_size_t(0)
    _check(load().fp8_gemm_workspace_bytes(ctypes.byref(n)), "fp8_gemm_workspace_bytes")
    return int(n.value)


def fp8_gemm_workspace(device=None) -> torch.Tensor:
    """A zeroed GEMM workspace for the current (or given) device, allocated
    by torch.  One launch at a time may use it."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return torch.zeros(fp8_gemm_workspace_bytes(), dtype=torch.uint8, device=dev)


def fp8_block_gemm_fprop(xq, sx, wq, sw, y=None, stream=None, workspace=None):
    """Y[M, N] = X W^T (bf16) from X codes [M, K] / scales [K/128, M] and W
    codes [N, K] / scales [N/128, K/128].  workspace: optional (see
    fp8_gemm_workspace)."""
    lib = load()
    M, K = xq.shape
    N = wq.shape[0]
    _want(xq, torch.uint8, (M, K), "xq")
    _want(sx, torch.float32, (K // 128, M), "sx")
    _want(wq, torch.uint8, (N, K), "wq")
    _want(sw, torch.float32, (N // 128, K // 128), "sw")
    allocated = y is None
    y = _out(y, torch.bfloat16, (M, N), xq.device, "y")
    _launch_checks([("xq", xq), ("sx", sx), ("wq", wq), ("sw", sw), ("y", y), ("workspace", workspace)],
                   stream)
    _record(stream, [y] if allocated else [])
    _check(lib.fp8_block_gemm_fprop(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(y), M, N, K,
                                    *_workspace(workspace), _stream(stream)),
           "fp8_block_gemm_fprop")
    return y


def fp8_block_gemm_dgrad(dyq, sdy, wqT, sw, dx=None, stream=None, workspace=None):
    """dX[M, K] = dY W (bf16) from dY codes [M, N] / scales [N/128, M], the
    transposed weight codes [K, N] and the weight scales [N/128, K/128]."""
    lib = load()
    M, N = dyq.shape
    K = wqT.shape[0]
    _want(dyq, torch.uint8, (M, N), "dyq")
    _want(sdy, torch.float32, (N // 128, M), "sdy")
    _want(wqT, torch.uint8, (K, N), "wqT")
    _want(sw, torch.float32, (N // 128, K // 128), "sw")
    allocated = dx is None
    dx = _out(dx, torch.bfloat16, (M, K), dyq.device, "dx")
    _launch_checks([("dyq", dyq), ("sdy", sdy), ("wqT", wqT), ("sw", sw), ("dx", dx),
                    ("workspace", workspace)], stream)
    _record(stream, [dx] if allocated else [])
    _check(lib.fp8_block_gemm_dgrad(_ptr(dyq), _ptr(sdy), _ptr(wqT), _ptr(sw), _ptr(dx), M, N, K,
                                    *_workspace(workspace), _stream(stream)),
           "fp8_block_gemm_dgrad")
    return dx


def fp8_block_gemm_wgrad(dyqT, sdyT, xqT, sxT, dw=None, stream=None, workspace=None):
    """dW[N, K] = dY^T X (bf16) from along-token codes: dY^T [N, M] / scales
    [M/128, N] and X^T [K, M] / scales [M/128, K]."""
    lib = load()
    N, M = dyqT.shape
    K = xqT.shape[0]
    _want(dyqT, torch.uint8, (N, M), "dyqT")
    _want(sdyT, torch.float32, (M // 128, N), "sdyT")
    _want(xqT, torch.uint8, (K, M), "xqT")
    _want(sxT, torch.float32, (M // 128, K), "sxT")
    allocated = dw is None
    dw = _out(dw, torch.bfloat16, (N, K), dyqT.device, "dw")
    _launch_checks([("dyqT", dyqT), ("sdyT", sdyT), ("xqT", xqT), ("sxT", sxT), ("dw", dw),
                    ("workspace", workspace)], stream)
    _record(stream, [dw] if allocated else [])
    _check(lib.fp8_block_gemm_wgrad(_ptr(dyqT), _ptr(sdyT), _ptr(xqT), _ptr(sxT), _ptr(dw), N, K, M,
                                    *_workspace(workspace), _stream(stream)),
           "fp8_block_gemm_wgrad")
    return dw


def fp8_block_gemm_wgrad_accum_f32(dyqT, sdyT, xqT, sxT, dw, stream=None, workspace=None):
    """dW[N, K] += dY^T X in FP32, in place, from the same along-token codes
    as fp8_block_gemm_wgrad; dw is a float32 [N, K] tensor (the main
    gradient).  Returns dw."""
    lib = load()
    N, M = dyqT.shape
    K = xqT.shape[0]
    _want(dyqT, torch.uint8, (N, M), "dyqT")
    _want(sdyT, torch.float32, (M // 128, N), "sdyT")
    _want(xqT, torch.uint8, (K, M), "xqT")
    _want(sxT, torch.float32, (M // 128, K), "sxT")
    _want(dw, torch.float32, (N, K), "dw")
    _launch_checks([("dyqT", dyqT), ("sdyT", sdyT), ("xqT", xqT), ("sxT", sxT), ("dw", dw),
                    ("workspace", workspace)], stream)
    _check(lib.fp8_block_gemm_wgrad_accum_f32(_ptr(dyqT), _ptr(sdyT), _ptr(xqT), _ptr(sxT), _ptr(dw),
                                              N, K, M, *_workspace(workspace), _stream(stream)),
           "fp8_block_gemm_wgrad_accum_f32")
    return dw


MAX_SHARDS = 8


def fp8_block_gemm_wgrad_reduce_scatter_f32(dyqT, sdyT, xqT, sxT, shards, stream=None, workspace=None):
    """dW = dY^T X of this rank's tokens, added in FP32 into the owners'
    shards: rows [q N / R, (q + 1) N / R) of dW into shards[q], a float32
    [N / R, K] tensor of rank q (this GPU's, or a peer's mapped into this
    process, see exchange_shards).  After every rank's call and a
    synchronization each shard holds its old contents plus the sum over
    ranks.  Returns shards."""
    lib = load()
    N, M = dyqT.shape
    K = xqT.shape[0]
    R = len(shards)
    if not 1 <= R <= MAX_SHARDS or N % R:
        raise ValueError(f"need 1..{MAX_SHARDS} shards dividing N = {N}, got {R}")
    _want(dyqT, torch.uint8, (N, M), "dyqT")
    _want(sdyT, torch.float32, (M // 128, N), "sdyT")
    _want(xqT, torch.uint8, (K, M), "xqT")
    _want(sxT, torch.float32, (M // 128, K), "sxT")
    for q, t in enumerate(shards):            # peers' shards may live on other devices
        _want(t, torch.float32, (N // R, K), f"shards[{q}]")
    _launch_checks([("dyqT", dyqT), ("sdyT", sdyT), ("xqT", xqT), ("sxT", sxT), ("workspace", workspace)], stream)
    table = (ctypes.c_void_p * R)(*[t.data_ptr() for t in shards])
    _check(lib.fp8_block_gemm_wgrad_reduce_scatter_f32(_ptr(dyqT), _ptr(sdyT), _ptr(xqT), _ptr(sxT),
                                                       ctypes.cast(table, ctypes.c_void_p), R, N, K, M,
                                                       *_workspace(workspace), _stream(stream)),
           "fp8_block_gemm_wgrad_reduce_scatter_f32")
    return shards


def exchange_shards(local, group=None, share=None, rebuild=None):
    """The shards of a data-parallel group as seen from this rank: every
    rank passes its own main-gradient shard; returns the list in rank order,
    this rank's own tensor at its place and the others mapped into this
    process through CUDA IPC (torch's tensor sharing).  share(t) turns a
    tensor into a picklable handle and rebuild(handle) maps one back; they
    default to torch.multiprocessing's CUDA reductions."""
    import torch.distributed as dist

    if share is None or rebuild is None:
        from torch.multiprocessing.reductions import reduce_tensor

        share = share or (lambda t: reduce_tensor(t))
        rebuild = rebuild or (lambda h: h[0](*h[1]))
    world = dist.get_world_size(group)
    me = dist.get_rank(group)
    handles = [None] * world
    dist.all_gather_object(handles, share(local), group=group)
    return [local if q == me else rebuild(handles[q]) for q in range(world)]


def fp8_block_gemm_wgrad_static_ws(dyqT, sdyT, xqT, sxT, dw=None, stream=None):
    """dW = dY^T X (bf16) like fp8_block_gemm_wgrad, with the split
    schedule's workspace inside the library (no device buffer passed), for
    callers that cannot allocate one; calls must not overlap on the GPU."""
    lib = load()
    N, M = dyqT.shape
    K = xqT.shape[0]
    _want(dyqT, torch.uint8, (N, M), "dyqT")
    _want(sdyT, torch.float32, (M // 128, N), "sdyT")
    _want(xqT, torch.uint8, (K, M), "xqT")
    _want(sxT, torch.float32, (M // 128, K), "sxT")
    allocated = dw is None
    dw = _out(dw, torch.bfloat16, (N, K), dyqT.device, "dw")
    _launch_checks([("dyqT", dyqT), ("sdyT", sdyT), ("xqT", xqT), ("sxT", sxT), ("dw", dw)], stream)
    _record(stream, [dw] if allocated else [])
    _check(lib.fp8_block_gemm_wgrad_static_ws(_ptr(dyqT), _ptr(sdyT), _ptr(xqT), _ptr(sxT), _ptr(dw), N, K, M,
                                              _stream(stream)),
           "fp8_block_gemm_wgrad_static_ws")
    return dw


def fp8_get_error() -> int:
    return int(load().fp8_get_error())


def fp8_clear_error() -> None:
    _check(load().fp8_clear_error(), "fp8_clear_error")


def fp8_set_wait_timeout_ns(ns: int) -> None:
    _check(load().fp8_set_wait_timeout_ns(int(ns)), "fp8_set_wait_timeout_ns")


def fp8_set_gemm_split_min_work(units_per_pair: int) -> None:
    _check(load().fp8_set_gemm_split_min_work(int(units_per_pair)), "fp8_set_gemm_split_min_work")


def fp8_status_string(status: int) -> str:
    return status_string(status)


def fp8_last_cuda_error() -> str:
    try:
        return load().fp8_last_cuda_error().decode()
    except OSError:
        return ""


def fp8_cast_e4m3_scaled(x, scale: float, q=None, stream=None):
    lib = load()
    n = x.numel()
    _want(x, torch.float32, tuple(x.shape), "x")
    allocated = q is None
    q = _out(q, torch.uint8, tuple(x.shape), x.device, "q")
    _launch_checks([("x", x), ("q", q)], stream)
    _record(stream, [q] if allocated else [])
    _check(lib.fp8_cast_e4m3_scaled(_ptr(x), ctypes.c_float(scale), _ptr(q), n, _stream(stream)),
           "fp8_cast_e4m3_scaled")
    return q


def fp8_selftest_division(stream=None):
    """Returns (code mismatches, first code mismatch, quotient-bit
    mismatches with |x/s| >= 2^-12, first such, quotient-bit mismatches
    below 2^-12)."""
    res = torch.zeros(6, dtype=torch.int64, device="cuda")
    _check(load().fp8_selftest_division(_ptr(res), _stream(stream)), "fp8_selftest_division")
    torch.cuda.synchronize()
    return tuple(res.cpu().tolist()[:5])


def fp8_selftest_wait_timeout(stream=None) -> None:
    _check(load().fp8_selftest_wait_timeout(_stream(stream)), "fp8_selftest_wait_timeout")


def fp8_selftest_stall_next(which: int) -> None:
    """Arm the next GEMM (1), tile quantizer (2) or both (3) launches to run
    into their bounded wait (test support)."""
    _check(load().fp8_selftest_stall_next(int(which)), "fp8_selftest_stall_next")


def fp8_selftest_silu_bf16(stream=None):
    """silu of every bfloat16 bit pattern as the fused SwiGLU producer
    computes it: a numpy uint16 array of 65536 bit patterns (index = input
    bits)."""
    out = torch.empty(65536, dtype=torch.int16, device="cuda")
    _check(load().fp8_selftest_silu_bf16(_ptr(out), _stream(stream)), "fp8_selftest_silu_bf16")
    torch.cuda.synchronize()
    return out.cpu().numpy().view("uint16")


def fp8_selftest_gemm_schedule(M: int, N: int, K: int, pairs: int, split: bool):
    """The GEMMs' work schedule as the library computes it (host code shared
    with the kernel): a list of (pair, tile, kb0, kb1, add_first, add_end)."""
    import numpy as np

    cap = 1 << 16
    rows = np.zeros((cap, 5), dtype=np.int32)
    n = ctypes.c_int64(0)
    _check(load().fp8_selftest_gemm_schedule(int(M), int(N), int(K), int(pairs), int(bool(split)),
                                            ctypes.c_void_p(rows.ctypes.data), cap, ctypes.byref(n)),
           "fp8_selftest_gemm_schedule")
    out = []
    for r in rows[: n.value]:
        out.append((int(r[0]), int(r[1]), int(r[2]), int(r[3]), int(r[4]) >> 16, int(r[4]) & 0xFFFF))
    return out
