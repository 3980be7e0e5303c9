"""The Python binding's marshalling (CPU): which pointers and sizes each
function hands to the C entry point, in the order include/fp8blk.h declares
them, and the device checks made before a launch.  The C library is replaced
by a recorder, so nothing is launched."""
import ctypes
from types import SimpleNamespace

import pytest
import torch

from blockwise_fp8_pretraining_b200 import _abi

STREAM = 0x5EED


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


def _value(arg):
    if isinstance(arg, ctypes.c_void_p):
        return arg.value or 0
    if isinstance(arg, ctypes.c_float):
        return arg.value
    return arg


def _want_cpu(t, dtype, shape, name):
    # the binding's checks minus the CUDA-residency one
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(name)
    return t


@pytest.fixture
def rec(monkeypatch):
    lib = _Recorder()
    checked = []
    monkeypatch.setattr(_abi, "load", lambda: lib)
    monkeypatch.setattr(_abi, "_want", _want_cpu)
    monkeypatch.setattr(_abi, "_stream", lambda s: ctypes.c_void_p(STREAM))
    monkeypatch.setattr(_abi, "_launch_checks", lambda named, stream: checked.append([n for n, _ in named]))
    lib.checked = checked
    return lib


def _args(rec):
    assert len(rec.calls) == 1
    name, args = rec.calls[0]
    return name, [_value(a) for a in args]


def p(t):
    return 0 if t is None else t.data_ptr()


@pytest.mark.parametrize("mode", [_abi.ROWWISE, _abi.COLWISE, _abi.BOTH])
def test_quantize_act_marshalling(rec, mode):
    x = torch.zeros((256, 384), dtype=torch.bfloat16)
    q_row, s_row, q_colT, s_col = _abi.fp8_quantize_act_1x128(x, mode)
    name, a = _args(rec)
    assert name == "fp8_quantize_act_1x128"
    assert a == [p(x), 256, 384, mode, p(q_row), p(s_row), p(q_colT), p(s_col), STREAM]
    if mode & _abi.ROWWISE:
        assert q_row.shape == (256, 384) and s_row.shape == (3, 256)
    else:
        assert q_row is None and s_row is None
    if mode & _abi.COLWISE:
        assert q_colT.shape == (384, 256) and s_col.shape == (2, 384)
    else:
        assert q_colT is None and s_col is None
    assert rec.checked == [["x", "q_row", "s_row", "q_colT", "s_col"]]


def test_quantize_act_uses_given_outputs(rec):
    x = torch.zeros((128, 256), dtype=torch.bfloat16)
    q = torch.empty((128, 256), dtype=torch.uint8)
    s = torch.empty((2, 128), dtype=torch.float32)
    out = _abi.fp8_quantize_act_1x128(x, _abi.ROWWISE, q_row=q, s_row=s)
    assert out[0] is q and out[1] is s
    with pytest.raises(ValueError):
        _abi.fp8_quantize_act_1x128(x, _abi.ROWWISE, q_row=torch.empty((128, 128), dtype=torch.uint8))


@pytest.mark.parametrize("transposed", [True, False])
def test_quantize_weight_marshalling(rec, transposed):
    w = torch.zeros((384, 256), dtype=torch.bfloat16)
    wq, sw, wqT = _abi.fp8_quantize_weight_128x128(w, transposed=transposed)
    name, a = _args(rec)
    assert name == "fp8_quantize_weight_128x128"
    assert a == [p(w), 384, 256, p(wq), p(sw), p(wqT), STREAM]
    assert wq.shape == (384, 256) and sw.shape == (3, 2)
    assert (wqT.shape == (256, 384)) if transposed else (wqT is None)


def test_fprop_marshalling(rec):
    M, N, K = 256, 384, 512
    xq = torch.zeros((M, K), dtype=torch.uint8)
    sx = torch.zeros((K // 128, M))
    wq = torch.zeros((N, K), dtype=torch.uint8)
    sw = torch.zeros((N // 128, K // 128))
    y = _abi.fp8_block_gemm_fprop(xq, sx, wq, sw)
    name, a = _args(rec)
    assert name == "fp8_block_gemm_fprop"
    assert a == [p(xq), p(sx), p(wq), p(sw), p(y), M, N, K, 0, 0, STREAM]
    assert y.shape == (M, N) and y.dtype == torch.bfloat16
    with pytest.raises(ValueError):        # scales in the other layout
        _abi.fp8_block_gemm_fprop(xq, sx.T.contiguous(), wq, sw)


def test_dgrad_marshalling(rec):
    M, N, K = 256, 384, 128                # dY [M, N], W [N, K]
    dyq = torch.zeros((M, N), dtype=torch.uint8)
    sdy = torch.zeros((N // 128, M))
    wqT = torch.zeros((K, N), dtype=torch.uint8)
    sw = torch.zeros((N // 128, K // 128))
    dx = _abi.fp8_block_gemm_dgrad(dyq, sdy, wqT, sw)
    name, a = _args(rec)
    assert name == "fp8_block_gemm_dgrad"
    assert a == [p(dyq), p(sdy), p(wqT), p(sw), p(dx), M, N, K, 0, 0, STREAM]
    assert dx.shape == (M, K)


def test_wgrad_marshalling(rec):
    N, K, M = 384, 128, 512                # dW [N, K] over M tokens
    dyqT = torch.zeros((N, M), dtype=torch.uint8)
    sdyT = torch.zeros((M // 128, N))
    xqT = torch.zeros((K, M), dtype=torch.uint8)
    sxT = torch.zeros((M // 128, K))
    dw = _abi.fp8_block_gemm_wgrad(dyqT, sdyT, xqT, sxT)
    name, a = _args(rec)
    assert name == "fp8_block_gemm_wgrad"
    assert a == [p(dyqT), p(sdyT), p(xqT), p(sxT), p(dw), N, K, M, 0, 0, STREAM]
    assert dw.shape == (N, K)


def test_cast_marshalling(rec):
    x = torch.zeros(1000)
    q = _abi.fp8_cast_e4m3_scaled(x, 0.5)
    name, a = _args(rec)
    assert name == "fp8_cast_e4m3_scaled"
    assert a == [p(x), 0.5, p(q), 1000, STREAM]


def test_nonzero_status_raises(monkeypatch):
    class Failing(_Recorder):
        def __getattr__(self, name):
            if name == "fp8_status_string":
                return lambda st: b"unsupported shape"
            return lambda *args: 2
    monkeypatch.setattr(_abi, "load", lambda: Failing())
    monkeypatch.setattr(_abi, "_want", _want_cpu)
    monkeypatch.setattr(_abi, "_stream", lambda s: ctypes.c_void_p(0))
    monkeypatch.setattr(_abi, "_launch_checks", lambda named, stream: None)
    z = torch.zeros((128, 128), dtype=torch.uint8)
    s = torch.zeros((1, 128))
    with pytest.raises(_abi.Fp8Error) as err:
        _abi.fp8_block_gemm_fprop(z, s, z, torch.zeros((1, 1)))
    assert err.value.status == 2 and "unsupported shape" in str(err.value)


def test_tensors_on_another_device_are_rejected():
    on = lambda i: SimpleNamespace(device=torch.device("cuda", i))   # noqa: E731
    _abi._check_devices([("a", on(1)), ("b", on(1)), ("c", None)], current=1)
    with pytest.raises(ValueError, match="b is on cuda:0"):
        _abi._check_devices([("a", on(1)), ("b", on(0))], current=1)
    with pytest.raises(ValueError, match="current CUDA device is cuda:0"):
        _abi._check_devices([("x", on(3))], current=0)


def test_gemm_workspace_marshalling(rec, monkeypatch):
    """An optional workspace tensor goes over as (pointer, bytes) right
    before the stream; a non-contiguous one is refused."""
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: True))
    N, K, M = 256, 128, 256
    dyqT = torch.zeros((N, M), dtype=torch.uint8)
    sdyT = torch.zeros((M // 128, N))
    xqT = torch.zeros((K, M), dtype=torch.uint8)
    sxT = torch.zeros((M // 128, K))
    dw = torch.zeros((N, K))
    ws = torch.zeros(4096, dtype=torch.uint8)
    _abi.fp8_block_gemm_wgrad_accum_f32(dyqT, sdyT, xqT, sxT, dw, workspace=ws)
    name, a = _args(rec)
    assert name == "fp8_block_gemm_wgrad_accum_f32"
    assert a == [p(dyqT), p(sdyT), p(xqT), p(sxT), p(dw), N, K, M, p(ws), 4096, STREAM]
    assert "workspace" in rec.checked[-1]
    with pytest.raises(ValueError):
        _abi.fp8_block_gemm_wgrad_accum_f32(dyqT, sdyT, xqT, sxT, dw,
                                            workspace=torch.zeros((64, 64), dtype=torch.uint8)[:, ::2])
