"""C-ABI checks that need no GPU: the library loads, exports every function
the header declares, and rejects bad arguments on the host before touching
the device (so the fake pointers below are never dereferenced)."""
import ctypes

import pytest

import blockwise_fp8_pretraining_b200 as fp8
from blockwise_fp8_pretraining_b200 import _abi

OK, NULL, SHAPE, ALIGN, MODE = 0, 1, 2, 3, 4


@pytest.fixture(scope="module")
def lib():
    from blockwise_fp8_pretraining_b200 import build

    build.build()
    return fp8.load()


def test_header_declares_the_expected_entry_points():
    names = set(fp8.header_functions())
    for want in ("fp8_quantize_act_1x128", "fp8_quantize_weight_128x128", "fp8_block_gemm_fprop",
                 "fp8_block_gemm_dgrad", "fp8_block_gemm_wgrad", "fp8_get_error",
                 "fp8_status_string"):
        assert want in names


def test_library_exports_every_header_function(lib):
    for name in fp8.header_functions():
        assert hasattr(lib, name), name


def test_python_binding_has_every_header_function():
    for name in fp8.header_functions():
        assert hasattr(fp8, name), name


def test_status_strings(lib):
    for st in range(7):
        assert lib.fp8_status_string(st)
    assert fp8.fp8_status_string(99) == "unknown status"


A16 = 0x10000          # fake, 16-byte aligned, never dereferenced
MIS = 0x10008          # fake, misaligned
S = ctypes.c_void_p(0)


def P(v):
    return ctypes.c_void_p(v)


def test_quantize_act_rejections(lib):
    q = lib.fp8_quantize_act_1x128
    assert q(P(A16), 256, 2048, 0, P(A16), P(A16), P(A16), P(A16), S) == MODE
    assert q(P(A16), 256, 2048, 5, P(A16), P(A16), P(A16), P(A16), S) == MODE
    assert q(P(A16), 256, 100, 1, P(A16), P(A16), None, None, S) == SHAPE
    assert q(P(A16), -1, 128, 1, P(A16), P(A16), None, None, S) == SHAPE
    assert q(P(A16), 100, 128, 2, None, None, P(A16), P(A16), S) == SHAPE   # colwise needs rows%128
    assert q(None, 256, 128, 1, P(A16), P(A16), None, None, S) == NULL
    assert q(P(A16), 256, 128, 1, None, P(A16), None, None, S) == NULL
    assert q(P(A16), 256, 128, 3, P(A16), P(A16), None, P(A16), S) == NULL
    assert q(P(MIS), 256, 128, 1, P(A16), P(A16), None, None, S) == ALIGN
    assert q(P(A16), 256, 128, 2, None, None, P(A16), P(MIS), S) == ALIGN
    # empty inputs are a no-op that launches nothing
    assert q(P(A16), 0, 128, 3, P(A16), P(A16), P(A16), P(A16), S) == OK
    assert q(P(A16), 5, 0, 1, P(A16), P(A16), None, None, S) == OK


def test_quantize_weight_rejections(lib):
    q = lib.fp8_quantize_weight_128x128
    assert q(P(A16), 100, 128, P(A16), P(A16), None, S) == SHAPE
    assert q(P(A16), 128, 129, P(A16), P(A16), None, S) == SHAPE
    assert q(P(A16), 128, 128, None, P(A16), None, S) == NULL
    assert q(P(A16), 128, 128, P(A16), P(A16), P(MIS), S) == ALIGN
    assert q(P(A16), 0, 128, P(A16), P(A16), None, S) == OK


@pytest.mark.parametrize("name", ["fp8_block_gemm_fprop", "fp8_block_gemm_dgrad"])
def test_fprop_dgrad_rejections(lib, name):
    g = getattr(lib, name)
    a = [P(A16)] * 5
    W = (None, 0)                                    # no workspace
    assert g(*a, 100, 256, 256, *W, S) == SHAPE      # M not a multiple of 128
    assert g(*a, 128, 0, 256, *W, S) == SHAPE
    assert g(*a, 128, 256, 0, *W, S) == SHAPE
    assert g(*a, 128, 200, 256, *W, S) == SHAPE
    big = fp8.MAX_CONTRACTION_FPROP + 128
    if name == "fp8_block_gemm_fprop":
        assert g(*a, 128, 256, big, *W, S) == SHAPE
    else:
        assert g(*a, 128, big, 256, *W, S) == SHAPE
    assert g(None, *a[1:], 128, 256, 256, *W, S) == NULL
    assert g(*a[:4], None, 128, 256, 256, *W, S) == NULL
    assert g(*a[:2], P(MIS), *a[3:], 128, 256, 256, *W, S) == ALIGN
    assert g(*a, 128, 256, 256, P(MIS), 1 << 30, S) == ALIGN     # misaligned workspace
    assert g(*a, 0, 256, 256, *W, S) == OK           # M == 0: nothing to do


def test_wgrad_rejections(lib):
    g = lib.fp8_block_gemm_wgrad
    a = [P(A16)] * 5
    W = (None, 0)
    assert g(*a, 256, 256, 0, *W, S) == SHAPE        # no tokens
    assert g(*a, 256, 256, 100, *W, S) == SHAPE
    assert g(*a, 200, 256, 256, *W, S) == SHAPE
    assert g(*a[:3], None, a[4], 256, 256, 256, *W, S) == NULL
    assert g(*a[:4], P(MIS), 256, 256, 256, *W, S) == ALIGN
    assert g(*a, 256, 256, 256, P(MIS), 1 << 30, S) == ALIGN


def test_workspace_size_query_rejects_null(lib):
    assert lib.fp8_gemm_workspace_bytes(None) == NULL


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(_abi._build, "LIB", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(OSError):
        _abi.load()


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "fp8blk.h"

#define EXPECT(call, want) do { fp8_status st_ = (call); \
    if (st_ != (want)) { printf("FAIL %s -> %d\n", #call, (int)st_); return 1; } } while (0)

int main(void) {
    void *a16 = (void *)(uintptr_t)0x10000;      /* never dereferenced */
    unsigned char *u = (unsigned char *)a16;
    float *f = (float *)a16;
    EXPECT(fp8_quantize_act_1x128(a16, 256, 2048, 0, u, f, u, f, NULL), FP8_ERR_MODE);
    EXPECT(fp8_quantize_act_1x128(a16, 100, 256, FP8_COLWISE, NULL, NULL, u, f, NULL), FP8_ERR_SHAPE);
    EXPECT(fp8_quantize_act_1x128(NULL, 0, 256, FP8_BOTH, NULL, NULL, NULL, NULL, NULL), FP8_OK);
    EXPECT(fp8_quantize_weight_128x128(a16, 128, 200, u, f, NULL, NULL), FP8_ERR_SHAPE);
    EXPECT(fp8_block_gemm_fprop(u, f, u, f, a16, 128, 128, FP8_MAX_CONTRACTION_FPROP + 128, NULL, 0,
                                NULL), FP8_ERR_SHAPE);
    EXPECT(fp8_block_gemm_dgrad(u, f, NULL, f, a16, 128, 128, 128, NULL, 0, NULL), FP8_ERR_NULL);
    EXPECT(fp8_block_gemm_wgrad(u, f, u, f, a16, 128, 128, 0, NULL, 0, NULL), FP8_ERR_SHAPE);
    EXPECT(fp8_gemm_workspace_bytes(NULL), FP8_ERR_NULL);
    EXPECT(fp8_set_wait_timeout_ns(0), FP8_OK);
    if (strcmp(fp8_status_string(FP8_ERR_ALIGN), "pointer not 16-byte aligned") != 0) return 1;
    if (fp8_last_cuda_error()[0] != '\0') return 1;
    puts("ok");
    return 0;
}
"""


def test_plain_c_client_compiles_links_and_gets_host_statuses(lib, tmp_path):
    """The header is plain C99 and a C program links the library directly."""
    import os
    import subprocess

    from blockwise_fp8_pretraining_b200 import build

    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(build.LIB)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.dirname(build.HEADER), str(src), "-o", str(exe),
                    "-L", libdir, "-lfp8blk", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"


def test_stall_switch_rejects_unknown_kernel_families(lib):
    for bad in (0, 4, -1):
        assert lib.fp8_selftest_stall_next(bad) == MODE


def test_wgrad_accum_rejections(lib):
    g = lib.fp8_block_gemm_wgrad_accum_f32
    a4 = [P(A16)] * 4
    W = (None, 0)
    assert g(*a4, P(A16), 128, 128, 0, *W, S) == SHAPE      # no tokens
    assert g(*a4, P(A16), 128, 100, 128, *W, S) == SHAPE
    assert g(*a4, None, 128, 128, 128, *W, S) == NULL
    assert g(*a4, P(MIS), 128, 128, 128, *W, S) == ALIGN
    assert g(*a4, P(A16), 128, 128, 128, P(MIS), 1 << 30, S) == ALIGN


def test_swiglu_quantize_rejections(lib):
    q = lib.fp8_swiglu_quantize_1x128
    assert q(P(A16), 256, 128, 0, P(A16), P(A16), None, None, S) == MODE
    assert q(P(A16), 100, 128, 1, P(A16), P(A16), None, None, S) == SHAPE      # rows % 128
    assert q(P(A16), 256, 100, 1, P(A16), P(A16), None, None, S) == SHAPE
    assert q(None, 256, 128, 1, P(A16), P(A16), None, None, S) == NULL
    assert q(P(A16), 256, 128, 2, None, None, P(A16), None, S) == NULL
    assert q(P(MIS), 256, 128, 1, P(A16), P(A16), None, None, S) == ALIGN
    assert q(P(A16), 0, 128, 3, None, None, None, None, S) == OK
    assert lib.fp8_selftest_silu_bf16(None, S) == NULL


def test_split_threshold_setter(lib):
    assert lib.fp8_set_gemm_split_min_work(-1) == SHAPE
    assert lib.fp8_set_gemm_split_min_work(0) == OK
    assert lib.fp8_set_gemm_split_min_work(fp8.GEMM_SPLIT_MIN_WORK_DEFAULT) == OK


def test_binding_constants_match_the_header():
    import re

    from blockwise_fp8_pretraining_b200 import build

    text = open(build.HEADER).read()
    defines = dict(re.findall(r"#define\s+(FP8_\w+)\s+(\d+)", text))
    assert int(defines["FP8_MAX_CONTRACTION_FPROP"]) == fp8.MAX_CONTRACTION_FPROP
    assert int(defines["FP8_GEMM_SPLIT_MIN_WORK_DEFAULT"]) == fp8.GEMM_SPLIT_MIN_WORK_DEFAULT


def test_rmsnorm_rejections(lib):
    r = lib.fp8_rmsnorm_rstd
    assert r(P(A16), 256, 100, 1e-6, P(A16), S) == SHAPE                   # cols % 8
    assert r(P(A16), 256, 128, -1.0, P(A16), S) == SHAPE                   # eps < 0
    assert r(None, 256, 128, 1e-6, P(A16), S) == NULL
    assert r(P(MIS), 256, 128, 1e-6, P(A16), S) == ALIGN
    assert r(P(A16), 0, 128, 1e-6, None, S) == OK
    q = lib.fp8_rmsnorm_quantize_1x128
    a = [P(A16)] * 3
    assert q(P(A16), 256, 128, P(A16), P(A16), 0, *a[:2], None, None, S) == MODE
    assert q(P(A16), 100, 128, P(A16), P(A16), 1, *a[:2], None, None, S) == SHAPE
    assert q(P(A16), 256, 100, P(A16), P(A16), 1, *a[:2], None, None, S) == SHAPE
    assert q(P(A16), 256, 128, None, P(A16), 1, *a[:2], None, None, S) == NULL
    assert q(P(A16), 256, 128, P(A16), None, 1, *a[:2], None, None, S) == NULL
    assert q(P(A16), 256, 128, P(A16), P(A16), 2, None, None, P(A16), None, S) == NULL
    assert q(P(A16), 256, 128, P(A16), P(MIS), 1, *a[:2], None, None, S) == ALIGN
    assert q(P(A16), 0, 128, None, None, 3, None, None, None, None, S) == OK


def test_wgrad_reduce_scatter_rejections(lib):
    g = lib.fp8_block_gemm_wgrad_reduce_scatter_f32
    a4 = [P(A16)] * 4
    W = (None, 0)
    table = (ctypes.c_void_p * 8)(*([A16] * 8))
    T = ctypes.cast(table, ctypes.c_void_p)
    assert g(*a4, T, 0, 256, 128, 128, *W, S) == SHAPE        # no ranks
    assert g(*a4, T, 9, 256, 128, 128, *W, S) == SHAPE        # more than 8
    assert g(*a4, T, 3, 256, 128, 128, *W, S) == SHAPE        # 3 does not divide 256
    assert g(*a4, T, 2, 256, 128, 0, *W, S) == SHAPE          # no tokens
    assert g(*a4, None, 2, 256, 128, 128, *W, S) == NULL
    bad = (ctypes.c_void_p * 2)(A16, MIS)
    assert g(*a4, ctypes.cast(bad, ctypes.c_void_p), 2, 256, 128, 128, *W, S) == ALIGN
    null = (ctypes.c_void_p * 2)(A16, 0)
    assert g(*a4, ctypes.cast(null, ctypes.c_void_p), 2, 256, 128, 128, *W, S) == NULL
