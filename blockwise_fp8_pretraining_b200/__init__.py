"""Blockwise-E4M3 FP8 Transformer linear layer for NVIDIA B200 (sm_100a).

The compute path is the CUDA library libfp8blk.so (C ABI in
include/fp8blk.h); this package is its Python binding.  The functions carry
the C entry points' names; see ``_abi`` for their arguments.  Nothing here
falls back to a CPU or library implementation: calling a function without
the built library raises.
"""
from ._abi import (  # noqa: F401
    BOTH,
    COLWISE,
    GEMM_SPLIT_MIN_WORK_DEFAULT,
    MAX_CONTRACTION_FPROP,
    ROWWISE,
    Fp8Error,
    fp8_block_gemm_dgrad,
    fp8_block_gemm_fprop,
    fp8_block_gemm_wgrad,
    fp8_block_gemm_wgrad_accum_f32,
    fp8_block_gemm_wgrad_reduce_scatter_f32,
    fp8_block_gemm_wgrad_static_ws,
    fp8_cast_e4m3_scaled,
    fp8_clear_error,
    fp8_gemm_workspace,
    fp8_gemm_workspace_bytes,
    fp8_get_error,
    fp8_last_cuda_error,
    fp8_quantize_act_1x128,
    fp8_quantize_weight_128x128,
    fp8_rmsnorm_quantize_1x128,
    fp8_rmsnorm_rstd,
    fp8_selftest_division,
    fp8_selftest_gemm_schedule,
    fp8_selftest_silu_bf16,
    fp8_selftest_stall_next,
    fp8_selftest_wait_timeout,
    fp8_set_gemm_split_min_work,
    fp8_set_wait_timeout_ns,
    fp8_status_string,
    fp8_swiglu_quantize_1x128,
    exchange_shards,
    header_functions,
    lib_path,
    load,
)
