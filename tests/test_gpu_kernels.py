"""GPU parity of every kernel against the CPU oracle at sizes the oracle
finishes in seconds: several tiles, ragged tails (row counts that are not a
multiple of a block's rows, N against 192-wide GEMM pair tiles, grids
with fewer tiles than SMs and with a partial last wave), heavy tails, zero
groups, and the degenerate cases of the method."""
import numpy as np
import pytest
import torch

import blockwise_fp8_pretraining_b200 as fp8
import oracle
from blockwise_fp8_pretraining_b200 import synthetic as syn

from _parity import (assert_bits_equal, assert_within_bound, check_act, check_dgrad, check_fprop,
                     check_wgrad, check_weight, dev, pick_rows, workspace)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fp8.load()
    fp8.fp8_clear_error()
    # The shapes here are small: let the split schedule apply to them too
    # whenever a workspace is given (its least-work threshold would keep
    # most of them whole).
    fp8.fp8_set_gemm_split_min_work(0)
    yield
    fp8.fp8_set_gemm_split_min_work(fp8.GEMM_SPLIT_MIN_WORK_DEFAULT)
    assert fp8.fp8_get_error() == 0


# ------------------------------------------------------------- element cast

def test_cast_matches_oracle_on_grid_midpoints_and_saturation():
    pos = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mid = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    vals = np.concatenate([
        pos.astype(np.float32), mid, np.nextafter(mid, np.float32(0)),
        np.nextafter(mid, np.float32(np.inf)),
        np.array([448, 463.99, 464, 470, 480, 1e4, 1e30, 3e38, 0.0, 1e-30, 1e-45], np.float32),
    ])
    vals = np.concatenate([vals, -vals]).astype(np.float32)
    for scale in (1.0, 0.5, 2.0 ** -20, 3.0, 1e-3, 7.0 / 448.0):
        q = fp8.fp8_cast_e4m3_scaled(torch.from_numpy(vals).to(dev()), scale)
        ref = oracle.e4m3_encode((vals / np.float32(scale)).astype(np.float32))
        assert_bits_equal(q, ref, f"cast scale={scale}")
    q0 = fp8.fp8_cast_e4m3_scaled(torch.from_numpy(vals).to(dev()), 0.0)
    assert torch.all(q0 == 0)


def test_cast_random_fp32_sweep():
    rng = np.random.default_rng(5)
    v = (np.exp(rng.uniform(np.log(1e-12), np.log(1e6), 2_000_000))
         * np.where(rng.random(2_000_000) < 0.5, -1, 1)).astype(np.float32)
    for scale in (1.0, 0.013, 1e-7):
        q = fp8.fp8_cast_e4m3_scaled(torch.from_numpy(v).to(dev()), scale)
        assert_bits_equal(q, oracle.e4m3_encode((v / np.float32(scale)).astype(np.float32)),
                          f"random cast {scale}")


def test_group_division_matches_ieee_division_exhaustively():
    """The quantizers divide by a group's scale with one reciprocal and two
    FMAs per element; every (bf16 amax, bf16 x) pair must give the same E4M3
    code, and the same float32 quotient, as IEEE division."""
    bad_code, first, bad_bits, first_bits, bad_tiny = fp8.fp8_selftest_division()
    print(f"division self-test: code mismatches {bad_code}, quotient mismatches >= 2^-12: "
          f"{bad_bits} (first 0x{first_bits:08x}), below 2^-12: {bad_tiny}")
    assert bad_code == 0, f"first mismatch amax=0x{first >> 16:04x} x=0x{first & 0xffff:04x}"
    assert bad_bits == 0, f"first quotient mismatch amax=0x{first_bits >> 16:04x} x=0x{first_bits & 0xffff:04x}"


# ------------------------------------------------------------- quantizers

@pytest.mark.parametrize("rows,cols", [(1, 128), (3, 384), (127, 256), (129, 2048), (1000, 640),
                                       (256, 2048)])
def test_rowwise_ragged_rows(rows, cols):
    x = syn.activation_bf16(rows, cols, max(1, cols // 100), 30.0, syn.generator(rows + cols))
    check_act(x, fp8.ROWWISE)


@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (384, 2048), (1024, 640)])
@pytest.mark.parametrize("mode", [fp8.COLWISE, fp8.BOTH])
def test_colwise_and_dual(rows, cols, mode):
    x = syn.activation_bf16(rows, cols, max(1, cols // 100), 30.0, syn.generator(rows * 3 + cols))
    check_act(x, mode)


def test_quantizers_heavy_tail_zero_and_negative_zero_groups():
    x = syn.student_t_bf16((512, 1024), seed=11).float()
    x[5, :] = 0.0                     # all-zero row groups
    x[6, :] = -0.0                    # groups of negative zeros
    x[:, 128:256] = 0.0               # all-zero column block
    x[7, 300] = 3.0e38                # near the top of the bf16 range
    x[8, 0:128] = 1e-40               # bf16 subnormals, scale becomes subnormal
    x[9, 0] = -1e-40
    x = x.to(torch.bfloat16)
    check_act(x, fp8.BOTH)
    check_act(x, fp8.ROWWISE)
    check_act(x, fp8.COLWISE)


@pytest.mark.parametrize("n,k", [(128, 128), (384, 256), (2048, 2048), (256, 6144)])
def test_weight_blocks(n, k):
    w = syn.normal_bf16((n, k), 0.02, syn.generator(n + k))
    check_weight(w)


def test_weight_without_transposed_copy_and_special_blocks():
    w = syn.normal_bf16((256, 384), 0.02, syn.generator(3)).float()
    w[:128, :128] = 0.0
    w[128:, 256:] = -0.0
    w = w.to(torch.bfloat16)
    wq, sw, wqT = fp8.fp8_quantize_weight_128x128(w.to(dev()), transposed=False)
    assert wqT is None
    q_o, s_o = oracle.quantize_weight(syn.bf16_bits(w))
    assert_bits_equal(wq, q_o, "codes")
    assert_bits_equal(sw, s_o, "scales")


# ------------------------------------------------------------------ GEMMs

GEMM_SHAPES = [
    (128, 128, 128),      # one tile, one slab
    (128, 384, 256),      # ragged N: one full and one half-width tile
    (256, 640, 512),
    (384, 256, 1152),     # odd number of slabs
    (1280, 2304, 384),    # 90 tiles: fewer tiles than SMs
    (4096, 2560, 256),    # 320 tiles: partial last wave
]


# With a workspace, shapes whose last wave of 256 x 256 tiles would leave
# pairs idle run the split schedule (slab ranges per pair, partial sums
# added by the pair holding each tile's first slab); without one, whole
# tiles.  Both must meet the bound.
SPLIT = [False, True]


@pytest.mark.parametrize("split", SPLIT)
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_fprop_small(M, N, K, split):
    g = syn.generator(M + N + K)
    x = syn.activation_bf16(M, K, max(1, K // 100), 30.0, g)
    w = syn.normal_bf16((N, K), 0.02, g)
    rows = None if M <= 384 else pick_rows(M, 96, M)
    check_fprop(x, w, rows, output_rounding=True, ws=workspace() if split else None)


@pytest.mark.parametrize("split", SPLIT)
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_dgrad_small(M, N, K, split):
    # dX [M, K] = dY [M, N] W [N, K]
    g = syn.generator(M * 7 + N + K)
    dy = syn.normal_bf16((M, N), 1e-3, g)
    w = syn.normal_bf16((N, K), 0.02, g)
    rows = None if M <= 384 else pick_rows(M, 96, M)
    check_dgrad(dy, w, rows, output_rounding=True, ws=workspace() if split else None)


@pytest.mark.parametrize("split", SPLIT)
@pytest.mark.parametrize("N,K,M", [(128, 128, 128), (384, 256, 256), (256, 640, 384),
                                   (1280, 2304, 256), (2560, 4096, 128), (2048, 2048, 1152)])
def test_wgrad_small(N, K, M, split):
    g = syn.generator(N * 5 + K + M)
    dy = syn.normal_bf16((M, N), 1e-3, g)
    x = syn.activation_bf16(M, K, max(1, K // 100), 30.0, g)
    rows = None if N <= 384 else pick_rows(N, 96, N)
    check_wgrad(dy, x, rows, output_rounding=True, ws=workspace() if split else None)


# Contractions of 32 slabs, where the split schedule applies: fewer tiles
# than CTA pairs (every tile cut across pairs) and a partly idle last wave.
SPLIT_SHAPES = [(256, 640, 4096), (1280, 2304, 4096), (4096, 2560, 4096)]


@pytest.mark.parametrize("split", SPLIT)
@pytest.mark.parametrize("M,N,K", SPLIT_SHAPES)
def test_split_schedule_fprop_dgrad(M, N, K, split):
    g = syn.generator(3 * M + N + K)
    ws = workspace() if split else None
    rows = None if M <= 256 else pick_rows(M, 96, M + 1)
    check_fprop(syn.activation_bf16(M, K, K // 100, 30.0, g), syn.normal_bf16((N, K), 0.02, g), rows,
                output_rounding=True, ws=ws)
    # dX [M, N] = dY [M, K] W [K, N]: a K-deep contraction onto N columns
    check_dgrad(syn.normal_bf16((M, K), 1e-3, g), syn.normal_bf16((K, N), 0.02, g), rows,
                output_rounding=True, ws=ws)


@pytest.mark.parametrize("split", SPLIT)
@pytest.mark.parametrize("N,K,M", [(1280, 2304, 4096), (2560, 4096, 4096), (256, 256, 8192)])
def test_split_schedule_wgrad(N, K, M, split):
    g = syn.generator(N + 5 * K + M)
    dy = syn.normal_bf16((M, N), 1e-3, g)
    x = syn.activation_bf16(M, K, max(1, K // 100), 30.0, g)
    rows = None if N <= 256 else pick_rows(N, 96, N + 2)
    check_wgrad(dy, x, rows, output_rounding=True, ws=workspace() if split else None)


@pytest.mark.parametrize("split", SPLIT)
def test_longest_contraction(split):
    """The longest contraction the fprop/dgrad entry points accept (256 slabs
    of 128), and a wgrad over as many tokens: every output element.  With the
    split schedule each of these single-tile GEMMs is cut into one slab range
    per CTA pair, and one pair adds all the others' partial sums."""
    K = fp8.MAX_CONTRACTION_FPROP
    g = syn.generator(31)
    ws = workspace() if split else None
    check_fprop(syn.activation_bf16(256, K, K // 100, 30.0, g), syn.normal_bf16((256, K), 0.02, g), ws=ws)
    # dX [128, 256] = dY [128, K] W [K, 256]: the contraction runs over K
    check_dgrad(syn.normal_bf16((128, K), 1e-3, g), syn.normal_bf16((K, 256), 0.02, g), ws=ws)
    # dW [256, 128] over K tokens
    check_wgrad(syn.normal_bf16((K, 256), 1e-3, g), syn.activation_bf16(K, 128, 1, 30.0, g), ws=ws)


def test_tiny_config_fprop_dgrad_wgrad_full():
    """X [256, 2048] (4 channels x50), W [2048, 2048], dY [256, 2048]: every
    output element of the three GEMMs against the oracle."""
    c = syn.tiny(seed=0)
    check_act(c["x"], fp8.BOTH)
    check_act(c["dy"], fp8.BOTH)
    check_weight(c["w"])
    check_fprop(c["x"], c["w"])
    check_dgrad(c["dy"], c["w"])
    check_wgrad(c["dy"], c["x"])


def test_gemm_degenerate_inputs():
    """All-zero operands give exact zeros; all-ones give the closed form."""
    d = dev()
    z = torch.zeros((256, 512), dtype=torch.bfloat16)
    w = syn.normal_bf16((384, 512), 0.02, syn.generator(9))
    y = check_fprop(z, w)
    assert torch.all(y == 0)
    ones = torch.ones((128, 128), dtype=torch.bfloat16)
    y = check_fprop(ones, ones, output_rounding=True)
    s = float(np.float32(1.0) / np.float32(448.0))
    want = torch.tensor(128 * (448 * s) ** 2, dtype=torch.float32).to(torch.bfloat16)
    assert torch.all(y.cpu() == want)


def test_empty_inputs_are_noops():
    d = dev()
    xq = torch.empty((0, 256), dtype=torch.uint8, device=d)
    sx = torch.empty((2, 0), dtype=torch.float32, device=d)
    wq = torch.zeros((128, 256), dtype=torch.uint8, device=d)
    sw = torch.zeros((1, 2), dtype=torch.float32, device=d)
    y = fp8.fp8_block_gemm_fprop(xq, sx, wq, sw)
    assert y.shape == (0, 128)
    wqT = torch.zeros((256, 128), dtype=torch.uint8, device=d)
    dx = fp8.fp8_block_gemm_dgrad(torch.empty((0, 128), dtype=torch.uint8, device=d),
                                  torch.empty((1, 0), dtype=torch.float32, device=d), wqT,
                                  torch.zeros((1, 2), dtype=torch.float32, device=d))
    assert dx.shape == (0, 256)
    q_row, s_row, q_colT, s_col = fp8.fp8_quantize_act_1x128(
        torch.empty((0, 256), dtype=torch.bfloat16, device=d), fp8.BOTH)
    assert q_row.shape == (0, 256) and s_col.shape == (0, 256)
    wq0, sw0, wqT0 = fp8.fp8_quantize_weight_128x128(torch.empty((0, 128), dtype=torch.bfloat16, device=d))
    assert wq0.shape == (0, 128) and wqT0.shape == (128, 0)
    torch.cuda.synchronize()


def test_outputs_do_not_depend_on_stream_or_repeat():
    """Same inputs on another stream and a second run give identical bits
    (each output element is produced by one thread in a fixed order, and
    split tiles add their partial sums in a fixed order)."""
    c = syn.tiny(seed=3)
    d = dev()
    x, w = c["x"].to(d), c["w"].to(d)
    xq, sx, _, _ = fp8.fp8_quantize_act_1x128(x, fp8.ROWWISE)
    wq, sw, _ = fp8.fp8_quantize_weight_128x128(w, transposed=False)
    y1 = fp8.fp8_block_gemm_fprop(xq, sx, wq, sw)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y2 = fp8.fp8_block_gemm_fprop(xq, sx, wq, sw)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    # the split schedule: repeated runs, and a second workspace on another stream
    ws2 = fp8.fp8_gemm_workspace()
    y3 = fp8.fp8_block_gemm_fprop(xq, sx, wq, sw, workspace=workspace())
    y4 = fp8.fp8_block_gemm_fprop(xq, sx, wq, sw, workspace=workspace())
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        y5 = fp8.fp8_block_gemm_fprop(xq, sx, wq, sw, workspace=ws2)
    s.synchronize()
    assert torch.equal(y3, y4) and torch.equal(y3, y5)
    # every flag is back to zero (the partial sums before them may remain):
    # the workspace holds, per CTA pair, 262144 bytes of partial sums, then
    # after all of those 2048 bytes of flags per pair
    for w in (workspace(), ws2):
        pairs = w.numel() // (262144 + 2048)
        flags = w[pairs * 262144: pairs * (262144 + 2048)]
        assert int(flags.count_nonzero()) == 0


# --------------------------------------------------------------- time-outs

def test_bounded_wait_times_out_and_reports():
    fp8.fp8_clear_error()
    fp8.fp8_set_wait_timeout_ns(2_000_000)          # 2 ms
    try:
        fp8.fp8_selftest_wait_timeout()
        assert fp8.fp8_get_error() == 6              # FP8_ERR_TIMEOUT
    finally:
        fp8.fp8_set_wait_timeout_ns(0)
        fp8.fp8_clear_error()
    # the context is still usable afterwards
    check_fprop(syn.normal_bf16((128, 128), 1.0, syn.generator(1)),
                syn.normal_bf16((128, 128), 0.02, syn.generator(2)))


# ------------------------------------------------------------ guard bands

GUARD_ROWS = 3


def _guarded(rows, cols, dtype, fill_bits):
    """A [rows, cols] view in the middle of a buffer whose GUARD_ROWS rows
    before and after are filled with a sentinel bit pattern."""
    itemsize = torch.empty((), dtype=dtype).element_size()
    int_t = {2: torch.int16, 4: torch.int32}[itemsize]
    buf = torch.full((rows + 2 * GUARD_ROWS, cols), fill_bits, dtype=int_t, device=dev()).view(dtype)
    return buf, buf[GUARD_ROWS:GUARD_ROWS + rows]


def _assert_guards(buf, rows, fill_bits, what):
    int_t = {2: torch.int16, 4: torch.int32}[buf.element_size()]
    raw = buf.view(int_t)
    for part, name in ((raw[:GUARD_ROWS], "before"), (raw[GUARD_ROWS + rows:], "after")):
        bad = int((part != fill_bits).sum())
        assert bad == 0, f"{what}: {bad} guard elements {name} the output were written"


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (384, 640, 256), (128, 256, 384), (640, 2560, 128)])
def test_gemm_writes_stay_inside_the_output(M, N, K):
    """Ragged tiles (N against 192-wide pair tiles, M = 128 against 256-row
    pair tiles): outputs are views inside sentinel-filled buffers, and every
    sentinel must survive fprop, dgrad and wgrad."""
    d = dev()
    g = syn.generator(M + 3 * N + 7 * K)
    x = syn.activation_bf16(M, K, max(1, K // 100), 30.0, g)
    w = syn.normal_bf16((N, K), 0.02, g)
    dy = syn.normal_bf16((M, N), 1e-3, g)
    sentinel = 0x7FA5          # a bfloat16 NaN pattern the kernels never produce
    xq, sx, _, _ = fp8.fp8_quantize_act_1x128(x.to(d), fp8.ROWWISE)
    wq, sw, wqT = fp8.fp8_quantize_weight_128x128(w.to(d))
    buf, y = _guarded(M, N, torch.bfloat16, sentinel)
    fp8.fp8_block_gemm_fprop(xq, sx, wq, sw, y=y, workspace=workspace())
    dyq, sdy, dyqT, sdyT = fp8.fp8_quantize_act_1x128(dy.to(d), fp8.BOTH)
    dbuf, dx = _guarded(M, K, torch.bfloat16, sentinel)
    fp8.fp8_block_gemm_dgrad(dyq, sdy, wqT, sw, dx=dx, workspace=workspace())
    _, _, xqT, sxT = fp8.fp8_quantize_act_1x128(x.to(d), fp8.COLWISE)
    wbuf, dw = _guarded(N, K, torch.bfloat16, sentinel)
    fp8.fp8_block_gemm_wgrad(dyqT, sdyT, xqT, sxT, dw=dw, workspace=workspace())
    fbuf, dwf = _guarded(N, K, torch.float32, 0x7FC0A5A5)
    dwf.zero_()
    fp8.fp8_block_gemm_wgrad_accum_f32(dyqT, sdyT, xqT, sxT, dwf, workspace=workspace())
    torch.cuda.synchronize()
    _assert_guards(buf, M, sentinel, "fprop")
    _assert_guards(dbuf, M, sentinel, "dgrad")
    _assert_guards(wbuf, N, sentinel, "wgrad")
    _assert_guards(fbuf, N, 0x7FC0A5A5, "wgrad accumulate")
    xq_o, sx_o = oracle.quantize_act_rowwise(syn.bf16_bits(x))
    wq_o, sw_o = oracle.quantize_weight(syn.bf16_bits(w))
    y_o, b_o = oracle.gemm_fprop(xq_o, sx_o, wq_o, sw_o)
    assert_within_bound(y, y_o, b_o, "fprop in a guarded buffer", output_rounding=True)


# -------------------------------------------- FP32 main-gradient accumulation

def _accumulate(N, K, M, micro_batches, seed, rows=None):
    """micro_batches wgrad products added into one FP32 main gradient on the
    GPU, and the same sum in FP64 by the oracle (both starting from the same
    seeded FP32 values).  Bound: each call's 2e-3 S + 1e-6, plus the FP32
    rounding of each addition on the GPU (half an ulp of the running value)."""
    d = dev()
    dw0 = torch.from_numpy(np.random.default_rng(seed).normal(scale=0.01, size=(N, K)).astype(np.float32))
    dw = dw0.to(d)
    running = dw0.numpy().astype(np.float64)
    tol = np.zeros((N, K) if rows is None else (len(rows), K))
    for b in range(micro_batches):
        g = syn.generator(seed * 1000 + b)
        dy = syn.normal_bf16((M, N), 1e-3, g)
        x = syn.activation_bf16(M, K, max(1, K // 100), 30.0, g)
        _, _, dyqT, sdyT = fp8.fp8_quantize_act_1x128(dy.to(d), fp8.COLWISE)
        _, _, xqT, sxT = fp8.fp8_quantize_act_1x128(x.to(d), fp8.COLWISE)
        fp8.fp8_block_gemm_wgrad_accum_f32(dyqT, sdyT, xqT, sxT, dw, workspace=workspace() if b % 2 else None)
        dyqT_o, sdyT_o = oracle.quantize_act_colwise(syn.bf16_bits(dy))
        xqT_o, sxT_o = oracle.quantize_act_colwise(syn.bf16_bits(x))
        new, bound = oracle.gemm_wgrad_accum(dyqT_o, sdyT_o, xqT_o, sxT_o, running)
        running = new
        sel = running if rows is None else running[rows]
        tol += 2e-3 * (bound if rows is None else bound[rows]) + 1e-6 + 2.0 ** -24 * np.abs(sel)
    torch.cuda.synchronize()
    got = dw.cpu().numpy().astype(np.float64)
    if rows is not None:
        got, running = got[rows], running[rows]
    err = np.abs(got - running)
    assert np.all(err <= tol), f"{int((err > tol).sum())} elements outside the accumulated bound"


@pytest.mark.parametrize("micro_batches", [2, 32])
def test_wgrad_accumulates_in_fp32_over_micro_batches(micro_batches):
    _accumulate(384, 640, 256, micro_batches, seed=micro_batches)


def test_wgrad_accumulates_with_the_split_schedule():
    """A 4096-token wgrad (32 slabs, split across CTA pairs on odd micro-batches)
    accumulated over 4 micro-batches."""
    _accumulate(512, 768, 4096, 4, seed=77)


@pytest.mark.slow
def test_wgrad_accumulates_in_fp32_at_the_qkv_shape():
    """Two 8192-token micro-batches into the fused-QKV main gradient
    [4096, 2048], every element."""
    _accumulate(syn.QKV_OUT, syn.HIDDEN, syn.TOKENS, 2, seed=5)


# ----------------------------------------------- time-outs of the real kernels

def test_gemm_and_quantizer_time_out_drain_and_recover():
    """An over-stated barrier byte count makes the first operand wait of every
    CTA run out: the GEMM and the tile quantizer must record FP8_ERR_TIMEOUT,
    drain what they issued and return, and the next launches must be
    correct."""
    d = dev()
    x = syn.activation_bf16(128, 128, 1, 30.0, syn.generator(41))
    w = syn.normal_bf16((128, 128), 0.02, syn.generator(42))
    xq, sx, _, _ = fp8.fp8_quantize_act_1x128(x.to(d), fp8.ROWWISE)
    wq, sw, _ = fp8.fp8_quantize_weight_128x128(w.to(d), transposed=False)
    torch.cuda.synchronize()
    fp8.fp8_clear_error()
    fp8.fp8_set_wait_timeout_ns(20_000_000)          # 20 ms
    try:
        fp8.fp8_selftest_stall_next(1)
        fp8.fp8_block_gemm_fprop(xq, sx, wq, sw)
        assert fp8.fp8_get_error() == 6               # FP8_ERR_TIMEOUT
        fp8.fp8_clear_error()
        fp8.fp8_selftest_stall_next(2)
        fp8.fp8_quantize_act_1x128(x.to(d), fp8.COLWISE)
        assert fp8.fp8_get_error() == 6
        fp8.fp8_clear_error()
    finally:
        fp8.fp8_set_wait_timeout_ns(0)
        fp8.fp8_clear_error()
    check_fprop(x, w, output_rounding=True)
    check_act(x, fp8.COLWISE)
    assert fp8.fp8_get_error() == 0


# ------------------------------------------------------ fused SwiGLU producer

def test_silu_matches_the_oracle_on_every_finite_bfloat16():
    """The fused producer's silu, rounded once to bfloat16, for all 65,024
    finite bfloat16 inputs against the oracle's correctly rounded silu."""
    got = fp8.fp8_selftest_silu_bf16()
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = ((bits.astype(np.uint32) >> 7) & 0xFF) != 0xFF
    want = oracle.silu_bf16(bits[finite])
    bad = np.nonzero(got[finite] != want)[0]
    assert bad.size == 0, (f"{bad.size} inputs differ, first g=0x{int(bits[finite][bad[0]]):04x}: "
                           f"gpu 0x{int(got[finite][bad[0]]):04x} oracle 0x{int(want[bad[0]]):04x}")


def _gate_up_case(rows, ffn, seed):
    """gate_up [rows, 2 ffn] bf16: N(0, 2) gate and N(0, 1) up, plus every
    kind of special value silu and the product meet: zeros of both signs,
    bfloat16 subnormals, values whose silu underflows FP32's exp, large
    magnitudes, and products below FP32's normal range."""
    g = syn.generator(seed)
    gate = torch.randn((rows, ffn), generator=g) * 2.0
    up = torch.randn((rows, ffn), generator=g)
    special = torch.tensor([0.0, -0.0, 1e-40, -1e-40, 3e-39, -9.2e-41, 2.0 ** -31, -(2.0 ** -25),
                            -90.0, -95.5, -100.0, -88.7, 85.0, -250.0, 300.0, 1e30, -1e30,
                            2.0 ** -8, -(2.0 ** -8), 0.5, -0.5, 7.0, -7.0, 80.0, -80.0])
    n = special.numel()
    gate[0, :n] = special
    gate[1, :n] = special
    up[1, :n] = torch.tensor([1e-30] * n)            # products below 2^-126
    gate[2, :n] = torch.full((n,), 1e-20)
    up[2, :n] = special                               # tiny silu times everything
    return torch.cat([gate, up], dim=1).to(torch.bfloat16)


@pytest.mark.parametrize("rows,ffn", [(128, 128), (256, 384), (384, 2048)])
@pytest.mark.parametrize("mode", [fp8.ROWWISE, fp8.COLWISE, fp8.BOTH])
def test_swiglu_quantize_matches_the_unfused_definition(rows, ffn, mode):
    gu = _gate_up_case(rows, ffn, rows + ffn + mode)
    q_row, s_row, q_colT, s_col = fp8.fp8_swiglu_quantize_1x128(gu.to(dev()), mode)
    torch.cuda.synchronize()
    h = oracle.swiglu_bf16(syn.bf16_bits(gu))
    if mode & fp8.ROWWISE:
        q_o, s_o = oracle.quantize_act_rowwise(h)
        assert_bits_equal(q_row, q_o, "fused row-wise codes")
        assert_bits_equal(s_row, s_o, "fused row-wise scales")
    if mode & fp8.COLWISE:
        q_o, s_o = oracle.quantize_act_colwise(h)
        assert_bits_equal(q_colT, q_o, "fused column-wise codes")
        assert_bits_equal(s_col, s_o, "fused column-wise scales")


# ------------------------------------------------------------ RMSNorm producer

def _norm_case(rows, cols, seed):
    """x with outlier channels, zero and tiny rows; gamma around 1 with
    zeros, negatives and magnitudes that make subnormal products."""
    g = syn.generator(seed)
    x = syn.activation_bf16(rows, cols, max(1, cols // 100), 30.0, g)
    x[0] = 0.0                                           # r = 1 / sqrt(eps)
    x[1] = x[1] * 1e-30                                  # tiny row, eps dominates
    x[2, :] = 3.0                                        # constant row
    gamma = (1.0 + 0.1 * torch.randn(cols, generator=g))
    gamma[:6] = torch.tensor([0.0, -1.0, 2.0 ** -120, -2.0 ** -126, 4.0, 2.0 ** 40])
    return x.to(torch.bfloat16), gamma.to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols", [(128, 128), (8, 2048), (300, 6144), (1, 8)])
def test_rmsnorm_rstd_matches_the_oracle(rows, cols):
    """The FP64 sum of squares in another order than the oracle's: equal, or
    one float32 ulp apart where the value sits next to a rounding midpoint."""
    x, _ = _norm_case(max(rows, 3), cols, rows + cols)
    x = x[:rows].contiguous()
    r = fp8.fp8_rmsnorm_rstd(x.to(dev()), 1e-6)
    torch.cuda.synchronize()
    want = oracle.rmsnorm_rstd(syn.bf16_bits(x), 1e-6)
    got = r.cpu().numpy()
    diff = np.abs(got.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
    assert diff.max() <= 1, diff.max()
    assert (diff != 0).mean() < 0.01


@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (384, 2048)])
@pytest.mark.parametrize("mode", [fp8.ROWWISE, fp8.COLWISE, fp8.BOTH])
def test_rmsnorm_quantize_matches_the_unfused_definition(rows, cols, mode):
    """Given the oracle's r, the fused producer's codes and scales equal the
    oracle's quantization of y = bf16(gamma * bf16(x * r)), bit for bit."""
    x, gamma = _norm_case(rows, cols, 3 * rows + cols + mode)
    xb, gb = syn.bf16_bits(x), syn.bf16_bits(gamma)
    r = oracle.rmsnorm_rstd(xb, 1e-6)
    q_row, s_row, q_colT, s_col = fp8.fp8_rmsnorm_quantize_1x128(
        x.to(dev()), torch.from_numpy(r).to(dev()), gamma.to(dev()), mode)
    torch.cuda.synchronize()
    y = oracle.rmsnorm_apply(xb, r, gb)
    if mode & fp8.ROWWISE:
        q_o, s_o = oracle.quantize_act_rowwise(y)
        assert_bits_equal(q_row, q_o, "norm row-wise codes")
        assert_bits_equal(s_row, s_o, "norm row-wise scales")
    if mode & fp8.COLWISE:
        q_o, s_o = oracle.quantize_act_colwise(y)
        assert_bits_equal(q_colT, q_o, "norm column-wise codes")
        assert_bits_equal(s_col, s_o, "norm column-wise scales")


# -------------------------------------- fused wgrad + data-parallel reduce-scatter

def _rank_inputs(N, K, M, seed):
    g = syn.generator(seed)
    dy = syn.normal_bf16((M, N), 1e-3, g)
    x = syn.activation_bf16(M, K, 4, 30.0, g)
    return dy, x


@pytest.mark.parametrize("nranks,M,split", [(1, 256, False), (2, 256, False), (4, 4096, True), (8, 256, False)])
def test_wgrad_reduce_scatter_into_emulated_ranks(nranks, M, split):
    """R ranks' wgrad products, each over its own M tokens, added by the
    fused epilogue into R FP32 shards (here all on this GPU; the addresses
    are what differ from peers' shards).  Each shard ends as its start plus
    the sum over ranks of its rows; against the oracle's FP64 sums, with each
    call's 2e-3 S + 1e-6 plus half an FP32 ulp of the running value per
    addition."""
    N, K, d = 1024, 384, dev()
    start = np.random.default_rng(nranks).normal(scale=0.01, size=(N, K)).astype(np.float32)
    rows = N // nranks
    shards = [torch.from_numpy(start[q * rows:(q + 1) * rows].copy()).to(d) for q in range(nranks)]
    running = start.astype(np.float64)
    tol = np.zeros((N, K))
    for r in range(nranks):
        dy, x = _rank_inputs(N, K, M, 5000 + 10 * nranks + r)
        _, _, dyqT, sdyT = fp8.fp8_quantize_act_1x128(dy.to(d), fp8.COLWISE)
        _, _, xqT, sxT = fp8.fp8_quantize_act_1x128(x.to(d), fp8.COLWISE)
        fp8.fp8_block_gemm_wgrad_reduce_scatter_f32(dyqT, sdyT, xqT, sxT, shards,
                                                    workspace=workspace() if split else None)
        dyqT_o, sdyT_o = oracle.quantize_act_colwise(syn.bf16_bits(dy))
        xqT_o, sxT_o = oracle.quantize_act_colwise(syn.bf16_bits(x))
        running, bound = oracle.gemm_wgrad_accum(dyqT_o, sdyT_o, xqT_o, sxT_o, running)
        tol += 2e-3 * bound + 1e-6 + 2.0 ** -24 * np.abs(running)
    torch.cuda.synchronize()
    got = np.concatenate([s.cpu().numpy() for s in shards]).astype(np.float64)
    err = np.abs(got - running)
    assert np.all(err <= tol), f"{int((err > tol).sum())} elements outside the bound"
