"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: torch's
float8_e4m3fn codec (an independent library implementation of E4M3FN),
the OCP format table, hand-worked groups (tests/golden), closed forms,
invariants of the definition and brute-force dequantize-then-matmul with
numpy.  See oracle/fp8_oracle.c for the definition being pinned.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from blockwise_fp8_pretraining_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
G = 128


# ------------------------------------------------------------------ helpers

def torch_decode(codes):
    """Library decode of E4M3FN codes (torch's float8_e4m3fn)."""
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def torch_encode(values):
    """Library RNE cast to E4M3FN.  torch saturates to 448 only up to the
    midpoint 464 and returns NaN beyond, so callers keep |v| <= 464."""
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def bits_of(values):
    return np.asarray(values, dtype=np.float32).view(np.uint32)


def to_bf16_bits(values):
    t = torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    return syn.bf16_bits(t)


def torch_quant_rowwise(x_bf16: torch.Tensor):
    """The quantizer definition written with torch library primitives:
    group amax, fp32 division by 448, fp32 division of each element, torch's
    E4M3 cast.  Used only for data whose |x/s| stays within torch's
    saturating range (always true for a group's own scale)."""
    rows, cols = x_bf16.shape
    xf = x_bf16.float().reshape(rows, cols // G, G)
    amax = xf.abs().amax(dim=2)                              # [rows, groups]
    s = amax / torch.tensor(448.0, dtype=torch.float32)
    safe = torch.where(s == 0, torch.ones_like(s), s)
    q = (xf / safe[:, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    q = torch.where((s == 0)[:, :, None], torch.zeros_like(q), q)
    return q.reshape(rows, cols).numpy(), s.T.contiguous().numpy()


def torch_quant_weight(w_bf16: torch.Tensor):
    n, k = w_bf16.shape
    wf = w_bf16.float().reshape(n // G, G, k // G, G)
    amax = wf.abs().amax(dim=(1, 3))                         # [n/128, k/128]
    s = amax / torch.tensor(448.0, dtype=torch.float32)
    safe = torch.where(s == 0, torch.ones_like(s), s)
    q = (wf / safe[:, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    q = torch.where((s == 0)[:, None, :, None], torch.zeros_like(q), q)
    return q.reshape(n, k).numpy(), s.numpy()


def dequant_rowwise(q, s):
    """[rows, cols] values from codes and [cols/128, rows] scales."""
    return torch_decode(q) * np.repeat(s.T.astype(np.float64), G, axis=1)


def dequant_weight(q, s):
    return torch_decode(q) * np.kron(s.astype(np.float64), np.ones((G, G)))


def assert_close_to_bound(y, ref, bound, rel):
    err = np.abs(y - ref)
    assert np.all(err <= rel * bound + 1e-300), float((err / np.maximum(bound, 1e-300)).max())


# -------------------------------------------------------------------- codec

def test_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch_decode(codes)
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_decode_spot_values_from_format_table():
    with open(os.path.join(GOLDEN, "e4m3_spot_values.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    for code_s, val_s in rows:
        got = oracle.e4m3_decode(np.array([int(code_s, 16)], np.uint8))[0]
        want = float(val_s)
        if np.isnan(want):
            assert np.isnan(got), code_s
        else:
            assert got == want and np.signbit(got) == np.signbit(want), code_s


def test_decode_grid_is_monotone_and_binade_spaced():
    vals = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))   # 0x00..0x7E
    assert np.all(np.diff(vals) > 0)
    gaps = np.diff(vals)
    # Subnormal steps and the step into the first normal binade are 2^-9;
    # each later binade's step is twice the previous one.
    assert np.all(gaps[:8] == 2.0 ** -9)
    for e in range(1, 16):
        seg = gaps[8 * e: 8 * e + 8]
        assert seg.size > 0 and np.all(seg == 2.0 ** (e - 10)), e


def test_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_encode_midpoints_tie_to_even_and_neighbours():
    pos = np.arange(0x7F, dtype=np.uint8)
    v = oracle.e4m3_decode(pos)
    lo, hi = v[:-1], v[1:]
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)   # exact in fp32
    even = np.where(pos[:-1] % 2 == 0, pos[:-1], pos[1:]).astype(np.uint8)
    below = np.nextafter(mid, np.float32(0))
    above = np.nextafter(mid, np.float32(np.inf))
    for sign in (1.0, -1.0):
        sb = np.uint8(0x80) if sign < 0 else np.uint8(0)
        assert np.array_equal(oracle.e4m3_encode(sign * mid), even | sb)
        assert np.array_equal(oracle.e4m3_encode(sign * below), pos[:-1] | sb)
        assert np.array_equal(oracle.e4m3_encode(sign * above), pos[1:] | sb)
        # the same decisions from the library cast
        assert np.array_equal(torch_encode(sign * mid), even | sb)
        assert np.array_equal(torch_encode(sign * below), pos[:-1] | sb)


def test_encode_saturates_at_448():
    big = np.array([448.0, 463.99, 464.0, 479.9, 480.0, 1e4, 1e30, 3.0e38], np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)


def test_encode_zero_and_tiny_keep_sign():
    v = np.array([0.0, -0.0, 1e-30, -1e-30, 2.0 ** -10, -(2.0 ** -10), 1e-45, -1e-45], np.float32)
    assert list(oracle.e4m3_encode(v)) == [0x00, 0x80, 0x00, 0x80, 0x00, 0x80, 0x00, 0x80]


def test_encode_matches_torch_on_dense_sweep():
    rng = np.random.default_rng(1)
    mag = np.exp(rng.uniform(np.log(1e-6), np.log(464.0), 400_000)).astype(np.float32)
    sign = np.where(rng.random(mag.size) < 0.5, -1, 1).astype(np.float32)
    v = np.concatenate([mag * sign, rng.uniform(-464, 464, 100_000).astype(np.float32)])
    assert np.array_equal(oracle.e4m3_encode(v), torch_encode(v))


# --------------------------------------------------------------- quantizers

def load_handworked():
    scales, elems = [], []
    with open(os.path.join(GOLDEN, "handworked_groups.txt")) as f:
        for ln in f:
            p = ln.split()
            if not p or p[0].startswith("#"):
                continue
            if p[0] == "scale":
                scales.append((int(p[1]), int(p[2]), int(p[3], 16)))
            else:
                elems.append((int(p[1]), int(p[2]), float(p[3]), int(p[4], 16)))
    return scales, elems


def test_handworked_groups_rowwise():
    scales, elems = load_handworked()
    x = np.zeros((2, 256), np.float32)
    for r, c, v, _ in elems:
        x[r, c] = v
    xb = to_bf16_bits(x)
    assert np.array_equal(oracle.bf16_to_float(xb), x)          # all exact in bf16
    q, s = oracle.quantize_act_rowwise(xb)
    want_q = np.zeros((2, 256), np.uint8)
    for r, c, _, code in elems:
        want_q[r, c] = code
    assert np.array_equal(q, want_q)
    assert s.shape == (2, 2)
    for r, g, b in scales:
        assert int(bits_of(s[g, r])) == b, (r, g)


def test_handworked_groups_colwise_and_weight():
    """The same groups placed along tokens (columns of X^T) and inside a
    128x128 weight block must give the same codes and scales."""
    scales, elems = load_handworked()
    x = np.zeros((2, 256), np.float32)
    for r, c, v, _ in elems:
        x[r, c] = v
    xt_bits = to_bf16_bits(x.T.copy())                           # [256, 2]
    qT, s = oracle.quantize_act_colwise(xt_bits)                 # [2, 256], [2, 2]
    q_row, s_row = oracle.quantize_act_rowwise(to_bf16_bits(x))
    assert np.array_equal(qT, q_row)
    assert np.array_equal(bits_of(s), bits_of(s_row))

    # weight: row 0 group 0's 128 values spread over a 128x128 block, with
    # an all-zero neighbour block.
    w = np.zeros((128, 256), np.float32)
    vals = x[0, :128]
    w[np.arange(128), (np.arange(128) * 37) % 128] = vals
    qw, sw = oracle.quantize_weight(to_bf16_bits(w))
    assert sw.shape == (1, 2)
    assert int(bits_of(sw[0, 0])) == 0x3F800000 and int(bits_of(sw[0, 1])) == 0
    got = qw[np.arange(128), (np.arange(128) * 37) % 128]
    assert np.array_equal(got, q_row[0, :128])
    mask = np.ones_like(qw, bool)
    mask[np.arange(128), (np.arange(128) * 37) % 128] = False
    assert np.all(qw[mask] == 0)


@pytest.mark.parametrize("maker", ["normal", "outlier", "student_t"])
def test_rowwise_matches_torch_library_definition(maker):
    if maker == "normal":
        x = syn.normal_bf16((96, 1024), 1.0, syn.generator(3))
    elif maker == "outlier":
        x = syn.activation_bf16(130, 2048, 20, 30.0, syn.generator(4))
    else:
        x = syn.student_t_bf16((64, 2048), seed=5)
    q, s = oracle.quantize_act_rowwise(syn.bf16_bits(x))
    q_ref, s_ref = torch_quant_rowwise(x)
    assert np.array_equal(bits_of(s), bits_of(s_ref))
    assert np.array_equal(q, q_ref)


def test_colwise_and_weight_match_torch_library_definition():
    x = syn.activation_bf16(256, 384, 4, 50.0, syn.generator(6))
    qT, s = oracle.quantize_act_colwise(syn.bf16_bits(x))
    q_ref, s_ref = torch_quant_rowwise(x.T.contiguous())
    assert np.array_equal(qT, q_ref)
    assert np.array_equal(bits_of(s), bits_of(s_ref))

    w = syn.normal_bf16((384, 256), 0.02, syn.generator(7))
    qw, sw = oracle.quantize_weight(syn.bf16_bits(w))
    qw_ref, sw_ref = torch_quant_weight(w)
    assert np.array_equal(qw, qw_ref)
    assert np.array_equal(bits_of(sw), bits_of(sw_ref))


def test_scaling_by_power_of_two_scales_s_and_keeps_codes():
    x = syn.activation_bf16(32, 512, 4, 50.0, syn.generator(8))
    q0, s0 = oracle.quantize_act_rowwise(syn.bf16_bits(x))
    for k in (-20, -3, 1, 7):
        xk = (x.float() * 2.0 ** k).to(torch.bfloat16)
        assert torch.equal(xk.float(), x.float() * 2.0 ** k)     # exact
        qk, sk = oracle.quantize_act_rowwise(syn.bf16_bits(xk))
        assert np.array_equal(qk, q0)
        assert np.array_equal(sk, s0 * np.float32(2.0 ** k))


def test_row_permutation_permutes_outputs():
    x = syn.activation_bf16(64, 256, 4, 50.0, syn.generator(9))
    perm = torch.randperm(64, generator=syn.generator(10))
    q, s = oracle.quantize_act_rowwise(syn.bf16_bits(x))
    qp, sp = oracle.quantize_act_rowwise(syn.bf16_bits(x[perm]))
    assert np.array_equal(qp, q[perm.numpy()])
    assert np.array_equal(sp, s[:, perm.numpy()])


def test_colwise_equals_rowwise_of_transpose():
    x = syn.activation_bf16(384, 256, 4, 50.0, syn.generator(11))
    qT, s = oracle.quantize_act_colwise(syn.bf16_bits(x))
    qr, sr = oracle.quantize_act_rowwise(syn.bf16_bits(x.T.contiguous()))
    assert np.array_equal(qT, qr) and np.array_equal(s, sr)


def test_weight_of_transpose_is_transpose():
    w = syn.normal_bf16((256, 384), 0.02, syn.generator(12))
    q, s = oracle.quantize_weight(syn.bf16_bits(w))
    qt, st = oracle.quantize_weight(syn.bf16_bits(w.T.contiguous()))
    assert np.array_equal(qt, q.T) and np.array_equal(st, s.T)


def test_all_zero_and_negative_zero_groups():
    x = np.zeros((3, 256), np.float32)
    x[1, :128] = -0.0
    x[2, 128:] = 1.0
    q, s = oracle.quantize_act_rowwise(to_bf16_bits(x))
    assert np.all(q[:2] == 0) and np.all(q[2, :128] == 0)
    assert np.all(s[:, :2] == 0) and s[0, 2] == 0
    assert np.all(q[2, 128:] == 0x7E)


def test_quantizer_bad_arguments():
    with pytest.raises(ValueError):
        oracle.quantize_act_rowwise(np.zeros((4, 100), np.uint16))
    with pytest.raises(ValueError):
        oracle.quantize_act_colwise(np.zeros((100, 128), np.uint16))
    with pytest.raises(ValueError):
        oracle.quantize_weight(np.zeros((128, 100), np.uint16))
    inf = to_bf16_bits(np.full((1, 128), np.inf, np.float32))
    with pytest.raises(ValueError):
        oracle.quantize_act_rowwise(inf)


def test_empty_rows():
    q, s = oracle.quantize_act_rowwise(np.zeros((0, 256), np.uint16))
    assert q.shape == (0, 256) and s.shape == (2, 0)


# -------------------------------------------------------------------- GEMMs

def _quant_case(seed, M, N, K):
    g = syn.generator(seed)
    x = syn.activation_bf16(M, K, 4, 30.0, g)
    w = syn.normal_bf16((N, K), 0.02, g)
    dy = syn.normal_bf16((M, N), 1e-3, g)
    return x, w, dy


def test_fprop_brute_force():
    x, w, _ = _quant_case(20, 200, 384, 512)
    xq, sx = oracle.quantize_act_rowwise(syn.bf16_bits(x))
    wq, sw = oracle.quantize_weight(syn.bf16_bits(w))
    y, bound = oracle.gemm_fprop(xq, sx, wq, sw)
    a = dequant_rowwise(xq, sx)
    b = dequant_weight(wq, sw)
    ref = a @ b.T
    ref_bound = np.abs(a) @ np.abs(b).T
    assert_close_to_bound(y, ref, ref_bound, 1e-12)
    assert_close_to_bound(bound, ref_bound, ref_bound, 1e-12)
    assert np.all(np.abs(y) <= bound * (1 + 1e-12))


def test_dgrad_brute_force():
    _, w, dy = _quant_case(21, 192, 384, 256)
    dyq, sdy = oracle.quantize_act_rowwise(syn.bf16_bits(dy))
    wq, sw = oracle.quantize_weight(syn.bf16_bits(w))
    dx, bound = oracle.gemm_dgrad(dyq, sdy, wq, sw)
    a = dequant_rowwise(dyq, sdy)          # [M, N]
    b = dequant_weight(wq, sw)             # [N, K]
    ref = a @ b
    ref_bound = np.abs(a) @ np.abs(b)
    assert dx.shape == (192, 256)
    assert_close_to_bound(dx, ref, ref_bound, 1e-12)
    assert_close_to_bound(bound, ref_bound, ref_bound, 1e-12)


def test_wgrad_brute_force():
    x, _, dy = _quant_case(22, 384, 256, 384)
    dyqT, sdyT = oracle.quantize_act_colwise(syn.bf16_bits(dy))   # [N, M]
    xqT, sxT = oracle.quantize_act_colwise(syn.bf16_bits(x))      # [K, M]
    dw, bound = oracle.gemm_wgrad(dyqT, sdyT, xqT, sxT)
    a = dequant_rowwise(dyqT, sdyT)        # [N, M]
    b = dequant_rowwise(xqT, sxT)          # [K, M]
    ref = a @ b.T
    ref_bound = np.abs(a) @ np.abs(b).T
    assert dw.shape == (256, 384)
    assert_close_to_bound(dw, ref, ref_bound, 1e-12)
    assert_close_to_bound(bound, ref_bound, ref_bound, 1e-12)


def test_fprop_all_ones_closed_form():
    ones = to_bf16_bits(np.ones((128, 128), np.float32))
    xq, sx = oracle.quantize_act_rowwise(ones)
    wq, sw = oracle.quantize_weight(ones)
    assert np.all(xq == 0x7E) and np.all(wq == 0x7E)
    s = Fraction(float(np.float32(1.0) / np.float32(448.0)))
    want = 128 * (448 * s) ** 2
    y, bound = oracle.gemm_fprop(xq, sx, wq, sw)
    assert np.all(np.abs(y - float(want)) <= 2.0 ** -52 * float(want))
    assert np.all(bound == y)


def test_fprop_block_identity_weight():
    x, _, _ = _quant_case(23, 128, 256, 256)
    eye = to_bf16_bits(np.eye(256, dtype=np.float32))
    xq, sx = oracle.quantize_act_rowwise(syn.bf16_bits(x))
    wq, sw = oracle.quantize_weight(eye)
    s_w = np.float32(1.0) / np.float32(448.0)
    assert sw[0, 1] == 0 and sw[1, 0] == 0 and sw[0, 0] == s_w and sw[1, 1] == s_w
    y, _ = oracle.gemm_fprop(xq, sx, wq, sw)
    want = dequant_rowwise(xq, sx) * (448.0 * float(s_w))
    assert np.all(np.abs(y - want) <= 1e-15 * np.abs(want))


def test_fprop_single_nonzero_per_row():
    rng = np.random.default_rng(24)
    M, N, K = 128, 256, 384
    xf = np.zeros((M, K), np.float32)
    cols = rng.integers(0, K, M)
    xf[np.arange(M), cols] = rng.normal(size=M).astype(np.float32)
    w = syn.normal_bf16((N, K), 0.02, syn.generator(25))
    xq, sx = oracle.quantize_act_rowwise(to_bf16_bits(xf))
    wq, sw = oracle.quantize_weight(syn.bf16_bits(w))
    y, _ = oracle.gemm_fprop(xq, sx, wq, sw)
    a = dequant_rowwise(xq, sx)
    b = dequant_weight(wq, sw)
    want = a[np.arange(M), cols][:, None] * b[:, cols].T
    assert np.all(np.abs(y - want) <= 1e-15 * np.abs(want))


def test_dgrad_equals_fprop_with_transposed_weight():
    _, w, dy = _quant_case(26, 128, 256, 384)
    dyq, sdy = oracle.quantize_act_rowwise(syn.bf16_bits(dy))
    wq, sw = oracle.quantize_weight(syn.bf16_bits(w))
    wtq, swt = oracle.quantize_weight(syn.bf16_bits(w.T.contiguous()))
    dx, b1 = oracle.gemm_dgrad(dyq, sdy, wq, sw)
    y, b2 = oracle.gemm_fprop(dyq, sdy, wtq, swt)
    assert np.array_equal(dx, y) and np.array_equal(b1, b2)


def test_row_subset_matches_full():
    x, w, dy = _quant_case(27, 256, 256, 256)
    xq, sx = oracle.quantize_act_rowwise(syn.bf16_bits(x))
    wq, sw = oracle.quantize_weight(syn.bf16_bits(w))
    y, b = oracle.gemm_fprop(xq, sx, wq, sw)
    rows = [255, 0, 17, 17]
    ys, bs = oracle.gemm_fprop(xq, sx, wq, sw, rows=rows)
    assert np.array_equal(ys, y[rows]) and np.array_equal(bs, b[rows])
    dyqT, sdyT = oracle.quantize_act_colwise(syn.bf16_bits(dy))
    xqT, sxT = oracle.quantize_act_colwise(syn.bf16_bits(x))
    dw, _ = oracle.gemm_wgrad(dyqT, sdyT, xqT, sxT)
    dws, _ = oracle.gemm_wgrad(dyqT, sdyT, xqT, sxT, rows=[3, 200])
    assert np.array_equal(dws, dw[[3, 200]])


def _exact(v):
    return Fraction(float(v))


def test_gemm_against_exact_rational_arithmetic():
    """fprop and wgrad of a 3-slab case against the exact value in rationals:
    every decoded code and every float32 scale is a dyadic rational, so the
    definition's sum can be formed with no rounding at all.  The oracle's
    FP64 result may differ from it only by its few final roundings."""
    x, w, _ = _quant_case(28, 128, 128, 384)
    xq, sx = oracle.quantize_act_rowwise(syn.bf16_bits(x))
    wq, sw = oracle.quantize_weight(syn.bf16_bits(w))
    rows = [0, 77]
    y, bound = oracle.gemm_fprop(xq, sx, wq, sw, rows=rows)
    dx_, dw_ = torch_decode(xq), torch_decode(wq)
    for ri, m in enumerate(rows):
        for n in (0, 5, 127):
            exact = Fraction(0)
            exact_abs = Fraction(0)
            for t in range(3):
                part = sum(_exact(dx_[m, k]) * _exact(dw_[n, k]) for k in range(t * G, (t + 1) * G))
                part_abs = sum(abs(_exact(dx_[m, k]) * _exact(dw_[n, k])) for k in range(t * G, (t + 1) * G))
                c = _exact(sx[t, m]) * _exact(sw[n // G, t])
                exact += c * part
                exact_abs += abs(c) * part_abs
            tol = 8 * 2.0 ** -53 * float(exact_abs)
            assert abs(Fraction(y[ri, n]) - exact) <= Fraction(tol)
            assert abs(Fraction(bound[ri, n]) - exact_abs) <= Fraction(tol)

    # wgrad contracts over the 384 tokens in 3 slabs with outer-product scales
    dyT = syn.normal_bf16((384, 128), 1e-3, syn.generator(29))
    xT = syn.activation_bf16(384, 128, 2, 30.0, syn.generator(30))
    dyqT, sdyT = oracle.quantize_act_colwise(syn.bf16_bits(dyT))       # [128, 384], [3, 128]
    xqT, sxT = oracle.quantize_act_colwise(syn.bf16_bits(xT))          # [128, 384], [3, 128]
    dw, dwb = oracle.gemm_wgrad(dyqT, sdyT, xqT, sxT, rows=[3, 100])
    da, db = torch_decode(dyqT), torch_decode(xqT)
    for ri, n in enumerate((3, 100)):
        for k in (0, 64, 127):
            exact = Fraction(0)
            exact_abs = Fraction(0)
            for t in range(3):
                for m in range(t * G, (t + 1) * G):
                    prod = _exact(sdyT[t, n]) * _exact(da[n, m]) * _exact(sxT[t, k]) * _exact(db[k, m])
                    exact += prod
                    exact_abs += abs(prod)
            tol = 8 * 2.0 ** -53 * float(exact_abs)
            assert abs(Fraction(dw[ri, k]) - exact) <= Fraction(tol)
            assert abs(Fraction(dwb[ri, k]) - exact_abs) <= Fraction(tol)


# ------------------------------------------------- main-gradient accumulation

def test_wgrad_accum_all_ones_closed_form_over_two_micro_batches():
    """dY = X = all-ones over 128 tokens: every along-token code is 0x7E (448)
    with s = fp32(1/448), so one micro-batch adds exactly 128 (448 s)^2 to
    every element.  Two micro-batches on a dyadic FP32 starting gradient give
    v + 2 * 128 (448 s)^2; selected rows read their own starting values."""
    ones = to_bf16_bits(np.ones((128, 256), np.float32))       # [tokens, N = K = 256]
    qT, sT = oracle.quantize_act_colwise(ones)                   # [256, 128], [1, 256]
    assert np.all(qT == 0x7E)
    s = Fraction(float(np.float32(1.0) / np.float32(448.0)))
    y = 128 * (448 * s) ** 2
    n_idx, k_idx = np.meshgrid(np.arange(256), np.arange(256), indexing="ij")
    v = ((n_idx - 100) * 0.25 + k_idx * 2.0 ** -10).astype(np.float32)
    rows = [5, 100, 255]
    out1, b1 = oracle.gemm_wgrad_accum(qT, sT, qT, sT, v.astype(np.float64))
    out2, _ = oracle.gemm_wgrad_accum(qT, sT, qT, sT, out1)
    sub, _ = oracle.gemm_wgrad_accum(qT, sT, qT, sT, out1, rows=rows)
    for n in rows:
        for k in (0, 1, 77, 255):
            want = Fraction(float(v[n, k])) + 2 * y
            assert abs(Fraction(out2[n, k]) - want) <= 2 * Fraction(2) ** -52 * abs(want)
    assert np.array_equal(sub, out2[rows])
    assert np.all(np.abs(b1 - float(y)) <= 2.0 ** -52 * float(y))
    zero, _ = oracle.gemm_wgrad_accum(qT, sT, qT, sT, None)
    assert np.all(np.abs(zero - float(y)) <= 2.0 ** -52 * float(y))


def test_wgrad_accum_against_exact_rational_arithmetic():
    """A 3-slab wgrad added to a random FP32 running gradient, selected rows,
    against the exact rational sum dw_in + sum_t sum_m s_a s_b a b."""
    dyT = syn.normal_bf16((384, 128), 1e-3, syn.generator(31))
    xT = syn.activation_bf16(384, 256, 2, 30.0, syn.generator(32))
    dyqT, sdyT = oracle.quantize_act_colwise(syn.bf16_bits(dyT))      # [128, 384]
    xqT, sxT = oracle.quantize_act_colwise(syn.bf16_bits(xT))         # [256, 384]
    v = np.random.default_rng(33).normal(scale=0.05, size=(128, 256)).astype(np.float32)
    rows = [100, 3]
    dw, _ = oracle.gemm_wgrad_accum(dyqT, sdyT, xqT, sxT, v.astype(np.float64), rows=rows)
    da, db = torch_decode(dyqT), torch_decode(xqT)
    for ri, n in enumerate(rows):
        for k in (0, 130, 255):
            exact = _exact(v[n, k])
            exact_abs = abs(exact)
            for t in range(3):
                for m in range(t * G, (t + 1) * G):
                    prod = _exact(sdyT[t, n]) * _exact(da[n, m]) * _exact(sxT[t, k]) * _exact(db[k, m])
                    exact += prod
                    exact_abs += abs(prod)
            assert abs(Fraction(dw[ri, k]) - exact) <= Fraction(8 * 2.0 ** -53 * float(exact_abs))


# -------------------------------------------------------------------- SwiGLU

def _bf16_rne_exact(v: Fraction, negative: bool) -> int:
    """Bit pattern of the bfloat16 nearest to the exact rational |v| with the
    given sign (ties to even), by rational arithmetic alone."""
    sign = 0x8000 if negative else 0
    mag = abs(v)
    if mag == 0:
        return sign
    e = mag.numerator.bit_length() - mag.denominator.bit_length()
    if Fraction(2) ** e > mag:
        e -= 1                                   # now 2^e <= mag < 2^(e+1)
    e = max(e, -126)
    step = Fraction(2) ** (e - 7)
    units = mag / step
    below = units.numerator // units.denominator
    rest = units - below
    pick = below + 1 if rest > Fraction(1, 2) or (rest == Fraction(1, 2) and below % 2) else below
    value = pick * step
    if value >= Fraction(2) ** 128:
        return sign | 0x7F80
    # encode: value = pick * 2^(e-7), pick <= 256
    if e == -126 and pick < 128:
        return sign | int(pick)                  # subnormal: mantissa = pick
    if pick == 256:
        pick, e = 128, e + 1
    return sign | ((e + 127) << 7) | (int(pick) - 128)


def test_bf16_from_double_matches_rational_rounding_and_torch():
    rng = np.random.default_rng(40)
    # float32 values (torch's float32 -> bfloat16 cast is RNE): normal,
    # subnormal, exact midpoints and their neighbours
    mids = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    vals = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-40, 38, 20000),
                           mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1)),
                           np.float32([0.0, -0.0, 1e-45, -1e-45, 3.3e38, -3.3e38])]).astype(np.float32)
    vals = vals[np.isfinite(vals)]
    want = syn.bf16_bits(torch.from_numpy(vals).to(torch.bfloat16))
    got = np.array([oracle.bf16_from_double(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want)
    # doubles that float32 cannot hold: rounding via float32 first would land
    # on a bfloat16 midpoint and go the wrong way
    for v, want_bits in [(1 + 2.0 ** -8 + 2.0 ** -30, 0x3F81), (1 + 2.0 ** -8 - 2.0 ** -30, 0x3F80),
                         (-(1 + 3 * 2.0 ** -8 - 2.0 ** -31), 0xBF81), (2.0 ** -133 * 0.5000001, 0x0001)]:
        assert oracle.bf16_from_double(v) == want_bits == _bf16_rne_exact(Fraction(v), v < 0)


def _silu_bits_reference(g: float, negative: bool) -> int:
    """bfloat16 of silu(g) from decimal arithmetic: the value is taken with
    a relative error far below 10^-(prec-5), and the result is accepted only
    when both ends of that interval round alike; otherwise the precision is
    raised (at |g| ~ 1e-40, g/2 can be a bfloat16 midpoint and the deciding
    term g^2/4 sits 40 digits further down)."""
    import decimal

    for prec in (40, 200):
        ctx = decimal.Context(prec=prec, Emax=decimal.MAX_EMAX, Emin=decimal.MIN_EMIN, traps=[])
        gd = decimal.Decimal(g)
        s = ctx.divide(gd, ctx.add(decimal.Decimal(1), ctx.exp(ctx.minus(gd))))
        if s.is_zero():
            return 0x8000 if negative else 0
        exact = Fraction(s)
        eps = Fraction(1, 10 ** (prec - 5))
        lo = _bf16_rne_exact(exact * (1 - eps), negative)
        hi = _bf16_rne_exact(exact * (1 + eps), negative)
        if lo == hi:
            return lo
    raise AssertionError(f"silu({g!r}) not decided at 200 digits")


def test_silu_every_bf16_input_against_exact_rounding():
    """All 65,024 finite bfloat16 g against silu(g) = g / (1 + e^-g) from
    decimal arithmetic, rounded to bfloat16 by rational arithmetic.  For
    |g| >= 200 the value is settled without exp: g > 0 gives
    g (1 - e^-g / (1 + e^-g)), below g by a relative 1e-87, so the bfloat16
    g itself; g < 0 gives a magnitude below 200 e^-200 < 1e-84, under half
    the smallest bfloat16 subnormal, so -0."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]
    got = oracle.silu_bf16(bits)
    g_vals = oracle.bf16_to_float(bits).astype(np.float64)
    for b, g, out in zip(bits, g_vals, got):
        negative = bool(b & 0x8000)
        if abs(g) >= 200:
            want = int(b) if g > 0 else 0x8000
        else:
            want = _silu_bits_reference(float(g), negative)
        assert int(out) == want, (hex(int(b)), float(g), hex(int(out)), hex(want))


def test_swiglu_layout_and_product_rounding():
    g = syn.generator(41)
    rows, ffn = 5, 200
    gate_up = syn.normal_bf16((rows, 2 * ffn), 1.0, g)
    bits = syn.bf16_bits(gate_up)
    h = oracle.swiglu_bf16(bits)
    assert h.shape == (rows, ffn)
    s = torch.from_numpy(oracle.silu_bf16(bits[:, :ffn]).astype(np.int16)).view(torch.bfloat16)
    up = gate_up[:, ffn:]
    # the product of two bfloat16 values is exact in float32; one RNE cast
    want = syn.bf16_bits((s.float() * up.float()).to(torch.bfloat16))
    assert np.array_equal(h, want)
    # up = 1 gives silu itself; large gates pass up through
    ones = np.full((1, 4), 0x3F80, np.uint16)
    gates = to_bf16_bits(np.float32([[1.0, -1.0, 100.0, -100.0]]))
    assert np.array_equal(oracle.swiglu_bf16(np.concatenate([gates, ones], axis=1)),
                          oracle.silu_bf16(gates))
    assert list(oracle.silu_bf16(gates)[0]) == [0x3F3B, 0xBE8A, 0x42C8, 0x8000]


def test_silu_rounding_margin_allows_fp64_evaluation():
    """For every bfloat16 g with 2^-30 <= |g| < 200, silu(g) lies at least
    2e-9 (relative) away from every bfloat16 rounding boundary.  So any
    evaluation with a smaller relative error, such as the double-precision
    quotient the oracle takes there (error of a few 1e-16), rounds exactly
    as the exact value does.  The other ranges are settled without that
    quotient: the g/2 + g^2/4 series below 2^-30, closed forms from 200 up."""
    import decimal

    ctx = decimal.Context(prec=60, Emax=decimal.MAX_EMAX, Emin=decimal.MIN_EMIN, traps=[])
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]
    g_vals = oracle.bf16_to_float(bits).astype(np.float64)
    smallest, count = 1.0, 0
    for g in g_vals:
        if not (2.0 ** -30 <= abs(g) < 200):
            continue
        gd = decimal.Decimal(float(g))
        s = Fraction(ctx.divide(gd, ctx.add(decimal.Decimal(1), ctx.exp(ctx.minus(gd)))))
        mag = abs(s)
        e = mag.numerator.bit_length() - mag.denominator.bit_length()
        if Fraction(2) ** e > mag:
            e -= 1
        step = Fraction(2) ** (max(e, -126) - 7)
        units = mag / step
        below = units.numerator // units.denominator
        # the rounding boundaries around mag: the midpoints below and above it
        d = min(abs(mag - (below + Fraction(1, 2)) * step), abs(mag - (below - Fraction(1, 2)) * step))
        smallest = min(smallest, float(d / mag))
        count += 1
    assert count > 9000
    assert smallest > 2e-9, smallest


# ---------------------------------------------------------------- RMSNorm

def _f32_nearest(v: Fraction):
    """The float32 nearest to the positive rational v (ties to the even
    significand), and whether v lies within 2^-38 (relative) of the midpoint
    between it and a neighbour (where a double evaluation may decide
    either way)."""
    f = np.float32(float(v))
    cands = {float(f), float(np.nextafter(f, np.float32(0))), float(np.nextafter(f, np.float32(np.inf)))}
    ranked = sorted(cands, key=lambda c: (abs(Fraction(c) - v), int(np.float32(c).view(np.uint32)) & 1))
    best, second = ranked[0], ranked[1]
    gap = abs(abs(Fraction(second) - v) - abs(Fraction(best) - v))
    return np.float32(best), gap < v * Fraction(1, 2 ** 38)


def _rstd_exact(row_bits: np.ndarray, eps: np.float32):
    import decimal

    vals = [Fraction(float(v)) for v in oracle.bf16_to_float(row_bits).astype(np.float64)]
    m = sum(v * v for v in vals) / len(vals) + Fraction(float(eps))
    ctx = decimal.Context(prec=50)
    d = ctx.divide(decimal.Decimal(1), ctx.sqrt(ctx.divide(decimal.Decimal(m.numerator), decimal.Decimal(m.denominator))))
    return _f32_nearest(Fraction(d))


def test_rmsnorm_rstd_closed_forms():
    """Rows of one repeated value c: mean c^2, so r = 1 / |c| with eps = 0
    (exact for powers of two); a zero row gives 1 / sqrt(eps)."""
    for k in range(-6, 7):
        c = np.float32(2.0 ** k)
        row = to_bf16_bits(np.full((2, 384), c, np.float32))
        row[1] |= 0x8000                             # the sign does not matter
        assert list(oracle.rmsnorm_rstd(row, 0.0)) == [np.float32(2.0 ** -k)] * 2
    three = to_bf16_bits(np.full((1, 256), 3.0, np.float32))
    assert oracle.rmsnorm_rstd(three, 0.0)[0] == _f32_nearest(Fraction(1, 3))[0]
    eps = np.float32(1e-6)
    zero = np.zeros((1, 128), np.uint16)
    assert oracle.rmsnorm_rstd(zero, float(eps))[0] == _rstd_exact(zero[0], eps)[0]
    # one nonzero value x among n: mean x^2 / n
    one = np.zeros((1, 512), np.uint16)
    one[0, 37] = to_bf16_bits(np.float32([[8.0]]))[0, 0]
    assert oracle.rmsnorm_rstd(one, 0.0)[0] == np.float32(np.sqrt(512.0) / 8.0)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_rmsnorm_rstd_against_exact_arithmetic(seed):
    """Random rows (normal with x30 outlier channels, Student-t tails, tiny
    magnitudes, 2048 and 6144 wide): the oracle's r equals the float32
    nearest to the exact 1 / sqrt(mean + eps), computed in rational and
    50-digit decimal arithmetic, except within 2^-38 of a rounding midpoint
    where either neighbour is accepted."""
    g = syn.generator(700 + seed)
    eps = np.float32(1e-6)
    rows = [syn.bf16_bits(syn.activation_bf16(3, 2048, 20, 30.0, g)),
            syn.bf16_bits(syn.student_t_bf16((2, 6144), seed=seed)),
            to_bf16_bits((np.random.default_rng(seed).standard_normal((2, 2048)) * 1e-3).astype(np.float32))]
    checked = 0
    for block in rows:
        got = oracle.rmsnorm_rstd(block, float(eps))
        for i in range(block.shape[0]):
            want, near = _rstd_exact(block[i], eps)
            if near:
                assert abs(int(got[i].view(np.uint32)) - int(want.view(np.uint32))) <= 1
            else:
                assert got[i] == want, (i, got[i], want)
            checked += 1
    assert checked == 7


def test_rmsnorm_apply_against_torch_and_exact_products():
    """y = bf16(gamma * bf16(fp32(x * r))): the FP32 product and the first
    rounding against torch's float32 multiply and bfloat16 cast, the second
    against torch's bfloat16 multiply (computed in float32 and rounded),
    which is exact wherever the float32 product is normal; subnormal
    products against exact rational rounding."""
    g = syn.generator(811)
    rows, cols = 6, 384
    x = syn.activation_bf16(rows, cols, 4, 30.0, g)
    r = torch.exp(torch.empty(rows).uniform_(-20.0, 20.0, generator=g)).float()
    gamma = (1.0 + 0.1 * torch.randn(cols, generator=g)).to(torch.bfloat16)
    gamma[:5] = torch.tensor([0.0, -1.0, 2.0 ** -120, -3.5, 2.0 ** 60]).to(torch.bfloat16)
    xb, gb = syn.bf16_bits(x), syn.bf16_bits(gamma)
    y = oracle.rmsnorm_apply(xb, r.numpy(), gb)
    t = (x.float() * r[:, None]).to(torch.bfloat16)
    prod = gamma.float()[None, :] * t.float()
    normal = (prod.abs() >= 2.0 ** -126) | (prod == 0)
    want = syn.bf16_bits(gamma[None, :] * t)
    assert np.array_equal(y[normal.numpy()], want[normal.numpy()])
    tb = syn.bf16_bits(t)
    for i, k in zip(*np.nonzero(~normal.numpy())):
        v = Fraction(float(oracle.bf16_to_float(gb[k:k + 1])[0])) * Fraction(float(oracle.bf16_to_float(tb[i, k:k + 1])[0]))
        assert int(y[i, k]) == _bf16_rne_exact(v, v < 0), (i, k)
    assert (~normal).sum() > 0                       # the subnormal case is exercised


def test_rmsnorm_is_invariant_to_power_of_two_row_scaling():
    """With eps = 0, scaling a row by 2^k scales r by 2^-k exactly, so the
    normalized and scaled output is unchanged."""
    g = syn.generator(919)
    x = syn.bf16_bits(syn.activation_bf16(4, 256, 3, 30.0, g))
    gamma = syn.bf16_bits((1.0 + 0.1 * torch.randn(256, generator=g)).to(torch.bfloat16))
    base = oracle.rmsnorm_apply(x, oracle.rmsnorm_rstd(x, 0.0), gamma)
    for k in (-5, 3, 11):
        xs = to_bf16_bits(oracle.bf16_to_float(x) * np.float32(2.0 ** k))
        assert np.array_equal(oracle.rmsnorm_apply(xs, oracle.rmsnorm_rstd(xs, 0.0), gamma), base), k


def test_rmsnorm_apply_fp32_product_near_bfloat16_midpoints():
    """x * r chosen to land within a few float32 units of bfloat16 rounding
    midpoints, where the bfloat16 result depends on the one float32
    rounding of the product: against torch's float32 multiply and casts."""
    rng = np.random.default_rng(5)
    rows, cols = 64, 128
    x = to_bf16_bits((rng.uniform(1.0, 2.0, (rows, cols)) * np.where(rng.random((rows, cols)) < 0.5, -1, 1))
                     .astype(np.float32))
    xf = oracle.bf16_to_float(x).astype(np.float64)
    # per row: a bfloat16 midpoint M near 1 (9 significant bits, odd last)
    # and r = fp32(M / x[row, 0]), so x[row, 0] * r is within an ulp of M;
    # the other columns land near other midpoints less tightly
    mids = (256 + 2 * rng.integers(0, 128, rows) + 1) / 512.0
    r = (mids / xf[:, 0]).astype(np.float32)
    gamma = np.full(cols, 0x3F80, np.uint16)          # gamma = 1: y is the first rounding
    y = oracle.rmsnorm_apply(x, r, gamma)
    t = (torch.from_numpy(xf.astype(np.float32)) * torch.from_numpy(r)[:, None]).to(torch.bfloat16)
    assert np.array_equal(y, syn.bf16_bits(t))
    prod = (xf.astype(np.float32) * r[:, None]).astype(np.float64)
    units = prod[:, 0] * 512.0                       # midpoints in [1/2, 1) are odd multiples of 2^-9
    assert np.mean((np.abs(units - np.round(units)) < 1e-4) & (np.round(units) % 2 == 1)) > 0.9
