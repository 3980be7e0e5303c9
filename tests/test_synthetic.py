"""The seeded synthetic inputs (CPU): shapes, determinism and the value
recipe.  These tensors feed both the CUDA path and the oracle, so a drift
here would silently change every parity case."""
import math

import numpy as np
import pytest
import torch

from blockwise_fp8_pretraining_b200 import synthetic as syn


def test_layer_shapes_follow_the_model():
    # hidden 2048, 16 + 8 + 8 heads of 128, FFN 6144 (gate and up fused)
    assert syn.LAYER_LINEARS == (("qkv", 4096, 2048), ("o_proj", 2048, 2048),
                                 ("gate_up", 12288, 2048), ("down", 2048, 6144))
    assert syn.TOKENS == 2 * 4096 and syn.LAYERS == 28
    layer = syn.layer(3, tokens=256)
    for name, n, k in syn.LAYER_LINEARS:
        t = layer[name]
        assert t["x"].shape == (256, k) and t["w"].shape == (n, k) and t["dy"].shape == (256, n)
        assert t["x"].dtype == t["w"].dtype == t["dy"].dtype == torch.bfloat16


def test_same_seed_same_tensors_other_seed_different():
    a = syn.tiny(seed=5)
    b = syn.tiny(seed=5)
    c = syn.tiny(seed=6)
    for key in ("x", "w", "dy"):
        assert torch.equal(a[key], b[key])
        assert not torch.equal(a[key], c[key])
    la, lb = syn.layer(11, tokens=128), syn.layer(11, tokens=128)
    for name, _, _ in syn.LAYER_LINEARS:
        for key in ("x", "w", "dy"):
            assert torch.equal(la[name][key], lb[name][key])


def test_outlier_channels_are_whole_columns_scaled():
    g = syn.generator(1)
    rows, cols, n_out, factor = 4096, 2048, syn.outlier_channels(2048), 30.0
    assert n_out == 20                                   # floor(1% of 2048)
    assert syn.outlier_channels(6144) == 61
    x = syn.activation_bf16(rows, cols, n_out, factor, g).float()
    col_std = x.std(dim=0)
    big = torch.nonzero(col_std > 10.0).flatten()
    assert big.numel() == n_out                         # exactly the scaled channels
    assert torch.all((col_std[big] > 25.0) & (col_std[big] < 35.0))
    rest = torch.ones(cols, dtype=torch.bool)
    rest[big] = False
    assert abs(col_std[rest].mean().item() - 1.0) < 0.02


@pytest.mark.parametrize("std", [1.0, 0.02, 1e-3])
def test_normal_std_is_the_second_parameter(std):
    x = syn.normal_bf16((512, 512), std, syn.generator(2)).float()
    assert abs(x.mean().item()) < 5 * std / 512
    assert abs(x.std().item() / std - 1.0) < 0.01


def test_values_are_rounded_to_bf16_from_float32():
    # the bf16 tensor is the RNE rounding of the same float32 draw
    g1, g2 = syn.generator(9), syn.generator(9)
    x = syn.normal_bf16((64, 64), 0.02, g1)
    ref = (torch.randn((64, 64), generator=g2, dtype=torch.float32) * 0.02).to(torch.bfloat16)
    assert torch.equal(x, ref)


def test_student_t_heavy_tail_fraction():
    shape = (1024, 1024)
    x = syn.student_t_bf16(shape, seed=4).float().numpy()
    n = x.size
    k = int(round(1e-3 * n))
    # the scaled positions dominate the tail: at least k values beyond what a
    # t(3) bulk reaches at that count
    big = np.sort(np.abs(x).ravel())[-k:]
    assert np.median(big) > 100.0
    bulk = np.sort(np.abs(x).ravel())[: n - 2 * k]
    assert bulk.max() < 100.0
    again = syn.student_t_bf16(shape, seed=4)
    assert torch.equal(torch.from_numpy(x).to(torch.bfloat16), again)


def test_swiglu_split_and_down_input_family():
    gate_up = syn.normal_bf16((32, 2 * 64), 1.0, syn.generator(7))
    h = syn.swiglu_bf16(gate_up)
    gate, up = gate_up[:, :64].float(), gate_up[:, 64:].float()
    ref = (torch.nn.functional.silu(gate).to(torch.bfloat16).float() * up).to(torch.bfloat16)
    assert h.shape == (32, 64) and torch.equal(h, ref)
    # the sweep's down-projection input is silu(g) * u of N(0,1) draws
    x = syn.layer(0, tokens=512)["down"]["x"].float()
    assert x.shape == (512, 6144)
    assert 0.3 < x.std().item() < 0.8            # E[(silu(g) u)^2]^(1/2) ~ 0.55


def test_bf16_bits_view():
    t = torch.tensor([1.0, -2.0, 0.0, -0.0], dtype=torch.bfloat16)
    assert syn.bf16_bits(t).tolist() == [0x3F80, 0xC000, 0x0000, 0x8000]
    assert math.isclose(float(t[0]), 1.0)
