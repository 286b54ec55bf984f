"""The seeded input generator: determinism, shapes, bf16 rounding (CPU only)."""
import numpy as np
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 65504.0, 1e-30, -3.3895e38, np.inf, -np.inf], np.float32)])
    mine = synth.f32_to_bf16_bits(a)
    theirs = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(mine, theirs)
    back = synth.bf16_bits_to_f32(mine)
    np.testing.assert_array_equal(back, torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_shapes_and_determinism():
    s = configs.TINY
    a = synth.make_inputs_bits(s)
    b = synth.make_inputs_bits(s)
    for k in synth.TENSOR_ORDER:
        np.testing.assert_array_equal(a[k], b[k])
    assert a["X"].shape == (64, 128) and a["w"].shape == (128,)
    assert a["Wg"].shape == (344, 128) and a["Wd"].shape == (128, 344)
    assert a["Ag"].shape == (8, 128) and a["Bg"].shape == (344, 8)
    assert a["Ad"].shape == (8, 344) and a["Bd"].shape == (128, 8)
    assert a["dY"].shape == (64, 128)
    # each tensor has its own stream: changing T does not change the weights
    s2 = synth.Shape(T=65, d=128, f=344, r=8)
    c = synth.make_inputs_bits(s2)
    np.testing.assert_array_equal(a["Wg"], c["Wg"])


def test_distributions():
    s = synth.Shape(T=512, d=256, f=512, r=16)
    x = synth.bits_to_f64(synth.make_inputs_bits(s))
    assert abs(x["X"].std() - 1.0) < 0.02
    assert abs(x["w"].mean() - 1.0) < 0.02 and abs(x["w"].std() - 0.1) < 0.02
    assert abs(x["Wg"].std() - 0.02) < 0.001
    b = 1 / np.sqrt(256)
    assert x["Ag"].max() <= b and x["Ag"].min() >= -b and abs(x["Ag"].std() - b / np.sqrt(3)) < 0.01 * b * 10
    assert abs(x["Bg"].std() - 0.01) < 0.001


def test_flops_formula():
    assert abs(configs.algorithmic_flops(configs.LLAMA3_8B) - 5.8159e12) / 5.8159e12 < 1e-4
    assert abs(configs.algorithmic_flops(configs.LLAMA32_1B) - 1.6734e12) / 1.6734e12 < 1e-4


def test_qkv_inputs_shapes_streams_and_determinism():
    s = synth.QkvShape(T=33, d=64, nq=64, nkv=16, r=8)
    a = synth.make_qkv_inputs_bits(s)
    b = synth.make_qkv_inputs_bits(s)
    shapes = {"X": (33, 64), "w": (64,), "Wq": (64, 64), "Wk": (16, 64), "Wv": (16, 64), "Aq": (8, 64),
              "Bq": (64, 8), "Ak": (8, 64), "Bk": (16, 8), "Av": (8, 64), "Bv": (16, 8), "dQ": (33, 64),
              "dK": (33, 16), "dV": (33, 16)}
    for k, sh in shapes.items():
        assert a[k].shape == sh and a[k].dtype == np.uint16, k
        assert np.array_equal(a[k], b[k]), k
    # streams of their own: not the MLP's X for the same seed and size
    mlp = synth.make_inputs_bits(synth.Shape(T=33, d=64, f=128, r=8), names=("X",))
    assert not np.array_equal(mlp["X"], a["X"])
    assert abs(s.scale - 2.0) < 1e-12
