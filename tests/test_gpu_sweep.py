"""GPU parity across the rank / length sweep at the 8B width (d = 4096, f = 14336,
alpha = 16): the full oracle at T = 512 for every rank, and at T = 32768 the outputs
the oracle can compute one by one (sampled rows of Y and dX; sampled columns of dBg,
dBu and dAd over all rows)."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import synth
from lora_fine_tuning_rmsnorm_b200.runner import GRADS, Problem
from oracle import lora_mlp_ref as ref
from tests.parity import assert_close, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def run_gpu(shape, bits):
    pb = Problem(shape, bits)
    pb.step()
    torch.cuda.synchronize()
    return pb


@pytest.mark.parametrize("r", [8, 16, 32, 64, 128])
def test_sweep_T512_full_oracle(cuda_ok, r):
    shape = synth.Shape(T=512, d=4096, f=14336, r=r, alpha=16.0)
    bits = synth.make_inputs_bits(shape)
    pb = run_gpu(shape, bits)
    R = ref.fwd_bwd(synth.bits_to_f64(bits), shape.scale, shape.eps, chunk=512, keep=("Y", "dX"))
    out = {"Y": to_np(pb.Y), "dX": to_np(pb.dX), **{k: to_np(v) for k, v in pb.g.items()}}
    for k in ("Y", "dX") + GRADS:
        assert_close(f"r{r} {k}", out[k], R[k])


@pytest.mark.parametrize("r", [8, 128])
def test_sweep_T32768_sampled(cuda_ok, r):
    shape = synth.Shape(T=32768, d=4096, f=14336, r=r, alpha=16.0)
    bits = synth.make_inputs_bits(shape)
    pb = run_gpu(shape, bits)
    rng = np.random.default_rng(r)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 16383, 32767], rng.integers(0, shape.T, 25)]))
    cols = np.unique(np.concatenate([[0, 1, 127, 14335], rng.integers(0, shape.f, 12)]))
    R = ref.sampled(synth.bits_to_f64(bits), shape.scale, shape.eps, rows, cols, chunk=4096)
    assert_close("Y rows", to_np(pb.Y)[rows], R["Y"])
    assert_close("dX rows", to_np(pb.dX)[rows], R["dX"])
    assert_close("dBg cols", to_np(pb.g["dBg"])[cols], R["dBg"])
    assert_close("dBu cols", to_np(pb.g["dBu"])[cols], R["dBu"])
    assert_close("dAd cols", to_np(pb.g["dAd"])[:, cols], R["dAd"])
