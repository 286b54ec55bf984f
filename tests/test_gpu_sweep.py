"""GPU parity across the whole rank / length sweep at the 8B width (d = 4096, f = 14336,
alpha = 16): every point r in {8, 16, 32, 64, 128} x T in {512, 2048, 8192, 32768}
against the full fp64 oracle, every element of Y, dX and the six adapter gradients.

The tile shape, the CTA pairing and the K-split counts of the rank-r projections and
of the adapter-gradient reductions are chosen from T (and N), so each length takes its
own launch configuration; at T = 32768 the adapter gradients are fp32-atomic sums over
four times the rows of the 8B workload."""
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, synth
from lora_fine_tuning_rmsnorm_b200.runner import GRADS, Problem
from oracle import lora_mlp_ref as ref
from tests.parity import assert_close, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

POINTS = [(s.T, s.r) for s in configs.SWEEP]


@pytest.mark.parametrize("T,r", POINTS, ids=[f"T{T}_r{r}" for T, r in POINTS])
def test_sweep_full_oracle(cuda_ok, T, r):
    shape = synth.Shape(T=T, d=4096, f=14336, r=r, alpha=16.0)
    bits = synth.make_inputs_bits(shape)
    pb = Problem(shape, bits)
    pb.step()
    torch.cuda.synchronize()
    out = {"Y": to_np(pb.Y), "dX": to_np(pb.dX), **{k: to_np(v) for k, v in pb.g.items()}}
    del pb
    torch.cuda.empty_cache()
    R = ref.fwd_bwd(synth.bits_to_f64(bits), shape.scale, shape.eps, chunk=2048, keep=("Y", "dX"))
    for k in ("Y", "dX") + GRADS:
        assert_close(f"T{T} r{r} {k}", out[k], R[k])
