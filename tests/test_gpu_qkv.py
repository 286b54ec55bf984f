"""GPU parity of the LoRA Q/K/V projections (lora_qkv_fwd / lora_qkv_bwd through the C
ABI) against the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, synth
from lora_fine_tuning_rmsnorm_b200.runner import QKV_GRADS, QkvProblem
from oracle import lora_qkv_ref as ref
from tests.parity import assert_close, to_np

pytestmark = pytest.mark.gpu


def run_and_check(shape, keep=("Q", "K", "V", "dX")):
    bits = synth.make_qkv_inputs_bits(shape)
    pb = QkvProblem(shape, bits)
    for v in pb.out.values():
        v.fill_(float("nan"))
    pb.dX.fill_(float("nan"))
    pb.ctx.fill_(0xFF)
    pb.ws.fill_(0xFF)
    pb.step()
    torch.cuda.synchronize()
    R = ref.fwd_bwd(synth.bits_to_f64(bits), shape.scale, shape.eps, chunk=1024, keep=keep)
    got = {**{k: to_np(v) for k, v in pb.out.items()}, "dX": to_np(pb.dX), **{k: to_np(v) for k, v in pb.g.items()}}
    for k in keep + QKV_GRADS:
        assert_close(k, got[k], R[k])
    return pb


SHAPES = [
    synth.QkvShape(T=200, d=136, nq=136, nkv=64, r=8),     # ragged T, d, nq; grouped K/V
    synth.QkvShape(T=64, d=128, nq=128, nkv=128, r=8),     # one M tile, no grouping
    synth.QkvShape(T=384, d=256, nq=256, nkv=64, r=16),
    synth.QkvShape(T=300, d=512, nq=512, nkv=128, r=32),
    synth.QkvShape(T=160, d=384, nq=384, nkv=96, r=128),   # largest rank
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"T{s.T}_d{s.d}_nq{s.nq}_nkv{s.nkv}_r{s.r}")
def test_qkv_parity_small(cuda_ok, shape):
    run_and_check(shape)


def test_qkv_zero_B(cuda_ok):
    """B = 0: the adapter-A gradients are exactly zero (Q_x = 0)."""
    shape = synth.QkvShape(T=256, d=256, nq=256, nkv=64, r=16)
    bits = synth.make_qkv_inputs_bits(shape)
    for k in ("Bq", "Bk", "Bv"):
        bits[k] = np.zeros_like(bits[k])
    pb = QkvProblem(shape, bits)
    pb.step()
    torch.cuda.synchronize()
    for k in ("dAq", "dAk", "dAv"):
        assert torch.all(pb.g[k] == 0), k


@pytest.mark.slow
def test_qkv_parity_llama3_8b(cuda_ok):
    """Full 8B attention shape (T = 8192, d = 4096, 32 + 8 + 8 heads of 128), every output
    against the oracle over all rows."""
    run_and_check(configs.QKV_8B)
