"""GPU parity of the LoRA-MLP forward + backward with 4-bit frozen weights (codes
expanded to bf16 inside the GEMMs) against the fp64 oracle run on the exactly
dequantised weights codebook[idx] * absmax.  The codes themselves must match the
oracle's quantiser bit for bit."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, synth
from lora_fine_tuning_rmsnorm_b200.runner import GRADS, Problem
from oracle import lora_mlp_ref as ref
from oracle import quant4_ref as q4
from tests.parity import assert_close, load_codebook, to_np

pytestmark = pytest.mark.gpu


def oracle_4bit_inputs(bits):
    inp = synth.bits_to_f64(bits)
    code = q4.codebook16()
    codes = {}
    for k in ("Wg", "Wu", "Wd"):
        idx, am = q4.quantize(inp[k], code)
        codes[k] = (idx, am)
        inp[k] = q4.dequantize(idx, am, code, inp[k].shape)
    return inp, codes


def run(shape, keep=("Y", "dX")):
    bits = synth.make_inputs_bits(shape)
    pb = Problem(shape, bits)
    pb.use_4bit(load_codebook())
    pb.Y.fill_(float("nan"))
    pb.dX.fill_(float("nan"))
    pb.step()
    torch.cuda.synchronize()
    inp, codes = oracle_4bit_inputs(bits)
    for k, name in (("g", "Wg"), ("u", "Wu"), ("d", "Wd")):
        gq, ga = pb.q4[0][k].cpu().numpy(), pb.q4[1][k].cpu().numpy()
        np.testing.assert_array_equal(q4.unpack(gq), codes[name][0], err_msg=name)
        np.testing.assert_array_equal(ga, codes[name][1], err_msg=name)
    R = ref.fwd_bwd(inp, shape.scale, shape.eps, chunk=1024, keep=keep)
    out = {"Y": to_np(pb.Y), "dX": to_np(pb.dX), **{k: to_np(v) for k, v in pb.g.items()}}
    for k in ("Y", "dX") + GRADS:
        assert_close(k, out[k], R[k])
    return pb


@pytest.mark.parametrize("shape", [
    synth.Shape(T=200, d=256, f=512, r=16, alpha=16.0),
    synth.Shape(T=300, d=512, f=768, r=32, alpha=16.0),
    synth.Shape(T=64, d=256, f=256, r=8, alpha=16.0),     # T <= 128: single-CTA tiles (no pairs)
    synth.Shape(T=2200, d=256, f=512, r=16, alpha=16.0),  # CTA pairs, banded tile order, ragged T
], ids=lambda s: f"T{s.T}_d{s.d}_f{s.f}_r{s.r}")
def test_fwd_bwd_parity_4bit_small(cuda_ok, shape):
    run(shape)


@pytest.mark.slow
def test_fwd_bwd_parity_4bit_llama3_8b(cuda_ok):
    run(configs.LLAMA3_8B)
