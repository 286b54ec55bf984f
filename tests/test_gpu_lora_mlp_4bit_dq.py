"""GPU parity with double-quantised 4-bit weights (LORA_WFMT_4BIT_DQ): the block
constants are themselves quantised to 8-bit codes with an fp32 scale per 256 of them
(lora_quantize_absmax8), and each call expands them before the 4-bit GEMMs.

The 4-bit codes, the 8-bit constant codes and the second-level scales must match the
oracle bit for bit; the outputs must match the fp64 oracle run on the exactly
dequantised weights codebook[idx] * (scale2 * k / 255)."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, ops, synth
from lora_fine_tuning_rmsnorm_b200.runner import GRADS, Problem
from oracle import lora_mlp_ref as ref
from oracle import quant4_ref as q4
from tests.parity import assert_close, load_codebook, to_np

pytestmark = pytest.mark.gpu


def run(shape):
    bits = synth.make_inputs_bits(shape)
    pb = Problem(shape, bits)
    pb.use_4bit(load_codebook(), double_quant=True)
    assert pb.dims.wfmt == ops.WFMT_4BIT_DQ
    pb.Y.fill_(float("nan"))
    pb.dX.fill_(float("nan"))
    pb.step()
    torch.cuda.synchronize()
    assert ops.status(pb.ws) == 0
    inp = synth.bits_to_f64(bits)
    code = q4.codebook16()
    for k, name in (("g", "Wg"), ("u", "Wu"), ("d", "Wd")):
        idx, am = q4.quantize(inp[name], code)
        np.testing.assert_array_equal(q4.unpack(pb.q4[0][k].cpu().numpy()), idx, err_msg=name)
        np.testing.assert_array_equal(pb.q4[1][k].cpu().numpy(), am, err_msg=name)
        c8, s2 = q4.quantize_absmax8(am)
        np.testing.assert_array_equal(pb.dq[0][k].cpu().numpy(), c8, err_msg=name + " codes8")
        np.testing.assert_array_equal(pb.dq[1][k].cpu().numpy(), s2, err_msg=name + " scale2")
        inp[name] = q4.dequantize(idx, q4.dequantize_absmax8(c8, s2).astype(np.float64), code, inp[name].shape)
    R = ref.fwd_bwd(inp, shape.scale, shape.eps, chunk=1024, keep=("Y", "dX"))
    out = {"Y": to_np(pb.Y), "dX": to_np(pb.dX), **{k: to_np(v) for k, v in pb.g.items()}}
    for k in ("Y", "dX") + GRADS:
        assert_close(k, out[k], R[k])


@pytest.mark.parametrize("shape", [
    synth.Shape(T=200, d=256, f=512, r=16, alpha=16.0),   # 2048 constants: 8 second-level blocks
    synth.Shape(T=64, d=256, f=768, r=8, alpha=16.0),     # single-CTA tiles; 3072 constants
    synth.Shape(T=300, d=512, f=1280, r=32, alpha=16.0),  # 10240 constants
], ids=lambda s: f"T{s.T}_d{s.d}_f{s.f}_r{s.r}")
def test_fwd_bwd_parity_4bit_dq_small(cuda_ok, shape):
    run(shape)


@pytest.mark.slow
def test_fwd_bwd_parity_4bit_dq_llama3_8b(cuda_ok):
    run(configs.LLAMA3_8B)


def test_absmax8_quantiser_ragged_and_zero_blocks(cuda_ok):
    """n not a multiple of 256, an all-zero block and exact ties (510 a = (2j - 1) s)."""
    rng = np.random.default_rng(5)
    a = (np.abs(rng.standard_normal(1000)) * 0.05).astype(np.float32)
    a[256:512] = 0.0
    a[512] = np.float32(510.0)                      # block 2's scale
    a[513:517] = np.array([1.0, 3.0, 199.0, 509.0], dtype=np.float32)   # exact midpoints
    at = torch.from_numpy(a).cuda()
    c8 = torch.empty(a.size, dtype=torch.uint8, device="cuda")
    s2 = torch.empty(4, dtype=torch.float32, device="cuda")
    ops.lora_quantize_absmax8(at, c8, s2)
    torch.cuda.synchronize()
    rc, rs = q4.quantize_absmax8(a)
    np.testing.assert_array_equal(c8.cpu().numpy(), rc)
    np.testing.assert_array_equal(s2.cpu().numpy(), rs)
    assert list(rc[513:517]) == [0, 1, 99, 254] and rs[1] == 0 and np.all(rc[256:512] == 0)
