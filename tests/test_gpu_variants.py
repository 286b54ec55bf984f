"""GPU parity of the variants around the path, against the fp64 oracle on the same seeded
inputs: the residual connection (Y = X + MLP(RMSNorm(X)), dX += dY), the norm-weight
gradient dw of a trainable-norm variant, and the weight merge W + s B A for export."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, ops, synth
from lora_fine_tuning_rmsnorm_b200.runner import GRADS, Problem
from oracle import lora_mlp_ref as ref
from oracle import quant4_ref as q4
from tests.parity import assert_close, load_codebook, to_np

pytestmark = pytest.mark.gpu


def run(shape, residual, norm_grad, bits4=False):
    bits = synth.make_inputs_bits(shape)
    pb = Problem(shape, bits, residual=residual, norm_grad=norm_grad)
    if bits4:
        pb.use_4bit(load_codebook())
    pb.Y.fill_(float("nan"))
    pb.dX.fill_(float("nan"))
    if pb.dw is not None:
        pb.dw.fill_(float("nan"))
    pb.step()
    torch.cuda.synchronize()
    inp = synth.bits_to_f64(bits)
    if bits4:
        code = q4.codebook16()
        for k in ("Wg", "Wu", "Wd"):
            idx, am = q4.quantize(inp[k], code)
            inp[k] = q4.dequantize(idx, am, code, inp[k].shape)
    R = ref.fwd_bwd(inp, shape.scale, shape.eps, chunk=1024, residual=residual)
    return pb, R


def check(pb, R, with_dw):
    out = {"Y": to_np(pb.Y), "dX": to_np(pb.dX), **{k: to_np(v) for k, v in pb.g.items()}}
    for k in ("Y", "dX") + GRADS:
        assert_close(k, out[k], R[k])
    if with_dw:
        assert_close("dw", to_np(pb.dw), R["dw"])


SHAPES = [
    synth.Shape(T=200, d=136, f=200, r=8, alpha=16.0),    # ragged, CTA pairs
    synth.Shape(T=64, d=256, f=344, r=16, alpha=16.0),    # one M tile
    synth.Shape(T=384, d=512, f=768, r=32, alpha=16.0),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"T{s.T}_d{s.d}_f{s.f}_r{s.r}")
def test_residual_and_norm_grad_parity(cuda_ok, shape):
    pb, R = run(shape, residual=True, norm_grad=True)
    check(pb, R, with_dw=True)


def test_norm_grad_without_residual(cuda_ok):
    pb, R = run(synth.Shape(T=300, d=256, f=512, r=16, alpha=16.0), residual=False, norm_grad=True)
    check(pb, R, with_dw=True)


def test_residual_4bit(cuda_ok):
    pb, R = run(synth.Shape(T=300, d=256, f=512, r=16, alpha=16.0), residual=True, norm_grad=False, bits4=True)
    check(pb, R, with_dw=False)


def test_residual_off_is_the_sub_block(cuda_ok):
    """residual = 1 changes Y by X and dX by dY (up to bf16 rounding of the sums) and
    leaves the adapter gradients as they are."""
    shape = synth.Shape(T=256, d=256, f=384, r=16, alpha=16.0)
    bits = synth.make_inputs_bits(shape)
    a = Problem(shape, bits)
    b = Problem(shape, bits, residual=True)
    a.step(); b.step()
    torch.cuda.synchronize()
    X, dY = a.t["X"].float(), a.t["dY"].float()
    torch.testing.assert_close(b.Y.float(), a.Y.float() + X, rtol=1e-2, atol=1e-2)
    torch.testing.assert_close(b.dX.float(), a.dX.float() + dY, rtol=1e-2, atol=1e-2)
    for k in GRADS:
        torch.testing.assert_close(b.g[k], a.g[k], rtol=1e-5, atol=1e-6 * float(a.g[k].abs().max()))


def _bf16(a):
    return torch.from_numpy(synth.f32_to_bf16_bits(a.astype(np.float32)).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("rows,cols,r", [(200, 136, 8), (512, 1024, 16), (33, 4096, 128), (7, 8, 1)])
def test_merge_weights_parity(cuda_ok, rows, cols, r):
    """Every element within one bf16 rounding of the exact W + s B A; in place equals out of
    place bit for bit."""
    rng = np.random.default_rng(rows * 131 + cols + r)
    W, A, B = (_bf16(rng.standard_normal(sh)) for sh in ((rows, cols), (r, cols), (rows, r)))
    s = 0.75
    Wd, Ad, Bd = W.cuda(), A.cuda(), B.cuda()
    out = ops.merge_weights(Wd, Ad, Bd, s)
    torch.cuda.synchronize()
    exact = ref.merge(W.double().numpy(), A.double().numpy(), B.double().numpy(), s)
    got = out.double().cpu().numpy()
    err = np.abs(got - exact)
    # bf16 round-to-nearest: <= 2^-9 relative, plus the fp32 sum's own error
    assert np.all(err <= 2.0 ** -8 * np.abs(exact) + 1e-6 * r), float((err / (np.abs(exact) + 1e-30)).max())
    inplace = Wd.clone()
    ops.merge_weights(inplace, Ad, Bd, s, out=inplace)
    torch.cuda.synchronize()
    assert torch.equal(inplace, out)


def test_merged_weights_reproduce_the_adapter_forward(cuda_ok):
    """The GPU forward with the GPU-merged weights (B = 0) matches the oracle on those
    merged weights, and they reproduce the adapter forward of the oracle within the
    bf16 storage rounding of the merged weights (W + s B A is exact only in fp64)."""
    shape = synth.Shape(T=256, d=256, f=512, r=16, alpha=16.0)
    bits = synth.make_inputs_bits(shape)
    # B ~ N(0, 0.5) instead of N(0, 0.01): the adapter term is then of the size of W, so a
    # wrong merge cannot hide inside the tolerance
    rng = np.random.default_rng(7)
    for k in ("Bg", "Bu", "Bd"):
        bits[k] = synth.f32_to_bf16_bits((0.5 * rng.standard_normal(bits[k].shape)).astype(np.float32))
    b = Problem(shape, bits)
    for W, A, B in (("Wg", "Ag", "Bg"), ("Wu", "Au", "Bu"), ("Wd", "Ad", "Bd")):
        ops.merge_weights(b.t[W], b.t[A], b.t[B], shape.scale, out=b.t[W])
        b.t[B].zero_()
    b.forward()
    torch.cuda.synchronize()
    inp = synth.bits_to_f64(bits)
    names = ("Wg", "Wu", "Wd", "Ag", "Bg", "Au", "Bu", "Ad", "Bd")
    with_adapters = ref.forward(inp["X"], inp["w"], shape.eps, *(inp[k] for k in names), shape.scale)["Y"]
    merged = dict(inp)
    for k in ("Wg", "Wu", "Wd", "Bg", "Bu", "Bd"):
        merged[k] = b.t[k].double().cpu().numpy()
    on_merged = ref.forward(inp["X"], inp["w"], shape.eps, *(merged[k] for k in names), shape.scale)["Y"]
    assert_close("Y (GPU, merged W)", to_np(b.Y), on_merged)
    assert_close("Y (oracle, merged bf16 W vs adapters)", on_merged, with_adapters)


@pytest.mark.slow
def test_residual_and_norm_grad_llama32_1b(cuda_ok):
    """1B shape (T = 8192, d = 2048, f = 8192), residual + dw, every output against the oracle."""
    pb, R = run(configs.LLAMA32_1B, residual=True, norm_grad=True)
    check(pb, R, with_dw=True)
