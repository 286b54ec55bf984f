"""GPU parity of the whole LoRA-MLP forward + backward (lora_mlp_fwd / lora_mlp_bwd
through the C ABI) against the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, synth
from lora_fine_tuning_rmsnorm_b200.runner import GRADS, Problem
from oracle import lora_mlp_ref as ref
from tests.parity import assert_close, to_np

pytestmark = pytest.mark.gpu

CHECKED = ("Y", "dX") + GRADS


def run_gpu(shape, bits=None, poison=True):
    pb = Problem(shape, bits)
    if poison:
        pb.Y.fill_(float("nan"))
        pb.dX.fill_(float("nan"))
        for g in pb.g.values():
            g.fill_(float("nan"))
        pb.ctx.fill_(0xFF)
        pb.ws.fill_(0xFF)
    pb.step()
    torch.cuda.synchronize()
    return pb


def oracle_all(shape, bits, keep=("Y", "dX", "G", "U", "Act", "rstd", "H")):
    inp = synth.bits_to_f64(bits)
    return ref.fwd_bwd(inp, shape.scale, shape.eps, chunk=1024, keep=keep)


def compare(pb, R, names=CHECKED):
    out = {"Y": to_np(pb.Y), "dX": to_np(pb.dX)}
    out.update({k: to_np(v) for k, v in pb.g.items()})
    res = {}
    for k in names:
        res[k] = assert_close(k, out[k], R[k])
    return res


SMALL_SHAPES = [
    configs.TINY,                                         # T=64 < one M tile, f=344 ragged
    synth.Shape(T=200, d=136, f=200, r=8, alpha=16.0),   # ragged T, d, f
    synth.Shape(T=384, d=256, f=512, r=16, alpha=16.0),
    synth.Shape(T=256, d=192, f=320, r=24, alpha=32.0),  # r not a multiple of 16
    synth.Shape(T=300, d=512, f=768, r=64, alpha=16.0),
    synth.Shape(T=160, d=384, f=256, r=128, alpha=16.0), # 2r = 256 rank rows: two M tiles
]


@pytest.mark.parametrize("shape", SMALL_SHAPES, ids=lambda s: f"T{s.T}_d{s.d}_f{s.f}_r{s.r}")
def test_fwd_bwd_parity_small(cuda_ok, shape):
    bits = synth.make_inputs_bits(shape)
    pb = run_gpu(shape, bits)
    R = oracle_all(shape, bits)
    compare(pb, R)
    sv = pb.saved()
    np.testing.assert_allclose(to_np(sv["rstd"]), R["rstd"], rtol=2e-6)
    for k in ("H", "G", "U", "Act"):
        assert_close(k, to_np(sv[k]), R[k])


def test_zero_B_invariant_on_gpu(cuda_ok):
    shape = synth.Shape(T=256, d=256, f=384, r=16)
    bits = synth.make_inputs_bits(shape)
    for k in ("Bg", "Bu", "Bd"):
        bits[k] = np.zeros_like(bits[k])
    pb = run_gpu(shape, bits)
    for k in ("dAg", "dAu", "dAd"):
        assert torch.all(pb.g[k] == 0), k
    R = oracle_all(shape, bits)
    compare(pb, R, names=("Y", "dX", "dBg", "dBu", "dBd"))


def test_repeat_calls_identical_outputs(cuda_ok):
    shape = synth.Shape(T=512, d=256, f=512, r=16)
    pb = run_gpu(shape)
    y0, dx0 = pb.Y.clone(), pb.dX.clone()
    g0 = {k: v.clone() for k, v in pb.g.items()}
    pb.step()
    torch.cuda.synchronize()
    assert torch.equal(pb.Y, y0) and torch.equal(pb.dX, dx0)
    for k in GRADS:   # atomics: equal up to summation order
        torch.testing.assert_close(pb.g[k], g0[k], rtol=1e-5, atol=1e-6 * float(g0[k].abs().max()))


@pytest.mark.slow
def test_fwd_bwd_parity_llama32_1b_full(cuda_ok):
    shape = configs.LLAMA32_1B
    bits = synth.make_inputs_bits(shape)
    pb = run_gpu(shape, bits, poison=False)
    R = oracle_all(shape, bits, keep=("Y", "dX"))
    compare(pb, R)


@pytest.mark.slow
def test_fwd_bwd_parity_llama3_8b(cuda_ok):
    """Full 8B shape in the bench's launch configuration: every output tensor,
    against the oracle over all 8192 rows."""
    shape = configs.LLAMA3_8B
    bits = synth.make_inputs_bits(shape)
    pb = run_gpu(shape, bits, poison=False)
    R = oracle_all(shape, bits, keep=("Y", "dX"))
    compare(pb, R)


def test_host_pipeline_matches_device_step(cuda_ok):
    """Host-buffer driver (double-buffered copies, one stream per direction) returns the
    same Y, dX and gradients as the device-resident step."""
    from lora_fine_tuning_rmsnorm_b200 import dist as ldist
    from lora_fine_tuning_rmsnorm_b200.runner import HostPipeline, bf16_tensor
    shape = synth.Shape(T=384, d=256, f=512, r=16)
    bits = synth.make_inputs_bits(shape)
    pb = run_gpu(shape, bits, poison=False)
    pipe = HostPipeline(pb, bf16_tensor(bits["X"], "cpu", pin=True), bf16_tensor(bits["dY"], "cpu", pin=True))
    pipe.start()
    for i in range(3):
        pipe.step(i, 3)
    pipe.finish()
    torch.cuda.synchronize()
    assert torch.equal(pipe.hY, pb.Y.cpu()) and torch.equal(pipe.hdX, pb.dX.cpu())
    _, views = ldist.flat_grads(shape.d, shape.f, shape.r)
    off = 0
    for k in ldist.GRAD_ORDER:
        n = views[k].numel()
        got = pipe.hflat[off:off + n].view_as(views[k])
        torch.testing.assert_close(got, pb.g[k].cpu(), rtol=1e-5, atol=1e-6 * float(pb.g[k].abs().max()))
        off += n
