"""Edge cases of the method on the GPU against the fp64 oracle, and the asynchronous
(non-debug) path at the 8B shape.

* Saturated SiLU: two gate columns reach |G| of several hundred, where sigmoid(G) is 0 or
  1 to fp32 precision on both sides (e^-G overflows or vanishes in the kernel's exp).
  Those columns of the down weight are scaled down by the same factor: with G stored in
  bf16 (as the method saves it), a gate of that size carries an absolute rounding error
  of about 2^-9 |G|, which moves silu' inside its transition band; left uncompensated,
  that alone takes the outputs past the 5e-3 bar whatever the kernel does (a CPU
  emulation of the bf16 storage chain reproduces it).
* RMSNorm rows at the edges of eps: an all-zero row (rstd = 1/sqrt(eps), H = 0), a row
  whose mean square is about eps, and a row a thousand times larger than the rest.
* The bench's launch configuration without LORA_MLP_DEBUG (no synchronisation or status
  read between the calls; the tests otherwise run in debug mode), in a fresh process
  because the library reads that setting once."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, synth
from lora_fine_tuning_rmsnorm_b200.runner import GRADS, Problem
from oracle import lora_mlp_ref as ref
from tests.parity import assert_close, to_np

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def edge_bits(shape, cols=(3, 101), scale=600.0):
    """The seeded inputs with two gate rows of Wg scaled by `scale` (so G reaches several
    hundred in those columns: sigmoid saturates and e^-G overflows fp32 past |G| = 88)
    and the same columns of Wd scaled by 1/scale (so Act Wd^T, dAct and dH stay at the
    scale of the other columns), plus four special rows of X."""
    raw = {n: synth.tensor_f64(n, shape) for n in synth.TENSOR_ORDER}
    raw["Wg"][list(cols)] *= scale
    raw["Wd"][:, list(cols)] /= scale
    raw["X"][0] = 0.0            # all-zero row
    raw["X"][1] *= 1e-3          # mean square ~ 1e-6 = eps
    raw["X"][2] *= 1e3           # large row
    raw["X"][shape.T - 1] = 0.0  # zero row in the ragged last tile
    return {k: synth.f32_to_bf16_bits(v.astype(np.float32)) for k, v in raw.items()}


@pytest.mark.parametrize("shape", [synth.Shape(T=300, d=256, f=384, r=16, alpha=16.0),
                                   synth.Shape(T=120, d=384, f=512, r=16, alpha=16.0)],
                         ids=["pair_T300", "single_T120"])
def test_saturated_silu_and_norm_edge_rows(cuda_ok, shape):
    bits = edge_bits(shape)
    pb = Problem(shape, bits)
    pb.step()
    torch.cuda.synchronize()
    R = ref.fwd_bwd(synth.bits_to_f64(bits), shape.scale, shape.eps, keep=("Y", "dX", "G", "rstd"))
    assert (R["G"] < -88).sum() > 20 and (R["G"] > 88).sum() > 20   # past the fp32 exp overflow, both signs
    np.testing.assert_allclose(R["rstd"][0], 1.0 / np.sqrt(shape.eps))
    sv = pb.saved()
    np.testing.assert_allclose(to_np(sv["rstd"]), R["rstd"], rtol=2e-6)
    assert torch.all(sv["H"][0] == 0) and torch.all(sv["H"][shape.T - 1] == 0)
    out = {"Y": to_np(pb.Y), "dX": to_np(pb.dX), **{k: to_np(v) for k, v in pb.g.items()}}
    for k in ("Y", "dX") + GRADS:
        assert_close(k, out[k], R[k])
    assert np.all(out["Y"][0] == 0) and np.all(out["dX"][0] == 0)   # exact zeros on both sides


@pytest.mark.slow
def test_nondebug_path_llama3_8b(cuda_ok, tmp_path):
    out = tmp_path / "mlp8b.npz"
    env = dict(os.environ, LORA_MLP_DEBUG="0")
    subprocess.run([sys.executable, "-m", "tests.gpu_worker", "mlp8b", str(out)], cwd=ROOT, env=env, check=True,
                   timeout=600)
    got = np.load(out)
    assert int(got["status"]) == 0
    shape = configs.LLAMA3_8B
    R = ref.fwd_bwd(synth.bits_to_f64(synth.make_inputs_bits(shape)), shape.scale, shape.eps, keep=("Y", "dX"))
    for k in ("Y", "dX") + GRADS:
        assert_close(f"non-debug {k}", got[k], R[k])
