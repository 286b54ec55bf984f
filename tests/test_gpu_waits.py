"""The bounded device waits, made to run out on purpose without faulting the GPU.

lora_gemm_bf16 with LORA_GEMM_TEST_NO_LOADS runs the single-CTA GEMM with a copy warp
that issues no loads and arms no barrier: nothing is ever in flight, so the MMA and
epilogue waits give up after LORA_MLP_WAIT_LIMIT_MS, the kernel records a status code,
frees its tensor memory and returns.  The call must report LORA_ERR_TIMEOUT (debug mode,
in this process) or leave the code for lora_mlp_status (non-debug, in a fresh process),
and the next normal call on the same stream must compute the right result."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import ops, synth
from lora_fine_tuning_rmsnorm_b200.runner import Problem, bf16_tensor
from oracle import lora_mlp_ref as ref
from tests.parity import assert_close, to_np

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WAIT_CODES = (0x100, 0x200, 0x300)   # producer, MMA or epilogue wait gave up (never a drain wait)


def gemm_inputs():
    rng = np.random.default_rng(7)
    Ab = synth.f32_to_bf16_bits(rng.standard_normal((256, 192)).astype(np.float32))
    Bb = synth.f32_to_bf16_bits(rng.standard_normal((128, 192)).astype(np.float32))
    return Ab, Bb


def gemm_ref(Ab, Bb):
    return synth.bf16_bits_to_f64(Ab) @ synth.bf16_bits_to_f64(Bb).T


def test_wait_runs_out_then_context_is_usable(cuda_ok, monkeypatch):
    Ab, Bb = gemm_inputs()
    A, B = bf16_tensor(Ab), bf16_tensor(Bb)
    C = torch.zeros(256, 128, dtype=torch.float32, device="cuda")
    monkeypatch.setenv("LORA_MLP_WAIT_LIMIT_MS", "50")
    with pytest.raises(ops.LoraError) as ei:
        ops.lora_gemm_bf16(A, 0, B, 0, C, test_no_loads=True)
    assert ei.value.code == -5
    assert ops.status() in WAIT_CODES
    monkeypatch.setenv("LORA_MLP_WAIT_LIMIT_MS", "3000")
    ops.lora_gemm_bf16(A, 0, B, 0, C)
    torch.cuda.synchronize()
    assert ops.status() == 0
    R = gemm_ref(Ab, Bb)
    np.testing.assert_allclose(to_np(C), R, rtol=0, atol=1e-5 * np.abs(R).max() * 2)
    # a whole fwd + bwd on the same stream afterwards
    shape = synth.Shape(T=200, d=136, f=200, r=8, alpha=16.0)
    bits = synth.make_inputs_bits(shape)
    pb = Problem(shape, bits)
    pb.step()
    torch.cuda.synchronize()
    assert ops.status(pb.ws) == 0
    Ro = ref.fwd_bwd(synth.bits_to_f64(bits), shape.scale, shape.eps, keep=("Y", "dX"))
    assert_close("Y after a timeout", to_np(pb.Y), Ro["Y"])
    assert_close("dX after a timeout", to_np(pb.dX), Ro["dX"])


def test_pair_tiles_refuse_the_test_flag(cuda_ok):
    x = torch.zeros(256, 64, dtype=torch.bfloat16, device="cuda")
    C = torch.zeros(256, 256, dtype=torch.float32, device="cuda")
    with pytest.raises(ops.LoraError) as ei:
        ops.lora_gemm_bf16(x, 0, x, 0, C, pair=True, test_no_loads=True)
    assert ei.value.code == -1


def test_status_query_outside_debug_mode(cuda_ok, tmp_path):
    out = tmp_path / "stall.npz"
    env = dict(os.environ, LORA_MLP_DEBUG="0", LORA_MLP_WAIT_LIMIT_MS="50")
    subprocess.run([sys.executable, "-m", "tests.gpu_worker", "stall", str(out)], cwd=ROOT, env=env, check=True,
                   timeout=300)
    got = np.load(out)
    assert int(got["code_stall"]) in WAIT_CODES
    assert int(got["code_after"]) == 0
    R = gemm_ref(got["A"], got["B"])
    np.testing.assert_allclose(got["C"], R, rtol=0, atol=1e-5 * np.abs(R).max() * 2)
