"""The single-pass rank-r streaming kernel against the fp64 oracle.  By default it computes
Q = s X B together with dB = X^T P from one read of the activation gradient X (the down
branch, and gate/up together) and the reduction dAd = Qd^T Act; with LORA_MLP_DUAL=2 it
also computes the forward projections P, Pd (the row product alone, K-major operand) and
dAg, dAu (the column product alone, written transposed).  Shapes chosen for its work split:

* several CTAs per (row region, problem), so Q goes through the fp32 partial slots and is
  summed by the last CTA to arrive (arrival order varies from run to run: the result may
  not), with ragged T and ragged column groups;
* one column group per problem (K <= 128), so each CTA owns whole rows and writes Q directly;
* r > 64 (MMA N = 128, two row blocks per region) and r = 8 (padded to 16);
* two calls in a row on one workspace (the arrival counters are left at zero).

The workspace and outputs start poisoned (NaN / 0xFF).  The two-pass form
(LORA_MLP_DUAL=0: a projection GEMM and a reduction GEMM) and the all-products form
(LORA_MLP_DUAL=2) run the small MLP, Q/K/V and o_proj suites and these shapes in fresh
processes, since the library reads that setting once.  The Q/K/V and o_proj backward use
the kernel too (Q with dB per branch; dA_q, dA_k, dA_v from one read of H)."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import synth
from lora_fine_tuning_rmsnorm_b200.runner import GRADS, Problem
from tests.test_gpu_lora_mlp import compare, oracle_all, run_gpu
from tests.parity import to_np

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

DUAL_SHAPES = [
    synth.Shape(T=300, d=256, f=384, r=16, alpha=16.0),     # 3 and 2 CTAs per region: partial slots
    synth.Shape(T=1000, d=520, f=1032, r=72, alpha=16.0),   # r > 64: N = 128, ragged K groups
    synth.Shape(T=20000, d=64, f=128, r=16, alpha=16.0),    # K <= 128: Q written directly
    synth.Shape(T=129, d=136, f=136, r=8, alpha=8.0),       # one row past a block, 8-column tails
    synth.Shape(T=2100, d=512, f=1024, r=128, alpha=32.0),  # many CTAs per region, r = 128
]


@pytest.mark.parametrize("shape", DUAL_SHAPES, ids=lambda s: f"T{s.T}_d{s.d}_f{s.f}_r{s.r}")
def test_rank_r_pass_parity(cuda_ok, shape):
    bits = synth.make_inputs_bits(shape)
    pb = run_gpu(shape, bits)
    R = oracle_all(shape, bits)
    compare(pb, R)
    # a second call on the same workspace (the counters were left at zero): dX repeats exactly,
    # the adapter gradients up to the order of their fp32 atomics
    first = {k: to_np(v).copy() for k, v in pb.g.items()}
    dX0 = to_np(pb.dX).copy()
    pb.step()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(pb.dX), dX0)   # Q is summed in slot order: bit-identical
    for k in GRADS:
        np.testing.assert_allclose(to_np(pb.g[k]), first[k], rtol=1e-5, atol=1e-6)
    compare(pb, R)


@pytest.mark.parametrize("mode", ["0", "2"], ids=["two_pass", "all_products"])
def test_other_forms(cuda_ok, mode):
    env = dict(os.environ, LORA_MLP_DUAL=mode)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_gpu_lora_mlp.py::test_fwd_bwd_parity_small",
                        "tests/test_gpu_dual.py::test_rank_r_pass_parity",
                        "tests/test_gpu_qkv.py::test_qkv_parity_small",
                        "tests/test_gpu_attn.py::test_o_proj_parity_small"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
