"""The GEMM mode with two M tiles per CTA-pair unit (MT = 2: every B stage shared by two
256-row tiles, one 512-column accumulator set in TMEM), forced on every GEMM that can take
it (gate/up, down, dAct, dH, bf16 and 4-bit, the cross-entropy's GEMMs, the Q/K/V and
o_proj GEMMs; the bf16 ones with their TMA-store epilogues) and run through the small
ragged parity suites against the oracle: units whose second M tile is partly or
wholly past the last row, ragged N, the LoRA K-extension, 4-bit expansion shared by both
tiles.  The tile choice only picks MT = 2 for large T, where the 8B and sweep tests cover
it; here the library reads LORA_MLP_MT=2 in a fresh process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SUITES = ["tests/test_gpu_lora_mlp.py::test_fwd_bwd_parity_small",
          "tests/test_gpu_lora_mlp_4bit.py::test_fwd_bwd_parity_4bit_small",
          "tests/test_gpu_lora_mlp_4bit_dq.py::test_fwd_bwd_parity_4bit_dq_small",
          "tests/test_gpu_ce.py::test_ce_parity_small",
          "tests/test_gpu_edge.py::test_saturated_silu_and_norm_edge_rows",
          "tests/test_gpu_qkv.py::test_qkv_parity_small",
          "tests/test_gpu_attn.py::test_o_proj_parity_small"]


def test_two_m_tiles_per_unit_forced(cuda_ok):
    env = dict(os.environ, LORA_MLP_MT="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", *SUITES], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
