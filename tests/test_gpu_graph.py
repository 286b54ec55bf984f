"""The C-ABI calls under CUDA stream capture: the MLP and Q/K/V fwd+bwd captured into one
CUDA graph on a side stream and replayed, against the same calls run eagerly (every call
enqueues only kernels and memsets on the caller's stream, so a step can be captured once
and replayed without per-call host work).  Outputs that no atomic touches must match
bit for bit; the adapter gradients (fp32 atomics) to rounding.  In a fresh non-debug
process: debug mode synchronises after every call, which a capture does not allow."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

EXACT = ("mlp_Y", "mlp_dX", "qkv_dX", "qkv_Q", "qkv_K", "qkv_V")


def test_capture_and_replay_match_eager(cuda_ok, tmp_path):
    out = tmp_path / "graph.npz"
    env = dict(os.environ, LORA_MLP_DEBUG="0")
    subprocess.run([sys.executable, "-m", "tests.gpu_worker", "graph", str(out)], cwd=ROOT, env=env, check=True,
                   timeout=600)
    got = np.load(out)
    assert int(got["status"]) == 0
    names = [k[len("eager_"):] for k in got.files if k.startswith("eager_")]
    assert set(EXACT) <= set(names) and len(names) > len(EXACT)
    for k in names:
        e, r = got["eager_" + k], got["replay_" + k]
        assert np.all(np.isfinite(e)), k
        if k in EXACT:
            np.testing.assert_array_equal(r, e, err_msg=k)
        else:
            np.testing.assert_allclose(r, e, rtol=1e-5, atol=1e-6 * float(np.abs(e).max()), err_msg=k)
