"""The allocation-free projection entry point, lora_lowrank_proj_noalloc.

It serves callers that cannot allocate device memory themselves: for example a plugin
inside a host framework that owns every device buffer and hands the plugin only its
inputs and outputs, so there is nowhere to put a workspace.  The entry point keeps its
K-split partial sums in a fixed array inside the library instead.

Checked here against the fp64 definition P = scale * X A^T on the same bf16 inputs (the
projection the forward stores for the LoRA term): two shapes with a ragged T and K
splits, called back to back and then repeated (every call shares the one scratch
array, so no state may carry over), a size exactly at the array's limit, and one just
past it that must be rejected.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import ops, synth
from lora_fine_tuning_rmsnorm_b200.runner import bf16_tensor
from tests.parity import assert_close, to_np

pytestmark = pytest.mark.gpu

SCRATCH_FLOATS = 4 << 20   # the library's fixed scratch: 16 MiB of fp32 partial sums


def inputs(T, K, r, seed):
    rng = np.random.default_rng(seed)
    Xb = synth.f32_to_bf16_bits(rng.standard_normal((T, K)).astype(np.float32))
    Ab = synth.f32_to_bf16_bits(rng.uniform(-1, 1, (r, K)).astype(np.float32) / np.float32(np.sqrt(K)))
    return Xb, Ab


def oracle_P(Xb, Ab, scale, rp):
    X, A = synth.bf16_bits_to_f64(Xb), synth.bf16_bits_to_f64(Ab)
    P = np.zeros((X.shape[0], rp))
    P[:, :A.shape[0]] = scale * (X @ A.T)
    return P


def call(Xb, Ab, scale):
    T, r = Xb.shape[0], Ab.shape[0]
    rp = (r + 15) // 16 * 16
    out = torch.full((T, rp), float("nan"), dtype=torch.bfloat16, device="cuda")
    ops.lora_lowrank_proj_noalloc(bf16_tensor(Xb), bf16_tensor(Ab), out, scale)
    torch.cuda.synchronize()
    assert ops.status() == 0
    return to_np(out), rp


# ragged T with 8 K splits; T not a multiple of 8 with 13 K splits (the split count
# follows T and K, so both shapes use most of the scratch's split structure)
SHAPES = [(1000, 512, 24, 2.0), (4099, 4096, 16, 1.0)]


def test_noalloc_matches_oracle_on_two_shapes_back_to_back(cuda_ok):
    data = [inputs(T, K, r, 11 + i) for i, (T, K, r, _) in enumerate(SHAPES)]
    order = [0, 1, 0]   # the repeat must not see anything the other shape left behind
    for call_no, i in enumerate(order):
        (Xb, Ab), scale = data[i], SHAPES[i][3]
        got, rp = call(Xb, Ab, scale)
        ref = oracle_P(Xb, Ab, scale, rp)
        r = Ab.shape[0]
        assert np.all(got[:, r:] == 0), f"call {call_no}: padding columns not zero"
        assert_close(f"noalloc call {call_no} (shape {i})", got, ref)


def test_noalloc_runs_exactly_at_the_scratch_limit(cuda_ok):
    # K = 64 is a single K block, hence one split: T x rp = 32768 x 128 = the whole array
    T, K, r = 32768, 64, 128
    assert T * 128 == SCRATCH_FLOATS
    Xb, Ab = inputs(T, K, r, 5)
    got, rp = call(Xb, Ab, 0.5)
    assert_close("noalloc at the limit", got, oracle_P(Xb, Ab, 0.5, rp))


def test_noalloc_rejects_sizes_past_the_scratch(cuda_ok):
    L = ops.lib()
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    p = ctypes.c_void_p(x.data_ptr())
    # one row more than fits (eight, to keep T a multiple of 8): rejected before any launch
    rc = L.lora_lowrank_proj_noalloc(32776, 64, 128, 1.0, p, p, p, None)
    assert rc == -3
    assert b"no-alloc scratch" in L.lora_mlp_last_error()
    rc = L.lora_lowrank_proj_noalloc(1 << 30, 64, 16, 1.0, p, p, p, None)
    assert rc == -3
