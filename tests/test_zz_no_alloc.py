"""The allocation-free projection entry point, for callers that cannot allocate
device memory themselves (for example a plugin whose host framework owns all device
memory and hands it only input and output buffers).

It must agree with the projection the forward writes into the saved context, on two
calls in a row (the calls share one fixed scratch array inside the library), and must
reject sizes beyond that array.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import ops, synth
from lora_fine_tuning_rmsnorm_b200.runner import Problem
from tests.parity import assert_close, to_np

pytestmark = pytest.mark.gpu


def test_noalloc_projection_matches_forward_context(cuda_ok):
    shape = synth.Shape(T=1000, d=512, f=768, r=24, alpha=16.0)
    pb = Problem(shape)
    pb.forward()
    torch.cuda.synchronize()
    sv = pb.saved()
    rp = ops.ctx_layout(pb.dims).rp
    H = sv["H"].contiguous()
    P_ref = sv["P"].float()
    for call, (adapter, col0) in enumerate((("Ag", 0), ("Au", rp))):
        out = torch.full((shape.T, rp), float("nan"), dtype=torch.bfloat16, device="cuda")
        ops.lora_lowrank_proj_noalloc(H, pb.t[adapter], out, shape.scale)
        torch.cuda.synchronize()
        ref = P_ref[:, col0:col0 + rp]
        assert torch.all(out[:, shape.r:] == 0), f"call {call}: padding columns not zero"
        assert_close(f"noalloc call {call}", to_np(out), to_np(ref), rel_fro=1e-3, max_rel=8e-3)


def test_noalloc_rejects_sizes_beyond_scratch(cuda_ok):
    L = ops.lib()
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    # 2^30 rows x 16 columns of fp32 partials is far above the fixed scratch
    rc = L.lora_lowrank_proj_noalloc(1 << 30, 64, 16, 1.0, ctypes.c_void_p(x.data_ptr()),
                                     ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(x.data_ptr()), None)
    assert rc == -3
    assert b"no-alloc scratch" in L.lora_mlp_last_error()
