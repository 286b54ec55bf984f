"""GPU parity of the attention-side next rows through the C ABI against the fp64 oracles:
LoRA on o_proj (lora_o_fwd / lora_o_bwd) and the rotary embedding of Q and K (lora_rope,
forward and the sine-negated backward), at small ragged shapes and at the Llama-3-8B
attention shapes."""
import numpy as np
import pytest
import torch

from lora_fine_tuning_rmsnorm_b200 import configs, ops, synth
from lora_fine_tuning_rmsnorm_b200.runner import OProblem, RopeProblem
from oracle import lora_o_ref, rope_ref
from tests.parity import assert_close, to_np

pytestmark = pytest.mark.gpu

O_SHAPES = [synth.OShape(T=64, n_in=128, n_out=344, r=8),       # T < one tile, ragged n_out
            synth.OShape(T=200, n_in=136, n_out=200, r=8),      # ragged everywhere
            synth.OShape(T=384, n_in=256, n_out=512, r=16),
            synth.OShape(T=300, n_in=512, n_out=768, r=64, alpha=32.0),
            synth.OShape(T=160, n_in=384, n_out=256, r=128)]


def o_check(shape, chunk=4096):
    bits = synth.make_o_inputs_bits(shape)
    pb = OProblem(shape, bits)
    pb.Y.fill_(float("nan"))
    pb.dX.fill_(float("nan"))
    pb.dAo.fill_(float("nan"))
    pb.dBo.fill_(float("nan"))
    pb.step()
    torch.cuda.synchronize()
    assert ops.status(pb.ws) == 0
    R = lora_o_ref.fwd_bwd(synth.bits_to_f64(bits), shape.scale, chunk=chunk)
    for k, v in (("Y", pb.Y), ("dX", pb.dX), ("dAo", pb.dAo), ("dBo", pb.dBo)):
        assert_close(f"o_proj {k}", to_np(v), R[k])


@pytest.mark.parametrize("shape", O_SHAPES, ids=lambda s: f"T{s.T}_in{s.n_in}_out{s.n_out}_r{s.r}")
def test_o_proj_parity_small(cuda_ok, shape):
    o_check(shape)


@pytest.mark.slow
def test_o_proj_parity_llama3_8b(cuda_ok):
    o_check(configs.O_8B)


def rope_check(shape, data):
    pb = RopeProblem(shape, data)
    pb.step()
    torch.cuda.synchronize()
    assert ops.status() == 0
    f64 = {k: synth.bf16_bits_to_f64(data[k]) for k in ("Q", "K", "dQ", "dK")}
    cos, sin = data["cos"].astype(np.float64), data["sin"].astype(np.float64)
    Qo, Ko = rope_ref.forward(f64["Q"], f64["K"], data["pos"], cos, sin, shape.hd)
    dQ, dK = rope_ref.backward(f64["dQ"], f64["dK"], data["pos"], cos, sin, shape.hd)
    for name, got, ref in (("Q", pb.t["Q"], Qo), ("K", pb.t["K"], Ko), ("dQ", pb.t["dQ"], dQ), ("dK", pb.t["dK"], dK)):
        assert_close(f"rope {name}", to_np(got), ref, rel_fro=4e-3, max_rel=8e-3)
    return pb


@pytest.mark.parametrize("T,hq,hk,hd", [(77, 4, 2, 64), (256, 3, 1, 128), (33, 2, 2, 16), (512, 8, 0, 32)])
def test_rope_parity_small_packed_positions(cuda_ok, T, hq, hk, hd):
    shape = synth.RopeShape(T=T, hq=hq, hk=max(hk, 1), hd=hd, seq_len=64, base=10000.0)
    data = synth.make_rope_inputs(shape)
    data["pos"] = np.random.default_rng(T).integers(0, 64, T).astype(np.int32)   # packed: arbitrary ids
    if hk == 0:   # queries only
        shape = synth.RopeShape(T=T, hq=hq, hk=0, hd=hd, seq_len=64, base=10000.0)
        data["K"] = data["K"][:, :0]
        data["dK"] = data["dK"][:, :0]
        pb = RopeProblem(shape, data)
        pb.t["K"] = pb.t["dK"] = None
        pb.step()
        torch.cuda.synchronize()
        Qo = rope_ref.rotate(synth.bf16_bits_to_f64(data["Q"]), data["pos"], data["cos"].astype(np.float64),
                             data["sin"].astype(np.float64), hd)
        assert_close("rope Q only", to_np(pb.t["Q"]), Qo, rel_fro=4e-3, max_rel=8e-3)
        return
    rope_check(shape, data)


@pytest.mark.slow
def test_rope_parity_llama3_8b(cuda_ok):
    shape = configs.ROPE_8B
    rope_check(shape, synth.make_rope_inputs(shape))


def test_rope_backward_inverts_forward(cuda_ok):
    shape = synth.RopeShape(T=300, hq=4, hk=2, hd=128, seq_len=300, base=500000.0)
    data = synth.make_rope_inputs(shape)
    pb = RopeProblem(shape, data)
    q0 = pb.t["Q"].clone()
    pb.forward()
    ops.lora_rope(pb.t["Q"], pb.t["K"], pb.pos, pb.cos, pb.sin, shape.hd, backward=True)
    torch.cuda.synchronize()
    assert_close("R^T R Q", to_np(pb.t["Q"]), to_np(q0), rel_fro=6e-3, max_rel=1.6e-2)   # two bf16 roundings
    assert torch.equal(pb.t["Q"][0], q0[0])   # position 0: the identity, exactly


def test_rope_rejects_out_of_range_positions(cuda_ok):
    shape = synth.RopeShape(T=40, hq=2, hk=1, hd=64, seq_len=40, base=10000.0)
    data = synth.make_rope_inputs(shape)
    data["pos"][7] = 40          # one past the table
    pb = RopeProblem(shape, data)
    before = pb.t["Q"][7].clone()
    with pytest.raises(ops.LoraError) as ei:
        pb.forward()
    assert ei.value.code == -1
    assert torch.equal(pb.t["Q"][7], before)   # that row is left as it was
