"""Runs one GPU workload in a fresh process and saves its outputs (.npz), for the tests
that need a process-wide setting the library reads once (LORA_MLP_DEBUG): the parity
run of the asynchronous, non-debug path and the status query outside debug mode.

    python -m tests.gpu_worker mlp8b OUT.npz      # 8B-shaped fwd+bwd, as bench.py runs it
    python -m tests.gpu_worker stall OUT.npz      # a GEMM whose waits run out, then a normal one
    python -m tests.gpu_worker graph OUT.npz      # fwd+bwd captured in a CUDA graph and replayed
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def mlp8b(out_path):
    import torch
    from lora_fine_tuning_rmsnorm_b200 import configs, ops, synth
    from lora_fine_tuning_rmsnorm_b200.runner import GRADS, Problem
    shape = configs.LLAMA3_8B
    pb = Problem(shape, synth.make_inputs_bits(shape))
    for _ in range(2):          # repeated steps, no synchronisation between the calls
        pb.step()
    code = ops.status(pb.ws)
    torch.cuda.synchronize()
    arrays = {"Y": pb.Y, "dX": pb.dX, **pb.g}
    np.savez(out_path, status=np.int32(code), **{k: v.float().cpu().numpy() for k, v in arrays.items()})


def stall(out_path):
    import torch
    from lora_fine_tuning_rmsnorm_b200 import ops, synth
    from lora_fine_tuning_rmsnorm_b200.runner import bf16_tensor
    rng = np.random.default_rng(7)
    Ab = synth.f32_to_bf16_bits(rng.standard_normal((256, 192)).astype(np.float32))
    Bb = synth.f32_to_bf16_bits(rng.standard_normal((128, 192)).astype(np.float32))
    A, B = bf16_tensor(Ab), bf16_tensor(Bb)
    C = torch.zeros(256, 128, dtype=torch.float32, device="cuda")
    ops.lora_gemm_bf16(A, 0, B, 0, C, test_no_loads=True)   # returns at once outside debug mode
    code_stall = ops.status()
    ops.lora_gemm_bf16(A, 0, B, 0, C)
    code_after = ops.status()
    np.savez(out_path, code_stall=np.int32(code_stall), code_after=np.int32(code_after), C=C.cpu().numpy(),
             A=Ab, B=Bb)


def graph(out_path):
    """The MLP and Q/K/V fwd+bwd called eagerly, then captured once into one CUDA graph on a
    side torch stream and replayed twice: outputs of the eager calls and of the replays."""
    import torch
    from lora_fine_tuning_rmsnorm_b200 import ops, synth
    from lora_fine_tuning_rmsnorm_b200.runner import QkvProblem, Problem
    mlp = Problem(synth.Shape(T=1000, d=256, f=640, r=16, alpha=16.0))
    qkv = QkvProblem(synth.QkvShape(T=600, d=256, nq=256, nkv=64, r=16))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())

    def step():
        mlp.step(stream=s)
        qkv.step(stream=s)

    def snapshot():
        torch.cuda.synchronize()
        out = {"mlp_Y": mlp.Y, "mlp_dX": mlp.dX, **{"mlp_" + k: v for k, v in mlp.g.items()},
               "qkv_dX": qkv.dX, **{"qkv_" + k: v for k, v in qkv.out.items()},
               **{"qkv_g_" + k: v for k, v in qkv.g.items()}}
        return {k: v.float().cpu().numpy().copy() for k, v in out.items()}

    with torch.cuda.stream(s):
        step()
    eager = snapshot()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for k in range(2):
        g.replay()
    replay = snapshot()
    code = ops.status(mlp.ws)
    np.savez(out_path, status=np.int32(code), **{"eager_" + k: v for k, v in eager.items()},
             **{"replay_" + k: v for k, v in replay.items()})


if __name__ == "__main__":
    {"mlp8b": mlp8b, "stall": stall, "graph": graph}[sys.argv[1]](sys.argv[2])
