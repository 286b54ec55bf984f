"""fp64 CPU oracle for a LoRA-augmented linear without a norm in front: the attention
output projection o_proj of a Llama decoder layer, forward and backward.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference arm may import or call anything under oracle/.  The CUDA
product path never does, and shares no code with it.

What it computes (plain definitions, float64, no rounding; bf16 inputs taken exactly):

  o_proj is one of the adapted modules of every LoRA configuration on the pages
  (target_modules q_proj, k_proj, v_proj, o_proj, gate_proj, up_proj, down_proj:
  "【编译】结合 Unsloth 与 🤗 TRL", §三.2; "Unsloth 深度实战", §3.2), and its adapter is the
  plain LoRA linear ("Unsloth 深度实战", §1.3, LoRALayer / LinearWithLoRA):

    Y = X Wo^T + s (X Ao^T) Bo^T,   X [T x n_in] (the attention output), Wo [n_out x n_in],
    Ao [r x n_in], Bo [n_out x r], s = alpha / r, Wo frozen, no dropout, no bias.

  Backward from dY (gradient of <dY, Y>), frozen Wo:
    Qo = dY Bo [T x r];  dX = dY Wo + s Qo Ao;  dAo = s Qo^T X;  dBo = s dY^T (X Ao^T).
"""
from __future__ import annotations

import numpy as np

from oracle.lora_mlp_ref import lora_linear


def forward(X, Wo, Ao, Bo, s):
    P = X @ Ao.T
    return dict(P=P, Y=lora_linear(X, Wo, Ao, Bo, s))


def backward(fw, dY, X, Wo, Ao, Bo, s):
    Qo = dY @ Bo
    return dict(Qo=Qo, dX=dY @ Wo + s * (Qo @ Ao), dAo=s * (Qo.T @ X), dBo=s * (dY.T @ fw["P"]))


def fwd_bwd(inp: dict, s: float, chunk: int = 4096):
    """Y and dX over all rows (in chunks), dAo and dBo summed over all rows."""
    X, dY = inp["X"], inp["dY"]
    Ys, dXs, dA, dB = [], [], 0.0, 0.0
    for t0 in range(0, X.shape[0], chunk):
        fw = forward(X[t0:t0 + chunk], inp["Wo"], inp["Ao"], inp["Bo"], s)
        bw = backward(fw, dY[t0:t0 + chunk], X[t0:t0 + chunk], inp["Wo"], inp["Ao"], inp["Bo"], s)
        Ys.append(fw["Y"])
        dXs.append(bw["dX"])
        dA = dA + bw["dAo"]
        dB = dB + bw["dBo"]
    return dict(Y=np.concatenate(Ys), dX=np.concatenate(dXs), dAo=dA, dBo=dB)
