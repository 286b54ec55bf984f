"""fp64 CPU oracle for the LoRA-augmented Q/K/V projections of a Llama attention block,
forward and backward.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference arm may import or call anything under oracle/.  The CUDA
product path never does, and shares no code with it.

What it computes (plain definitions, float64, no rounding; bf16 inputs taken exactly):

  The decoder layer's attention half starts with the RMSNorm kernel and then the Q/K/V
  projections with the LoRA forward written by hand ("Unsloth — 用手写 Triton kernel 给 HF
  微调换心脏", §2.3, the per-layer forward order, and §7, LoRA_QKV / apply_lora_qkv; the
  adapted modules q_proj, k_proj, v_proj: "Unsloth 深度实战", §4):

    H = RMSNorm(X) (cached rstd, as for the MLP)
    Q = H Wq^T + s (H Aq^T) Bq^T,  K = H Wk^T + s (H Ak^T) Bk^T,  V = H Wv^T + s (H Av^T) Bv^T

  Wq [nq x d], Wk, Wv [nkv x d] (nkv < nq: grouped-query attention), A [r x d], B [n x r].

  Backward from dQ, dK, dV (what the attention backward returns): the chain rule of the
  same expressions, frozen W and norm weight, gradients for X and the six adapters.
"""
from __future__ import annotations

import numpy as np

from oracle.lora_mlp_ref import rmsnorm_bwd, rmsnorm_fwd

_NAMES = ("q", "k", "v")


def forward(X, w, eps, Wq, Wk, Wv, Aq, Bq, Ak, Bk, Av, Bv, s):
    H, rstd = rmsnorm_fwd(X, w, eps)
    out = dict(rstd=rstd, H=H)
    for n, W, A, B in zip(_NAMES, (Wq, Wk, Wv), (Aq, Ak, Av), (Bq, Bk, Bv)):
        P = H @ A.T
        out["P" + n] = P
        out[n.upper()] = H @ W.T + s * (P @ B.T)
    return out


def backward(fw, dQ, dK, dV, X, w, Wq, Wk, Wv, Aq, Bq, Ak, Bk, Av, Bv, s):
    H = fw["H"]
    out = {}
    dH = np.zeros_like(H)
    for n, dZ, W, A, B in zip(_NAMES, (dQ, dK, dV), (Wq, Wk, Wv), (Aq, Ak, Av), (Bq, Bk, Bv)):
        Qx = dZ @ B                               # [T x r]
        out["dB" + n] = s * (dZ.T @ fw["P" + n])  # [n x r]
        out["dA" + n] = s * (Qx.T @ H)            # [r x d]
        dH += dZ @ W + s * (Qx @ A)
    out["dH"] = dH
    out["dX"] = rmsnorm_bwd(dH, X, w, fw["rstd"])
    return out


GRADS = ("dAq", "dBq", "dAk", "dBk", "dAv", "dBv")
_W = ("w", "Wq", "Wk", "Wv", "Aq", "Bq", "Ak", "Bk", "Av", "Bv")


def fwd_bwd(inp: dict, s: float, eps: float, chunk: int = 2048, keep=("Q", "K", "V", "dX")):
    """Forward + backward over all rows in chunks; per-row tensors in `keep` concatenated,
    the six adapter gradients summed over all rows."""
    X = inp["X"]
    grads = None
    rows = {k: [] for k in keep}
    for t0 in range(0, X.shape[0], chunk):
        sl = slice(t0, t0 + chunk)
        fw = forward(X[sl], inp["w"], eps, *(inp[k] for k in _W[1:]), s)
        bw = backward(fw, inp["dQ"][sl], inp["dK"][sl], inp["dV"][sl], X[sl], *(inp[k] for k in _W), s)
        both = {**fw, **bw}
        for k in keep:
            rows[k].append(both[k])
        if grads is None:
            grads = {k: bw[k].copy() for k in GRADS}
        else:
            for k in GRADS:
                grads[k] += bw[k]
    out = {k: np.concatenate(v, axis=0) for k, v in rows.items()}
    out.update(grads)
    return out
