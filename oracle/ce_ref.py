"""fp64 CPU oracle for the language-model head's cross-entropy loss, forward and backward,
as the fused chunked kernel computes it (the logits are a definition here, not an
output).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference arm may import or call anything under oracle/.  The CUDA
product path never does, and shares no code with it.

What the pages fix: the training forward ends with the loss computed from the final
hidden states in chunks, the logits tensor never existing in full and the model
returning a placeholder instead of logits; the cross-entropy kernel is one of the
hand-written kernels with a hand-derived backward ("Unsloth — 用手写 Triton kernel 给 HF
微调换心脏", §2.3 step 6, §4, §7: Fast_CrossEntropyLoss, unsloth_fused_ce_loss).

Readings taken (the pages print no formula; this is the Hugging Face causal-LM loss the
fused kernel replaces):
  * logits z = H W^T, H [T x d] the final normalised hidden states, W [V x d] the frozen
    LM head (not an adapted module), no bias;
  * per token, loss_t = logsumexp_v z_tv - z_{t, y_t}; a label outside [0, V) (the usual
    ignore index -100 included) leaves the token out;
  * the reduction is the mean over the tokens that are not left out (reduction "mean"),
    or their sum (reduction "sum"); with no token left, the loss and gradient are 0;
  * backward for an upstream gradient g of the reduced loss:
        dH_t = (g / n) sum_v (softmax(z_t)_v - [v = y_t]) W_v    (n = #tokens kept, or 1 for sum)
    and dH_t = 0 for tokens left out.  The labels are already shifted by the caller.
"""
from __future__ import annotations

import numpy as np


def logsumexp(z):
    m = z.max(axis=1, keepdims=True)
    return (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))[:, 0]


def valid(labels, V):
    return (labels >= 0) & (labels < V)


def forward(H, W, labels, reduction="mean"):
    """Per-token loss (0 where left out), lse, the reduced loss and the kept count."""
    V = W.shape[0]
    z = H @ W.T
    lse = logsumexp(z)
    ok = valid(labels, V)
    loss = np.zeros(H.shape[0])
    rows = np.nonzero(ok)[0]
    loss[rows] = lse[rows] - z[rows, labels[rows]]
    n = int(ok.sum())
    total = loss.sum()
    red = (total / n if n else 0.0) if reduction == "mean" else total
    return dict(loss_rows=loss, lse=lse, loss=red, n_valid=n)


def backward(H, W, labels, g=1.0, reduction="mean"):
    V = W.shape[0]
    ok = valid(labels, V)
    n = int(ok.sum())
    if n == 0:
        return np.zeros_like(H)
    scale = g / n if reduction == "mean" else g
    z = H @ W.T
    p = np.exp(z - logsumexp(z)[:, None])
    rows = np.nonzero(ok)[0]
    p[rows, labels[rows]] -= 1.0
    p[~ok] = 0.0
    return scale * (p @ W)


def rows_fwd_bwd(H, W, labels, rows, n_valid, g=1.0, reduction="mean"):
    """loss_t, lse_t and dH_t of selected rows only (every quantity is row-local given
    the kept count n_valid of the whole batch), for long inputs."""
    sub = forward(H[rows], W, labels[rows], reduction="sum")
    scale = (g / n_valid if n_valid else 0.0) if reduction == "mean" else g
    z = H[rows] @ W.T
    p = np.exp(z - sub["lse"][:, None])
    ok = valid(labels[rows], W.shape[0])
    idx = np.nonzero(ok)[0]
    p[idx, labels[rows][idx]] -= 1.0
    p[~ok] = 0.0
    return dict(loss_rows=sub["loss_rows"], lse=sub["lse"], dH=scale * (p @ W))
