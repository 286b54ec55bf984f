"""fp64 CPU oracle for the LoRA-augmented Llama MLP sub-block, forward and backward.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference arm may import or call anything under oracle/.  The CUDA
product path never does, and shares no code with it.

What it computes (plain definitions, float64, no rounding anywhere; bf16 inputs
are taken exactly):

  RMSNorm with cached rstd ("Unsloth提速秘诀：Triton内核如何加速反向传播", §3.2,
  the _rms_norm_forward_kernel description): mean of squares over the true column
  count, eps inside the square root, rstd kept for the backward, y = x * rstd * w.
  No bias (Llama), norm weight frozen.

  LoRA linear ("Unsloth 深度实战", §1.3, LoRALayer / LinearWithLoRA):
  y = x W^T + s (x A^T) B^T with A [r x in], B [out x r], s = alpha / r, base W frozen,
  no dropout (the fast path needs lora_dropout == 0: "Unsloth — 用手写 Triton kernel
  给 HF 微调换心脏", §5).

  SwiGLU MLP ("Unsloth — 用手写 Triton kernel 给 HF 微调换心脏", §2.3 and §7,
  swiglu_fg_kernel / LoRA_MLP): act = silu(gate) * up, silu(z) = z * sigmoid(z),
  then the LoRA-augmented down projection.  No residual connection: Y = MLP(RMSNorm(X)).

  Backward: the closed-form chain rule of the same expressions (the pages name a
  hand-derived LoRA_MLP backward that writes gradients directly, §4 of the same
  page, and the SiLU derivative, "Unsloth提速秘诀…", §2.2); gradients for X and for
  the six adapter matrices only (W and the norm weight are frozen).

Variants around the path (off by default):

  residual: the decoder layer adds the sub-block's output to its input, Y = X + MLP(RMSNorm(X)),
  so the backward adds dY to dX ("Unsloth加速原理揭秘", §3.1, the LoRA forward that ends in a
  residual add; the Llama residual stream).

  dw: gradient of the norm weight, for a trainable-norm variant (the norm weight is frozen in
  LoRA fine-tuning): H = X * rstd * w gives dw_j = sum_t dH_tj x_tj rstd_t
  ("Unsloth提速秘诀…", §3.2, the norm kernel's weight operand).

  merge: the adapter folded into the frozen weight for export, W + s B A ("Unsloth提速秘诀…",
  §3.1, "LoRA Update + Weight Merge"; "Unsloth 深度实战", §5.1, the merged 16-bit save).

Rows are independent in every step except the adapter-gradient reductions over T,
so long inputs are processed in row chunks with fp64 accumulation across chunks.
"""
from __future__ import annotations

import numpy as np


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    return z * sigmoid(z)


def silu_grad(z):
    """d/dz [z * sigmoid(z)] = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    sg = sigmoid(z)
    return sg * (1.0 + z * (1.0 - sg))


def rmsnorm_fwd(X, w, eps):
    """rstd_t = 1/sqrt(mean_j x_tj^2 + eps);  H = X * rstd[:, None] * w."""
    ms = np.mean(X * X, axis=1)
    rstd = 1.0 / np.sqrt(ms + eps)
    H = X * rstd[:, None] * w[None, :]
    return H, rstd


def rmsnorm_bwd(dH, X, w, rstd):
    """dX for H = X * rstd * w (rstd depending on X), using the cached rstd.

    With g = dH * w and xhat = X * rstd:  dX = rstd * (g - xhat * mean_j(g * xhat)).
    """
    g = dH * w[None, :]
    xhat = X * rstd[:, None]
    c = np.mean(g * xhat, axis=1)
    return rstd[:, None] * (g - xhat * c[:, None])


def lora_linear(x, W, A, B, s):
    """x W^T + s * (x A^T) B^T, in the pages' order (x @ A.T @ B.T * scaling)."""
    return x @ W.T + s * ((x @ A.T) @ B.T)


def merge(W, A, B, s):
    """The adapter folded into the frozen weight: W + s B A (W [out x in], B [out x r],
    A [r x in])."""
    return W + s * (B @ A)


def forward(X, w, eps, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual=False):
    """Full forward; returns every intermediate the backward needs.  With `residual`
    the sub-block's input is added to its output."""
    H, rstd = rmsnorm_fwd(X, w, eps)
    Pg = H @ Ag.T
    Pu = H @ Au.T
    G = H @ Wg.T + s * (Pg @ Bg.T)
    U = H @ Wu.T + s * (Pu @ Bu.T)
    Act = silu(G) * U
    Pd = Act @ Ad.T
    Y = Act @ Wd.T + s * (Pd @ Bd.T)
    if residual:
        Y = Y + X
    return dict(rstd=rstd, H=H, G=G, U=U, Act=Act, Pg=Pg, Pu=Pu, Pd=Pd, Y=Y)


def backward(fw, dY, X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual=False):
    """Gradients of <dY, Y> w.r.t. X, the six adapter matrices and the norm weight (dw,
    for the trainable-norm variant)."""
    H, G, U, Act = fw["H"], fw["G"], fw["U"], fw["Act"]
    Pg, Pu, Pd = fw["Pg"], fw["Pu"], fw["Pd"]
    # down projection  Y = Act Wd^T + s (Act Ad^T) Bd^T
    Qd = dY @ Bd                      # [T x r]
    dBd = s * (dY.T @ Pd)             # [d x r]
    dAd = s * (Qd.T @ Act)            # [r x f]
    dAct = dY @ Wd + s * (Qd @ Ad)    # [T x f]
    # SwiGLU  Act = silu(G) * U
    dG = dAct * U * silu_grad(G)
    dU = dAct * silu(G)
    # gate / up projections  G = H Wg^T + s (H Ag^T) Bg^T  (same for U)
    Qg = dG @ Bg
    Qu = dU @ Bu
    dBg = s * (dG.T @ Pg)
    dBu = s * (dU.T @ Pu)
    dAg = s * (Qg.T @ H)
    dAu = s * (Qu.T @ H)
    dH = dG @ Wg + dU @ Wu + s * (Qg @ Ag + Qu @ Au)
    dX = rmsnorm_bwd(dH, X, w, fw["rstd"])
    if residual:
        dX = dX + dY
    dw = np.sum(dH * X * fw["rstd"][:, None], axis=0)
    return dict(dX=dX, dAg=dAg, dBg=dBg, dAu=dAu, dBu=dBu, dAd=dAd, dBd=dBd, dw=dw,
                dAct=dAct, dG=dG, dU=dU, dH=dH, Qd=Qd, Qg=Qg, Qu=Qu)


_GRADS = ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd", "dw")


def fwd_bwd(inp: dict, s: float, eps: float, chunk: int = 2048, keep=("Y", "dX"), residual=False):
    """Forward + backward over all rows in chunks of `chunk` tokens.

    `inp` holds fp64 arrays X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, dY.
    Returns the per-row tensors named in `keep` (concatenated over chunks) and the
    six adapter gradients and dw summed over all rows.
    """
    X, dY = inp["X"], inp["dY"]
    W = {k: inp[k] for k in ("w", "Wg", "Wu", "Wd", "Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    T = X.shape[0]
    grads = None
    rows = {k: [] for k in keep}
    for t0 in range(0, T, chunk):
        xs, dys = X[t0:t0 + chunk], dY[t0:t0 + chunk]
        fw = forward(xs, W["w"], eps, W["Wg"], W["Wu"], W["Wd"], W["Ag"], W["Bg"],
                     W["Au"], W["Bu"], W["Ad"], W["Bd"], s, residual)
        bw = backward(fw, dys, xs, W["w"], W["Wg"], W["Wu"], W["Wd"], W["Ag"], W["Bg"],
                      W["Au"], W["Bu"], W["Ad"], W["Bd"], s, residual)
        both = {**fw, **bw}
        for k in keep:
            rows[k].append(both[k])
        if grads is None:
            grads = {k: bw[k].copy() for k in _GRADS}
        else:
            for k in _GRADS:
                grads[k] += bw[k]
    out = {k: np.concatenate(v, axis=0) for k, v in rows.items()}
    out.update(grads)
    return out


def sampled(inp: dict, s: float, eps: float, rows, cols, chunk: int = 4096):
    """Selected outputs of the same forward/backward, computed without the full
    [T x f] products, for long inputs:

      Y[rows], dX[rows]                 (every step is row-local given the weights)
      dBg[cols], dBu[cols], dAd[:, cols] (need only the columns `cols` of G, U, Act
                                          and dAct, over all T rows)

    Written from the same definitions as forward()/backward(), restricted to the
    requested rows / columns.
    """
    X, dY = inp["X"], inp["dY"]
    w, Wg, Wu, Wd = inp["w"], inp["Wg"], inp["Wu"], inp["Wd"]
    Ag, Bg, Au, Bu, Ad, Bd = (inp[k] for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd"))
    rows = np.asarray(rows)
    cols = np.asarray(cols)
    # row-local outputs
    fw = forward(X[rows], w, eps, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s)
    bw = backward(fw, dY[rows], X[rows], w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s)
    out = {"Y": fw["Y"], "dX": bw["dX"]}
    # column-restricted reductions over all rows
    dBg = np.zeros((cols.size, Bg.shape[1]))
    dBu = np.zeros((cols.size, Bu.shape[1]))
    dAd = np.zeros((Ad.shape[0], cols.size))
    for t0 in range(0, X.shape[0], chunk):
        H, _ = rmsnorm_fwd(X[t0:t0 + chunk], w, eps)
        dy = dY[t0:t0 + chunk]
        Pg, Pu = H @ Ag.T, H @ Au.T
        G = H @ Wg[cols].T + s * (Pg @ Bg[cols].T)
        U = H @ Wu[cols].T + s * (Pu @ Bu[cols].T)
        Act = silu(G) * U
        Qd = dy @ Bd
        dAct = dy @ Wd[:, cols] + s * (Qd @ Ad[:, cols])
        dG = dAct * U * silu_grad(G)
        dU = dAct * silu(G)
        dBg += s * (dG.T @ Pg)
        dBu += s * (dU.T @ Pu)
        dAd += s * (Qd.T @ Act)
    out.update(dBg=dBg, dBu=dBu, dAd=dAd)
    return out
