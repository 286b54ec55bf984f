"""fp64 CPU oracle for the rotary position embedding (RoPE) applied to the query and key
heads, forward and backward.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference arm may import or call anything under oracle/.  The CUDA
product path never does, and shares no code with it.

What the pages fix: each decoder layer runs a RoPE kernel on Q and K right after the
Q/K/V projections, writing in place ("Unsloth — 用手写 Triton kernel 给 HF 微调换心脏",
§2.3), the rotation of q at its position and of k at its position is fused into one
kernel that looks the tables up by position ("Unsloth加速原理揭秘", §2.2), and the
backward is the same kernel run again with the sine negated (same page as the first,
§4).  The pages do not print the pairing of the dimensions or how the tables are built.

Readings taken (plainest reading; they are the Llama convention the Triton kernel copies
from Hugging Face):
  * a head of hd features is rotated as hd/2 pairs (x_i, x_{i + hd/2}), i < hd/2
    ("rotate half"), by the angle of frequency i at the token's position:
        y_i          = x_i c - x_{i+hd/2} s
        y_{i+hd/2}   = x_{i+hd/2} c + x_i s,        c = cos[pos, i], s = sin[pos, i];
  * cos and sin are tables [n_pos x hd/2] indexed by a per-token position id (an input:
    packed sequences restart their positions), with the usual frequencies
    theta_i = base^(-2i/hd) when built here (tables(): angle = pos * theta_i);
  * the backward of y = R x is dx = R^T dy, the same rotation with the sine negated.
"""
from __future__ import annotations

import numpy as np


def tables(n_pos: int, hd: int, base: float):
    """cos, sin [n_pos x hd/2] in fp64: angle(p, i) = p * base^(-2i/hd)."""
    theta = base ** (-2.0 * np.arange(hd // 2) / hd)
    ang = np.outer(np.arange(n_pos, dtype=np.float64), theta)
    return np.cos(ang), np.sin(ang)


def rotate(x, pos, cos, sin, hd, sign=1.0):
    """Rotate every head of x [T x (H * hd)] at its row's position; sign = -1 applies the
    inverse rotation (the backward)."""
    T, n = x.shape
    xh = x.reshape(T, n // hd, hd)
    c = cos[pos][:, None, :]
    s = sign * sin[pos][:, None, :]
    a, b = xh[..., :hd // 2], xh[..., hd // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1).reshape(T, n)


def forward(Q, K, pos, cos, sin, hd):
    return rotate(Q, pos, cos, sin, hd), rotate(K, pos, cos, sin, hd)


def backward(dQ, dK, pos, cos, sin, hd):
    """Gradients of <dQo, RoPE(Q)> + <dKo, RoPE(K)>: the transposed (inverse) rotation."""
    return rotate(dQ, pos, cos, sin, hd, -1.0), rotate(dK, pos, cos, sin, hd, -1.0)
