"""Reference 4-bit blockwise quantisation of the frozen weights (plain definitions).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The pages describe QLoRA's 4-bit NormalFloat storage: weights compressed to 4 bits
with a codebook taken from quantiles of the normal distribution
("Unsloth 深度实战", §1.4; "Unsloth提速秘诀：Triton内核如何加速反向传播", §4.1 table:
NF4), dequantised before the matmul and fused with it
("Unsloth加速原理揭秘：为何训练快5-8倍？", §5.2).  The pages fix neither the
codebook's exact values nor the assignment rule, so this module takes these readings:

  codebook: q_i = Phi^{-1}((i + 0.5) / 16), i = 0..15, normalised by max|q|, rounded
            to fp32 (ascending, symmetric, c_0 = -1, c_15 = +1, no exact zero);
  blocks:   64 consecutive elements of the row-major [out x in] matrix, one fp32 absmax
            per block (double quantisation of the absmax constants: see below);
  codes:    nearest code to w / absmax, ties to the lower index, computed exactly as
            idx = #{ i in 0..14 : w > absmax * m_i },  m_i = fl32((c_i + c_{i+1}) / 2);
            an all-zero block has absmax 0 and codes 0;
  packing:  two codes per byte, the even element in the low nibble;
  dequant:  w_hat = c[idx] * absmax (exact in fp64 here).

The comparison w > absmax * m_i is exact in fp64, since the product of two fp32
values fits in a double's 53-bit significand.

Double quantisation ("Unsloth 深度实战", §1.4: the quantisation constants are themselves
quantised).  The pages give no format; the plainest reading, taken here:

  blocks2:  256 consecutive absmax constants (the last block may be shorter), one fp32
            scale2 per block = the largest constant of the block (they are >= 0);
  codes8:   each constant a -> the nearest of the 256 levels scale2 * k / 255, ties to the
            lower level, decided exactly as k = #{ j in 1..255 : 510 a > (2j - 1) scale2 }
            (both products are exact in fp64: a 24-bit significand times a 9-bit
            integer); an all-zero block has scale2 0 and codes 0;
  dequant:  a_hat = scale2 * k / 255 (exact here), then w_hat = c[idx] * a_hat.
"""
from __future__ import annotations

import statistics

import numpy as np


def codebook16() -> np.ndarray:
    nd = statistics.NormalDist()
    q = np.array([nd.inv_cdf((i + 0.5) / 16.0) for i in range(16)], dtype=np.float64)
    return (q / np.max(np.abs(q))).astype(np.float32)


def midpoints(code: np.ndarray) -> np.ndarray:
    c = code.astype(np.float64)
    return ((c[:-1] + c[1:]) / 2.0).astype(np.float32)


def quantize(Wf: np.ndarray, code: np.ndarray, block: int = 64):
    """Wf: values (exactly representable in fp32) of a row-major [out x in] matrix.

    Returns (idx uint8 [numel], absmax float32 [numel/block]).
    """
    flat = np.asarray(Wf, dtype=np.float64).reshape(-1)
    if flat.size % block:
        raise ValueError("numel must be a multiple of the block size")
    blk = flat.reshape(-1, block)
    absmax = np.max(np.abs(blk), axis=1).astype(np.float32)     # exact (max of fp32 values)
    thr = absmax.astype(np.float64)[:, None, None] * midpoints(code).astype(np.float64)[None, None, :]
    gt = blk[:, :, None] > thr                                  # [nblk, block, 15]
    idx = gt.sum(axis=2).astype(np.uint8)
    return idx.reshape(-1), absmax


def pack(idx: np.ndarray) -> np.ndarray:
    idx = np.asarray(idx, dtype=np.uint8).reshape(-1)
    return (idx[0::2] | (idx[1::2] << 4)).astype(np.uint8)


def unpack(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out


def dequantize(idx: np.ndarray, absmax: np.ndarray, code: np.ndarray, shape, block: int = 64):
    c = code.astype(np.float64)[np.asarray(idx, dtype=np.int64)]
    a = np.repeat(absmax.astype(np.float64), block)
    return (c * a).reshape(shape)


def quantize_absmax8(absmax: np.ndarray, block2: int = 256):
    """Second-level quantisation of the fp32 absmax constants.

    Returns (codes8 uint8 [n], scale2 float32 [ceil(n / block2)])."""
    a = np.asarray(absmax, dtype=np.float32).reshape(-1)
    n = a.size
    nb = (n + block2 - 1) // block2
    scale2 = np.array([a[b * block2:(b + 1) * block2].max() for b in range(nb)], dtype=np.float32)
    s = np.repeat(scale2.astype(np.float64), block2)[:n]
    lhs = 510.0 * a.astype(np.float64)                               # exact
    thr = np.arange(1, 510, 2, dtype=np.float64)                     # 2j - 1, j = 1..255
    codes8 = np.empty(n, dtype=np.uint8)
    for i0 in range(0, n, 65536):                                    # row chunks bound the memory
        sl = slice(i0, i0 + 65536)
        codes8[sl] = (lhs[sl, None] > s[sl, None] * thr[None, :]).sum(axis=1)  # exact; strict: ties go down
    return codes8, scale2


def dequantize_absmax8(codes8: np.ndarray, scale2: np.ndarray, block2: int = 256) -> np.ndarray:
    """a_hat = scale2 * k / 255 in fp64."""
    k = np.asarray(codes8, dtype=np.float64).reshape(-1)
    s = np.repeat(np.asarray(scale2, dtype=np.float64), block2)[:k.size]
    return s * k / 255.0
