"""Seeded synthetic inputs for the LoRA-MLP sub-block.

This module is shared by the CUDA path's tests/bench and by the fp64 oracle's
tests.  It draws random numbers and rounds them to bf16; it contains none of the
method's arithmetic (no norm, no projection, no activation).

Recipe (one stream per tensor, fixed order):
  base seed 3407 (the seed the pages use in their training scripts,
  "Unsloth 深度实战", §3.2 and "【编译】结合 Unsloth 与 🤗 TRL", §三);
  tensor k in the order X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, dY draws from
  numpy Generator(PCG64(SeedSequence([3407, k]))).

Distributions (the workload descriptions of the LoRA-MLP configs):
  X ~ N(0,1) [T x d];  w ~ 1 + N(0, 0.1) [d];
  Wg, Wu ~ N(0, 0.02) [f x d];  Wd ~ N(0, 0.02) [d x f];
  A ~ kaiming-uniform(a=sqrt(5)) on [r x in] = U(-1/sqrt(in), 1/sqrt(in))
      ("Unsloth 深度实战", §1.3: A random Kaiming-uniform, B zero at init);
  B ~ N(0, 0.01) [out x r] (non-zero so the adapter gradients are non-trivial);
  dY ~ N(0, 1) [T x d].
Every value is drawn in fp64, rounded to fp32, then to bf16 with
round-to-nearest-even on the bit pattern; the same bits go to both sides.
"""
from __future__ import annotations

import dataclasses
import numpy as np

BASE_SEED = 3407
TENSOR_ORDER = ("X", "w", "Wg", "Wu", "Wd", "Ag", "Bg", "Au", "Bu", "Ad", "Bd", "dY")


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even), returned as uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # u + 0x7FFF + lsb stays below 2^32 for every non-NaN pattern (at most 0xFF80_7FFF)
    r = ((u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


@dataclasses.dataclass(frozen=True)
class Shape:
    T: int
    d: int
    f: int
    r: int
    alpha: float = 16.0
    eps: float = 1e-6

    @property
    def scale(self) -> float:
        # the LoRA scaling alpha / r ("Unsloth 深度实战", §1.3, LoRALayer)
        return self.alpha / self.r


def _rng(k: int, seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, k])))


def _normal(k, seed, shape, mean, std):
    return mean + std * _rng(k, seed).standard_normal(size=shape, dtype=np.float64)


def _uniform(k, seed, shape, bound):
    return _rng(k, seed).uniform(-bound, bound, size=shape)


def tensor_f64(name: str, s: Shape, seed: int = BASE_SEED) -> np.ndarray:
    """Draw one tensor in fp64, before bf16 rounding."""
    k = TENSOR_ORDER.index(name)
    T, d, f, r = s.T, s.d, s.f, s.r
    if name == "X":
        return _normal(k, seed, (T, d), 0.0, 1.0)
    if name == "w":
        return _normal(k, seed, (d,), 1.0, 0.1)
    if name in ("Wg", "Wu"):
        return _normal(k, seed, (f, d), 0.0, 0.02)
    if name == "Wd":
        return _normal(k, seed, (d, f), 0.0, 0.02)
    if name in ("Ag", "Au"):
        return _uniform(k, seed, (r, d), 1.0 / np.sqrt(d))
    if name == "Ad":
        return _uniform(k, seed, (r, f), 1.0 / np.sqrt(f))
    if name in ("Bg", "Bu"):
        return _normal(k, seed, (f, r), 0.0, 0.01)
    if name == "Bd":
        return _normal(k, seed, (d, r), 0.0, 0.01)
    if name == "dY":
        return _normal(k, seed, (T, d), 0.0, 1.0)
    raise KeyError(name)


def make_inputs_bits(s: Shape, seed: int = BASE_SEED, names=TENSOR_ORDER) -> dict:
    """All inputs as bf16 bit arrays (uint16), keyed by name."""
    return {n: f32_to_bf16_bits(tensor_f64(n, s, seed).astype(np.float32)) for n in names}


def bits_to_f64(bits: dict) -> dict:
    return {k: bf16_bits_to_f64(v) for k, v in bits.items()}


def row_slice_bits(bits: dict, rows) -> dict:
    """Restrict the per-token tensors (X, dY) to a subset of rows."""
    out = dict(bits)
    for k in ("X", "dY"):
        if k in out:
            out[k] = np.ascontiguousarray(out[k][rows])
    return out


# ---------------------------------------------------------------- attention Q/K/V projections
QKV_TENSOR_ORDER = ("X", "w", "Wq", "Wk", "Wv", "Aq", "Bq", "Ak", "Bk", "Av", "Bv", "dQ", "dK", "dV")
# streams of their own (k offset), so the MLP inputs of the same seed are not reused
_QKV_STREAM0 = 100


@dataclasses.dataclass(frozen=True)
class QkvShape:
    """T tokens, hidden d, nq query features, nkv key/value features (grouped-query
    attention when nkv < nq), LoRA rank r."""
    T: int
    d: int
    nq: int
    nkv: int
    r: int
    alpha: float = 16.0
    eps: float = 1e-6

    @property
    def scale(self) -> float:
        return self.alpha / self.r


def qkv_tensor_f64(name: str, s: QkvShape, seed: int = BASE_SEED) -> np.ndarray:
    """One Q/K/V-projection input in fp64, before bf16 rounding (the same distributions
    as the MLP's: activations N(0,1), norm weight 1 + N(0,0.1), W N(0,0.02),
    A U(+-1/sqrt(in)), B N(0,0.01))."""
    k = _QKV_STREAM0 + QKV_TENSOR_ORDER.index(name)
    T, d, nq, nkv, r = s.T, s.d, s.nq, s.nkv, s.r
    n_out = {"q": nq, "k": nkv, "v": nkv}
    if name == "X":
        return _normal(k, seed, (T, d), 0.0, 1.0)
    if name == "w":
        return _normal(k, seed, (d,), 1.0, 0.1)
    if name[0] == "W":
        return _normal(k, seed, (n_out[name[1]], d), 0.0, 0.02)
    if name[0] == "A":
        return _uniform(k, seed, (r, d), 1.0 / np.sqrt(d))
    if name[0] == "B":
        return _normal(k, seed, (n_out[name[1]], r), 0.0, 0.01)
    if name[0] == "d":
        return _normal(k, seed, (T, n_out[name[1].lower()]), 0.0, 1.0)
    raise KeyError(name)


def make_qkv_inputs_bits(s: QkvShape, seed: int = BASE_SEED, names=QKV_TENSOR_ORDER) -> dict:
    return {n: f32_to_bf16_bits(qkv_tensor_f64(n, s, seed).astype(np.float32)) for n in names}


# ---------------------------------------------------------------- attention output projection o_proj
O_TENSOR_ORDER = ("X", "Wo", "Ao", "Bo", "dY")
_O_STREAM0 = 200


@dataclasses.dataclass(frozen=True)
class OShape:
    """T tokens, n_in input features (the attention output, heads x head dim), n_out
    output features (the hidden size), LoRA rank r."""
    T: int
    n_in: int
    n_out: int
    r: int
    alpha: float = 16.0

    @property
    def scale(self) -> float:
        return self.alpha / self.r


def o_tensor_f64(name: str, s: OShape, seed: int = BASE_SEED) -> np.ndarray:
    """One o_proj input in fp64 (the MLP's distributions: activations and upstream
    gradients N(0,1), W N(0,0.02), A U(+-1/sqrt(in)), B N(0,0.01))."""
    k = _O_STREAM0 + O_TENSOR_ORDER.index(name)
    if name == "X":
        return _normal(k, seed, (s.T, s.n_in), 0.0, 1.0)
    if name == "Wo":
        return _normal(k, seed, (s.n_out, s.n_in), 0.0, 0.02)
    if name == "Ao":
        return _uniform(k, seed, (s.r, s.n_in), 1.0 / np.sqrt(s.n_in))
    if name == "Bo":
        return _normal(k, seed, (s.n_out, s.r), 0.0, 0.01)
    if name == "dY":
        return _normal(k, seed, (s.T, s.n_out), 0.0, 1.0)
    raise KeyError(name)


def make_o_inputs_bits(s: OShape, seed: int = BASE_SEED) -> dict:
    return {n: f32_to_bf16_bits(o_tensor_f64(n, s, seed).astype(np.float32)) for n in O_TENSOR_ORDER}


# ---------------------------------------------------------------- RoPE on the query / key heads
_ROPE_STREAM0 = 300


@dataclasses.dataclass(frozen=True)
class RopeShape:
    """T tokens in sequences of seq_len (position ids t mod seq_len), hq query heads and
    hk key heads of hd features, rotary base."""
    T: int
    hq: int
    hk: int
    hd: int
    seq_len: int
    base: float = 500000.0


def rope_tables(n_pos: int, hd: int, base: float):
    """The cos / sin caches the RoPE kernel looks up by position: [n_pos x hd/2] fp32,
    angle(p, i) = p * base^(-2 i / hd), computed in fp64 and rounded once (how a model
    builds its rotary caches; they are inputs of the kernel)."""
    theta = base ** (-2.0 * np.arange(hd // 2, dtype=np.float64) / hd)
    ang = np.outer(np.arange(n_pos, dtype=np.float64), theta)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def make_rope_inputs(s: RopeShape, seed: int = BASE_SEED) -> dict:
    """Q [T x hq hd], K [T x hk hd] and their upstream gradients dQ, dK as bf16 bits
    (N(0,1)), position ids int32 [T] = t mod seq_len, cos / sin tables fp32."""
    out = {}
    for i, (name, h) in enumerate((("Q", s.hq), ("K", s.hk), ("dQ", s.hq), ("dK", s.hk))):
        out[name] = f32_to_bf16_bits(_normal(_ROPE_STREAM0 + i, seed, (s.T, h * s.hd), 0.0, 1.0).astype(np.float32))
    out["pos"] = (np.arange(s.T) % s.seq_len).astype(np.int32)
    out["cos"], out["sin"] = rope_tables(s.seq_len, s.hd, s.base)
    return out


# ---------------------------------------------------------------- LM-head cross-entropy
_CE_STREAM0 = 400
IGNORE_INDEX = -100


@dataclasses.dataclass(frozen=True)
class CeShape:
    """T tokens, hidden d, vocabulary V; a fraction of the labels is the ignore index
    (prompt tokens left out of the loss)."""
    T: int
    d: int
    V: int
    ignored: float = 0.05


def make_ce_inputs(s: CeShape, seed: int = BASE_SEED) -> dict:
    """H [T x d] (final normalised hidden states) N(0,1) and the frozen LM head W [V x d]
    N(0,0.02) as bf16 bits; labels int32 [T] uniform over the vocabulary with the given
    fraction set to the ignore index."""
    H = f32_to_bf16_bits(_normal(_CE_STREAM0, seed, (s.T, s.d), 0.0, 1.0).astype(np.float32))
    W = f32_to_bf16_bits(_normal(_CE_STREAM0 + 1, seed, (s.V, s.d), 0.0, 0.02).astype(np.float32))
    g = _rng(_CE_STREAM0 + 2, seed)
    labels = g.integers(0, s.V, s.T).astype(np.int32)
    labels[g.random(s.T) < s.ignored] = IGNORE_INDEX
    return {"H": H, "W": W, "labels": labels}
