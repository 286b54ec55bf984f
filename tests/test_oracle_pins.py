"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
finite differences, closed forms, invariants, brute force, library routines and the
numbers the pages print.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

from lora_fine_tuning_rmsnorm_b200 import synth
from oracle import lora_mlp_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
NAMES = ("w", "Wg", "Wu", "Wd", "Ag", "Bg", "Au", "Bu", "Ad", "Bd")


def tiny_inputs(T=5, d=8, f=12, r=3, seed=11, bf16=False):
    s = synth.Shape(T=T, d=d, f=f, r=r, alpha=2.0 * r)
    if bf16:
        return s, synth.bits_to_f64(synth.make_inputs_bits(s, seed=seed))
    return s, {k: synth.tensor_f64(k, s, seed) for k in synth.TENSOR_ORDER}


def run(inp, s, eps=1e-6, residual=False):
    fw = ref.forward(inp["X"], inp["w"], eps, *(inp[k] for k in NAMES[1:]), s.scale, residual)
    bw = ref.backward(fw, inp["dY"], inp["X"], *(inp[k] for k in NAMES), s.scale, residual)
    return fw, bw


def loss(inp, s, eps=1e-6, residual=False):
    fw = ref.forward(inp["X"], inp["w"], eps, *(inp[k] for k in NAMES[1:]), s.scale, residual)
    return float(np.sum(inp["dY"] * fw["Y"]))


GRAD_OF = {"X": "dX", "Ag": "dAg", "Bg": "dBg", "Au": "dAu", "Bu": "dBu", "Ad": "dAd", "Bd": "dBd",
           "w": "dw"}


def fd_errors(inp, s, eps=1e-6, h=1e-5, seed=5, residual=False):
    """Relative error of <grad, V> against a central difference of L = <dY, Y>."""
    _, bw = run(inp, s, eps, residual)
    rng = np.random.default_rng(seed)
    errs = {}
    for name, gname in GRAD_OF.items():
        V = rng.standard_normal(inp[name].shape)
        plus = dict(inp); plus[name] = inp[name] + h * V
        minus = dict(inp); minus[name] = inp[name] - h * V
        fd = (loss(plus, s, eps, residual) - loss(minus, s, eps, residual)) / (2 * h)
        an = float(np.sum(bw[gname] * V))
        errs[name] = abs(fd - an) / max(abs(fd), 1e-300)
    return errs


# ---------------------------------------------------------------- finite differences

def test_backward_matches_finite_differences():
    s, inp = tiny_inputs()
    errs = fd_errors(inp, s)
    assert max(errs.values()) < 1e-7, errs


def test_residual_variant_matches_finite_differences():
    """Y = X + MLP(RMSNorm(X)): the dY term in dX (and every other gradient) against FD."""
    s, inp = tiny_inputs(seed=31)
    errs = fd_errors(inp, s, residual=True)
    # <dY, X> adds a large constant to L for every direction but X, so the central
    # difference cancels more digits there; the X direction carries the residual term
    assert errs["X"] < 1e-8, errs
    assert max(errs.values()) < 5e-6, errs
    fr, br = run(inp, s, residual=True)
    f0, b0 = run(inp, s)
    np.testing.assert_allclose(fr["Y"] - f0["Y"], inp["X"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(br["dX"] - b0["dX"], inp["dY"], rtol=1e-12, atol=1e-14)
    for k in ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd", "dw"):
        np.testing.assert_array_equal(br[k], b0[k])


def test_norm_weight_grad_closed_form_scale_invariance():
    """With eps = 0 the norm output does not depend on the scale of a row, so dw from
    rows scaled by c > 0 equals dw of the unscaled rows."""
    s, inp = tiny_inputs(seed=32)
    _, b1 = run(inp, s, eps=0.0)
    scaled = dict(inp)
    scaled["X"] = inp["X"] * np.linspace(0.5, 3.0, inp["X"].shape[0])[:, None]
    _, b2 = run(scaled, s, eps=0.0)
    np.testing.assert_allclose(b2["dw"], b1["dw"], rtol=1e-11, atol=1e-14)


def test_merge_brute_force_loops():
    """ref.merge against an element-by-element loop of W_ij + s sum_k B_ik A_kj."""
    rng = np.random.default_rng(33)
    W, A, B = rng.standard_normal((5, 7)), rng.standard_normal((3, 7)), rng.standard_normal((5, 3))
    s = 0.75
    M = ref.merge(W, A, B, s)
    for i in range(5):
        for j in range(7):
            acc = 0.0
            for k in range(3):
                acc += B[i, k] * A[k, j]
            assert abs(M[i, j] - (W[i, j] + s * acc)) < 1e-13


def test_backward_matches_finite_differences_bf16_inputs_eps_large():
    s, inp = tiny_inputs(T=4, d=16, f=24, r=2, seed=3, bf16=True)
    errs = fd_errors(inp, s, eps=0.5)
    assert max(errs.values()) < 1e-7, errs


# -------------------------------------------------------------------- closed forms

def test_silu_closed_forms():
    assert ref.silu(0.0) == 0.0
    assert ref.silu_grad(0.0) == 0.5
    z = np.linspace(-12, 12, 97)
    # library routine: scipy's logistic sigmoid
    np.testing.assert_allclose(ref.silu(z), z * scipy.special.expit(z), rtol=1e-14, atol=1e-300)
    h = 1e-6
    fd = (ref.silu(z + h) - ref.silu(z - h)) / (2 * h)
    np.testing.assert_allclose(ref.silu_grad(z), fd, rtol=1e-8, atol=1e-10)
    # large |z| limits: silu -> z (z >> 0), -> 0 (z << 0)
    assert abs(ref.silu(40.0) - 40.0) < 1e-12
    assert abs(ref.silu(-40.0)) < 1e-12


def test_rmsnorm_forward_closed_forms():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((7, 33)) * 3.0
    w = 1 + 0.1 * rng.standard_normal(33)
    eps = 1e-3
    H, rstd = ref.rmsnorm_fwd(X, w, eps)
    ms = np.mean(X ** 2, axis=1)
    # mean over the TRUE column count (not a padded block): mean((H/w)^2) = ms/(ms+eps)
    np.testing.assert_allclose(np.mean((H / w) ** 2, axis=1), ms / (ms + eps), rtol=1e-13)
    # eps = 0: output is invariant to scaling the row
    H0, _ = ref.rmsnorm_fwd(X, w, 0.0)
    H1, _ = ref.rmsnorm_fwd(5.5 * X, w, 0.0)
    np.testing.assert_allclose(H0, H1, rtol=1e-13)
    # single-element row: |H| = |x| / sqrt(x^2 + eps) * w
    Hs, _ = ref.rmsnorm_fwd(np.array([[2.0]]), np.array([3.0]), 1.0)
    assert abs(Hs[0, 0] - 2.0 / math.sqrt(5.0) * 3.0) < 1e-15


def test_rmsnorm_backward_closed_forms():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((6, 40))
    w = 1 + 0.1 * rng.standard_normal(40)
    dH = rng.standard_normal((6, 40))
    # eps = 0: scale invariance => sum_j dX_j x_j = 0 per row
    _, r0 = ref.rmsnorm_fwd(X, w, 0.0)
    dX0 = ref.rmsnorm_bwd(dH, X, w, r0)
    np.testing.assert_allclose(np.sum(dX0 * X, axis=1), 0.0, atol=1e-12)
    # eps > 0: sum_j dX_j x_j = rstd * eps * rstd^2 * sum_j g_j x_j
    eps = 0.7
    _, r = ref.rmsnorm_fwd(X, w, eps)
    dX = ref.rmsnorm_bwd(dH, X, w, r)
    g = dH * w
    np.testing.assert_allclose(np.sum(dX * X, axis=1), r * eps * r ** 2 * np.sum(g * X, axis=1), rtol=1e-11)
    # elementwise finite differences of the norm alone
    h = 1e-6
    for (i, j) in [(0, 0), (3, 17), (5, 39)]:
        Xp = X.copy(); Xp[i, j] += h
        Xm = X.copy(); Xm[i, j] -= h
        fd = (np.sum(dH * ref.rmsnorm_fwd(Xp, w, eps)[0]) - np.sum(dH * ref.rmsnorm_fwd(Xm, w, eps)[0])) / (2 * h)
        assert abs(fd - dX[i, j]) < 1e-8 * max(1.0, abs(fd))


# ---------------------------------------------------------------------- invariants

def frozen_mlp(inp, eps=1e-6):
    H, _ = ref.rmsnorm_fwd(inp["X"], inp["w"], eps)
    g = H @ inp["Wg"].T
    u = H @ inp["Wu"].T
    return (g / (1 + np.exp(-g)) * u) @ inp["Wd"].T


def test_zero_B_gives_frozen_output_and_zero_dA():
    s, inp = tiny_inputs(seed=21)
    for k in ("Bg", "Bu", "Bd"):
        inp[k] = np.zeros_like(inp[k])
    fw, bw = run(inp, s)
    np.testing.assert_allclose(fw["Y"], frozen_mlp(inp), rtol=1e-13, atol=1e-15)
    for k in ("dAg", "dAu", "dAd"):
        assert np.all(bw[k] == 0.0), k
    for k in ("dBg", "dBu", "dBd"):
        assert np.abs(bw[k]).max() > 0


def test_zero_A_gives_zero_dB():
    s, inp = tiny_inputs(seed=22)
    for k in ("Ag", "Au", "Ad"):
        inp[k] = np.zeros_like(inp[k])
    fw, bw = run(inp, s)
    np.testing.assert_allclose(fw["Y"], frozen_mlp(inp), rtol=1e-13, atol=1e-15)
    for k in ("dBg", "dBu", "dBd"):
        assert np.all(bw[k] == 0.0), k


def test_zero_scale_gives_frozen_output():
    s, inp = tiny_inputs(seed=23)
    fw = ref.forward(inp["X"], inp["w"], 1e-6, *(inp[k] for k in NAMES[1:]), 0.0)
    np.testing.assert_allclose(fw["Y"], frozen_mlp(inp), rtol=1e-13, atol=1e-15)


def test_merge_equivalence():
    """Y(W, A, B, s) = Y(W + s B A, 0, 0) and the same dX (weight merge for export)."""
    s, inp = tiny_inputs(seed=24)
    sc = s.scale
    fw, bw = run(inp, s)
    merged = dict(inp)
    merged["Wg"] = ref.merge(inp["Wg"], inp["Ag"], inp["Bg"], sc)
    merged["Wu"] = ref.merge(inp["Wu"], inp["Au"], inp["Bu"], sc)
    merged["Wd"] = ref.merge(inp["Wd"], inp["Ad"], inp["Bd"], sc)
    for k in ("Ag", "Au", "Ad", "Bg", "Bu", "Bd"):
        merged[k] = np.zeros_like(inp[k])
    fm, bm = run(merged, s)
    np.testing.assert_allclose(fw["Y"], fm["Y"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(bw["dX"], bm["dX"], rtol=1e-11, atol=1e-13)
    # adapter grads follow from the merged weight's grad dWeff = dZ^T x:
    #   dA = s B^T dWeff, dB = s dWeff A^T
    dWg = bm["dG"].T @ fm["H"]
    np.testing.assert_allclose(bw["dAg"], sc * inp["Bg"].T @ dWg, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(bw["dBg"], sc * dWg @ inp["Ag"].T, rtol=1e-11, atol=1e-14)
    dWd = inp["dY"].T @ fm["Act"]
    np.testing.assert_allclose(bw["dAd"], sc * inp["Bd"].T @ dWd, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(bw["dBd"], sc * dWd @ inp["Ad"].T, rtol=1e-11, atol=1e-14)


def test_linearity_in_dY():
    s, inp = tiny_inputs(seed=25)
    rng = np.random.default_rng(2)
    d1 = rng.standard_normal(inp["dY"].shape)
    d2 = rng.standard_normal(inp["dY"].shape)
    outs = []
    for dy in (d1, d2, d1 + 2 * d2):
        q = dict(inp); q["dY"] = dy
        outs.append(run(q, s)[1])
    for k in ("dX", "dAg", "dBg", "dAu", "dBu", "dAd", "dBd"):
        np.testing.assert_allclose(outs[2][k], outs[0][k] + 2 * outs[1][k], rtol=1e-10, atol=1e-13)


def test_chunked_fwd_bwd_equals_whole():
    s, inp = tiny_inputs(T=23, seed=26)
    a = ref.fwd_bwd(inp, s.scale, 1e-6, chunk=5, keep=("Y", "dX", "G"))
    b = ref.fwd_bwd(inp, s.scale, 1e-6, chunk=1000, keep=("Y", "dX", "G"))
    for k in a:
        np.testing.assert_allclose(a[k], b[k], rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------- brute force

def test_forward_brute_force_loops():
    s, inp = tiny_inputs(T=3, d=4, f=6, r=2, seed=27)
    eps, sc = 1e-6, s.scale
    X, w = inp["X"], inp["w"]
    T, d, f, r = 3, 4, 6, 2

    def lin(x, W, A, B, n_out, n_in):
        out = [0.0] * n_out
        xa = [sum(x[i] * A[k][i] for i in range(n_in)) for k in range(r)]
        for o in range(n_out):
            acc = sum(x[i] * W[o][i] for i in range(n_in))
            acc += sc * sum(xa[k] * B[o][k] for k in range(r))
            out[o] = acc
        return out

    Yb = []
    for t in range(T):
        ms = sum(X[t][j] ** 2 for j in range(d)) / d
        rs = 1.0 / math.sqrt(ms + eps)
        h = [X[t][j] * rs * w[j] for j in range(d)]
        g = lin(h, inp["Wg"], inp["Ag"], inp["Bg"], f, d)
        u = lin(h, inp["Wu"], inp["Au"], inp["Bu"], f, d)
        a = [g[j] / (1.0 + math.exp(-g[j])) * u[j] for j in range(f)]
        Yb.append(lin(a, inp["Wd"], inp["Ad"], inp["Bd"], d, f))
    fw, _ = run(inp, s)
    np.testing.assert_allclose(fw["Y"], np.array(Yb), rtol=1e-12, atol=1e-15)


# ------------------------------------------------------------- the pages' numbers

def test_page_numbers_lora_shapes():
    with open(os.path.join(GOLDEN, "page_facts.json")) as fh:
        facts = json.load(fh)
    pc = facts["lora_param_count"]
    n, m, r = pc["n"], pc["m"], pc["r"]
    # A [r x in], B [out x r]: r*(n+m) trainable values vs n*m
    s = synth.Shape(T=1, d=m, f=n, r=r)
    A = synth.tensor_f64("Ag", s)
    B = synth.tensor_f64("Bg", s)
    assert A.size + B.size == pc["lora"]
    assert n * m == pc["full"]
    assert n * m // (A.size + B.size) == pc["ratio"]
    xa = facts["x_a_fraction"]
    s2 = synth.Shape(T=4, d=xa["d"], f=32, r=xa["r"])
    inp = {k: synth.tensor_f64(k, s2) for k in synth.TENSOR_ORDER}
    fw = ref.forward(inp["X"], inp["w"], 1e-6, *(inp[k] for k in NAMES[1:]), s2.scale)
    frac = fw["Pg"].size / inp["X"].size
    assert round(100 * frac, 1) == xa["percent"]


def test_sampled_outputs_equal_full_oracle():
    s, inp = tiny_inputs(T=37, d=16, f=24, r=3, seed=41)
    full = ref.fwd_bwd(inp, s.scale, 1e-6, chunk=1000, keep=("Y", "dX"))
    rows = [0, 5, 36]
    cols = [1, 7, 23]
    smp = ref.sampled(inp, s.scale, 1e-6, rows, cols, chunk=10)
    np.testing.assert_allclose(smp["Y"], full["Y"][rows], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(smp["dX"], full["dX"][rows], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(smp["dBg"], full["dBg"][cols], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(smp["dBu"], full["dBu"][cols], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(smp["dAd"], full["dAd"][:, cols], rtol=1e-12, atol=1e-15)
