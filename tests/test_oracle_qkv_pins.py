"""Pins of the fp64 Q/K/V-projection oracle against facts that do not come from the
oracle itself: finite differences, brute-force loops, invariants.  CPU only."""
import math

import numpy as np

from lora_fine_tuning_rmsnorm_b200 import synth
from oracle import lora_qkv_ref as ref

W_NAMES = ("Wq", "Wk", "Wv", "Aq", "Bq", "Ak", "Bk", "Av", "Bv")


def tiny(T=5, d=8, nq=8, nkv=4, r=3, seed=41):
    s = synth.QkvShape(T=T, d=d, nq=nq, nkv=nkv, r=r, alpha=2.0 * r)
    return s, {k: synth.qkv_tensor_f64(k, s, seed) for k in synth.QKV_TENSOR_ORDER}


def run(inp, s, eps=1e-6):
    fw = ref.forward(inp["X"], inp["w"], eps, *(inp[k] for k in W_NAMES), s.scale)
    bw = ref.backward(fw, inp["dQ"], inp["dK"], inp["dV"], inp["X"], inp["w"], *(inp[k] for k in W_NAMES), s.scale)
    return fw, bw


def loss(inp, s, eps=1e-6):
    fw, _ = run(inp, s, eps)
    return float(np.sum(inp["dQ"] * fw["Q"]) + np.sum(inp["dK"] * fw["K"]) + np.sum(inp["dV"] * fw["V"]))


def test_backward_matches_finite_differences():
    """L = <dQ, Q> + <dK, K> + <dV, V>: every gradient against a central difference."""
    s, inp = tiny()
    _, bw = run(inp, s)
    rng = np.random.default_rng(3)
    h = 1e-5
    for name, g in (("X", "dX"), ("Aq", "dAq"), ("Bq", "dBq"), ("Ak", "dAk"), ("Bk", "dBk"), ("Av", "dAv"),
                    ("Bv", "dBv")):
        V = rng.standard_normal(inp[name].shape)
        p = dict(inp); p[name] = inp[name] + h * V
        m = dict(inp); m[name] = inp[name] - h * V
        fd = (loss(p, s) - loss(m, s)) / (2 * h)
        an = float(np.sum(bw[g] * V))
        assert abs(fd - an) <= 1e-7 * max(abs(fd), 1e-12), (name, fd, an)


def test_forward_brute_force_loops():
    """Q, K, V from explicit loops over the definitions (norm, then x W^T + s (x A^T) B^T)."""
    s, inp = tiny(T=3, d=4, nq=4, nkv=2, r=2, seed=42)
    fw, _ = run(inp, s)
    X, w = inp["X"], inp["w"]
    for t in range(3):
        ms = sum(X[t, j] ** 2 for j in range(4)) / 4
        rs = 1.0 / math.sqrt(ms + 1e-6)
        h = [X[t, j] * rs * w[j] for j in range(4)]
        for name, W, A, B in (("Q", "Wq", "Aq", "Bq"), ("K", "Wk", "Ak", "Bk"), ("V", "Wv", "Av", "Bv")):
            for o in range(inp[W].shape[0]):
                base = sum(h[j] * inp[W][o, j] for j in range(4))
                p = [sum(h[j] * inp[A][k, j] for j in range(4)) for k in range(2)]
                lora = sum(p[k] * inp[B][o, k] for k in range(2))
                assert abs(fw[name][t, o] - (base + s.scale * lora)) < 1e-12


def test_zero_B_and_merge_equivalence():
    """B = 0: frozen projections and dA = 0.  W + s B A with zero adapters reproduces the
    adapter forward and dX."""
    s, inp = tiny(seed=43)
    z = dict(inp)
    for k in ("Bq", "Bk", "Bv"):
        z[k] = np.zeros_like(inp[k])
    fz, bz = run(z, s)
    for n, W in (("Q", "Wq"), ("K", "Wk"), ("V", "Wv")):
        np.testing.assert_allclose(fz[n], fz["H"] @ inp[W].T, rtol=1e-13, atol=1e-15)
    for k in ("dAq", "dAk", "dAv"):
        assert np.all(bz[k] == 0)
    fw, bw = run(inp, s)
    m = dict(inp)
    for W, A, B in (("Wq", "Aq", "Bq"), ("Wk", "Ak", "Bk"), ("Wv", "Av", "Bv")):
        m[W] = inp[W] + s.scale * inp[B] @ inp[A]
        m[B] = np.zeros_like(inp[B])
    fm, bm = run(m, s)
    for n in ("Q", "K", "V"):
        np.testing.assert_allclose(fm[n], fw[n], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(bm["dX"], bw["dX"], rtol=1e-11, atol=1e-13)


def test_chunked_equals_whole():
    s = synth.QkvShape(T=37, d=16, nq=16, nkv=8, r=4)
    inp = synth.bits_to_f64(synth.make_qkv_inputs_bits(s))
    a = ref.fwd_bwd(inp, s.scale, s.eps, chunk=8)
    b = ref.fwd_bwd(inp, s.scale, s.eps, chunk=64)
    for k in a:
        np.testing.assert_allclose(a[k], b[k], rtol=1e-12, atol=1e-14)
