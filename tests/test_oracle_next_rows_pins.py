"""Pins of the oracles of the next rows (CPU only): the o_proj LoRA linear, RoPE and the
LM-head cross-entropy.  Each is checked against something other than itself: finite
differences, brute-force loops, a complex-number restatement, library routines
(scipy's logsumexp), closed forms and invariants; planted mistakes must fail them."""
import math

import numpy as np
import pytest
import scipy.special

from lora_fine_tuning_rmsnorm_b200 import synth
from oracle import ce_ref, lora_o_ref, rope_ref
from oracle.lora_mlp_ref import merge


def rnd(rng, *shape, scale=1.0):
    return scale * rng.standard_normal(shape)


# ------------------------------------------------------------------ o_proj LoRA linear
def o_inputs(seed=0, T=5, n_in=12, n_out=10, r=3):
    rng = np.random.default_rng(seed)
    return dict(X=rnd(rng, T, n_in), Wo=rnd(rng, n_out, n_in, scale=0.3), Ao=rnd(rng, r, n_in, scale=0.5),
                Bo=rnd(rng, n_out, r, scale=0.5), dY=rnd(rng, T, n_out))


def o_loss(inp, s):
    return float(np.sum(inp["dY"] * lora_o_ref.forward(inp["X"], inp["Wo"], inp["Ao"], inp["Bo"], s)["Y"]))


@pytest.mark.parametrize("name,gname", [("X", "dX"), ("Ao", "dAo"), ("Bo", "dBo")])
def test_o_backward_matches_finite_differences(name, gname):
    inp, s, h = o_inputs(1), 1.7, 1e-5
    g = lora_o_ref.fwd_bwd(inp, s)[gname]
    V = np.random.default_rng(9).standard_normal(inp[name].shape)
    up, dn = dict(inp), dict(inp)
    up[name] = inp[name] + h * V
    dn[name] = inp[name] - h * V
    fd = (o_loss(up, s) - o_loss(dn, s)) / (2 * h)
    assert abs(fd - np.sum(g * V)) <= 1e-7 * max(1.0, abs(fd))


def test_o_forward_brute_force():
    inp, s = o_inputs(2), 0.75
    X, Wo, Ao, Bo = inp["X"], inp["Wo"], inp["Ao"], inp["Bo"]
    Y = lora_o_ref.forward(X, Wo, Ao, Bo, s)["Y"]
    for t in range(X.shape[0]):
        for o in range(Wo.shape[0]):
            acc = sum(X[t, i] * Wo[o, i] for i in range(X.shape[1]))
            for k in range(Ao.shape[0]):
                acc += s * Bo[o, k] * sum(X[t, i] * Ao[k, i] for i in range(X.shape[1]))
            assert abs(Y[t, o] - acc) <= 1e-12 * max(1.0, abs(acc))


def test_o_zero_B_and_merge():
    inp, s = o_inputs(3), 2.0
    z = dict(inp, Bo=np.zeros_like(inp["Bo"]))
    R = lora_o_ref.fwd_bwd(z, s)
    np.testing.assert_allclose(R["Y"], inp["X"] @ inp["Wo"].T, rtol=1e-14, atol=1e-14)
    assert np.all(R["dAo"] == 0)
    full = lora_o_ref.fwd_bwd(inp, s)
    Wm = merge(inp["Wo"], inp["Ao"], inp["Bo"], s)
    np.testing.assert_allclose(full["Y"], inp["X"] @ Wm.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(full["dX"], inp["dY"] @ Wm, rtol=1e-12, atol=1e-12)


def test_o_planted_mistakes_fail_the_fd_pin(monkeypatch):
    inp, s, h = o_inputs(4), 1.3, 1e-5
    V = np.random.default_rng(5).standard_normal(inp["X"].shape)
    up, dn = dict(inp), dict(inp)
    up["X"], dn["X"] = inp["X"] + h * V, inp["X"] - h * V
    fd = (o_loss(up, s) - o_loss(dn, s)) / (2 * h)

    def bad_backward(fw, dY, X, Wo, Ao, Bo, s):   # adapter term of dX dropped
        Qo = dY @ Bo
        return dict(Qo=Qo, dX=dY @ Wo, dAo=s * (Qo.T @ X), dBo=s * (dY.T @ fw["P"]))
    monkeypatch.setattr(lora_o_ref, "backward", bad_backward)
    g = lora_o_ref.fwd_bwd(inp, s)["dX"]
    assert abs(fd - np.sum(g * V)) > 1e-4 * max(1.0, abs(fd))


# ------------------------------------------------------------------ RoPE
HD = 8


def rope_inputs(seed=0, T=6, hq=3, hk=1, n_pos=16):
    rng = np.random.default_rng(seed)
    cos, sin = rope_ref.tables(n_pos, HD, 10000.0)
    pos = rng.integers(0, n_pos, T)
    return rnd(rng, T, hq * HD), rnd(rng, T, hk * HD), pos, cos, sin


def test_rope_tables_closed_form():
    cos, sin = rope_ref.tables(40, 128, 500000.0)
    assert cos.shape == (40, 64)
    for p in (0, 1, 7, 39):
        for i in (0, 1, 31, 63):
            ang = p * 500000.0 ** (-2.0 * i / 128)
            assert math.isclose(cos[p, i], math.cos(ang), rel_tol=1e-13, abs_tol=1e-15)
            assert math.isclose(sin[p, i], math.sin(ang), rel_tol=1e-13, abs_tol=1e-15)


def test_rope_equals_complex_multiplication():
    """Each pair (x_i, x_{i+hd/2}) as the complex number x_i + j x_{i+hd/2} is multiplied by
    e^{j angle}: an independent restatement of the rotation."""
    Q, _, pos, cos, sin = rope_inputs(1)
    out = rope_ref.rotate(Q, pos, cos, sin, HD)
    T, n = Q.shape
    for t in range(T):
        for h in range(n // HD):
            for i in range(HD // 2):
                z = complex(Q[t, h * HD + i], Q[t, h * HD + i + HD // 2])
                ang = pos[t] * 10000.0 ** (-2.0 * i / HD)
                w = z * complex(math.cos(ang), math.sin(ang))
                assert abs(out[t, h * HD + i] - w.real) < 1e-12
                assert abs(out[t, h * HD + i + HD // 2] - w.imag) < 1e-12


def test_rope_norm_inverse_identity_and_composition():
    Q, K, pos, cos, sin = rope_inputs(2)
    Qo, Ko = rope_ref.forward(Q, K, pos, cos, sin, HD)
    a, b = Q.reshape(len(Q), -1, HD), Qo.reshape(len(Q), -1, HD)
    np.testing.assert_allclose(a[..., :4] ** 2 + a[..., 4:] ** 2, b[..., :4] ** 2 + b[..., 4:] ** 2, rtol=1e-12)
    dQ, dK = rope_ref.backward(Qo, Ko, pos, cos, sin, HD)       # R^T R = I
    np.testing.assert_allclose(dQ, Q, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dK, K, rtol=1e-12, atol=1e-12)
    zero = np.zeros_like(pos)
    np.testing.assert_array_equal(rope_ref.rotate(Q, zero, cos, sin, HD), Q)   # position 0: identity
    p1, p2 = np.full_like(pos, 3), np.full_like(pos, 5)                        # R(3) R(5) = R(8)
    twice = rope_ref.rotate(rope_ref.rotate(Q, p1, cos, sin, HD), p2, cos, sin, HD)
    np.testing.assert_allclose(twice, rope_ref.rotate(Q, p1 + p2, cos, sin, HD), rtol=1e-12, atol=1e-12)


def test_rope_backward_matches_finite_differences():
    Q, K, pos, cos, sin = rope_inputs(3)
    rng = np.random.default_rng(4)
    dQo, dKo = rnd(rng, *Q.shape), rnd(rng, *K.shape)
    dQ, dK = rope_ref.backward(dQo, dKo, pos, cos, sin, HD)
    VQ, VK, h = rnd(rng, *Q.shape), rnd(rng, *K.shape), 1e-5

    def L(q, k):
        qo, ko = rope_ref.forward(q, k, pos, cos, sin, HD)
        return np.sum(dQo * qo) + np.sum(dKo * ko)
    fd = (L(Q + h * VQ, K + h * VK) - L(Q - h * VQ, K - h * VK)) / (2 * h)
    assert abs(fd - (np.sum(dQ * VQ) + np.sum(dK * VK))) < 1e-8 * max(1.0, abs(fd))


def test_rope_planted_sign_mistake_fails_the_complex_pin(monkeypatch):
    Q, _, pos, cos, sin = rope_inputs(5)
    orig = rope_ref.rotate
    monkeypatch.setattr(rope_ref, "rotate", lambda x, p, c, s, hd, sign=1.0: orig(x, p, c, s, hd, -sign))
    with pytest.raises(AssertionError):
        test_rope_equals_complex_multiplication()


def test_synth_rope_tables_are_the_definition():
    """The product's input generator builds the same tables (to fp32)."""
    c32, s32 = synth.rope_tables(2048, 128, 500000.0)
    cos, sin = rope_ref.tables(2048, 128, 500000.0)
    assert c32.dtype == np.float32 and s32.dtype == np.float32
    np.testing.assert_allclose(c32, cos, rtol=0, atol=2e-7)
    np.testing.assert_allclose(s32, sin, rtol=0, atol=2e-7)


# ------------------------------------------------------------------ cross-entropy
def ce_inputs(seed=0, T=7, d=6, V=11):
    rng = np.random.default_rng(seed)
    labels = rng.integers(0, V, T)
    labels[1] = -100          # the usual ignore index
    labels[4] = V + 3         # out of range: left out as well
    return rnd(rng, T, d), rnd(rng, V, d, scale=0.7), labels


def test_ce_logsumexp_matches_scipy():
    H, W, _ = ce_inputs(1)
    z = H @ W.T
    np.testing.assert_allclose(ce_ref.logsumexp(z), scipy.special.logsumexp(z, axis=1), rtol=1e-14)


def test_ce_brute_force_loss():
    H, W, labels = ce_inputs(2)
    R = ce_ref.forward(H, W, labels)
    total, n = 0.0, 0
    for t in range(H.shape[0]):
        z = [sum(H[t, i] * W[v, i] for i in range(H.shape[1])) for v in range(W.shape[0])]
        lse = math.log(sum(math.exp(x) for x in z))
        assert abs(R["lse"][t] - lse) < 1e-12
        if 0 <= labels[t] < W.shape[0]:
            assert abs(R["loss_rows"][t] - (lse - z[labels[t]])) < 1e-12
            total += lse - z[labels[t]]
            n += 1
        else:
            assert R["loss_rows"][t] == 0.0
    assert R["n_valid"] == n == 5
    assert abs(R["loss"] - total / n) < 1e-12


def test_ce_uniform_logits_give_log_V():
    H, W, labels = ce_inputs(3)
    R = ce_ref.forward(H, np.zeros_like(W), labels)
    ok = ce_ref.valid(labels, W.shape[0])
    np.testing.assert_allclose(R["loss_rows"][ok], math.log(W.shape[0]), rtol=1e-15)


def test_ce_invariant_to_a_constant_logit_shift():
    """A constant added to every logit of a row (a ones column in H against a constant
    column in W) changes neither the loss nor dH's original columns."""
    H, W, labels = ce_inputs(4)
    H2 = np.concatenate([H, np.ones((H.shape[0], 1))], axis=1)
    W2 = np.concatenate([W, np.full((W.shape[0], 1), 3.25)], axis=1)
    np.testing.assert_allclose(ce_ref.forward(H2, W2, labels)["loss"], ce_ref.forward(H, W, labels)["loss"],
                               rtol=1e-13)
    np.testing.assert_allclose(ce_ref.backward(H2, W2, labels)[:, :-1], ce_ref.backward(H, W, labels),
                               rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("reduction", ["mean", "sum"])
def test_ce_backward_matches_finite_differences(reduction):
    H, W, labels = ce_inputs(5)
    g, h = 0.8, 1e-6
    dH = ce_ref.backward(H, W, labels, g, reduction)
    V = np.random.default_rng(6).standard_normal(H.shape)
    L = lambda x: g * ce_ref.forward(x, W, labels, reduction)["loss"]   # noqa: E731
    fd = (L(H + h * V) - L(H - h * V)) / (2 * h)
    assert abs(fd - np.sum(dH * V)) < 1e-7 * max(1.0, abs(fd))
    ok = ce_ref.valid(labels, W.shape[0])
    assert np.all(dH[~ok] == 0)


def test_ce_softmax_rows_sum_to_one():
    """With every LM-head row equal, sum_v (softmax - onehot) = 0 gives dH = 0."""
    H, W, labels = ce_inputs(6)
    Weq = np.tile(W[:1], (W.shape[0], 1))
    np.testing.assert_allclose(ce_ref.backward(H, Weq, labels), 0.0, atol=1e-14)


def test_ce_rows_equal_full_and_no_kept_tokens():
    H, W, labels = ce_inputs(7, T=9)
    full_f, full_b = ce_ref.forward(H, W, labels), ce_ref.backward(H, W, labels)
    rows = np.array([0, 1, 4, 8])
    sub = ce_ref.rows_fwd_bwd(H, W, labels, rows, full_f["n_valid"])
    np.testing.assert_allclose(sub["loss_rows"], full_f["loss_rows"][rows], rtol=1e-14)
    np.testing.assert_allclose(sub["dH"], full_b[rows], rtol=1e-13, atol=1e-16)
    none = np.full_like(labels, -100)
    assert ce_ref.forward(H, W, none)["loss"] == 0.0 and np.all(ce_ref.backward(H, W, none) == 0)


def test_ce_planted_mistake_fails_the_fd_pin(monkeypatch):
    """The label term dropped from the backward (softmax alone) fails the FD pin."""
    H, W, labels = ce_inputs(8)
    h = 1e-6
    V = np.random.default_rng(9).standard_normal(H.shape)
    L = lambda x: ce_ref.forward(x, W, labels)["loss"]   # noqa: E731
    fd = (L(H + h * V) - L(H - h * V)) / (2 * h)

    def bad(H, W, labels, g=1.0, reduction="mean"):
        ok = ce_ref.valid(labels, W.shape[0])
        z = H @ W.T
        p = np.exp(z - ce_ref.logsumexp(z)[:, None])
        p[~ok] = 0.0
        return g / ok.sum() * (p @ W)
    monkeypatch.setattr(ce_ref, "backward", bad)
    assert abs(fd - np.sum(ce_ref.backward(H, W, labels) * V)) > 1e-3
