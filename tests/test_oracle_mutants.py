"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch
each one: a dropped term, a wrong sign, a wrong index, a transposed operand."""
import numpy as np
import pytest

from oracle import lora_mlp_ref as ref
from tests.test_oracle_pins import fd_errors, tiny_inputs


def _bwd_drop_lora_dH(fw, dY, X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual=False):
    out = ORIG_BWD(fw, dY, X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual)
    dH = out["dG"] @ Wg + out["dU"] @ Wu          # missing s (Qg Ag + Qu Au)
    out["dX"] = ref.rmsnorm_bwd(dH, X, w, fw["rstd"])
    return out


def _bwd_swap_pg_pu(fw, dY, X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual=False):
    out = ORIG_BWD(fw, dY, X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual)
    out["dBg"] = s * (out["dG"].T @ fw["Pu"])      # wrong index (up instead of gate)
    return out


def _bwd_transposed_dAd(fw, dY, X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual=False):
    out = ORIG_BWD(fw, dY, X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual)
    Qd = dY @ Bd
    out["dAd"] = s * (Qd.T @ (out["dAct"]))        # wrong operand
    return out


def _bwd_no_scale_dBd(fw, dY, X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual=False):
    out = ORIG_BWD(fw, dY, X, w, Wg, Wu, Wd, Ag, Bg, Au, Bu, Ad, Bd, s, residual)
    out["dBd"] = dY.T @ fw["Pd"]                    # dropped scaling
    return out


def _rms_bwd_sign(dH, X, w, rstd):
    g = dH * w[None, :]
    xhat = X * rstd[:, None]
    c = np.mean(g * xhat, axis=1)
    return rstd[:, None] * (g + xhat * c[:, None])  # wrong sign


def _rms_bwd_no_w(dH, X, w, rstd):
    xhat = X * rstd[:, None]
    c = np.mean(dH * xhat, axis=1)
    return rstd[:, None] * (dH - xhat * c[:, None])  # dropped the weight


def _silu_grad_wrong(z):
    sg = ref.sigmoid(z)
    return sg * (1.0 + (1.0 - sg))                  # dropped z


ORIG_BWD = ref.backward

MUTANTS = {
    "drop_lora_term_in_dH": ("backward", _bwd_drop_lora_dH),
    "gate_grad_uses_up_P": ("backward", _bwd_swap_pg_pu),
    "dAd_wrong_operand": ("backward", _bwd_transposed_dAd),
    "dBd_missing_scale": ("backward", _bwd_no_scale_dBd),
    "rmsnorm_bwd_sign": ("rmsnorm_bwd", _rms_bwd_sign),
    "rmsnorm_bwd_drops_w": ("rmsnorm_bwd", _rms_bwd_no_w),
    "silu_grad_drops_z": ("silu_grad", _silu_grad_wrong),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_finite_difference_pin_catches_mutant(monkeypatch, name):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(ref, attr, fn)
    s, inp = tiny_inputs(seed=31)
    errs = fd_errors(inp, s, eps=0.1)
    assert max(errs.values()) > 1e-4, (name, errs)


def test_unmutated_oracle_passes_same_check():
    s, inp = tiny_inputs(seed=31)
    assert max(fd_errors(inp, s, eps=0.1).values()) < 1e-7


# ---------------------------------------------------------------- Q/K/V projections
from oracle import lora_qkv_ref as qref  # noqa: E402
from tests.test_oracle_qkv_pins import loss as qkv_loss, run as qkv_run, tiny as qkv_tiny  # noqa: E402

QKV_ORIG_BWD = qref.backward


def _qkv_bwd_drop_lora_k(fw, dQ, dK, dV, X, w, Wq, Wk, Wv, Aq, Bq, Ak, Bk, Av, Bv, s):
    out = QKV_ORIG_BWD(fw, dQ, dK, dV, X, w, Wq, Wk, Wv, Aq, Bq, Ak, Bk, Av, Bv, s)
    dH = out["dH"] - s * ((dK @ Bk) @ Ak)          # the K adapter's term missing from dH
    out["dX"] = qref.rmsnorm_bwd(dH, X, w, fw["rstd"])
    return out


def _qkv_bwd_dBv_no_scale(fw, dQ, dK, dV, X, w, Wq, Wk, Wv, Aq, Bq, Ak, Bk, Av, Bv, s):
    out = QKV_ORIG_BWD(fw, dQ, dK, dV, X, w, Wq, Wk, Wv, Aq, Bq, Ak, Bk, Av, Bv, s)
    out["dBv"] = dV.T @ fw["Pv"]                    # dropped scaling
    return out


def _qkv_bwd_dAq_wrong_operand(fw, dQ, dK, dV, X, w, Wq, Wk, Wv, Aq, Bq, Ak, Bk, Av, Bv, s):
    out = QKV_ORIG_BWD(fw, dQ, dK, dV, X, w, Wq, Wk, Wv, Aq, Bq, Ak, Bk, Av, Bv, s)
    out["dAq"] = s * ((dQ @ Bq).T @ X)              # raw X instead of the normalised H
    return out


QKV_MUTANTS = {"drop_lora_k_in_dH": _qkv_bwd_drop_lora_k, "dBv_missing_scale": _qkv_bwd_dBv_no_scale,
               "dAq_uses_X_not_H": _qkv_bwd_dAq_wrong_operand}


def _qkv_fd_max_err(inp, s):
    _, bw = qkv_run(inp, s)
    rng = np.random.default_rng(3)
    h = 1e-5
    worst = 0.0
    for name, g in (("X", "dX"), ("Aq", "dAq"), ("Bq", "dBq"), ("Ak", "dAk"), ("Bk", "dBk"), ("Av", "dAv"),
                    ("Bv", "dBv")):
        V = rng.standard_normal(inp[name].shape)
        p = dict(inp); p[name] = inp[name] + h * V
        m = dict(inp); m[name] = inp[name] - h * V
        fd = (qkv_loss(p, s) - qkv_loss(m, s)) / (2 * h)
        an = float(np.sum(bw[g] * V))
        worst = max(worst, abs(fd - an) / max(abs(fd), 1e-300))
    return worst


@pytest.mark.parametrize("name", sorted(QKV_MUTANTS))
def test_qkv_finite_difference_pin_catches_mutant(monkeypatch, name):
    monkeypatch.setattr(qref, "backward", QKV_MUTANTS[name])
    s, inp = qkv_tiny(seed=44)
    assert _qkv_fd_max_err(inp, s) > 1e-4, name


def test_qkv_unmutated_oracle_passes_same_check():
    s, inp = qkv_tiny(seed=44)
    assert _qkv_fd_max_err(inp, s) < 1e-7
