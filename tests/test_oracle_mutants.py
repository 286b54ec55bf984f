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
