"""Parity helpers: the tolerance of the LoRA-MLP outputs against the fp64 oracle.

Per output tensor (bf16 I/O, fp32 accumulation):
  relative Frobenius error ||O - R||_F / ||R||_F <= 5e-3, and
  max |O - R| <= 2e-2 * max |R|.
"""
import numpy as np

REL_FRO = 5e-3
MAX_REL = 2e-2


def errors(out, ref):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    err = out - ref
    nref = np.linalg.norm(ref)
    rf = np.linalg.norm(err) / nref if nref > 0 else np.linalg.norm(err)
    mref = np.abs(ref).max()
    ma = np.abs(err).max() / mref if mref > 0 else np.abs(err).max()
    return float(rf), float(ma)


def assert_close(name, out, ref, rel_fro=REL_FRO, max_rel=MAX_REL):
    out = np.asarray(out, dtype=np.float64)
    assert np.all(np.isfinite(out)), f"{name}: non-finite values"
    rf, ma = errors(out, ref)
    assert rf <= rel_fro and ma <= max_rel, f"{name}: rel_fro={rf:.3e} (<= {rel_fro}), max/max={ma:.3e} (<= {max_rel})"
    return rf, ma


def to_np(t):
    import torch
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype != torch.float64 else t.cpu().numpy()


def load_codebook() -> list:
    """The 16-entry 4-bit codebook written by tests/golden/make_codebook.py (an input of
    the 4-bit kernels, computed once by the oracle)."""
    import json
    import os
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "codebook16.json")) as fh:
        return [float.fromhex(h) for h in json.load(fh)["codebook_f32_hex"]]
