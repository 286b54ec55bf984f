"""Pins of the oracle's 4-bit codebook and quantiser (CPU only)."""
from fractions import Fraction

import numpy as np
import scipy.stats

from lora_fine_tuning_rmsnorm_b200 import synth
from oracle import quant4_ref as q4


def test_codebook_matches_library_normal_quantiles():
    c = q4.codebook16()
    q = scipy.stats.norm.ppf((np.arange(16) + 0.5) / 16.0)
    np.testing.assert_array_equal(c, (q / np.abs(q).max()).astype(np.float32))


def test_codebook_shape_properties():
    c = q4.codebook16().astype(np.float64)
    assert c.dtype == np.float64 and c.shape == (16,)
    assert np.all(np.diff(c) > 0)
    assert c[0] == -1.0 and c[15] == 1.0
    np.testing.assert_array_equal(c, -c[::-1])
    assert not np.any(c == 0.0)


def _blocks(seed=0, nblk=40, block=64):
    rng = np.random.default_rng(seed)
    w = (0.02 * rng.standard_normal((nblk, block))).astype(np.float32)
    w = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(w))
    w[3] = 0.0                                  # an all-zero block
    w[4, :] = -0.0
    w[5, 7] = w[5].max() * 3                    # a positive absmax element
    w[6, 9] = -abs(w[6]).max() * 3              # a negative absmax element
    return w


def test_rule_equals_exact_rational_count():
    """idx = #{i : w > absmax * m_i}, evaluated in exact rational arithmetic."""
    c = q4.codebook16()
    m = q4.midpoints(c)
    w = _blocks(seed=1, nblk=8)
    idx, absmax = q4.quantize(w, c)
    idx = idx.reshape(w.shape)
    for b in range(w.shape[0]):
        a = Fraction(float(absmax[b]))
        assert a == max(abs(Fraction(float(v))) for v in w[b])
        for j in range(w.shape[1]):
            x = Fraction(float(w[b, j]))
            cnt = sum(1 for mi in m if x > a * Fraction(float(mi)))
            assert idx[b, j] == cnt


def test_nearest_code_with_lower_tie():
    c = q4.codebook16().astype(np.float64)
    w = _blocks(seed=2)
    idx, absmax = q4.quantize(w, c.astype(np.float32))
    idx = idx.reshape(w.shape)
    for b in range(w.shape[0]):
        if absmax[b] == 0:
            assert np.all(idx[b] == 0)
            continue
        v = w[b].astype(np.float64) / absmax[b]
        dist = np.abs(v[:, None] - c[None, :])
        best = dist.min(axis=1)
        chosen = dist[np.arange(v.size), idx[b]]
        # nearest up to the fp32 rounding of the midpoints
        assert np.all(chosen <= best + 1e-6)
    # exact midpoints go to the lower index
    m = q4.midpoints(c.astype(np.float32)).astype(np.float64)
    blk = np.zeros(64); blk[0] = 1.0; blk[1:16] = m
    idx2, _ = q4.quantize(blk.astype(np.float32).astype(np.float64), c.astype(np.float32))
    np.testing.assert_array_equal(idx2[1:16], np.arange(15))


def test_absmax_element_maps_to_end_codes_and_idempotence():
    c = q4.codebook16()
    w = _blocks(seed=3)
    idx, absmax = q4.quantize(w, c)
    idx = idx.reshape(w.shape)
    for b in range(w.shape[0]):
        if absmax[b] == 0:
            continue
        j = int(np.argmax(np.abs(w[b])))
        assert idx[b, j] == (15 if w[b, j] > 0 else 0)
    wh = q4.dequantize(idx.reshape(-1), absmax, c, w.shape)
    idx2, absmax2 = q4.quantize(wh, c)
    np.testing.assert_array_equal(idx2, idx.reshape(-1))
    np.testing.assert_array_equal(absmax2, absmax)


def test_dequant_error_bound():
    c = q4.codebook16().astype(np.float64)
    gap = np.max(np.diff(c))
    w = _blocks(seed=4)
    idx, absmax = q4.quantize(w, c.astype(np.float32))
    wh = q4.dequantize(idx, absmax, c.astype(np.float32), w.shape)
    bound = np.repeat(absmax.astype(np.float64), 64).reshape(w.shape) * gap / 2
    assert np.all(np.abs(w - wh) <= bound * (1 + 1e-6))


def test_pack_nibble_order_roundtrip():
    idx = np.arange(32, dtype=np.uint8) % 16
    p = q4.pack(idx)
    assert p[0] == (0 | (1 << 4)) and p[7] == (14 | (15 << 4))
    np.testing.assert_array_equal(q4.unpack(p), idx)


def test_golden_codebook_file_matches_oracle():
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "codebook16.json")) as fh:
        j = json.load(fh)
    got = np.array([float.fromhex(h) for h in j["codebook_f32_hex"]], dtype=np.float64)
    np.testing.assert_array_equal(got, q4.codebook16().astype(np.float64))


def test_stored_codebook_is_the_oracles():
    """tests/golden/codebook16.json (the 4-bit kernels' codebook input) holds exactly the
    oracle's fp32 codebook, as written by tests/golden/make_codebook.py."""
    from tests.parity import load_codebook
    np.testing.assert_array_equal(np.asarray(load_codebook(), dtype=np.float64),
                                  q4.codebook16().astype(np.float64))
