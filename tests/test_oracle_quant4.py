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


# ------------------------------------------------------------ double quantisation of absmax
def _absmax_sample(n=1000, seed=3):
    rng = np.random.default_rng(seed)
    a = np.abs(rng.standard_normal(n)).astype(np.float32) * np.float32(0.05)
    a[17] = 0.0
    a[300:556] = 0.0                  # one whole second-level block of zeros
    return a


def test_absmax8_rule_in_exact_rational_arithmetic():
    a = _absmax_sample(600)
    codes, s2 = q4.quantize_absmax8(a)
    for i in range(0, 600, 7):
        s = Fraction(float(s2[i // 256]))
        x = Fraction(float(a[i]))
        # the nearest level s k / 255, ties to the lower one
        best = min(range(256), key=lambda k: (abs(x - s * k / 255), k))
        assert codes[i] == best, (i, codes[i], best)


def test_absmax8_block_max_gets_255_and_zero_blocks_give_zero():
    a = _absmax_sample()
    codes, s2 = q4.quantize_absmax8(a)
    assert s2.size == 4 and s2[1] >= 0
    for b in range(4):
        blk = a[b * 256:(b + 1) * 256]
        if blk.max() > 0:
            assert codes[b * 256 + int(np.argmax(blk))] == 255
    assert np.all(codes[300:556][a[300:556] == 0] == 0)
    zero_block = np.zeros(256, dtype=np.float32)
    c0, s0 = q4.quantize_absmax8(zero_block)
    assert s0[0] == 0 and np.all(c0 == 0)


def test_absmax8_error_bound_and_idempotence():
    a = _absmax_sample(2000, 9)
    codes, s2 = q4.quantize_absmax8(a)
    ahat = q4.dequantize_absmax8(codes, s2)
    s = np.repeat(s2.astype(np.float64), 256)[:a.size]
    assert np.all(np.abs(ahat - a.astype(np.float64)) <= s / 510.0 * (1 + 1e-12))
    # re-quantising the levels themselves (rounded to fp32) returns the same codes
    codes2, s22 = q4.quantize_absmax8(ahat.astype(np.float32))
    np.testing.assert_array_equal(s22, s2)
    np.testing.assert_array_equal(codes2, codes)


def test_absmax8_ties_go_to_the_lower_level():
    s = np.float32(1.0)
    # a constant exactly halfway between levels 3/255 and 4/255 (3.5/255 = 7/510) when representable:
    a = np.array([s, np.float32(7.0 / 510.0)], dtype=np.float32)
    codes, _ = q4.quantize_absmax8(a)
    x = Fraction(float(a[1]))
    if x == Fraction(7, 510):
        assert codes[1] == 3
    else:   # not representable: nearest level by exact comparison
        assert codes[1] == (4 if x > Fraction(7, 510) else 3)
    # exact ties by construction: scale2 = 510 * 2^-k makes 510 a = (2j - 1) scale2 representable
    s = np.float32(510.0)
    a = np.array([s] + [np.float32(2 * j - 1) for j in (1, 2, 100, 255)], dtype=np.float32)
    codes, _ = q4.quantize_absmax8(a)
    np.testing.assert_array_equal(codes, [255, 0, 1, 99, 254])
