"""Pins for the oracle's FP8 (E4M3) cache codec: the format's closed forms,
round-to-nearest-even ties, saturation, underflow, the per-page scale and the
round trip's error bound.  (CPU only.)"""
import numpy as np
import pytest

import oracle
from oracle import fp8


def test_decode_closed_forms():
    v = fp8.e4m3_decode
    assert v(0x38) == 1.0 and v(0xB8) == -1.0
    assert v(0x7E) == 448.0 and v(0xFE) == -448.0          # largest finite: 2^8 * 1.75
    assert v(0x08) == 2.0 ** -6                            # smallest normal
    assert v(0x01) == 2.0 ** -9 and v(0x07) == 7 * 2.0 ** -9  # subnormals m * 2^-9
    assert v(0x00) == 0.0 and np.signbit(v(0x80))
    assert v(0x40) == 2.0 and v(0x3C) == 1.5 and v(0x30) == 0.5
    assert np.isnan(v(0x7F)) and np.isnan(v(0xFF))
    vals = v(np.arange(256))
    assert np.isnan(vals).sum() == 2
    pos = vals[:0x7F]
    assert np.all(np.diff(pos) > 0)                       # codes 0x00..0x7E increase
    # every finite magnitude is m * 2^k with m in [8, 16) (normals) or m < 8 (subnormals)
    e = (np.arange(0x7F) >> 3) & 0xF
    m = np.arange(0x7F) & 7
    ref = np.where(e == 0, m * 2.0 ** -9, (8 + m) * 2.0 ** (e - 10))
    np.testing.assert_array_equal(pos, ref)


def test_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    np.testing.assert_array_equal(fp8.e4m3_encode(fp8.e4m3_decode(codes)), codes)


def test_encode_ties_go_to_the_even_code():
    enc = fp8.e4m3_encode
    assert enc(1.0625) == 0x38          # halfway 1.0 (0x38) / 1.125 (0x39): even
    assert enc(1.1875) == 0x3A          # halfway 1.125 / 1.25: 0x3A is even
    assert enc(np.float32(1.0625) + np.float32(2.0 ** -20)) == 0x39   # just past halfway: up
    assert enc(-1.0625) == 0xB8
    assert enc(2.0 ** -10) == 0x00      # halfway 0 / 2^-9: even (zero)
    assert enc(1.5 * 2.0 ** -9) == 0x02 # halfway 2^-9 / 2^-8: 0x02 is even
    assert enc(3 * 2.0 ** -11) == 0x01  # nearest subnormal


def test_encode_saturates_and_underflows():
    enc = fp8.e4m3_encode
    assert enc(448.0) == 0x7E and enc(464.0) == 0x7E and enc(1e30) == 0x7E
    assert enc(-1e6) == 0xFE
    assert enc(2.0 ** -12) == 0x00 and enc(-2.0 ** -12) == 0x80
    assert enc(np.nan) & 0x7F == 0x7F


def test_page_scale_and_round_trip_bound():
    rng = np.random.default_rng(5)
    pool = (rng.standard_normal((3, 64, 96)) * np.array([1.0, 30.0, 1e-3])[:, None, None]).astype(np.float32)
    pool[1, 10:, :] = np.nan                                  # poisoned unused slots
    codes, scales = fp8.quantize_pages(pool)
    for p in range(3):
        fin = np.isfinite(pool[p])
        amax = np.abs(pool[p][fin]).max()
        assert scales[p] == np.float32(np.float32(amax) / np.float32(448))
        # the page's largest magnitude lands on +-448 exactly
        i = np.unravel_index(np.argmax(np.where(fin, np.abs(pool[p]), -1)), pool[p].shape)
        assert fp8.e4m3_decode(codes[p][i]) == np.sign(pool[p][i]) * 448.0
    deq = fp8.dequantize_pages(codes, scales)
    fin = np.isfinite(pool)
    assert np.all(np.isnan(deq[~fin]))
    s = np.asarray(scales, dtype=np.float64)[:, None, None] * np.ones_like(pool, dtype=np.float64)
    err = np.abs(deq - pool.astype(np.float64))[fin]
    # half a unit in the last place: 2^-4 relative for normals, 2^-10 * scale for subnormals
    bound = np.maximum(np.abs(pool.astype(np.float64))[fin] * 2.0 ** -4, s[fin] * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)
    assert fp8.page_scale(np.zeros((4, 4))) == 1.0


def test_unrotate_inverts_the_cache_rotation():
    rng = np.random.default_rng(6)
    k = rng.standard_normal((50, 64))
    pos = rng.integers(0, 100000, 50)
    np.testing.assert_allclose(fp8.unrotate(oracle.cache_rows_rotated(k, pos), pos), k, atol=1e-9)


@pytest.mark.parametrize("slip", ["half_up", "no_saturation", "scale_by_max"])
def test_planted_codec_mistakes_fail_a_pin(slip, monkeypatch):
    """A plausible mistake in the codec fails one of the pins above."""
    good_encode, good_scale = fp8.e4m3_encode, fp8.page_scale
    if slip == "half_up":
        def bad(x):
            c = good_encode(x)
            xv = np.asarray(x, dtype=np.float64)
            tie = np.abs(fp8.e4m3_decode(c) - xv) == np.abs(fp8.e4m3_decode((c & 0x7F) + 1) - xv)
            return np.where(tie & (np.abs(xv) > np.abs(fp8.e4m3_decode(c))) | tie, (c + 1).astype(np.uint8), c)
        monkeypatch.setattr(fp8, "e4m3_encode", bad)
        with pytest.raises(AssertionError):
            test_encode_ties_go_to_the_even_code()
    elif slip == "no_saturation":
        monkeypatch.setattr(fp8, "e4m3_encode",
                            lambda x: np.where(np.abs(np.asarray(x, np.float64)) > 448, np.uint8(0x7F),
                                               good_encode(x)).astype(np.uint8))
        with pytest.raises(AssertionError):
            test_encode_saturates_and_underflows()
    else:
        monkeypatch.setattr(fp8, "page_scale", lambda x: np.float32(np.nanmax(np.abs(np.asarray(x, np.float32)))))
        with pytest.raises(AssertionError):
            test_page_scale_and_round_trip_bound()
