"""Pins for the oracle's FP8 latent-cache read-back (``e4m3_value``, ``latent_cache_dequant``).

e4m3_value is checked code by code against hand-worked values of the format and against torch's
float8_e4m3fn decode of all 256 codes (a library routine, independent of the oracle's arithmetic).
latent_cache_dequant is checked on constructed caches whose dequantised values are known in closed
form.  Planted mistakes (mutants built here, on the CPU) must each fail at least one pin."""

import numpy as np
import pytest
import torch

from oracle import mla_oracle as O


# ------------------------------------------------------------------------------------------
# Mutants of the two functions
# ------------------------------------------------------------------------------------------

def _decode(c, bias=7, mant_div=8.0, subnormal=True):
    c = np.asarray(c, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / mant_div) * np.exp2(e - float(bias))
    val = np.where(e == 0, m / mant_div * 2.0 ** (1 - bias), normal) if subnormal else normal
    return np.where((c & 0x7F) == 0x7F, np.nan, sign * val)


def dec_bias8(c):
    return _decode(c, bias=8)


def dec_mant16(c):
    return _decode(c, mant_div=16.0)


def dec_no_subnormals(c):
    return _decode(c, subnormal=False)


def dq_ok(c8, s):
    return O.latent_cache_dequant(c8, s)


def dq_block64(c8, s):
    """Scale column f // 64 (clipped) instead of f // 128."""
    v = O.e4m3_value(c8)
    idx = np.minimum(np.arange(v.shape[-1]) // 64, s.shape[-1] - 1)
    return v * np.asarray(s, dtype=np.float64)[..., idx]


def dq_divide(c8, s):
    """Dividing by the scale instead of multiplying."""
    v = O.e4m3_value(c8)
    return v / np.asarray(s, dtype=np.float64)[..., np.arange(v.shape[-1]) // 128]


def dq_first_row_scale(c8, s):
    """Every row read with the first row's scales."""
    v = O.e4m3_value(c8)
    s = np.asarray(s, dtype=np.float64)
    return v * s[:1, np.arange(v.shape[-1]) // 128]


DECODERS = [O.e4m3_value, dec_bias8, dec_mant16, dec_no_subnormals]
DEQUANTS = [dq_ok, dq_block64, dq_divide, dq_first_row_scale]


# ------------------------------------------------------------------------------------------
# Pins of the decoder
# ------------------------------------------------------------------------------------------

def pin_hand_values(dec):
    """Worked by hand from the format: 0x38 = 1, 0x40 = 2, 0x7E = 1.75 * 2^8 = 448 (largest
    finite), 0x01 = 2^-9 (smallest subnormal), 0x08 = 2^-6 (smallest normal), 0x07 = 7 * 2^-9,
    0xC4 = -(1.5 * 2^1) = -3, 0x80 = -0."""
    codes = [0x38, 0x40, 0x7E, 0x01, 0x08, 0x07, 0xC4, 0x80]
    want = [1.0, 2.0, 448.0, 2.0 ** -9, 2.0 ** -6, 7 * 2.0 ** -9, -3.0, -0.0]
    got = dec(codes)
    return np.array_equal(got, want) and np.signbit(got[-1])


def pin_nan_codes(dec):
    """Exactly two codes are NaN: 0x7F and 0xFF."""
    v = dec(np.arange(256, dtype=np.uint8))
    return set(np.flatnonzero(np.isnan(v)).tolist()) == {0x7F, 0xFF}


def pin_torch_decode(dec):
    """All 256 codes against torch's float8_e4m3fn decode."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = dec(codes)
    return bool(np.all((got == ref) | (np.isnan(got) & np.isnan(ref))))


DEC_PINS = [pin_hand_values, pin_nan_codes, pin_torch_decode]


@pytest.mark.parametrize("pin", DEC_PINS, ids=lambda p: p.__name__)
def test_decoder_pins_hold(pin):
    assert pin(O.e4m3_value)


@pytest.mark.parametrize("mutant", DECODERS[1:], ids=lambda m: m.__name__)
def test_decoder_mistakes_are_caught(mutant):
    assert not all(p(mutant) for p in DEC_PINS)


# ------------------------------------------------------------------------------------------
# Pins of the cache read-back
# ------------------------------------------------------------------------------------------

def pin_unit_codes(dq):
    """Every code 0x38 (= 1): the read-back is the scale grid itself, broadcast over each
    128-feature block of its row."""
    L = 5
    s = np.arange(1, 4 * L + 1, dtype=np.float32).reshape(L, 4) * 0.25
    c8 = np.full((L, 512), 0x38, dtype=np.uint8)
    want = np.repeat(s.astype(np.float64), 128, axis=1)
    return np.array_equal(dq(c8, s), want)


def pin_one_hot(dq):
    """A single non-zero code per row, at feature 300 of row t (block 2): only that element is
    non-zero and it equals 2 * scale[t, 2]."""
    L = 3
    s = np.array([[1, 2, 3, 4], [5, 6, 7, 8], [0.5, 0.25, 0.125, 0.0625]], dtype=np.float32)
    c8 = np.zeros((L, 512), dtype=np.uint8)
    c8[:, 300] = 0x40
    got = dq(c8, s)
    want = np.zeros((L, 512))
    want[:, 300] = 2.0 * s[:, 2]
    return np.array_equal(got, want)


def pin_round_trip(dq):
    """Quantised with scale = block max / 448 (torch's float8 cast of x / scale), the read-back is
    within the format's relative precision (2^-4 for normal values) of x."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((6, 512)) * np.exp(rng.uniform(-3, 3, (6, 1)))
    blocks = x.reshape(6, 4, 128)
    s = (np.abs(blocks).max(axis=-1) / 448.0).astype(np.float32)
    q = torch.from_numpy((blocks / s[..., None].astype(np.float64)).reshape(6, 512)).to(torch.float8_e4m3fn)
    c8 = q.view(torch.uint8).numpy()
    got = dq(c8, s)
    big = np.abs(x) > 4 * np.repeat(s.astype(np.float64), 128, axis=1) * 2.0 ** -6
    return bool(np.all(np.abs(got - x)[big] <= 2.0 ** -4 * np.abs(x)[big]))


DQ_PINS = [pin_unit_codes, pin_one_hot, pin_round_trip]


@pytest.mark.parametrize("pin", DQ_PINS, ids=lambda p: p.__name__)
def test_dequant_pins_hold(pin):
    assert pin(dq_ok)


@pytest.mark.parametrize("mutant", DEQUANTS[1:], ids=lambda m: m.__name__)
def test_dequant_mistakes_are_caught(mutant):
    assert not all(p(mutant) for p in DQ_PINS)
