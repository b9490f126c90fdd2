"""Pins of the cache-append oracle (``rms_norm``, ``rope_interleaved``, ``cache_append``) against
what the pages and the mathematics fix, independent of the oracle's own formulas: a library
routine (torch's fp64 ``rms_norm``), invariants of a rotation, hand-computed values, and planted
mistakes that must fail them."""

import math

import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(11)


# ------------------------------------------------------------------------------------------
# RMSNorm ("Key-value latent RMSNorm": fp32, x rsqrt(mean(x^2) + eps), one gain per feature)
# ------------------------------------------------------------------------------------------

def _rms_checks(fn):
    x = RNG.standard_normal((5, 512))
    g = RNG.uniform(0.5, 1.5, 512)
    # the library routine, in fp64
    want = torch.nn.functional.rms_norm(torch.from_numpy(x), (512,), torch.from_numpy(g), eps=1e-6).numpy()
    assert np.allclose(fn(x, g, 1e-6), want, rtol=1e-12, atol=1e-12)
    # a constant row c * 1 normalises to c / sqrt(c^2 + eps) (textbook special case)
    c = np.full((1, 8), 0.01)
    assert np.allclose(fn(c, None, 1e-4), 0.01 / math.sqrt(1e-4 + 1e-4), rtol=1e-12)
    # without eps the output has unit mean square and does not depend on the row's scale
    y = fn(x, None, 0.0)
    assert np.allclose(np.mean(y * y, -1), 1.0, rtol=1e-12)
    assert np.allclose(fn(-3.5 * x, None, 0.0), -y, rtol=1e-12)
    # the gain scales the normalised row feature by feature (it is not normalised away)
    assert np.allclose(fn(x, g, 1e-6), g * fn(x, None, 1e-6), rtol=1e-12)


def test_rms_norm_pins():
    _rms_checks(O.rms_norm)


def rms_no_eps(x, g, eps):
    return O.rms_norm(x, g, 0.0)


def rms_gain_first(x, g, eps):
    x = np.asarray(x, dtype=np.float64)
    return O.rms_norm(x if g is None else x * g, None, eps)


def rms_mean_abs(x, g, eps):
    x = np.asarray(x, dtype=np.float64)
    y = x / (np.mean(np.abs(x), -1, keepdims=True) + eps)
    return y if g is None else y * g


@pytest.mark.parametrize("mutant", [rms_no_eps, rms_gain_first, rms_mean_abs], ids=lambda m: m.__name__)
def test_rms_norm_planted_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        _rms_checks(mutant)


# ------------------------------------------------------------------------------------------
# Rotary embedding of the shared key (reading: interleaved pairs, angle pos base^(-2i/d))
# ------------------------------------------------------------------------------------------

def _rope_checks(fn):
    d = 64
    y = RNG.standard_normal((6, d))
    pos = np.array([0, 1, 7, 1000, 4095, 65535])
    r = fn(y, pos, 10000.0)
    # position 0 is the identity
    assert np.allclose(r[0], y[0], rtol=0, atol=1e-15)
    # every pair keeps its length (a rotation)
    assert np.allclose(np.hypot(r[:, 0::2], r[:, 1::2]), np.hypot(y[:, 0::2], y[:, 1::2]), rtol=1e-12)
    # rotating by a then by b equals rotating by a + b
    a, b = np.array([3, 500, 17, 2]), np.array([11, 29, 4000, 60000])
    yy = y[:4]
    assert np.allclose(fn(fn(yy, a, 10000.0), b, 10000.0), fn(yy, a + b, 10000.0), rtol=1e-9, atol=1e-9)
    # scores depend on the relative position only: <R(m) q, R(n) k> = <R(m - n) q, k>
    q, k = RNG.standard_normal((1, d)), RNG.standard_normal((1, d))
    for m, n in ((5, 2), (100, 37), (4000, 4000)):
        lhs = (fn(q, [m], 10000.0) @ fn(k, [n], 10000.0).T).item()
        rhs = (fn(q, [m - n], 10000.0) @ k.T).item()
        assert abs(lhs - rhs) < 1e-9 * (1 + abs(lhs))
    # hand-computed values: pair 0 turns by pos radians counter-clockwise, (1, 0) -> (cos 1, sin 1);
    # pair 1 of a 4-wide key turns by pos * base^(-1/2): at base 10000 and pos 100, one radian
    one = fn(np.array([[1.0, 0.0, 1.0, 0.0]]), [1], 10000.0)[0]
    assert np.allclose(one[:2], [math.cos(1.0), math.sin(1.0)], rtol=0, atol=1e-15)
    hundred = fn(np.array([[0.0, 0.0, 1.0, 0.0]]), [100], 10000.0)[0]
    assert np.allclose(hundred[2:], [math.cos(1.0), math.sin(1.0)], rtol=0, atol=1e-12)


def test_rope_pins():
    _rope_checks(O.rope_interleaved)


def rope_clockwise(y, pos, base):
    return O.rope_interleaved(y, -np.asarray(pos), base)


def rope_freq_i_over_d(y, pos, base):
    return O.rope_interleaved(y, pos, base * base)  # base^(-2i/d) squared = base^(-4i/d): wrong ladder


def rope_half_split(y, pos, base):
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    inter = np.empty_like(y)
    inter[:, 0::2], inter[:, 1::2] = y[:, : d // 2], y[:, d // 2:]
    r = O.rope_interleaved(inter, pos, base)
    return np.concatenate([r[:, 0::2], r[:, 1::2]], -1)


def rope_sign_slip(y, pos, base):
    # the sine term of the odd output mis-signed: [[c, -s], [-s, c]] is no rotation
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[:, None] * base ** (-np.arange(0, d, 2) / d)
    c, s = np.cos(ang), np.sin(ang)
    r = np.empty_like(y)
    r[:, 0::2] = y[:, 0::2] * c - y[:, 1::2] * s
    r[:, 1::2] = -y[:, 0::2] * s + y[:, 1::2] * c
    return r


@pytest.mark.parametrize("mutant", [rope_clockwise, rope_freq_i_over_d, rope_half_split, rope_sign_slip],
                         ids=lambda m: m.__name__)
def test_rope_planted_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        _rope_checks(mutant)


# ------------------------------------------------------------------------------------------
# The split ("Key-value down-projection": latent first, rotary key last)
# ------------------------------------------------------------------------------------------

def test_cache_append_split():
    d_c, d_r = 512, 64
    kv = RNG.standard_normal((3, d_c + d_r))
    g = RNG.uniform(0.5, 1.5, d_c)
    c, k = O.cache_append(kv, [0, 0, 0], d_c, d_r, g, 1e-6)
    # position 0: the rotary part passes through unchanged, the latent part is normalised alone
    assert np.array_equal(k, kv[:, d_c:])
    want = torch.nn.functional.rms_norm(torch.from_numpy(kv[:, :d_c]), (d_c,), torch.from_numpy(g), eps=1e-6)
    assert np.allclose(c, want.numpy(), rtol=1e-12, atol=1e-12)
    # the rotary part never leaks into the latent's norm
    kv2 = kv.copy()
    kv2[:, d_c:] *= 100.0
    c2, _ = O.cache_append(kv2, [5, 6, 7], d_c, d_r, g, 1e-6)
    assert np.array_equal(c, c2)
