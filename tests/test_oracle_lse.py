"""Pins for the oracle's log-sum-exp output (the ``lse`` of ``latent_attention``,
``absorbed_decode`` and ``multi_token_decode``): the natural log of sum_t exp(s_t) over the kept
positions, s already multiplied by the softmax scale ("DeepSeek-V3.2-Exp - Absorb key weights",
decode excerpt: scaled scores, optional top-k -inf mask, softmax over positions).

Each pin fixes lse against something other than the oracle's own formula: a closed form, a
hand-built score set, or a brute force written as plain Python sums.  Planted mistakes (each a
mutant of the oracle built here, on the CPU) must each be rejected by at least one pin."""

import math

import numpy as np
import pytest

from oracle import mla_oracle as O


def _x(seed=0, n_h=3, d_c=8, d_r=4, L=7):
    r = np.random.default_rng(seed)
    return dict(q_tilde=r.standard_normal((n_h, d_c)), q_pe=r.standard_normal((n_h, d_r)),
                c_kv=r.standard_normal((L, d_c)), k_r=r.standard_normal((L, d_r)),
                scale=1.0 / math.sqrt(3 * d_c + d_r))


# ------------------------------------------------------------------------------------------
# The oracle and plausible mistakes in it
# ------------------------------------------------------------------------------------------

def lse_ok(x, topk=None):
    return O.latent_attention(x["q_tilde"], x["q_pe"], x["c_kv"], x["k_r"], x["scale"], topk)[1]


def lse_via_multi_token(x, topk=None):
    """The same quantity through multi_token_decode with T = 1 (its lse must agree).  W^UK is the
    identity on the latent so that q~ = q_nope exactly."""
    n_h, d_c = x["q_tilde"].shape
    w = np.zeros((n_h, 2 * d_c, d_c))
    for i in range(n_h):
        w[i, :d_c, :] = np.eye(d_c)
    tk = None if topk is None else np.asarray(topk)[None, :]
    out = O.multi_token_decode(x["q_tilde"][None], x["q_pe"][None], x["c_kv"], x["k_r"],
                               w.reshape(-1, d_c), x["scale"], d_c, tk)
    return out["lse"][0]


def lse_log2_units(x, topk=None):
    """log2 of the sum instead of the natural log."""
    return lse_ok(x, topk) / math.log(2.0)


def lse_unscaled(x, topk=None):
    """Scores taken before the softmax scale."""
    return lse_ok(dict(x, scale=1.0), topk)


def lse_of_mean(x, topk=None):
    """log of the mean of exp(s) instead of the sum."""
    n = x["c_kv"].shape[0] if topk is None else len(set(int(i) for i in topk))
    return lse_ok(x, topk) - math.log(n)


def lse_unmasked(x, topk=None):
    """The top-k mask left out of the normaliser."""
    return lse_ok(x, None)


def lse_no_rope(x, topk=None):
    """The rotary score term left out."""
    return lse_ok(dict(x, q_pe=np.zeros_like(x["q_pe"])), topk)


def lse_no_shift(x, topk=None):
    """log(sum(exp(s))) taken without subtracting the maximum: overflows for large scores."""
    q, p, c, k = (np.asarray(x[n], dtype=np.float64) for n in ("q_tilde", "q_pe", "c_kv", "k_r"))
    s = x["scale"] * (q @ c.T + p @ k.T)
    if topk is not None:
        s = s + O.index_mask(c.shape[0], topk)[None, :]
    with np.errstate(over="ignore"):
        return np.log(np.sum(np.exp(s), axis=-1))


MUTANTS = [lse_log2_units, lse_unscaled, lse_of_mean, lse_unmasked, lse_no_rope, lse_no_shift]


# ------------------------------------------------------------------------------------------
# Pins
# ------------------------------------------------------------------------------------------

def _scores_by_hand(x, h):
    """Head h's scaled scores written out as plain sums (math.fsum), one per cached position."""
    q, p, c, k = (np.asarray(x[n], dtype=np.float64) for n in ("q_tilde", "q_pe", "c_kv", "k_r"))
    return [x["scale"] * (math.fsum(q[h, j] * c[t, j] for j in range(c.shape[1])) +
                          math.fsum(p[h, j] * k[t, j] for j in range(k.shape[1])))
            for t in range(c.shape[0])]


def pin_single_position(fn):
    """One cached row: lse = s_0 itself (the sum has one term, exp then log)."""
    x = _x(1, L=1)
    want = np.array([_scores_by_hand(x, h)[0] for h in range(3)])
    return np.allclose(fn(x), want, rtol=1e-12, atol=1e-13)


def pin_two_keys(fn):
    """Two rows with scores fixed by construction: c_0 = 0, c_1 = e_0, k^R_0 = e_0, k^R_1 = 0,
    q~ = a e_0, q^R = b e_0, so s_0 = scale b and s_1 = scale a, and
    lse = log(exp(scale a) + exp(scale b))."""
    a, b, d_c, d_r, n_h = 1.3, -0.6, 8, 4, 2
    scale = 1.0 / math.sqrt(6.0)
    c = np.zeros((2, d_c)); c[1, 0] = 1.0
    k = np.zeros((2, d_r)); k[0, 0] = 1.0
    q = np.zeros((n_h, d_c)); q[:, 0] = a
    p = np.zeros((n_h, d_r)); p[:, 0] = b
    x = dict(q_tilde=q, q_pe=p, c_kv=c, k_r=k, scale=scale)
    want = math.log(math.exp(scale * a) + math.exp(scale * b))
    return np.allclose(fn(x), want, rtol=1e-13, atol=1e-14)


def pin_zero_query(fn):
    """q = 0: every score is 0, so lse = log L."""
    x = _x(2, L=9)
    x = dict(x, q_tilde=np.zeros_like(x["q_tilde"]), q_pe=np.zeros_like(x["q_pe"]))
    return np.allclose(fn(x), math.log(9), rtol=1e-13, atol=1e-14)


def pin_common_rotary_shift(fn):
    """Every cached rotary row equal to u: the rotary term adds the same scale (q^R . u) to every
    score of a head, so lse(q^R) = lse(q^R = 0) + scale (q^R . u) (log-sum-exp shift rule)."""
    x = _x(3, L=6)
    u = np.random.default_rng(30).standard_normal(x["k_r"].shape[1])
    x = dict(x, k_r=np.broadcast_to(u, x["k_r"].shape).copy())
    base = fn(dict(x, q_pe=np.zeros_like(x["q_pe"])))
    want = base + x["scale"] * (x["q_pe"] @ u)
    return np.allclose(fn(x), want, rtol=1e-12, atol=1e-13)


def pin_large_scores(fn):
    """Scores near 1000 (exp overflows in fp64): one row scores 1000 + d_0 and the others
    1000 + d_t, so lse = 1000 + log(sum_t exp(d_t)), computed from the small offsets."""
    d = np.array([0.25, -1.5, 0.75, 0.0])
    L, d_c = d.size, 4
    c = np.zeros((L, d_c)); c[:, 0] = 1.0; c[:, 1] = d
    q = np.zeros((1, d_c)); q[0, 0] = 1000.0; q[0, 1] = 1.0
    x = dict(q_tilde=q, q_pe=np.zeros((1, 2)), c_kv=c, k_r=np.zeros((L, 2)), scale=1.0)
    want = 1000.0 + math.log(math.fsum(math.exp(v) for v in d))
    return np.allclose(fn(x), want, rtol=1e-15, atol=1e-12)


def pin_brute_force(fn):
    """Small random inputs: lse_h = log(fsum_t exp(s_t)), the scores written out as sums."""
    x = _x(4, n_h=4, d_c=6, d_r=2, L=11)
    want = np.array([math.log(math.fsum(math.exp(s) for s in _scores_by_hand(x, h))) for h in range(4)])
    return np.allclose(fn(x), want, rtol=1e-12, atol=1e-13)


def pin_brute_force_topk(fn):
    """With a top-k set: the sum runs over the selected rows only (a set: a repeated index
    counts once)."""
    x = _x(5, n_h=3, d_c=6, d_r=2, L=13)
    topk = [7, 2, 11, 2, 0]
    keep = sorted(set(topk))
    want = np.array([math.log(math.fsum(math.exp(_scores_by_hand(x, h)[t]) for t in keep)) for h in range(3)])
    got = fn(x, topk)
    return np.allclose(got, want, rtol=1e-12, atol=1e-13)


PINS = [pin_single_position, pin_two_keys, pin_zero_query, pin_common_rotary_shift, pin_large_scores,
        pin_brute_force, pin_brute_force_topk]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
@pytest.mark.parametrize("fn", [lse_ok, lse_via_multi_token], ids=["latent_attention", "multi_token_T1"])
def test_lse_pins_hold(pin, fn):
    assert pin(fn)


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_lse_planted_mistakes_are_caught(mutant):
    assert not all(p(mutant) for p in PINS), f"no pin catches {mutant.__name__}"


def test_lse_matches_the_softmax_normaliser():
    """exp(s_t - lse) is the softmax weight the oracle returns (the two outputs agree)."""
    x = _x(6, n_h=2, L=5)
    ctx, lse, alpha = O.latent_attention(x["q_tilde"], x["q_pe"], x["c_kv"], x["k_r"], x["scale"])
    for h in range(2):
        s = _scores_by_hand(x, h)
        assert np.allclose([math.exp(v - lse[h]) for v in s], alpha[h], rtol=1e-12, atol=1e-15)
