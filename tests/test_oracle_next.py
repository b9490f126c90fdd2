"""Pins of the oracles for the rows ranked next: several new tokens per decode, the sparse
prefill, and the FP8 block-scaled wkv_b.  Each is checked against a form it does not share code
with (the naive prefill, the one-token decode, a brute-force gather, torch's float8 conversion)
or against facts of the number format, and planted mistakes must fail the same checks."""

import numpy as np
import pytest
import torch

import oracle as O

N_H, D_C, D_R, D_H, D_V = 4, 48, 16, 24, 20
SCALE = O.softmax_scale(D_H, D_R)


def make_seq(L, seed):
    rng = np.random.default_rng(seed)
    return dict(
        q=rng.standard_normal((L, N_H, D_H + D_R)),
        c=rng.standard_normal((L, D_C)),
        kr=rng.standard_normal((L, D_R)),
        w=rng.standard_normal((N_H * (D_H + D_V), D_C)) * 0.2,
    )


# ------------------------------------------------------------------------------------------
# Several new tokens per decode (reading: the prefill's causal rule among the new tokens)
# ------------------------------------------------------------------------------------------

def _multi_checks(fn):
    L, T = 37, 5
    x = make_seq(L, 1)
    q_nope, q_pe = x["q"][L - T:, :, :D_H], x["q"][L - T:, :, D_H:]
    got = fn(q_nope, q_pe, x["c"], x["kr"], x["w"], SCALE, D_V)
    # the naive prefill over the same rows, its last T query rows (reconstructed keys and values)
    want = O.naive_prefill(x["q"], x["c"], x["kr"], x["w"], SCALE, N_H, D_H, D_V, rows=list(range(L - T, L)))
    assert np.allclose(got["o"], want, rtol=1e-10, atol=1e-12)
    # T = 1 is the one-token absorbed decode over all L rows
    one = fn(q_nope[-1:], q_pe[-1:], x["c"], x["kr"], x["w"], SCALE, D_V)
    dec = O.absorbed_decode(q_nope[-1], q_pe[-1], x["c"], x["kr"], x["w"], SCALE, D_V)
    assert np.allclose(one["ctx"][0], dec["ctx"], rtol=1e-12, atol=1e-14)
    assert np.allclose(one["lse"][0], dec["lse"], rtol=1e-12)
    # sparse: each query's selected set, then the causal rule, equals a gather of those rows
    rng = np.random.default_rng(2)
    topk = np.stack([rng.choice(L, 9, replace=False) for _ in range(T)])
    topk[:, 0] = 0                                      # every set holds a visible row
    sp = fn(q_nope, q_pe, x["c"], x["kr"], x["w"], SCALE, D_V, topk=topk)
    for i in range(T):
        keep = np.array(sorted(t for t in set(topk[i].tolist()) if t <= L - T + i))
        o, _ = O.naive_decode(q_nope[i], q_pe[i], x["c"][keep], x["kr"][keep], x["w"], SCALE)
        assert np.allclose(sp["o"][i], o, rtol=1e-10, atol=1e-12)


def test_multi_token_decode_pins():
    _multi_checks(O.multi_token_decode)


def multi_no_causal(q_nope, q_pe, c, kr, w, scale, d_v, topk=None):
    # every new token sees all L rows: the later tokens leak into the earlier queries
    T = q_nope.shape[0]
    outs = [O.absorbed_decode(q_nope[i], q_pe[i], c, kr, w, scale, d_v,
                              None if topk is None else topk[i]) for i in range(T)]
    return {k: np.stack([o[k] for o in outs]) for k in ("ctx", "lse", "o")}


def multi_strict(q_nope, q_pe, c, kr, w, scale, d_v, topk=None):
    # off by one: query s attends t < its own position
    T, L = q_nope.shape[0], c.shape[0]
    outs = []
    for i in range(T):
        lim = max(L - T + i, 1)
        tk = None if topk is None else [t for t in topk[i] if t < lim] or [0]
        outs.append(O.absorbed_decode(q_nope[i], q_pe[i], c[:lim], kr[:lim], w, scale, d_v, tk))
    return {k: np.stack([o[k] for o in outs]) for k in ("ctx", "lse", "o")}


@pytest.mark.parametrize("mutant", [multi_no_causal, multi_strict], ids=lambda m: m.__name__)
def test_multi_token_decode_planted_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        _multi_checks(mutant)


# ------------------------------------------------------------------------------------------
# Sparse prefill (the V3.2 MHA-prefill excerpt: index mask + causal mask)
# ------------------------------------------------------------------------------------------

def _sparse_checks(fn):
    S = 29
    x = make_seq(S, 3)
    rng = np.random.default_rng(4)
    # selected sets that include future positions (the causal mask must remove them)
    topk = np.stack([rng.choice(S, 7, replace=False) for _ in range(S)])
    topk[:, 0] = np.arange(S)                           # each row selects itself
    got = fn(x["q"], x["c"], x["kr"], x["w"], SCALE, topk)
    for s in range(S):
        keep = np.array(sorted(t for t in set(topk[s].tolist()) if t <= s))
        o, _ = O.naive_decode(x["q"][s, :, :D_H], x["q"][s, :, D_H:], x["c"][keep], x["kr"][keep], x["w"], SCALE)
        assert np.allclose(got[s], o, rtol=1e-10, atol=1e-12)
    # every position selected: the dense causal prefill
    full = np.tile(np.arange(S), (S, 1))
    assert np.allclose(fn(x["q"], x["c"], x["kr"], x["w"], SCALE, full),
                       O.naive_prefill(x["q"], x["c"], x["kr"], x["w"], SCALE, N_H, D_H, D_V), rtol=1e-12)
    # only position 0 selected: every row's output is head i's value of row 0, W^UV_i c_0
    only0 = np.zeros((S, 1), dtype=np.int64)
    _, w_uv = O.split_wkv_b(x["w"], N_H, D_H, D_V)
    v0 = np.einsum("hdc,c->hd", w_uv, x["c"][0])
    assert np.allclose(fn(x["q"], x["c"], x["kr"], x["w"], SCALE, only0), np.broadcast_to(v0, (S, N_H, D_V)),
                       rtol=1e-12, atol=1e-14)


def sparse_oracle(q, c, kr, w, scale, topk):
    return O.naive_prefill(q, c, kr, w, scale, N_H, D_H, D_V, topk=topk)


def test_sparse_prefill_pins():
    _sparse_checks(sparse_oracle)


def sparse_no_causal(q, c, kr, w, scale, topk):
    return O.naive_prefill(q, c, kr, w, scale, N_H, D_H, D_V, causal=False, topk=topk)


def sparse_ignores_topk(q, c, kr, w, scale, topk):
    return O.naive_prefill(q, c, kr, w, scale, N_H, D_H, D_V)


@pytest.mark.parametrize("mutant", [sparse_no_causal, sparse_ignores_topk], ids=lambda m: m.__name__)
def test_sparse_prefill_planted_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        _sparse_checks(mutant)


# ------------------------------------------------------------------------------------------
# FP8 wkv_b with one fp32 scale per 128 x 128 block (linear excerpt; dequantised once for decode)
# ------------------------------------------------------------------------------------------

def _dequant_checks(fn):
    # e4m3 values fixed by the format (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
    # infinities, 448 the largest normal, 2^-9 the smallest subnormal), read through torch
    bits = torch.tensor([0x38, 0x40, 0x7E, 0x01, 0xB8, 0x39, 0x08], dtype=torch.uint8)
    vals = bits.view(torch.float8_e4m3fn).reshape(1, -1)
    deq = fn(vals, np.ones((1, 1)), 128)
    assert np.array_equal(deq[0], [1.0, 2.0, 448.0, 2.0 ** -9, -1.0, 1.125, 2.0 ** -6])
    # a weight that is not a whole number of blocks: the grid is ceil(out/128) x ceil(in/128)
    out_f, in_f = 300, 200
    assert O.fp8_block_scale_shape(out_f, in_f) == (3, 2)
    w_q = torch.ones((out_f, in_f)).to(torch.float8_e4m3fn)
    sc = np.arange(1.0, 7.0).reshape(3, 2)
    d = fn(w_q, sc, 128)
    for bi in range(3):
        for bj in range(2):
            blk = d[128 * bi:128 * (bi + 1), 128 * bj:128 * (bj + 1)]
            assert np.all(blk == sc[bi, bj]), (bi, bj)
    # dequantising the wkv_b of the decode: scale 1 is the identity on the fp8 values
    rng = np.random.default_rng(5)
    w = torch.from_numpy(rng.standard_normal((512, 256)).astype(np.float32) * 0.05).to(torch.float8_e4m3fn)
    assert np.array_equal(fn(w, np.ones(O.fp8_block_scale_shape(512, 256)), 128), w.float().numpy())


def test_weight_dequant_pins():
    _dequant_checks(O.weight_dequant)


def dequant_transposed(w_q, scale, block):
    w = w_q.float().numpy().astype(np.float64) if hasattr(w_q, "float") else np.asarray(w_q, dtype=np.float64)
    s = np.asarray(scale, dtype=np.float64)
    r, c = np.arange(w.shape[0]) // block, np.arange(w.shape[1]) // block
    return w * s.T[c][:, r].T if s.shape[0] == s.shape[1] else w * s.reshape(s.shape[::-1]).T[r][:, c]


def dequant_block64(w_q, scale, block):
    w = w_q.float().numpy().astype(np.float64)
    s = np.asarray(scale, dtype=np.float64)
    r = np.minimum(np.arange(w.shape[0]) // 64, s.shape[0] - 1)
    c = np.minimum(np.arange(w.shape[1]) // 64, s.shape[1] - 1)
    return w * s[r][:, c]


@pytest.mark.parametrize("mutant", [dequant_transposed, dequant_block64], ids=lambda m: m.__name__)
def test_weight_dequant_planted_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        _dequant_checks(mutant)
