"""Pins for the CPU oracle: facts the pages print, closed forms, library special cases and
brute force.  Each pin is also run against a planted mistake (a mutant of the oracle built
here, on the CPU) to show that the pin would catch it."""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _tiny(seed=0, n_h=3, d_c=8, d_r=4, d_h=5, d_v=6, L=7):
    r = _rng(seed)
    return dict(
        q_nope=r.standard_normal((n_h, d_h)), q_pe=r.standard_normal((n_h, d_r)),
        c_kv=r.standard_normal((L, d_c)), k_r=r.standard_normal((L, d_r)),
        w_kv_b=r.standard_normal((n_h * (d_h + d_v), d_c)) * 0.3,
        scale=1.0 / math.sqrt(d_h + d_r), d_v=d_v)


# ------------------------------------------------------------------------------------------
# Mutants: plausible mistakes, each of which some pin below must reject
# ------------------------------------------------------------------------------------------

def _swap_uk_uv(w, n_h, d_h, d_v):
    """W^UK and W^UV slices exchanged ("KV Reconstruction", "Watch-outs")."""
    assert d_h == d_v
    w = np.asarray(w, dtype=np.float64).reshape(n_h, d_h + d_v, -1)
    return np.concatenate([w[:, d_h:], w[:, :d_h]], axis=1).reshape(n_h * (d_h + d_v), -1)


def decode_ok(x, topk=None):
    return O.absorbed_decode(x["q_nope"], x["q_pe"], x["c_kv"], x["k_r"], x["w_kv_b"], x["scale"],
                             x["d_v"], topk)["o"]


def decode_naive(x, topk=None):
    return O.naive_decode(x["q_nope"], x["q_pe"], x["c_kv"], x["k_r"], x["w_kv_b"], x["scale"], topk)[0]


def decode_swapped(x, topk=None):
    n_h, d_h = x["q_nope"].shape
    y = dict(x, w_kv_b=_swap_uk_uv(x["w_kv_b"], n_h, d_h, x["d_v"]))
    return decode_ok(y, topk)


def decode_no_rope(x, topk=None):
    return decode_ok(dict(x, q_pe=np.zeros_like(x["q_pe"])), topk)


def decode_head_scale(x, topk=None):
    d_h = x["q_nope"].shape[1]
    return decode_ok(dict(x, scale=1.0 / math.sqrt(d_h)), topk)


def decode_rope_full_key(x, topk=None):
    """Rotary applied over the whole reconstructed key ("KV Reconstruction", "Watch-outs"):
    here, a fixed rotation of every adjacent pair of the 192-wide key by position t."""
    q_nope, q_pe, c, kr, w, scale = (np.asarray(x[k], dtype=np.float64)
                                     for k in ("q_nope", "q_pe", "c_kv", "k_r", "w_kv_b", "scale"))
    n_h, d_h = q_nope.shape
    w_uk, w_uv = O.split_wkv_b(w, n_h, d_h, x["d_v"])
    k = np.concatenate([np.einsum("hdc,tc->thd", w_uk, c),
                        np.broadcast_to(kr[:, None, :], (c.shape[0], n_h, kr.shape[1]))], -1)
    t = np.arange(c.shape[0])[:, None, None]
    ke, ko = k[..., 0::2].copy(), k[..., 1::2].copy()
    k[..., 0::2] = ke * np.cos(t * 0.5) - ko * np.sin(t * 0.5)
    k[..., 1::2] = ke * np.sin(t * 0.5) + ko * np.cos(t * 0.5)
    s = scale * np.einsum("hd,thd->ht", np.concatenate([q_nope, q_pe], -1), k)
    a = O.softmax(s)
    return np.einsum("ht,thd->hd", a, np.einsum("hdc,tc->thd", w_uv, c))


MUTANTS = [decode_swapped, decode_no_rope, decode_head_scale, decode_rope_full_key]


# ------------------------------------------------------------------------------------------
# Facts the pages print
# ------------------------------------------------------------------------------------------

def test_page_counts_and_shapes():
    g = json.load(open(GOLDEN))
    d = g["deepseek_v3_dims"]["value"]
    assert O.value_up_params(d["n_h"], d["d_v"], d["d_c"]) == g["value_up_params_per_instance"]["value"]
    assert 58 * O.value_up_params(d["n_h"], d["d_v"], d["d_c"]) == g["value_up_params_58_blocks"]["value"]
    w = np.zeros(tuple(g["wkv_b_shape"]["value"]), dtype=np.float32)
    w_uk, w_uv = O.split_wkv_b(w, d["n_h"], d["d_h"], d["d_v"])
    up = tuple(g["up_projection_shape_671b"]["value"])
    assert (w_uk.shape[0] * w_uk.shape[1], w_uk.shape[2]) == up
    assert (w_uv.shape[0] * w_uv.shape[1], w_uv.shape[2]) == up
    assert w_uv.size == g["value_up_params_per_instance"]["value"]
    assert d["d_h"] + 64 == g["key_width"]["value"]
    assert abs(O.softmax_scale(128, 64) - 192 ** -0.5) < 1e-15


def test_cache_size_formulas_match_real_buffers():
    """"Decoupled RoPE": the MLA cache is B N (d_c + d_R) s bytes, MHA's is 2 B N h_q d_h s.
    Checked against the byte size of actual cache buffers of those shapes."""
    B, N = 3, 17
    for dt, s in ((torch.bfloat16, 2), (torch.float32, 4)):
        mla = torch.empty((B, N, 512 + 64), dtype=dt)
        assert mla.numel() * mla.element_size() == O.mla_cache_bytes(B, N, 512, 64, s)
        k = torch.empty((B, N, 128, 128), dtype=dt)
        v = torch.empty((B, N, 128, 128), dtype=dt)
        kv_bytes = (k.numel() * k.element_size()) + (v.numel() * v.element_size())
        assert kv_bytes == O.mha_cache_bytes(B, N, 128, 128, s)
    # the decode workload: 32 x 4096 rows of 576 bf16 values
    assert O.mla_cache_bytes(32, 4096, 512, 64, 2) == 150_994_944


# ------------------------------------------------------------------------------------------
# The absorb identity ("KV Reconstruction", "Absorb path")
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("seed,dims", [(0, (3, 8, 4, 5, 6, 7)), (1, (4, 64, 16, 32, 32, 64)),
                                       (2, (2, 16, 2, 16, 3, 1)), (3, (5, 12, 8, 7, 7, 33))])
def test_absorb_equals_naive(seed, dims):
    n_h, d_c, d_r, d_h, d_v, L = dims
    x = _tiny(seed, n_h, d_c, d_r, d_h, d_v, L)
    on, an = O.naive_decode(x["q_nope"], x["q_pe"], x["c_kv"], x["k_r"], x["w_kv_b"], x["scale"])
    ab = O.absorbed_decode(x["q_nope"], x["q_pe"], x["c_kv"], x["k_r"], x["w_kv_b"], x["scale"], d_v)
    assert np.allclose(on, ab["o"], rtol=1e-12, atol=1e-13)
    assert np.allclose(an, ab["alpha"], rtol=1e-12, atol=1e-14)


def test_absorb_equals_naive_sparse():
    x = _tiny(4, L=40)
    idx = _rng(9).choice(40, 11, replace=False)
    assert np.allclose(decode_naive(x, idx), decode_ok(x, idx), rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------------------------------
# Closed forms
# ------------------------------------------------------------------------------------------

def pin_single_position(fn):
    """One cached position: alpha = 1, so o_i = W^UV_i c_0 (rows d_h..d_h+d_v of head i)."""
    x = _tiny(5, n_h=3, d_c=8, d_r=4, d_h=6, d_v=6, L=1)
    w = x["w_kv_b"].reshape(3, 12, 8)
    want = np.stack([w[i, 6:12, :] @ x["c_kv"][0] for i in range(3)])
    return np.allclose(fn(x), want, rtol=1e-12, atol=1e-13)


def pin_two_keys(fn):
    """Two positions with known scores: W^UK_i = identity on the first d_h latent features,
    q^C = a e_0, c_0 = 0, c_1 = e_0, q^R = b e_0, k^R_0 = e_0, k^R_1 = 0.  Then
    s_0 = scale b, s_1 = scale a and alpha_1 = 1 / (1 + exp(scale (b - a)))."""
    n_h, d_c, d_r, d_h, d_v = 2, 8, 4, 6, 6
    a, b = 1.7, -0.4
    w = np.zeros((n_h, d_h + d_v, d_c))
    for i in range(n_h):
        w[i, :d_h, :d_h] = np.eye(d_h)
        w[i, d_h:, :] = _rng(11 + i).standard_normal((d_v, d_c))
    c = np.zeros((2, d_c)); c[1, 0] = 1.0
    kr = np.zeros((2, d_r)); kr[0, 0] = 1.0
    qn = np.zeros((n_h, d_h)); qn[:, 0] = a
    qp = np.zeros((n_h, d_r)); qp[:, 0] = b
    scale = 1.0 / math.sqrt(d_h + d_r)
    x = dict(q_nope=qn, q_pe=qp, c_kv=c, k_r=kr, w_kv_b=w.reshape(-1, d_c), scale=scale, d_v=d_v)
    a1 = 1.0 / (1.0 + math.exp(scale * (b - a)))
    want = np.stack([w[i, d_h:, :] @ ((1 - a1) * c[0] + a1 * c[1]) for i in range(n_h)])
    return np.allclose(fn(x), want, rtol=1e-12, atol=1e-14)


def pin_zero_query(fn):
    """q = 0: every score is 0, alpha = 1/L, o_i = W^UV_i mean_t(c_t)."""
    x = _tiny(6, L=9)
    x = dict(x, q_nope=np.zeros_like(x["q_nope"]), q_pe=np.zeros_like(x["q_pe"]))
    n_h, d_h = x["q_nope"].shape
    w = x["w_kv_b"].reshape(n_h, d_h + x["d_v"], -1)
    want = np.stack([w[i, d_h:, :] @ x["c_kv"].mean(0) for i in range(n_h)])
    return np.allclose(fn(x), want, rtol=1e-12, atol=1e-13)


def pin_sdpa(fn):
    """Library special case: build k = [W^UK c; k^R] and v = W^UV c with torch's linear and
    view/split as in the prefill excerpt, then torch's scaled_dot_product_attention (fp64)."""
    x = _tiny(7, n_h=4, d_c=10, d_r=4, d_h=6, d_v=6, L=13)
    n_h, d_h = x["q_nope"].shape
    c = torch.tensor(x["c_kv"]); w = torch.tensor(x["w_kv_b"])
    kv = torch.nn.functional.linear(c, w).view(c.shape[0], n_h, d_h + x["d_v"])
    k_nope, v = torch.split(kv, [d_h, x["d_v"]], dim=-1)
    k = torch.cat([k_nope, torch.tensor(x["k_r"])[:, None, :].expand(-1, n_h, -1)], -1)
    q = torch.cat([torch.tensor(x["q_nope"]), torch.tensor(x["q_pe"])], -1)
    o = torch.nn.functional.scaled_dot_product_attention(
        q[:, None, :], k.transpose(0, 1), v.transpose(0, 1), scale=x["scale"])[:, 0, :]
    return np.allclose(fn(x), o.numpy(), rtol=1e-12, atol=1e-13)


PINS = [pin_single_position, pin_two_keys, pin_zero_query, pin_sdpa]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
@pytest.mark.parametrize("fn", [decode_ok, decode_naive], ids=["absorbed", "naive"])
def test_pins_hold(pin, fn):
    assert pin(fn)


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_planted_mistakes_are_caught(mutant):
    assert not all(p(mutant) for p in PINS), f"no pin catches {mutant.__name__}"


def test_dominant_score():
    """One position far above the rest: alpha concentrates there, ctx equals that row."""
    x = _tiny(8, L=6)
    qt = np.zeros((3, 8)); qt[:, 2] = 1.0
    c = np.asarray(x["c_kv"]).copy(); c[4, 2] = 2000.0
    ctx, lse, a = O.latent_attention(qt, np.zeros((3, 4)), c, x["k_r"], 1.0)
    assert np.allclose(ctx, np.broadcast_to(c[4], ctx.shape), rtol=0, atol=1e-300)
    assert np.allclose(lse, 2000.0, rtol=1e-15)


def test_absorb_q_and_out_up_closed_forms():
    """q^C = e_j selects row j of W^UK_i; ctx = e_c selects column c of W^UV_i."""
    n_h, d_c, d_h, d_v = 3, 10, 4, 5
    w = _rng(12).standard_normal((n_h * (d_h + d_v), d_c))
    wr = w.reshape(n_h, d_h + d_v, d_c)
    for j in range(d_h):
        q = np.zeros((n_h, d_h)); q[:, j] = 1.0
        assert np.array_equal(O.absorb_q(q, w, n_h, d_h, d_v), wr[:, j, :])
    for cc in range(d_c):
        ctx = np.zeros((2, n_h, d_c)); ctx[:, :, cc] = 1.0
        assert np.array_equal(O.out_up(ctx, w, n_h, d_h, d_v), np.broadcast_to(wr[:, d_h:, cc], (2, n_h, d_v)))


# ------------------------------------------------------------------------------------------
# Softmax, masks, top-k (brute force)
# ------------------------------------------------------------------------------------------

def test_softmax_rows():
    from scipy.special import softmax as sp_softmax
    s = _rng(13).standard_normal((5, 40)) * 7
    a = O.softmax(s)
    assert np.allclose(a.sum(-1), 1.0, rtol=0, atol=1e-12) and (a >= 0).all()
    assert np.allclose(a, sp_softmax(s, axis=-1), rtol=1e-13, atol=1e-16)
    s[:, 3] = -np.inf
    assert (O.softmax(s)[:, 3] == 0).all()


def test_topk_brute_force():
    """The -inf scatter mask over all positions equals attention over the gathered rows."""
    x = _tiny(14, L=50)
    qt = O.absorb_q(x["q_nope"], x["w_kv_b"], 3, 5, 6)
    for k in (1, 7, 50):
        idx = _rng(15 + k).choice(50, k, replace=False)
        ctx_m, lse_m, _ = O.latent_attention(qt, x["q_pe"], x["c_kv"], x["k_r"], x["scale"], idx)
        ctx_g, lse_g, _ = O.latent_attention(qt, x["q_pe"], x["c_kv"][idx], x["k_r"][idx], x["scale"])
        assert np.allclose(ctx_m, ctx_g, rtol=1e-13, atol=1e-14)
        assert np.allclose(lse_m, lse_g, rtol=1e-13)
        if k == 1:  # a single kept row is returned exactly
            assert np.array_equal(ctx_m, np.broadcast_to(x["c_kv"][idx[0]], ctx_m.shape))
    full = O.latent_attention(qt, x["q_pe"], x["c_kv"], x["k_r"], x["scale"], np.arange(50))[0]
    dense = O.latent_attention(qt, x["q_pe"], x["c_kv"], x["k_r"], x["scale"])[0]
    assert np.allclose(full, dense, rtol=1e-14, atol=1e-15)


def test_topk_set_semantics_and_order():
    assert np.array_equal(O.index_mask(6, [1, 1, 4]), O.index_mask(6, [4, 1]))
    x = _tiny(16, L=30)
    idx = _rng(17).choice(30, 9, replace=False)
    a = decode_ok(x, idx)
    b = decode_ok(x, idx[::-1].copy())
    assert np.allclose(a, b, rtol=1e-14, atol=1e-15)
    with pytest.raises(AssertionError):
        O.index_mask(6, [6])


# ------------------------------------------------------------------------------------------
# Prefill
# ------------------------------------------------------------------------------------------

def _prefill_inputs(seed=18, S=9, n_h=3, d_c=8, d_r=4, d_h=5, d_v=6):
    r = _rng(seed)
    return dict(q=r.standard_normal((S, n_h, d_h + d_r)), c_kv=r.standard_normal((S, d_c)),
                k_r=r.standard_normal((S, d_r)), w=r.standard_normal((n_h * (d_h + d_v), d_c)) * 0.3,
                dims=(n_h, d_h, d_v), scale=1.0 / math.sqrt(d_h + d_r))


def test_prefill_last_row_equals_absorbed_decode():
    p = _prefill_inputs()
    n_h, d_h, d_v = p["dims"]
    out = O.naive_prefill(p["q"], p["c_kv"], p["k_r"], p["w"], p["scale"], n_h, d_h, d_v)
    last = O.absorbed_decode(p["q"][-1, :, :d_h], p["q"][-1, :, d_h:], p["c_kv"], p["k_r"], p["w"],
                             p["scale"], d_v)["o"]
    assert np.allclose(out[-1], last, rtol=1e-12, atol=1e-13)
    # a middle row equals decode over the prefix
    mid = O.absorbed_decode(p["q"][4, :, :d_h], p["q"][4, :, d_h:], p["c_kv"][:5], p["k_r"][:5], p["w"],
                            p["scale"], d_v)["o"]
    assert np.allclose(out[4], mid, rtol=1e-12, atol=1e-13)


def test_prefill_first_row_and_sdpa():
    p = _prefill_inputs(19)
    n_h, d_h, d_v = p["dims"]
    out = O.naive_prefill(p["q"], p["c_kv"], p["k_r"], p["w"], p["scale"], n_h, d_h, d_v)
    w = p["w"].reshape(n_h, d_h + d_v, -1)
    assert np.allclose(out[0], np.stack([w[i, d_h:] @ p["c_kv"][0] for i in range(n_h)]), rtol=1e-12)
    # library special case: causal SDPA over k/v built with torch ops
    c = torch.tensor(p["c_kv"]); S = c.shape[0]
    kv = torch.nn.functional.linear(c, torch.tensor(p["w"])).view(S, n_h, d_h + d_v)
    k_nope, v = torch.split(kv, [d_h, d_v], -1)
    k = torch.cat([k_nope, torch.tensor(p["k_r"])[:, None, :].expand(-1, n_h, -1)], -1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(p["q"]).transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1),
        is_causal=True, scale=p["scale"]).transpose(0, 1)
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-13)
    # row/head subsets are the same definition
    sub = O.naive_prefill(p["q"], p["c_kv"], p["k_r"], p["w"], p["scale"], n_h, d_h, d_v,
                          rows=[2, 7], heads=[1])
    assert np.allclose(sub, out[[2, 7]][:, [1]], rtol=1e-14)
    # non-causal prefill is full attention: every row equals decode over all S positions
    nc = O.naive_prefill(p["q"], p["c_kv"], p["k_r"], p["w"], p["scale"], n_h, d_h, d_v, causal=False, rows=[0])
    d0 = O.absorbed_decode(p["q"][0, :, :d_h], p["q"][0, :, d_h:], p["c_kv"], p["k_r"], p["w"], p["scale"], d_v)["o"]
    assert np.allclose(nc[0], d0, rtol=1e-12, atol=1e-13)


def test_naive_heads_subset():
    x = _tiny(20, n_h=4, L=12)
    full, _ = O.naive_decode(x["q_nope"], x["q_pe"], x["c_kv"], x["k_r"], x["w_kv_b"], x["scale"])
    part, _ = O.naive_decode(x["q_nope"], x["q_pe"], x["c_kv"], x["k_r"], x["w_kv_b"], x["scale"], heads=[3, 1])
    assert np.allclose(part, full[[3, 1]], rtol=1e-14)
