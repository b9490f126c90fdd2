"""Several new tokens per sequence in one decode call (mla_decode_absorb_multi) against the oracle,
and T = 1 against the one-token decode bit for bit.

The oracle's multi_token_decode applies the causal rule among the new tokens (token s of T sees the
cached rows t <= L - T + s).  The GPU call is fed the oracle's absorbed queries rounded to bf16, so the
reference here is the oracle's latent attention of each token over its visible rows, with that same
query; a separate check ties it to multi_token_decode."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import V3_DECODE
from head_latent_attention_absorb_b200.inputs import make_decode_inputs

from _util import check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_absorb_b200.build import build
    build(quiet=True)
    api.lib()
    return torch.device("cuda:0")


def _queries(B, T, cfg, seed):
    rng = np.random.default_rng(seed)
    q_nope = torch.from_numpy(rng.standard_normal((B, T, cfg.n_h, cfg.d_h), dtype=np.float32)).to(torch.bfloat16)
    q_pe = torch.from_numpy(rng.standard_normal((B, T, cfg.n_h, cfg.d_r), dtype=np.float32)).to(torch.bfloat16)
    return q_nope, q_pe


@pytest.mark.parametrize("T", [2, 4])
def test_multi_token_decode_against_oracle(dev, T):
    B = 6
    lengths = torch.tensor([T, 64, 129, 300, 777, 129 + T], dtype=torch.int32)
    cfg = V3_DECODE.with_(B=B, n_max=777)
    x = make_decode_inputs(cfg, lengths=lengths)
    q_nope, q_pe = _queries(B, T, cfg, 70 + T)
    qt = torch.from_numpy(O.absorb_q(q_nope, x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16)
    cache = x["cache"].to(dev)
    lse = torch.empty((B * T, cfg.n_h), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ctx = api.mla_decode_absorb_multi(cfg.dims, qt.to(dev), q_pe.to(dev), cache[..., :cfg.d_c], cache[..., cfg.d_c:],
                                      lengths.to(dev), cfg.scale, lse=lse, dev_err=err)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err) == 0
    lse = lse.reshape(B, T, cfg.n_h)
    for b in range(B):
        L = int(lengths[b])
        want_ctx, want_lse = [], []
        for s in range(T):
            vis = L - T + s + 1
            c, l, _ = O.latent_attention(qt[b, s], q_pe[b, s], x["c_kv"][b, :vis], x["k_r"][b, :vis], cfg.scale)
            want_ctx.append(c)
            want_lse.append(l)
        check_close(ctx[b], np.stack(want_ctx), torch.bfloat16, f"multi T={T} b={b} ctx")
        check_close(lse[b], np.stack(want_lse), torch.bfloat16, f"multi T={T} b={b} lse")


def test_multi_token_reference_is_the_oracle_definition():
    """The per-token reference used above equals the oracle's multi_token_decode (given the same
    absorbed query), so the GPU is checked against that definition."""
    cfg = V3_DECODE.with_(B=1, n_max=90, n_h=4)
    x = make_decode_inputs(cfg, lengths=torch.tensor([90], dtype=torch.int32))
    q_nope, q_pe = _queries(1, 3, cfg, 5)
    out = O.multi_token_decode(q_nope[0], q_pe[0], x["c_kv"][0], x["k_r"][0], x["w_kv_b"], cfg.scale, cfg.d_v)
    for s in range(3):
        vis = 90 - 3 + s + 1
        c, l, _ = O.latent_attention(out["q_tilde"][s], q_pe[0, s], x["c_kv"][0, :vis], x["k_r"][0, :vis], cfg.scale)
        assert np.allclose(c, out["ctx"][s], rtol=1e-12, atol=1e-14)
        assert np.allclose(l, out["lse"][s], rtol=1e-12, atol=1e-12)


def test_one_token_is_the_decode(dev):
    cfg = V3_DECODE.with_(B=3, n_max=500)
    x = make_decode_inputs(cfg, lengths=torch.tensor([500, 1, 130], dtype=torch.int32))
    qt = torch.from_numpy(O.absorb_q(x["q_nope"], x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16).to(dev)
    cache, lens, qp = x["cache"].to(dev), x["lengths"].to(dev), x["q_pe"].to(dev)
    a = api.mla_decode_absorb(cfg.dims, qt, qp, cache[..., :512], cache[..., 512:], lens, cfg.scale)
    b = api.mla_decode_absorb_multi(cfg.dims, qt[:, None], qp[:, None], cache[..., :512], cache[..., 512:], lens,
                                    cfg.scale)
    torch.cuda.synchronize()
    assert torch.equal(a, b[:, 0])


def test_too_short_sequence_is_flagged(dev):
    T = 3
    cfg = V3_DECODE.with_(B=2, n_max=200)
    lengths = torch.tensor([2, 200], dtype=torch.int32)  # sequence 0 holds fewer rows than new tokens
    x = make_decode_inputs(cfg, lengths=torch.tensor([200, 200], dtype=torch.int32))
    q_nope, q_pe = _queries(2, T, cfg, 9)
    qt = torch.from_numpy(O.absorb_q(q_nope, x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16).to(dev)
    cache = x["cache"].to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    lse = torch.empty((2 * T, cfg.n_h), dtype=torch.float32, device=dev)
    ctx = api.mla_decode_absorb_multi(cfg.dims, qt, q_pe.to(dev), cache[..., :512], cache[..., 512:],
                                      lengths.to(dev), cfg.scale, lse=lse, dev_err=err)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err) == 7  # MLA_ERR_LENGTH
    # the first token of sequence 0 would see no row: zero context, lse = -inf
    assert bool((ctx[0, 0].float() == 0).all())
    assert bool(torch.isinf(lse[0]).all())
    # sequence 1 is unaffected
    for s in range(T):
        vis = 200 - T + s + 1
        c, _, _ = O.latent_attention(qt[1, s].cpu(), q_pe[1, s], x["c_kv"][1, :vis], x["k_r"][1, :vis], cfg.scale)
        check_close(ctx[1, s], c, torch.bfloat16, f"sequence 1 token {s}")
