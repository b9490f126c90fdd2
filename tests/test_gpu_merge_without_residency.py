"""The split-KV merge when the clusters of a launch may not all be resident at once.

With many partials per sequence the decode kernels use a sliced merge: every cluster holding a piece
of the sequence publishes its partial and waits for all the others.  That needs every cluster of the
launch resident together.  The host allows it only when the occupancy query confirmed that the grid
fits in one wave, and MLA_DECODE_SLICED_MERGE=0 turns it off.  Without it the last cluster to arrive
merges every partial (it waits only on clusters that have already run).  Both merges must give the
oracle's result, for the one-token decode and the multi-token decode."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import RAGGED_LONG, SPARSE_V32, V3_DECODE
from head_latent_attention_absorb_b200.inputs import make_decode_inputs

from _util import check_close

pytestmark = pytest.mark.gpu

ENV = "MLA_DECODE_SLICED_MERGE"


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_absorb_b200.build import build
    build(quiet=True)
    api.lib()
    return torch.device("cuda:0")


def _both_merges(monkeypatch, call):
    """Runs `call` with the sliced merge allowed, then turned off; returns both results."""
    monkeypatch.delenv(ENV, raising=False)
    a = call()
    torch.cuda.synchronize()
    monkeypatch.setenv(ENV, "0")
    b = call()
    torch.cuda.synchronize()
    monkeypatch.delenv(ENV, raising=False)
    return a, b


def test_one_token_decode_ragged_long(dev, monkeypatch):
    """B = 8, lengths up to 64k: the longest sequence spans many clusters (many partials)."""
    cfg = RAGGED_LONG
    x = make_decode_inputs(cfg)
    qt = torch.from_numpy(O.absorb_q(x["q_nope"], x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16)
    cache = x["cache"].to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        lse = torch.empty((cfg.B, cfg.n_h), dtype=torch.float32, device=dev)
        ctx = api.mla_decode_absorb(cfg.dims, qt.to(dev), x["q_pe"].to(dev), cache[..., :cfg.d_c],
                                    cache[..., cfg.d_c:], x["lengths"].to(dev), cfg.scale, lse=lse, dev_err=err)
        return ctx.clone(), lse.clone()

    (ctx_s, lse_s), (ctx_l, lse_l) = _both_merges(monkeypatch, call)
    assert api.mla_get_device_error(err) == 0
    b = int(torch.argmax(x["lengths"]))
    L = int(x["lengths"][b])
    want_ctx, want_lse, _ = O.latent_attention(qt[b], x["q_pe"][b], x["c_kv"][b, :L], x["k_r"][b, :L], cfg.scale)
    for name, ctx, lse in (("sliced", ctx_s, lse_s), ("last-arrival", ctx_l, lse_l)):
        check_close(ctx[b], want_ctx, torch.bfloat16, f"{name} merge ctx, L={L}")
        check_close(lse[b], want_lse, torch.bfloat16, f"{name} merge lse, L={L}")
    check_close(ctx_l, ctx_s.float().cpu().numpy(), torch.bfloat16, "the two merges agree")


def test_multi_token_decode_long_sequence(dev, monkeypatch):
    """One sequence of 20,000 rows and two new tokens: two pseudo-sequences over every cluster."""
    T, L = 2, 20000
    cfg = V3_DECODE.with_(B=1, n_max=L)
    x = make_decode_inputs(cfg, lengths=torch.tensor([L], dtype=torch.int32))
    rng = np.random.default_rng(2020)
    q_nope = torch.from_numpy(rng.standard_normal((1, T, cfg.n_h, cfg.d_h), dtype=np.float32)).to(torch.bfloat16)
    q_pe = torch.from_numpy(rng.standard_normal((1, T, cfg.n_h, cfg.d_r), dtype=np.float32)).to(torch.bfloat16)
    qt = torch.from_numpy(O.absorb_q(q_nope, x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16)
    cache = x["cache"].to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        lse = torch.empty((T, cfg.n_h), dtype=torch.float32, device=dev)
        ctx = api.mla_decode_absorb_multi(cfg.dims, qt.to(dev), q_pe.to(dev), cache[..., :cfg.d_c],
                                          cache[..., cfg.d_c:], x["lengths"].to(dev), cfg.scale, lse=lse,
                                          dev_err=err)
        return ctx.clone(), lse.clone()

    (ctx_s, lse_s), (ctx_l, lse_l) = _both_merges(monkeypatch, call)
    assert api.mla_get_device_error(err) == 0
    for s in range(T):
        vis = L - T + s + 1
        want_ctx, want_lse, _ = O.latent_attention(qt[0, s], q_pe[0, s], x["c_kv"][0, :vis], x["k_r"][0, :vis],
                                                   cfg.scale)
        for name, ctx, lse in (("sliced", ctx_s, lse_s), ("last-arrival", ctx_l, lse_l)):
            check_close(ctx[0, s], want_ctx, torch.bfloat16, f"{name} merge token {s} ctx")
            check_close(lse[s], want_lse, torch.bfloat16, f"{name} merge token {s} lse")


def test_topk_decode_four_partials(dev, monkeypatch):
    """Top-k decode, B = 16 sequences of 2048 selected rows over 74 clusters: four partials per
    sequence.  Sliced (every cluster merges a quarter of the heads) and, with the sliced merge off,
    the last cluster bulk-loading the three others; both against the oracle on two sequences."""
    cfg = SPARSE_V32
    x = make_decode_inputs(cfg)
    qt = torch.from_numpy(O.absorb_q(x["q_nope"], x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16)
    cache = x["cache"].to(dev)
    topk = x["topk"].to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        lse = torch.empty((cfg.B, cfg.n_h), dtype=torch.float32, device=dev)
        ctx = api.mla_decode_absorb(cfg.dims, qt.to(dev), x["q_pe"].to(dev), cache[..., :cfg.d_c],
                                    cache[..., cfg.d_c:], x["lengths"].to(dev), cfg.scale, topk_idx=topk,
                                    lse=lse, dev_err=err)
        return ctx.clone(), lse.clone()

    (ctx_s, lse_s), (ctx_l, lse_l) = _both_merges(monkeypatch, call)
    assert api.mla_get_device_error(err) == 0
    for b in (0, cfg.B - 1):
        L = int(x["lengths"][b])
        want_ctx, want_lse, _ = O.latent_attention(qt[b], x["q_pe"][b], x["c_kv"][b, :L], x["k_r"][b, :L],
                                                   cfg.scale, x["topk"][b].numpy())
        for name, ctx, lse in (("sliced", ctx_s, lse_s), ("last-arrival", ctx_l, lse_l)):
            check_close(ctx[b], want_ctx, torch.bfloat16, f"{name} merge ctx b={b}")
            check_close(lse[b], want_lse, torch.bfloat16, f"{name} merge lse b={b}")
