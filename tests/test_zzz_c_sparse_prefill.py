"""Sparse prefill (each query row's top-k set plus the causal mask) on the GPU against the oracle."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import PREFILL
from head_latent_attention_absorb_b200.inputs import make_prefill_inputs

from _util import check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch.device("cuda")


def draw_topk(B, S, k, seed):
    # each row selects itself plus k - 1 positions drawn over the whole sequence (future ones too:
    # the causal mask must remove them)
    rng = np.random.default_rng(seed)
    idx = np.stack([np.stack([np.concatenate([[s], rng.choice(S, k - 1, replace=False)]) for s in range(S)])
                    for _ in range(B)]).astype(np.int32)
    return idx


@pytest.mark.parametrize("S,k", [(200, 16), (640, 64)])
def test_sparse_prefill_against_oracle(dev, S, k):
    cfg = PREFILL.with_(B=2, n_max=S)
    p = make_prefill_inputs(cfg)
    topk = draw_topk(cfg.B, S, k, 40 + S)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = api.mla_prefill_sparse(cfg.dims, p["q"].cuda(), p["c_kv"].cuda(), p["k_r"].cuda(), p["w_kv_b"].cuda(),
                                 cfg.scale, torch.from_numpy(topk).cuda(), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    heads = [0, 77, 127]
    for b in range(cfg.B):
        want = O.naive_prefill(p["q"][b], p["c_kv"][b], p["k_r"][b], p["w_kv_b"], cfg.scale, cfg.n_h, cfg.d_h,
                               cfg.d_v, heads=heads, topk=topk[b])
        check_close(out[b][:, heads], want, torch.bfloat16, f"sparse prefill S={S} b={b}")


def test_every_position_selected_matches_dense(dev):
    cfg = PREFILL.with_(B=1, n_max=384)
    p = make_prefill_inputs(cfg)
    S = cfg.n_max
    topk = np.tile(np.arange(S, dtype=np.int32), (1, S, 1))
    args = (cfg.dims, p["q"].cuda(), p["c_kv"].cuda(), p["k_r"].cuda(), p["w_kv_b"].cuda(), cfg.scale)
    sp = api.mla_prefill_sparse(*args, torch.from_numpy(topk).cuda())
    dense = api.mla_prefill_naive(*args)
    torch.cuda.synchronize()
    # the same arithmetic in the same order; the two kernel instantiations may still contract a
    # multiply-add differently, so allow one bf16 ulp
    diff = (sp.float() - dense.float()).abs()
    assert bool((diff <= dense.float().abs() * 2.0 ** -7 + 1e-6).all()), float(diff.max())


@pytest.mark.parametrize("k", [512, 2048])
def test_sparse_prefill_2048_sampled_rows(dev, k):
    """The prefill workload's length (S = 2048, 16 query tiles): each row selects k positions (k = S:
    every position, in a random order per row), checked on rows sampled across all query tiles,
    including the first and last row of several tiles."""
    cfg = PREFILL.with_(B=1, n_max=2048)
    p = make_prefill_inputs(cfg)
    S = cfg.n_max
    rng = np.random.default_rng(7 + k)
    if k < S:
        topk = draw_topk(1, S, k, 90 + k)
    else:
        topk = np.stack([rng.permutation(S) for _ in range(S)])[None].astype(np.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = api.mla_prefill_sparse(cfg.dims, p["q"].cuda(), p["c_kv"].cuda(), p["k_r"].cuda(), p["w_kv_b"].cuda(),
                                 cfg.scale, torch.from_numpy(topk).cuda(), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = sorted({0, 1, 63, 127, 128, 255, 511, 512, 1000, 1023, 1024, 1535, 1536, 2000, 2046, 2047} |
                  set(rng.choice(S, 8, replace=False).tolist()))
    heads = [0, 63, 127]
    want = O.naive_prefill(p["q"][0], p["c_kv"][0], p["k_r"][0], p["w_kv_b"], cfg.scale, cfg.n_h, cfg.d_h, cfg.d_v,
                           rows=rows, heads=heads, topk=topk[0])
    check_close(out[0][rows][:, heads], want, torch.bfloat16, f"sparse prefill S=2048 k={k}")
