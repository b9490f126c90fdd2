"""Sparse prefill on invalid index sets.  Rows whose set holds no visible position (every selected
t > s) are written as zeros with MLA_ERR_INDEX set, the other rows unchanged: one query tile has no
visible key in any row (its key-tile list would be empty), another has empty rows among valid ones.
Indices outside [0, S) set MLA_ERR_INDEX and drop out of their rows' sets."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import PREFILL
from head_latent_attention_absorb_b200.inputs import make_prefill_inputs

from _util import check_close

pytestmark = pytest.mark.gpu

MLA_ERR_INDEX = 4


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch.device("cuda")


def draw_topk_with_empty_rows(S, k, seed):
    """Rows of query tile 1 (positions 128..255) select only future positions; even rows of query
    tile 2 select only s + 1; every other row selects itself plus k - 1 random positions."""
    rng = np.random.default_rng(seed)
    idx = np.empty((S, k), dtype=np.int32)
    empty = np.zeros(S, dtype=bool)
    for s in range(S):
        if 128 <= s < 256:
            idx[s] = rng.choice(np.arange(s + 1, S), k, replace=False)
            empty[s] = True
        elif 256 <= s < S - 1 and s % 2 == 0:
            idx[s] = s + 1  # one future position, repeated (a set: counts once)
            empty[s] = True
        else:
            idx[s] = np.concatenate([[s], rng.choice(S, k - 1, replace=False)])
    return idx, empty


def test_empty_rows_are_zero_and_flagged(dev):
    cfg = PREFILL.with_(B=1, n_max=384)
    p = make_prefill_inputs(cfg)
    S = cfg.n_max
    topk, empty = draw_topk_with_empty_rows(S, 16, 123)
    # the oracle's own reading of the mask: an empty row has no position with a finite mask
    for s in range(S):
        assert bool(np.isfinite(O.index_mask(S, topk[s])[: s + 1]).any()) != bool(empty[s])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = api.mla_prefill_sparse(cfg.dims, p["q"].cuda(), p["c_kv"].cuda(), p["k_r"].cuda(), p["w_kv_b"].cuda(),
                                 cfg.scale, torch.from_numpy(topk[None]).cuda(), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == MLA_ERR_INDEX
    o = out[0].float().cpu()
    assert bool((o[torch.from_numpy(empty)] == 0).all())
    rows = [s for s in (0, 1, 100, 127, 257, 259, 301, 383) if not empty[s]]
    heads = [0, 64, 127]
    want = O.naive_prefill(p["q"][0], p["c_kv"][0], p["k_r"][0], p["w_kv_b"], cfg.scale, cfg.n_h, cfg.d_h, cfg.d_v,
                           rows=rows, heads=heads, topk=topk)
    check_close(out[0][rows][:, heads], want, torch.bfloat16, "sparse prefill beside empty rows")


def test_out_of_range_indices_are_flagged_and_ignored(dev):
    """An index outside [0, S) sets MLA_ERR_INDEX and drops out of its row's set; the rest of the row
    (and every other row) is the oracle's result on the set without it."""
    cfg = PREFILL.with_(B=1, n_max=300)
    p = make_prefill_inputs(cfg)
    S, k = cfg.n_max, 16
    rng = np.random.default_rng(77)
    good = np.stack([np.concatenate([[s], rng.choice(S, k - 1, replace=False)]) for s in range(S)]).astype(np.int32)
    bad = good.copy()
    bad_rows = [3, 130, 299]
    for s in bad_rows:
        bad[s, 5] = -1 - s    # negative
        bad[s, 9] = S + s     # past the sequence
    # the set without the dropped entries: the row's own position stands in for them (a repeat,
    # which the set semantics ignore)
    clean = bad.copy()
    for s in bad_rows:
        clean[s, 5] = s
        clean[s, 9] = s
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = api.mla_prefill_sparse(cfg.dims, p["q"].cuda(), p["c_kv"].cuda(), p["k_r"].cuda(), p["w_kv_b"].cuda(),
                                 cfg.scale, torch.from_numpy(bad[None]).cuda(), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == MLA_ERR_INDEX
    rows = [0, 3, 64, 130, 131, 255, 299]
    heads = [0, 99]
    want = O.naive_prefill(p["q"][0], p["c_kv"][0], p["k_r"][0], p["w_kv_b"], cfg.scale, cfg.n_h, cfg.d_h, cfg.d_v,
                           rows=rows, heads=heads, topk=clean)
    check_close(out[0][rows][:, heads], want, torch.bfloat16, "sparse prefill with dropped indices")
