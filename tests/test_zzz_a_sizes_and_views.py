"""Sizes, layouts and checks past the other GPU files' cases: batches larger than one projection
CTA's tile, more decode sequences than clusters (and than the planner keeps in registers), the
query halves as strided views of one tensor, and the device check of top-k index arrays.  This file
sorts last, so a failure here never hides the results of the other GPU files."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import SPARSE_V32, V3_DECODE
from head_latent_attention_absorb_b200.inputs import make_decode_inputs

from _util import check_close
from test_gpu_parity import check_decode_call, dev, upload, v3  # noqa: F401 (fixtures)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------------------------------
# Batch and sequence counts past one CTA's share
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("B", [97, 200, 300])
def test_projections_large_batches(v3, B):
    # batches past one CTA's tile: out_up takes 96 rows per CTA, absorb_q 256; rows on both sides of
    # each tile boundary and the last row are checked against the oracle
    cfg = V3_DECODE
    rng = np.random.default_rng(B)
    q_nope = torch.from_numpy(rng.standard_normal((B, cfg.n_h, cfg.d_h), dtype=np.float32)).to(torch.bfloat16)
    ctx = torch.from_numpy(rng.standard_normal((B, cfg.n_h, cfg.d_c), dtype=np.float32) * 0.05).to(torch.bfloat16)
    qt = api.mla_absorb_q(cfg.dims, q_nope.cuda(), v3["w_d"])
    o = api.mla_out_up(cfg.dims, ctx.cuda(), v3["w_d"])
    torch.cuda.synchronize()
    rows = sorted({0, 95, 96, 191, 192, 255, 256, B - 1} & set(range(B)))
    check_close(qt[rows], O.absorb_q(q_nope[rows], v3["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v), torch.bfloat16,
                f"absorb_q B={B}")
    check_close(o[rows], O.out_up(ctx[rows], v3["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v), torch.bfloat16,
                f"out_up B={B}")


def test_decode_many_sequences(dev):
    # more sequences than clusters (contiguous tile ranges, several sequences per cluster, split
    # sequences at range ends) and more than 256 (the work plan re-reads tile counts from memory)
    B = 300
    lengths = torch.from_numpy(np.random.default_rng(300).integers(1, 301, B).astype(np.int32))
    cfg = V3_DECODE.with_(B=B, n_max=300)
    x = upload(make_decode_inputs(cfg, lengths=lengths), dev)
    check_decode_call(x, cfg.dims, torch.bfloat16)



# ------------------------------------------------------------------------------------------
# Query halves as views of one tensor
# ------------------------------------------------------------------------------------------

def test_query_as_views_of_one_tensor(v3):
    # the query projection yields [B, n_h, d_h + d_r]; q_nope and q_pe are strided views of it
    # (row stride 192): the step must give the same bits as with contiguous copies
    cfg = V3_DECODE
    q = torch.cat([v3["q_nope_d"], v3["q_pe_d"]], dim=-1)
    assert q.shape[-1] == cfg.d_h + cfg.d_r
    qt_v = api.mla_absorb_q(cfg.dims, q[..., :cfg.d_h], v3["w_d"])
    ctx_v = api.mla_decode_absorb(cfg.dims, qt_v, q[..., cfg.d_h:], v3["c_kv_d"], v3["k_r_d"], v3["len_d"], cfg.scale)
    qt_c = api.mla_absorb_q(cfg.dims, v3["q_nope_d"].contiguous(), v3["w_d"])
    ctx_c = api.mla_decode_absorb(cfg.dims, qt_c, v3["q_pe_d"].contiguous(), v3["c_kv_d"], v3["k_r_d"], v3["len_d"],
                                  cfg.scale)
    torch.cuda.synchronize()
    assert torch.equal(qt_v, qt_c)
    assert torch.equal(ctx_v, ctx_c)



# ------------------------------------------------------------------------------------------
# Device check of top-k index arrays (range and distinctness per sequence)
# ------------------------------------------------------------------------------------------

MLA_ERR_INDEX, MLA_ERR_LENGTH = 4, 7


def host_index_status(idx: np.ndarray, lengths, n_max: int) -> int:
    """What the flag must hold: 0, or the first error class a scan of the rows finds (the kernel
    raises every error it sees, the first to land wins, so the test cases carry one class each)."""
    for b, row in enumerate(idx):
        L = n_max if lengths is None else int(lengths[b])
        if not 1 <= L <= n_max:
            return MLA_ERR_LENGTH
        if (row < 0).any() or (row >= L).any() or len(set(row.tolist())) != len(row):
            return MLA_ERR_INDEX
    return 0


def device_index_status(idx: np.ndarray, lengths, n_max: int) -> int:
    t = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
    ln = None if lengths is None else torch.as_tensor(np.asarray(lengths, dtype=np.int32)).cuda()
    err = api.mla_check_topk(t, n_max, ln)
    return api.mla_get_device_error(err)


def test_sparse_workload_indices_are_valid(dev):
    cfg = SPARSE_V32
    x = make_decode_inputs(cfg)
    idx, lengths = x["topk"].numpy(), x["lengths"].numpy()
    assert host_index_status(idx, lengths, cfg.n_max) == 0
    assert device_index_status(idx, lengths, cfg.n_max) == 0


@pytest.mark.parametrize("case", ["duplicate", "too_large", "negative", "zero_length", "no_lengths_ok"])
def test_each_error_class(dev, case):
    rng = np.random.default_rng(8)
    B, k, n_max = 6, 300, 5000
    lengths = rng.integers(k, n_max + 1, B)
    idx = np.stack([rng.choice(L, k, replace=False) for L in lengths])
    if case == "duplicate":
        idx[3, 7] = idx[3, 200]
    elif case == "too_large":
        idx[1, 0] = lengths[1]
    elif case == "negative":
        idx[5, 299] = -1
    elif case == "zero_length":
        lengths[2] = 0
    elif case == "no_lengths_ok":
        lengths = None
    want = host_index_status(idx, lengths, n_max)
    assert want == {"duplicate": MLA_ERR_INDEX, "too_large": MLA_ERR_INDEX, "negative": MLA_ERR_INDEX,
                    "zero_length": MLA_ERR_LENGTH, "no_lengths_ok": 0}[case]
    assert device_index_status(idx, lengths, n_max) == want


def test_long_cache_bitmap(dev):
    # a million positions: a 122 KB bitmap, past the default 48 KB of shared memory
    rng = np.random.default_rng(9)
    n_max, k = 1_000_000, 2048
    idx = np.stack([rng.choice(n_max, k, replace=False) for _ in range(3)])
    assert device_index_status(idx, None, n_max) == 0
    idx[2, 1000] = idx[2, 5]
    assert device_index_status(idx, None, n_max) == MLA_ERR_INDEX
