"""The split-KV merge must not depend on which cluster of a split sequence arrives last: the last
to arrive merges, and repeated calls on the same inputs must agree bit for bit (two-partial merges
round both weighted products on their own; several partials are summed in slot order)."""

import numpy as np
import pytest
import torch

from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import RAGGED_LONG, V3_DECODE
from head_latent_attention_absorb_b200.inputs import make_decode_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_absorb_b200.build import build
    build(quiet=True)
    api.lib()
    return torch.device("cuda:0")


def repeat_equal(cfg, x, dev, calls=6):
    cache = x["cache"].to(dev)
    qt = api.mla_absorb_q(cfg.dims, x["q_nope"].to(dev), x["w_kv_b"].to(dev))
    lse = torch.empty((cfg.B, cfg.n_h), dtype=torch.float32, device=dev)
    args = (cfg.dims, qt, x["q_pe"].to(dev), cache[..., :cfg.d_c], cache[..., cfg.d_c:], x["lengths"].to(dev),
            cfg.scale)
    first = api.mla_decode_absorb(*args, lse=lse).clone()
    first_lse = lse.clone()
    for _ in range(calls - 1):
        assert torch.equal(api.mla_decode_absorb(*args, lse=lse), first), "ctx differs between calls"
        assert torch.equal(lse, first_lse), "lse differs between calls"


def test_two_and_three_partial_merges_repeat_exactly(dev):
    """B = 33, lengths up to 130: one-tile chunks, so most sequences are merged from two or three
    partials."""
    cfg = V3_DECODE.with_(B=33, n_max=130)
    lengths = torch.from_numpy(np.random.default_rng(33).integers(1, 131, size=33).astype(np.int32))
    repeat_equal(cfg, make_decode_inputs(cfg, lengths=lengths), dev)


def test_ragged_long_repeats_exactly(dev):
    """The ragged workload: sequences up to 64k spread over contiguous tile ranges (many partials)."""
    repeat_equal(RAGGED_LONG, make_decode_inputs(RAGGED_LONG), dev, calls=3)
