"""Several new tokens per sequence with more query groups than clusters (mla_decode_absorb_multi).

50 sequences of 2..300 cached rows with two new tokens each are 100 query groups over 128-position
tiles: the work plan cuts the concatenated tiles into contiguous ranges and a cluster walks several
query groups, so the query of a later group is loaded while the previous group's epilogue and merge
decision are in flight.  Against the oracle on the first, a middle and the last sequence, and the
device error flag stays clear."""

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


def test_two_tokens_many_sequences_range_plan(dev):
    B, T = 50, 2
    lengths = torch.from_numpy(np.random.default_rng(2050).integers(T, 301, size=B).astype(np.int32))
    cfg = V3_DECODE.with_(B=B, n_max=300)
    x = make_decode_inputs(cfg, lengths=lengths)
    rng = np.random.default_rng(2051)
    q_nope = torch.from_numpy(rng.standard_normal((B, T, cfg.n_h, cfg.d_h), dtype=np.float32)).to(torch.bfloat16)
    q_pe = torch.from_numpy(rng.standard_normal((B, T, cfg.n_h, cfg.d_r), dtype=np.float32)).to(torch.bfloat16)
    qt = torch.from_numpy(O.absorb_q(q_nope, x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16)
    cache = x["cache"].to(dev)
    lse = torch.empty((B * T, cfg.n_h), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ctx = api.mla_decode_absorb_multi(cfg.dims, qt.to(dev), q_pe.to(dev), cache[..., :cfg.d_c], cache[..., cfg.d_c:],
                                      lengths.to(dev), cfg.scale, lse=lse, dev_err=err)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err) == 0
    lse = lse.reshape(B, T, cfg.n_h)
    for b in (0, 24, B - 1):
        L = int(lengths[b])
        for s in range(T):
            vis = L - T + s + 1
            want_ctx, want_lse, _ = O.latent_attention(qt[b, s], q_pe[b, s], x["c_kv"][b, :vis], x["k_r"][b, :vis],
                                                       cfg.scale)
            check_close(ctx[b, s], want_ctx, torch.bfloat16, f"multi range plan b={b} s={s} ctx")
            check_close(lse[b, s], want_lse, torch.bfloat16, f"multi range plan b={b} s={s} lse")
