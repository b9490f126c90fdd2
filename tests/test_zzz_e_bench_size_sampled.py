"""The two secondary workloads the bench times at sizes no other test reaches, checked against the
oracle on sampled outputs in the same launch configuration: the multi-token decode at B = 32, T = 2,
N = 4096 and the sparse prefill at B = 1, S = 8192 with 2048 selected positions per row."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import PREFILL, V3_DECODE
from head_latent_attention_absorb_b200.inputs import make_decode_inputs, make_prefill_inputs

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


def test_multi_token_decode_bench_size(dev):
    B, T = 32, 2
    cfg = V3_DECODE
    x = make_decode_inputs(cfg)
    rng = np.random.default_rng(3232)
    q_nope = torch.from_numpy(rng.standard_normal((B, T, cfg.n_h, cfg.d_h), dtype=np.float32)).to(torch.bfloat16)
    q_pe = torch.from_numpy(rng.standard_normal((B, T, cfg.n_h, cfg.d_r), dtype=np.float32)).to(torch.bfloat16)
    qt = torch.from_numpy(O.absorb_q(q_nope, x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16)
    cache = x["cache"].to(dev)
    lse = torch.empty((B * T, cfg.n_h), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ctx = api.mla_decode_absorb_multi(cfg.dims, qt.to(dev), q_pe.to(dev), cache[..., :cfg.d_c], cache[..., cfg.d_c:],
                                      x["lengths"].to(dev), cfg.scale, lse=lse, dev_err=err)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err) == 0
    lse = lse.reshape(B, T, cfg.n_h)
    for b in (0, 17, B - 1):
        L = int(x["lengths"][b])
        for s in range(T):
            vis = L - T + s + 1
            want_ctx, want_lse, _ = O.latent_attention(qt[b, s], q_pe[b, s], x["c_kv"][b, :vis], x["k_r"][b, :vis],
                                                       cfg.scale)
            check_close(ctx[b, s], want_ctx, torch.bfloat16, f"multi bench size b={b} s={s} ctx")
            check_close(lse[b, s], want_lse, torch.bfloat16, f"multi bench size b={b} s={s} lse")


def test_sparse_prefill_bench_size_sampled_rows(dev):
    cfg = PREFILL.with_(B=1, n_max=8192)
    p = make_prefill_inputs(cfg)
    S, k = cfg.n_max, 2048
    rng = np.random.default_rng(cfg.seed + 300)
    topk = np.empty((1, S, k), dtype=np.int32)
    for s_ in range(S):  # each row: itself plus 2047 positions over the whole sequence (later ones masked)
        topk[0, s_, 0] = s_
        topk[0, s_, 1:] = rng.choice(S, k - 1, replace=False)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out = api.mla_prefill_sparse(cfg.dims, p["q"].to(dev), p["c_kv"].to(dev), p["k_r"].to(dev), p["w_kv_b"].to(dev),
                                 cfg.scale, torch.from_numpy(topk).to(dev), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = [0, 1, 127, 128, 2047, 4096, 6143, 8191]
    heads = [0, 127]
    want = O.naive_prefill(p["q"][0], p["c_kv"][0], p["k_r"][0], p["w_kv_b"], cfg.scale, cfg.n_h, cfg.d_h, cfg.d_v,
                           rows=rows, heads=heads, topk=topk[0])
    check_close(out[0][rows][:, heads], want, torch.bfloat16, "sparse prefill S=8192 k=2048")
