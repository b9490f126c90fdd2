"""Several new tokens per sequence, each with its own top-k set (mla_decode_absorb_multi_topk), against
the oracle: token s of a sequence of L cached rows attends the rows of its set with t <= L - T + s
(the sets include later positions on purpose; the causal rule removes them).  bf16 at the DeepSeek
dimensions and fp32 at the tiny ones; T = 1 is the one-token top-k decode; a sequence shorter than
T new tokens is flagged and its tokens get ctx = 0, lse = -inf."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import TINY_F32, V3_DECODE
from head_latent_attention_absorb_b200.inputs import make_decode_inputs

from _util import check_close

pytestmark = pytest.mark.gpu

MLA_ERR_LENGTH = 7


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_absorb_b200.build import build
    build(quiet=True)
    api.lib()
    return torch.device("cuda:0")


def draw_sets(lengths, T, k, seed):
    """Row b * T + s: the token's own position L - T + s, then k - 1 distinct positions drawn over all
    L rows (T > 1: later new tokens' rows included, for the causal rule to remove)."""
    rng = np.random.default_rng(seed)
    B = len(lengths)
    idx = np.empty((B, T, k), dtype=np.int32)
    for b, L in enumerate(lengths):
        for s in range(T):
            own = L - T + s
            others = rng.permutation(np.delete(np.arange(L), own))[: k - 1]
            idx[b, s] = np.concatenate([[own], others])
    return idx


def reference(qt, q_pe, x, lengths, idx, T, scale):
    """Per token: the oracle's latent attention over its visible rows, masked to its visible set."""
    ctx, lse = {}, {}
    for b, L in enumerate(lengths):
        for s in range(T):
            vis = L - T + s + 1
            sel = [int(t) for t in idx[b, s] if t < vis]
            c, l, _ = O.latent_attention(qt[b, s], q_pe[b, s], x["c_kv"][b, :vis], x["k_r"][b, :vis], scale,
                                         topk=sel)
            ctx[b, s], lse[b, s] = c, l
    return ctx, lse


def run(cfg, lengths, T, k, dtype, seed, dev):
    B = len(lengths)
    x = make_decode_inputs(cfg, lengths=torch.tensor(lengths, dtype=torch.int32))
    rng = np.random.default_rng(seed)
    q_nope = torch.from_numpy(rng.standard_normal((B, T, cfg.n_h, cfg.d_h), dtype=np.float32)).to(dtype)
    q_pe = torch.from_numpy(rng.standard_normal((B, T, cfg.n_h, cfg.d_r), dtype=np.float32)).to(dtype)
    qt = torch.from_numpy(O.absorb_q(q_nope, x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(dtype)
    idx = draw_sets(lengths, T, k, seed + 1)
    cache = x["cache"].to(dev)
    lse = torch.empty((B * T, cfg.n_h), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ctx = api.mla_decode_absorb_multi_topk(cfg.dims, qt.to(dev), q_pe.to(dev), cache[..., :cfg.d_c],
                                           cache[..., cfg.d_c:], x["lengths"].to(dev), torch.from_numpy(idx).to(dev),
                                           cfg.scale, lse=lse, dev_err=err)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err) == 0
    want_ctx, want_lse = reference(qt, q_pe, x, lengths, idx, T, cfg.scale)
    lse = lse.reshape(B, T, cfg.n_h)
    for (b, s), c in want_ctx.items():
        check_close(ctx[b, s], c, dtype, f"multi top-k T={T} b={b} s={s} ctx")
        check_close(lse[b, s], want_lse[b, s], dtype, f"multi top-k T={T} b={b} s={s} lse")


@pytest.mark.parametrize("T", [1, 2, 4])
def test_bf16_sets_against_oracle(dev, T):
    run(V3_DECODE.with_(B=3, n_max=300), [T + 60, 150, 300], T, 48, torch.bfloat16, 600 + T, dev)


@pytest.mark.parametrize("T", [2, 3])
def test_fp32_tiny_sets_against_oracle(dev, T):
    run(TINY_F32.with_(B=2, n_max=64), [40, 64], T, 16, torch.float32, 700 + T, dev)


def test_short_sequence_is_flagged(dev):
    T, k = 3, 8
    cfg = V3_DECODE.with_(B=2, n_max=200)
    x = make_decode_inputs(cfg, lengths=torch.tensor([200, 200], dtype=torch.int32))
    lengths = torch.tensor([2, 200], dtype=torch.int32)  # sequence 0 holds fewer rows than new tokens
    rng = np.random.default_rng(11)
    q_nope = torch.from_numpy(rng.standard_normal((2, T, cfg.n_h, cfg.d_h), dtype=np.float32)).to(torch.bfloat16)
    q_pe = torch.from_numpy(rng.standard_normal((2, T, cfg.n_h, cfg.d_r), dtype=np.float32)).to(torch.bfloat16)
    qt = torch.from_numpy(O.absorb_q(q_nope, x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16)
    idx = draw_sets([200, 200], T, k, 12)
    idx[0] = np.minimum(idx[0], 1)  # in range for the short sequence too
    cache = x["cache"].to(dev)
    lse = torch.empty((2 * T, cfg.n_h), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ctx = api.mla_decode_absorb_multi_topk(cfg.dims, qt.to(dev), q_pe.to(dev), cache[..., :512], cache[..., 512:],
                                           lengths.to(dev), torch.from_numpy(idx).to(dev), cfg.scale, lse=lse,
                                           dev_err=err)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err) == MLA_ERR_LENGTH
    assert bool((ctx[0].float() == 0).all())
    assert bool(torch.isinf(lse[:T]).all())
    want_ctx, _ = reference(qt[1:], q_pe[1:], {"c_kv": x["c_kv"][1:], "k_r": x["k_r"][1:]}, [200], idx[1:], T,
                            cfg.scale)
    for (_, s), c in want_ctx.items():
        check_close(ctx[1, s], c, torch.bfloat16, f"sequence 1 token {s}")
