"""FP8 wkv_b projections on the GPU: against the oracle with the dequantised weight, and bit-equal
to the bf16 projections given that weight rounded to bf16 (the kernel rounds the same way)."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import V3_DECODE

from _util import check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch.device("cuda")


def quantize_blocks(w: torch.Tensor, block: int = 128):
    """e4m3 weight and fp32 scale per block x block tile (scale = tile amax / 448)."""
    R, C = w.shape
    gr, gc = O.fp8_block_scale_shape(R, C, block)
    tiles = w.reshape(gr, block, gc, block).abs().amax(dim=(1, 3)).clamp_min(1e-12)
    scale = (tiles / 448.0).float()
    wq = (w / scale.repeat_interleave(block, 0).repeat_interleave(block, 1)).to(torch.float8_e4m3fn)
    return wq, scale


@pytest.mark.parametrize("B", [1, 32, 200])
def test_fp8_projections(dev, B):
    cfg = V3_DECODE
    rng = np.random.default_rng(900 + B)
    w = torch.from_numpy(rng.standard_normal((cfg.n_h * (cfg.d_h + cfg.d_v), cfg.d_c), dtype=np.float32) * 0.02)
    wq, scale = quantize_blocks(w)
    w_deq = (wq.float() * scale.repeat_interleave(128, 0).repeat_interleave(128, 1))  # fp32, then rounded below
    q_nope = torch.from_numpy(rng.standard_normal((B, cfg.n_h, cfg.d_h), dtype=np.float32)).to(torch.bfloat16)
    ctx = torch.from_numpy(rng.standard_normal((B, cfg.n_h, cfg.d_c), dtype=np.float32) * 0.05).to(torch.bfloat16)
    wq_d, sc_d = wq.cuda(), scale.cuda()
    qt8 = api.mla_absorb_q_fp8(cfg.dims, q_nope.cuda(), wq_d, sc_d)
    o8 = api.mla_out_up_fp8(cfg.dims, ctx.cuda(), wq_d, sc_d)
    w_bf = w_deq.to(torch.bfloat16).cuda()
    qt16 = api.mla_absorb_q(cfg.dims, q_nope.cuda(), w_bf)
    o16 = api.mla_out_up(cfg.dims, ctx.cuda(), w_bf)
    torch.cuda.synchronize()
    assert torch.equal(qt8, qt16)
    assert torch.equal(o8, o16)
    rows = sorted({0, B // 2, B - 1})
    w_oracle = O.weight_dequant(wq, scale.numpy())
    check_close(qt8[rows], O.absorb_q(q_nope[rows], w_oracle, cfg.n_h, cfg.d_h, cfg.d_v), torch.bfloat16, "absorb fp8")
    check_close(o8[rows], O.out_up(ctx[rows], w_oracle, cfg.n_h, cfg.d_h, cfg.d_v), torch.bfloat16, "out_up fp8")
