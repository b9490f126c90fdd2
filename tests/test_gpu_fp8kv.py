"""The absorbed decode over an FP8 latent cache (mla_decode_absorb_fp8kv) on the GPU.

The kernel dequantises each E4M3 code on chip as bf16(float(code) * scale) and then runs the same
attention as the bf16 decode, so its results must equal mla_decode_absorb on the bf16 cache built
the same way on the host, bit for bit.  Against the oracle (latent_cache_dequant, then the latent
attention in fp64) they must agree within the bf16 tolerance."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import V3_DECODE
from head_latent_attention_absorb_b200.inputs import make_decode_inputs, pack_fp8_cache, quantize_latent_fp8

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


def kernel_read_back(c8: torch.Tensor, sc: torch.Tensor, block: int = 128) -> torch.Tensor:
    """The bf16 cache the FP8-cache kernel reads back: bf16(float(code) * scale), one fp32 product
    and one rounding (the oracle's latent_cache_dequant rounds once from the exact product instead)."""
    shp = c8.shape
    f = c8.view(torch.float8_e4m3fn).to(torch.float32).reshape(*shp[:-1], shp[-1] // block, block)
    return (f * sc[..., None]).reshape(shp).to(torch.bfloat16)


def _case(cfg, lengths=None, seed_q=11):
    x = make_decode_inputs(cfg, lengths=lengths)
    c8, sc = quantize_latent_fp8(x["c_kv"])
    deq = kernel_read_back(c8, sc)
    qt = torch.from_numpy(O.absorb_q(x["q_nope"], x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16)
    return x, c8, sc, deq, qt


def _fp8_call(cfg, dev, qt, q_pe, c8, sc, k_r, lengths, packed=True):
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    lse = torch.empty((qt.shape[0], cfg.n_h), dtype=torch.float32, device=dev)
    if packed:
        rows = pack_fp8_cache(c8, sc, k_r).to(dev)
        c8d = rows[..., :512]
        scd = rows[..., 512:528].view(torch.float32)
        krd = rows[..., 528:].view(torch.bfloat16)
    else:
        c8d, scd, krd = c8.to(dev), sc.to(dev), k_r.to(torch.bfloat16).contiguous().to(dev)
    ctx = api.mla_decode_absorb_fp8kv(cfg.dims, qt.to(dev), q_pe.to(dev), c8d, scd, krd, lengths.to(dev), cfg.scale,
                                      lse=lse, dev_err=err)
    torch.cuda.synchronize()
    return ctx, lse, api.mla_get_device_error(err)


def test_fp8kv_equals_bf16_decode_on_dequantised_cache(dev):
    """B = 32, N = 4096 (the benchmarked shape), packed 656-byte rows: ctx and lse bit-equal to the
    bf16 decode over bf16(float(code) * scale)."""
    cfg = V3_DECODE
    x, c8, sc, deq, qt = _case(cfg)
    ctx8, lse8, e = _fp8_call(cfg, dev, qt, x["q_pe"], c8, sc, x["k_r"], x["lengths"])
    assert e == 0
    lse = torch.empty_like(lse8)
    ctx = api.mla_decode_absorb(cfg.dims, qt.to(dev), x["q_pe"].to(dev), deq.to(dev), x["k_r"].contiguous().to(dev),
                                x["lengths"].to(dev), cfg.scale, lse=lse)
    torch.cuda.synchronize()
    assert torch.equal(ctx8, ctx)
    assert torch.equal(lse8, lse)


def test_fp8kv_against_oracle_ragged(dev):
    """Lengths 1, 63, 64, 65, 300 and 777 (single rows, tile tails, split sequences), separate
    arrays: against the oracle's read-back of the FP8 cache and its latent attention."""
    lengths = torch.tensor([1, 63, 64, 65, 300, 777], dtype=torch.int32)
    cfg = V3_DECODE.with_(B=6, n_max=777)
    x, c8, sc, deq, qt = _case(cfg, lengths=lengths)
    ctx8, lse8, e = _fp8_call(cfg, dev, qt, x["q_pe"], c8, sc, x["k_r"], lengths, packed=False)
    assert e == 0
    for b in range(6):
        L = int(lengths[b])
        c_kv = O.latent_cache_dequant(c8[b, :L].numpy(), sc[b, :L].numpy())
        want_ctx, want_lse, _ = O.latent_attention(qt[b], x["q_pe"][b], c_kv, x["k_r"][b, :L], cfg.scale)
        check_close(ctx8[b], want_ctx, torch.bfloat16, f"fp8 cache ctx b={b} L={L}")
        check_close(lse8[b], want_lse, torch.bfloat16, f"fp8 cache lse b={b} L={L}")


def test_fp8kv_packed_equals_separate(dev):
    cfg = V3_DECODE.with_(B=5, n_max=640)
    lengths = torch.tensor([640, 1, 129, 300, 511], dtype=torch.int32)
    x, c8, sc, deq, qt = _case(cfg, lengths=lengths)
    a = _fp8_call(cfg, dev, qt, x["q_pe"], c8, sc, x["k_r"], lengths, packed=True)
    b = _fp8_call(cfg, dev, qt, x["q_pe"], c8, sc, x["k_r"], lengths, packed=False)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fp8kv_bad_length_and_host_checks(dev):
    cfg = V3_DECODE.with_(B=3, n_max=200)
    x, c8, sc, deq, qt = _case(cfg, lengths=torch.tensor([200, 5, 120], dtype=torch.int32))
    ctx, lse, e = _fp8_call(cfg, dev, qt, x["q_pe"], c8, sc, x["k_r"], torch.tensor([200, 0, 120], dtype=torch.int32))
    assert e == 7  # MLA_ERR_LENGTH
    assert bool((ctx[1].float() == 0).all())
    # a row stride of the codes that is not a multiple of 16 bytes is refused before any launch
    c8d = torch.zeros((3, 200, 520), dtype=torch.uint8, device=dev)[..., :512]
    with pytest.raises(RuntimeError):
        api.mla_decode_absorb_fp8kv(cfg.dims, qt.to(dev), x["q_pe"].to(dev), c8d, sc.to(dev),
                                    x["k_r"].contiguous().to(dev), x["lengths"].to(dev), cfg.scale)


def test_fp8kv_many_sequences_range_plan(dev):
    """B = 100 sequences of 1..300 rows: more sequences than clusters, so the work plan cuts the
    concatenated tiles into ranges and a cluster walks several sequences.  The conversion runs on a
    tile counter that carries over the segments; bit-equal to the bf16 decode as above."""
    B = 100
    lengths = torch.from_numpy(np.random.default_rng(100).integers(1, 301, size=B).astype(np.int32))
    cfg = V3_DECODE.with_(B=B, n_max=300)
    x, c8, sc, deq, qt = _case(cfg, lengths=lengths)
    ctx8, lse8, e = _fp8_call(cfg, dev, qt, x["q_pe"], c8, sc, x["k_r"], lengths, packed=True)
    assert e == 0
    lse = torch.empty_like(lse8)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ctx = api.mla_decode_absorb(cfg.dims, qt.to(dev), x["q_pe"].to(dev), deq.to(dev), x["k_r"].contiguous().to(dev),
                                lengths.to(dev), cfg.scale, lse=lse, dev_err=err)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err) == 0
    assert torch.equal(ctx8, ctx)
    assert torch.equal(lse8, lse)
