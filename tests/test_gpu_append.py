"""Cache append on the GPU against the oracle (RMSNorm of the latent, rotary embedding of the
shared key, both written at the token's position), through the C ABI."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api

from _util import to_np

# The append is elementwise (after one fp32 reduction), and its outputs are cache values of any
# size, so the bound is relative, not the attention outputs' absolute 2e-2.  bf16 keeps 7 mantissa
# bits: rounding to nearest moves a value by up to half an ulp, at most 2^-8 |ref|.  The bound
# allows a full ulp, 2^-7 |ref|, to cover the fp32 arithmetic before the rounding.  fp32: a few
# ulp of rsqrt and of the rotation, 1e-5 |ref|.  The absolute 1e-5 covers the rotation's
# cancellation (x0 cos - x1 sin near zero carries ~1e-7 |x| of fp32 error, inputs here |x| < 20).
ULP_TOL = {torch.bfloat16: (2.0 ** -7, 1e-5), torch.float32: (1e-5, 1e-5)}


def check_close(got, want, dtype, what=""):
    g, w = to_np(got), np.asarray(want, dtype=np.float64)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    rel, ab = ULP_TOL[dtype]
    bad = np.abs(g - w) > rel * np.abs(w) + ab
    assert not bad.any(), f"{what}: {int(bad.sum())} elements off, worst {np.abs(g - w)[bad].max():.3e}"

pytestmark = pytest.mark.gpu

DS = (128, 512, 64, 128, 128)
TINY = (4, 64, 16, 32, 32)
DEV = "cuda"


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch.device("cuda")


def run_append(dims, dtype, B, n_max, positions, seed, gain=True):
    d_c, d_r = dims[1], dims[2]
    rng = np.random.default_rng(seed)
    kv_a = torch.from_numpy(rng.standard_normal((B, d_c + d_r), dtype=np.float32) * 3).to(dtype)
    g = torch.from_numpy(rng.uniform(0.5, 1.5, d_c).astype(np.float32)) if gain else None
    cache = torch.from_numpy(rng.standard_normal((B, n_max, d_c + d_r), dtype=np.float32)).to(dtype).to(DEV)
    before = cache.clone()
    pos = torch.tensor(positions, dtype=torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    api.mla_cache_append(dims, kv_a.to(DEV), pos.to(DEV), cache[..., :d_c], cache[..., d_c:],
                         None if g is None else g.to(DEV), 1e-6, 10000.0, dev_err=err)
    if DEV == "cuda":
        torch.cuda.synchronize()
    return kv_a, g, pos, cache, before, int(err.item())


def check_rows(dims, dtype, kv_a, g, pos, cache, before, valid):
    d_c, d_r = dims[1], dims[2]
    bs = [b for b in range(kv_a.shape[0]) if valid[b]]
    want_c, want_k = O.cache_append(kv_a[bs], pos[bs].numpy(), d_c, d_r, g, 1e-6, 10000.0)
    ib = torch.tensor(bs, dtype=torch.long, device=cache.device)
    ip = pos[bs].long().to(cache.device)
    rows = cache[ib, ip].cpu()
    check_close(rows[:, :d_c], want_c, dtype, "latent rows")
    check_close(rows[:, d_c:], want_k, dtype, "rotary rows")
    # every other row is untouched, bit for bit
    after, ref = cache.clone(), before.clone()
    after[ib, ip] = 0
    ref[ib, ip] = 0
    assert torch.equal(after, ref)


def test_append_decode_shape(dev):
    # the decode workload's cache: 32 sequences of 4096 rows, positions across it (first and last row)
    B, n_max = 32, 4096
    positions = [0, n_max - 1] + list(np.random.default_rng(5).integers(0, n_max, B - 2))
    kv_a, g, pos, cache, before, err = run_append(DS, torch.bfloat16, B, n_max, positions, 31)
    assert err == 0
    check_rows(DS, torch.bfloat16, kv_a, g, pos, cache, before, [True] * B)


def test_append_long_positions(dev):
    # positions up to 64K: the rotary angle must stay accurate far from the origin
    B, n_max = 4, 65536
    kv_a, g, pos, cache, before, err = run_append(DS, torch.bfloat16, B, n_max, [0, 1, 40000, 65535], 32)
    assert err == 0
    check_rows(DS, torch.bfloat16, kv_a, g, pos, cache, before, [True] * B)


def test_append_fp32_any_dims_no_gain(dev):
    B, n_max = 5, 70
    kv_a, g, pos, cache, before, err = run_append(TINY, torch.float32, B, n_max, [3, 0, 69, 12, 12], 33,
                                                  gain=False)
    assert err == 0
    check_rows(TINY, torch.float32, kv_a, g, pos, cache, before, [True] * B)


def test_append_bad_position_sets_flag_and_writes_nothing(dev):
    B, n_max = 4, 256
    kv_a, g, pos, cache, before, err = run_append(DS, torch.bfloat16, B, n_max, [7, -1, n_max, 200], 34)
    assert err == 4  # MLA_ERR_INDEX
    check_rows(DS, torch.bfloat16, kv_a, g, pos, cache, before, [True, False, False, True])
