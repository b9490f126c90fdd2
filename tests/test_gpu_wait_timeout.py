"""Failure detection without a fault: the bounded mbarrier wait that every kernel of the library
uses, made to run out.  One CTA waits on an mbarrier that nothing arrives on; after the limit the
kernel gives up, the device flag reads MLA_ERR_TIMEOUT, and the context keeps working: a decode run
right after it still matches the oracle."""

import time

import numpy as np
import pytest
import torch

from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import V3_DECODE
from head_latent_attention_absorb_b200.inputs import make_decode_inputs

from _util import check_close, oracle_latent
import oracle as O

pytestmark = pytest.mark.gpu

MLA_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_absorb_b200.build import build
    build(quiet=True)
    api.lib()
    return torch.device("cuda:0")


def test_wait_runs_out_and_context_survives(dev):
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    t0 = time.time()
    api.check(api.lib().mla_selftest_wait_timeout(20_000_000, err.data_ptr(), None), "selftest")  # 20 ms
    assert api.mla_get_device_error(err) == MLA_ERR_TIMEOUT
    assert time.time() - t0 < 5.0
    x = torch.arange(1024, device=dev, dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2

    # a decode right after the timed-out kernel: same result as the oracle, no flag raised
    cfg = V3_DECODE.with_(B=3, n_max=700)
    inp = make_decode_inputs(cfg)
    qt = torch.from_numpy(O.absorb_q(inp["q_nope"], inp["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)).to(torch.bfloat16)
    cache = inp["cache"].to(dev)
    lse = torch.empty((3, 128), dtype=torch.float32, device=dev)
    err2 = torch.zeros(1, dtype=torch.int32, device=dev)
    ctx = api.mla_decode_absorb(cfg.dims, qt.to(dev), inp["q_pe"].to(dev), cache[..., :cfg.d_c], cache[..., cfg.d_c:],
                                inp["lengths"].to(dev), cfg.scale, lse=lse, dev_err=err2)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err2) == 0
    want_ctx, want_lse = oracle_latent(qt, inp["q_pe"], inp["c_kv"], inp["k_r"], inp["lengths"], cfg.scale)
    check_close(ctx, want_ctx, torch.bfloat16, "ctx after a timeout")
    check_close(lse, want_lse, torch.bfloat16, "lse after a timeout")


def test_wait_limit_is_checked_on_the_host(dev):
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for bad in (0, 999, 2_000_000_000):
        assert api.lib().mla_selftest_wait_timeout(bad, err.data_ptr(), None) == 1  # MLA_ERR_INVALID_ARG
    assert api.lib().mla_selftest_wait_timeout(1_000_000, None, None) == 1
    assert api.mla_get_device_error(err) == 0
