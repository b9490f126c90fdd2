"""mla_decode_absorb_static: the decode entry point for callers that cannot allocate device memory
(it uses the library's built-in scratch instead of a caller workspace).  Checked through the C ABI
against mla_decode_absorb with a caller workspace, on consecutive calls that reuse the scratch and on
replays of a CUDA graph that captured the call.  It also passes when run on its own in a fresh
process."""

import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200._capi import MLAError
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


def _case(B, n_max, lengths=None):
    cfg = V3_DECODE.with_(B=B, n_max=n_max)
    x = make_decode_inputs(cfg, lengths=None if lengths is None else torch.tensor(lengths, dtype=torch.int32))
    cache = x["cache"].cuda()
    qt = torch.from_numpy(O.absorb_q(x["q_nope"], x["w_kv_b"], 128, 128, 128)).to(torch.bfloat16).cuda()
    return cfg, dict(qt=qt, qp=x["q_pe"].cuda(), c=cache[..., :512], k=cache[..., 512:], lens=x["lengths"].cuda())


# B=4 with 19 tiles over the device's clusters splits every multi-tile sequence, so the scratch
# holds partials; B=32 x 4096 is the full benchmarked decode.
CASES = [(4, 700, [700, 1, 333, 64]), (32, 4096, None)]


@pytest.mark.parametrize("B,n_max,lengths", CASES)
def test_static_scratch_matches_workspace_decode(dev, B, n_max, lengths):
    cfg, t = _case(B, n_max, lengths)
    lse_ref = torch.empty((B, 128), dtype=torch.float32, device=dev)
    ref = api.mla_decode_absorb(cfg.dims, t["qt"], t["qp"], t["c"], t["k"], t["lens"], cfg.scale, lse=lse_ref)
    torch.cuda.synchronize()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for call in range(2):  # two calls in a row share (and reuse) the built-in scratch
        ctx = torch.full((B, 128, 512), float("nan"), dtype=torch.bfloat16, device=dev)
        lse = torch.full((B, 128), float("nan"), dtype=torch.float32, device=dev)
        api.mla_decode_absorb_static(cfg.dims, t["qt"], t["qp"], t["c"], t["k"], t["lens"], cfg.scale,
                                     ctx=ctx, lse=lse, dev_err=err)
        torch.cuda.synchronize()
        # the same kernel on the same inputs, and its split-KV merge does not depend on the order in
        # which clusters arrive: the results agree bit for bit (a stale partial or flag left in the
        # shared scratch by the previous call would show here)
        assert torch.equal(ctx, ref), f"ctx call {call}"
        assert torch.equal(lse, lse_ref), f"lse call {call}"
        check_close(ctx, ref.float().cpu().numpy(), torch.bfloat16, f"ctx call {call}")
    assert api.mla_get_device_error(err) == 0


def test_static_scratch_rejects_other_paths(dev):
    cfg, t = _case(2, 128)
    with pytest.raises(MLAError, match="UNSUPPORTED"):
        api.mla_decode_absorb_static(cfg.dims, t["qt"].float(), t["qp"].float(), t["c"].float(), t["k"].float(),
                                     t["lens"], cfg.scale)


def test_static_scratch_in_a_cuda_graph(dev):
    """The use the entry point is for: a warm call (it looks up the scratch), then the call captured
    in a CUDA graph and replayed twice.  B = 4 with split sequences, so every replay publishes and
    merges partials in the shared scratch with the same launch tag; both replays equal the
    workspace decode bit for bit."""
    B, n_max, lengths = CASES[0]
    cfg, t = _case(B, n_max, lengths)
    lse_ref = torch.empty((B, 128), dtype=torch.float32, device=dev)
    ref = api.mla_decode_absorb(cfg.dims, t["qt"], t["qp"], t["c"], t["k"], t["lens"], cfg.scale, lse=lse_ref)
    ctx = torch.empty((B, 128, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, 128), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    api.mla_decode_absorb_static(cfg.dims, t["qt"], t["qp"], t["c"], t["k"], t["lens"], cfg.scale,
                                 ctx=ctx, lse=lse, dev_err=err)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            api.mla_decode_absorb_static(cfg.dims, t["qt"], t["qp"], t["c"], t["k"], t["lens"], cfg.scale,
                                         ctx=ctx, lse=lse, dev_err=err)
    torch.cuda.synchronize()
    for rep in range(2):
        ctx.fill_(float("nan"))
        lse.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(ctx, ref), f"ctx replay {rep}"
        assert torch.equal(lse, lse_ref), f"lse replay {rep}"
    assert api.mla_get_device_error(err) == 0
    del graph
