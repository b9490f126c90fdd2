"""GPU parity: every entry point of libmla_b200.so against the CPU oracle on the same seeded
inputs, through the C ABI (via the ctypes binding).  Full workload sizes plus small cases that
span several tiles with ragged tails, and the degenerate cases of the method."""

import numpy as np
import pytest
import torch

import oracle as O
from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import PREFILL, RAGGED_LONG, SPARSE_V32, TINY_F32, V3_DECODE
from head_latent_attention_absorb_b200.inputs import make_decode_inputs, make_prefill_inputs

from _util import check_close, oracle_latent, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_absorb_b200.build import build
    build(quiet=True)
    api.lib()
    return torch.device("cuda:0")


def upload(inp, dev):
    out = dict(inp)
    cache = inp["cache"].to(dev)
    d_c = inp["cfg"].d_c
    out.update(cache_d=cache, c_kv_d=cache[..., :d_c], k_r_d=cache[..., d_c:], w_d=inp["w_kv_b"].to(dev),
               q_nope_d=inp["q_nope"].to(dev), q_pe_d=inp["q_pe"].to(dev), len_d=inp["lengths"].to(dev),
               topk_d=None if inp["topk"] is None else inp["topk"].to(dev))
    return out


def gpu_step(x, dims, err=None):
    qt = api.mla_absorb_q(dims, x["q_nope_d"], x["w_d"])
    lse = torch.empty(qt.shape[:2], dtype=torch.float32, device=qt.device)
    ctx = api.mla_decode_absorb(dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], x["scale"],
                                topk_idx=x["topk_d"], lse=lse, dev_err=err)
    o = api.mla_out_up(dims, ctx, x["w_d"])
    torch.cuda.synchronize()
    return qt, ctx, lse, o


def oracle_qt(x):
    cfg = x["cfg"]
    return O.absorb_q(x["q_nope"], x["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v)


def check_decode_call(x, dims, dt, batches=None):
    """mla_decode_absorb alone: fed the oracle's q~ (rounded to the input dtype)."""
    qt = torch.from_numpy(oracle_qt(x)).to(dt)
    lse = torch.empty((qt.shape[0], qt.shape[1]), dtype=torch.float32, device="cuda")
    ctx = api.mla_decode_absorb(dims, qt.cuda(), x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], x["scale"],
                                topk_idx=x["topk_d"], lse=lse)
    torch.cuda.synchronize()
    bs = list(range(qt.shape[0])) if batches is None else batches
    want_ctx, want_lse = oracle_latent(qt, x["q_pe"], x["c_kv"], x["k_r"], x["lengths"], x["scale"], x["topk"], bs)
    check_close(ctx[bs], want_ctx, dt, "ctx")
    # lse: same bound as every other output of its dtype.  (On the bf16 path the softmax sum is
    # taken over the bf16-rounded weights that the P*V product uses, each within 2^-9 relative,
    # so lse can differ from the exact value by up to ~2e-3.)
    check_close(lse[bs], want_lse, dt, "lse")
    return ctx


# ------------------------------------------------------------------------------------------
# Tiny fp32 workload: every entry point at 1e-4
# ------------------------------------------------------------------------------------------

def test_tiny_f32_every_entry_point(dev):
    cfg = TINY_F32
    x = upload(make_decode_inputs(cfg), dev)
    dims = cfg.dims
    qt, ctx, lse, o = gpu_step(x, dims)
    check_close(qt, oracle_qt(x), torch.float32, "q_tilde")
    check_decode_call(x, dims, torch.float32)
    ref = O.absorbed_decode(x["q_nope"][0], x["q_pe"][0], x["c_kv"][0], x["k_r"][0], x["w_kv_b"], cfg.scale, cfg.d_v)
    naive, _ = O.naive_decode(x["q_nope"][0], x["q_pe"][0], x["c_kv"][0], x["k_r"][0], x["w_kv_b"], cfg.scale)
    check_close(o[0], naive, torch.float32, "o vs naive")
    check_close(ctx[0], ref["ctx"], torch.float32, "ctx")
    o2 = api.mla_out_up(dims, torch.from_numpy(ref["ctx"][None]).float().cuda(), x["w_d"])
    check_close(o2[0], ref["o"], torch.float32, "out_up")


@pytest.mark.parametrize("causal", [True, False])
def test_tiny_f32_prefill(dev, causal):
    cfg = TINY_F32.with_(kind="prefill", B=2, n_max=37)
    p = make_prefill_inputs(cfg)
    out = api.mla_prefill_naive(cfg.dims, p["q"].cuda(), p["c_kv"].cuda(), p["k_r"].cuda(), p["w_kv_b"].cuda(),
                                cfg.scale, causal=causal)
    torch.cuda.synchronize()
    for b in range(cfg.B):
        want = O.naive_prefill(p["q"][b], p["c_kv"][b], p["k_r"][b], p["w_kv_b"], cfg.scale, cfg.n_h, cfg.d_h,
                               cfg.d_v, causal=causal)
        check_close(out[b], want, torch.float32, f"prefill b={b}")


# ------------------------------------------------------------------------------------------
# DeepSeek-V3 decode, B=32, N=4096 (the benchmarked workload)
# ------------------------------------------------------------------------------------------

@pytest.fixture(scope="module")
def v3(dev):
    return upload(make_decode_inputs(V3_DECODE), dev)


def test_v3_absorb_q(v3):
    qt = api.mla_absorb_q(V3_DECODE.dims, v3["q_nope_d"], v3["w_d"])
    torch.cuda.synchronize()
    check_close(qt, oracle_qt(v3), torch.bfloat16, "q_tilde")


def test_v3_decode_call(v3):
    check_decode_call(v3, V3_DECODE.dims, torch.bfloat16)


def test_v3_out_up(v3):
    cfg = V3_DECODE
    ctx = np.random.default_rng(7).standard_normal((cfg.B, cfg.n_h, cfg.d_c)) * 0.05
    ctx_t = torch.from_numpy(ctx).to(torch.bfloat16)
    o = api.mla_out_up(cfg.dims, ctx_t.cuda(), v3["w_d"])
    torch.cuda.synchronize()
    check_close(o, O.out_up(ctx_t, v3["w_kv_b"], cfg.n_h, cfg.d_h, cfg.d_v), torch.bfloat16, "out_up")


def test_v3_whole_step_vs_oracle(v3):
    cfg = V3_DECODE
    qt, ctx, lse, o = gpu_step(v3, cfg.dims)
    want = np.stack([O.absorbed_decode(v3["q_nope"][b], v3["q_pe"][b], v3["c_kv"][b], v3["k_r"][b], v3["w_kv_b"],
                                       cfg.scale, cfg.d_v)["o"] for b in range(cfg.B)])
    check_close(o, want, torch.bfloat16, "o (absorbed oracle)")
    heads = list(range(0, 128, 9))
    for b in (0, 13, 31):  # the literal naive equations on a sub-sample
        naive, _ = O.naive_decode(v3["q_nope"][b], v3["q_pe"][b], v3["c_kv"][b], v3["k_r"][b], v3["w_kv_b"],
                                  cfg.scale, heads=heads)
        check_close(o[b, heads], naive, torch.bfloat16, f"o vs naive b={b}")


# ------------------------------------------------------------------------------------------
# Tiles and ragged tails at small sizes, layouts, degenerate cases
# ------------------------------------------------------------------------------------------

TAIL_LENGTHS = [1, 2, 63, 64, 65, 127, 128, 129, 255, 1000, 1024, 1100]


def test_decode_ragged_tails(dev):
    cfg = V3_DECODE.with_(B=len(TAIL_LENGTHS), n_max=1100)
    x = upload(make_decode_inputs(cfg, lengths=torch.tensor(TAIL_LENGTHS, dtype=torch.int32)), dev)
    check_decode_call(x, cfg.dims, torch.bfloat16)


def test_decode_separate_and_packed_layouts_agree(dev):
    cfg = V3_DECODE.with_(B=3, n_max=700)
    x = upload(make_decode_inputs(cfg, lengths=torch.tensor([700, 333, 64], dtype=torch.int32)), dev)
    qt = torch.from_numpy(oracle_qt(x)).to(torch.bfloat16).cuda()
    a = api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale)
    c_sep = x["c_kv_d"].contiguous()
    k_sep = x["k_r_d"].contiguous()
    b = api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], c_sep, k_sep, x["len_d"], cfg.scale)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_single_position_is_exact(dev):
    """One cached row: alpha = 1 and ctx equals c_0 bit for bit."""
    cfg = V3_DECODE.with_(B=4, n_max=256)
    x = upload(make_decode_inputs(cfg, lengths=torch.ones(4, dtype=torch.int32)), dev)
    qt = torch.from_numpy(oracle_qt(x)).to(torch.bfloat16).cuda()
    lse = torch.empty((4, 128), dtype=torch.float32, device="cuda")
    ctx = api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale, lse=lse)
    torch.cuda.synchronize()
    assert torch.equal(ctx, x["c_kv_d"][:, 0:1, :].expand(-1, 128, -1))


def test_zero_query_is_uniform_average(dev):
    cfg = V3_DECODE.with_(B=2, n_max=777)
    x = upload(make_decode_inputs(cfg), dev)
    qt = torch.zeros((2, 128, 512), dtype=torch.bfloat16, device="cuda")
    qp = torch.zeros((2, 128, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 128), dtype=torch.float32, device="cuda")
    ctx = api.mla_decode_absorb(cfg.dims, qt, qp, x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale, lse=lse)
    torch.cuda.synchronize()
    want = to_np(x["c_kv"][:, :777]).mean(1)[:, None, :].repeat(128, 1)
    check_close(ctx, want, torch.bfloat16, "uniform average")
    assert np.allclose(to_np(lse), np.log(777.0), rtol=1e-6)


# ------------------------------------------------------------------------------------------
# Long ragged decode (B=8, lengths ~ U[1024, 65536])
# ------------------------------------------------------------------------------------------

def test_ragged_long(dev):
    x = upload(make_decode_inputs(RAGGED_LONG), dev)
    check_decode_call(x, RAGGED_LONG.dims, torch.bfloat16)
    _, _, _, o = gpu_step(x, RAGGED_LONG.dims)
    b = int(torch.argmin(x["lengths"]))
    L = int(x["lengths"][b])
    want = O.absorbed_decode(x["q_nope"][b], x["q_pe"][b], x["c_kv"][b, :L], x["k_r"][b, :L], x["w_kv_b"],
                             RAGGED_LONG.scale, 128)["o"]
    check_close(o[b], want, torch.bfloat16, "o shortest sequence")


# ------------------------------------------------------------------------------------------
# Sparse (top-k) decode, B=16, N=32768, k=2048
# ------------------------------------------------------------------------------------------

@pytest.fixture(scope="module")
def sparse(dev):
    return upload(make_decode_inputs(SPARSE_V32), dev)


def test_sparse_decode(sparse):
    check_decode_call(sparse, SPARSE_V32.dims, torch.bfloat16)


def test_sparse_whole_step_vs_naive(sparse):
    cfg = SPARSE_V32
    _, _, _, o = gpu_step(sparse, cfg.dims)
    heads = list(range(0, 128, 5))
    for b in (0, 15):
        naive, _ = O.naive_decode(sparse["q_nope"][b], sparse["q_pe"][b], sparse["c_kv"][b], sparse["k_r"][b],
                                  sparse["w_kv_b"], cfg.scale, topk=sparse["topk"][b].numpy(), heads=heads)
        check_close(o[b, heads], naive, torch.bfloat16, f"sparse o vs naive b={b}")


def test_topk_single_index_is_exact_gather(sparse):
    """k = 1: the context is the selected cache row, bit for bit (the gather is exact)."""
    cfg = SPARSE_V32
    idx = sparse["topk_d"][:, :1].contiguous()
    qt = torch.from_numpy(oracle_qt(sparse)).to(torch.bfloat16).cuda()
    ctx = api.mla_decode_absorb(cfg.dims, qt, sparse["q_pe_d"], sparse["c_kv_d"], sparse["k_r_d"], sparse["len_d"],
                                cfg.scale, topk_idx=idx)
    torch.cuda.synchronize()
    rows = sparse["c_kv_d"][torch.arange(cfg.B, device="cuda"), idx[:, 0].long()]
    assert torch.equal(ctx, rows[:, None, :].expand(-1, 128, -1))


def test_topk_full_set_equals_dense_and_order_free(dev):
    cfg = SPARSE_V32.with_(B=2, n_max=600, topk=600)
    x = upload(make_decode_inputs(cfg), dev)
    qt = torch.from_numpy(oracle_qt(x)).to(torch.bfloat16).cuda()
    sp = api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale,
                               topk_idx=x["topk_d"])
    dense = api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale)
    rev = api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale,
                                topk_idx=x["topk_d"].flip(1).contiguous())
    torch.cuda.synchronize()
    check_close(sp, to_np(dense), torch.bfloat16, "top-k full set vs dense")
    check_close(rev, to_np(sp), torch.bfloat16, "top-k reversed order")


def test_topk_many_sequences_range_plan(dev):
    """B = 100 sequences of 200 rows with every position selected, in order: more sequences than
    clusters, so both gathering warps walk several sequences per cluster.  Same result as the dense
    decode, and the oracle on three sequences."""
    B, L = 100, 200
    cfg = SPARSE_V32.with_(B=B, n_max=L, topk=L)
    x = upload(make_decode_inputs(cfg, lengths=torch.full((B,), L, dtype=torch.int32)), dev)
    qt = torch.from_numpy(oracle_qt(x)).to(torch.bfloat16).cuda()
    tk = torch.arange(L, dtype=torch.int32).repeat(B, 1).contiguous().cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp = api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale,
                               topk_idx=tk, dev_err=err)
    dense = api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err) == 0
    check_close(sp, to_np(dense), torch.bfloat16, "top-k every position vs dense, B=100")
    for b in (0, 57, B - 1):
        want, _, _ = O.latent_attention(qt[b].cpu(), x["q_pe"][b], x["c_kv"][b, :L], x["k_r"][b, :L], cfg.scale,
                                        np.arange(L))
        check_close(sp[b], want, torch.bfloat16, f"top-k range plan b={b}")


def test_dense_many_sequences_range_plan(dev):
    """B = 100 sequences of 1..300 rows: a cluster's range crosses many sequences, short ones whole
    and the ones at its ends split with a neighbour cluster, so split-KV arrivals of consecutive
    segments follow each other closely.  Against the oracle on every sequence's first head row and
    in full on four sequences (the shortest, the longest, two split ones)."""
    B = 100
    lengths = torch.from_numpy(np.random.default_rng(101).integers(1, 301, size=B).astype(np.int32))
    cfg = V3_DECODE.with_(B=B, n_max=300)
    x = upload(make_decode_inputs(cfg, lengths=lengths), dev)
    qt = torch.from_numpy(oracle_qt(x)).to(torch.bfloat16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lse = torch.empty((B, cfg.n_h), dtype=torch.float32, device="cuda")
    ctx = api.mla_decode_absorb(cfg.dims, qt.cuda(), x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale,
                                lse=lse, dev_err=err)
    torch.cuda.synchronize()
    assert api.mla_get_device_error(err) == 0
    Ls = lengths.numpy()
    full = {int(np.argmin(Ls)), int(np.argmax(Ls)), 37, 62}
    for b in range(B):
        L = int(Ls[b])
        heads = slice(None) if b in full else slice(0, 1)
        want_ctx, want_lse, _ = O.latent_attention(qt[b, heads], x["q_pe"][b, heads], x["c_kv"][b, :L],
                                                   x["k_r"][b, :L], cfg.scale)
        check_close(ctx[b, heads], want_ctx, torch.bfloat16, f"ctx b={b} L={L}")
        check_close(lse[b, heads], want_lse, torch.bfloat16, f"lse b={b} L={L}")


# ------------------------------------------------------------------------------------------
# Naive causal prefill, B=2, S=2048
# ------------------------------------------------------------------------------------------

def test_prefill_full_size_sampled_rows(dev):
    cfg = PREFILL
    p = make_prefill_inputs(cfg)
    out = api.mla_prefill_naive(cfg.dims, p["q"].cuda(), p["c_kv"].cuda(), p["k_r"].cuda(), p["w_kv_b"].cuda(),
                                cfg.scale)
    torch.cuda.synchronize()
    rows = [0, 1, 2, 63, 64, 127, 128, 129, 1000, 1023, 1024, 2046, 2047]
    for b in range(cfg.B):
        want = O.naive_prefill(p["q"][b], p["c_kv"][b], p["k_r"][b], p["w_kv_b"], cfg.scale, cfg.n_h, cfg.d_h,
                               cfg.d_v, rows=rows)
        check_close(out[b, rows], want, torch.bfloat16, f"prefill b={b}")
    # the last prefill row equals the absorbed decode over the whole sequence (GPU against GPU
    # is not a parity claim; both are checked against the oracle above / in the decode tests)
    S = cfg.n_max
    dec = O.absorbed_decode(p["q"][0, S - 1, :, :128], p["q"][0, S - 1, :, 128:], p["c_kv"][0], p["k_r"][0],
                            p["w_kv_b"], cfg.scale, 128)["o"]
    check_close(out[0, S - 1], dec, torch.bfloat16, "prefill last row vs absorbed decode")


def test_prefill_small_ragged(dev):
    cfg = PREFILL.with_(B=3, n_max=333)
    p = make_prefill_inputs(cfg)
    out = api.mla_prefill_naive(cfg.dims, p["q"].cuda(), p["c_kv"].cuda(), p["k_r"].cuda(), p["w_kv_b"].cuda(),
                                cfg.scale)
    torch.cuda.synchronize()
    for b in range(cfg.B):
        want = O.naive_prefill(p["q"][b], p["c_kv"][b], p["k_r"][b], p["w_kv_b"], cfg.scale, cfg.n_h, cfg.d_h,
                               cfg.d_v, heads=list(range(0, 128, 7)))
        check_close(out[b][:, list(range(0, 128, 7))], want, torch.bfloat16, f"prefill b={b}")


@pytest.mark.parametrize("S,causal", [(100, True), (256, True), (600, True), (600, False), (384, False)])
def test_prefill_query_tile_pairings(dev, S, causal):
    # a CTA runs query tile n_qt-1-i and then tile i: one tile (S=100), an even tile count (256),
    # an odd count whose middle tile runs alone (384, 600), causal and bidirectional
    cfg = PREFILL.with_(B=2, n_max=S)
    p = make_prefill_inputs(cfg)
    out = api.mla_prefill_naive(cfg.dims, p["q"].cuda(), p["c_kv"].cuda(), p["k_r"].cuda(), p["w_kv_b"].cuda(),
                                cfg.scale, causal=causal)
    torch.cuda.synchronize()
    heads = [0, 37, 127]
    for b in range(cfg.B):
        want = O.naive_prefill(p["q"][b], p["c_kv"][b], p["k_r"][b], p["w_kv_b"], cfg.scale, cfg.n_h, cfg.d_h,
                               cfg.d_v, causal=causal, heads=heads)
        check_close(out[b][:, heads], want, torch.bfloat16, f"prefill S={S} causal={causal} b={b}")


# ------------------------------------------------------------------------------------------
# Device-side error flag (no trap: the offending row is skipped)
# ------------------------------------------------------------------------------------------

def test_device_error_flags(dev):
    cfg = SPARSE_V32.with_(B=2, n_max=512, topk=16)
    x = upload(make_decode_inputs(cfg), dev)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qt = torch.from_numpy(oracle_qt(x)).to(torch.bfloat16).cuda()
    bad = x["topk_d"].clone()
    bad[1, 3] = 512  # == length: outside [0, length)
    api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], x["len_d"], cfg.scale,
                          topk_idx=bad, dev_err=err)
    assert api.mla_get_device_error(err) == 4
    api.mla_clear_device_error(err)
    assert api.mla_get_device_error(err) == 0
    lens = torch.tensor([512, 600], dtype=torch.int32, device="cuda")  # > n_max
    api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], lens, cfg.scale, dev_err=err)
    assert api.mla_get_device_error(err) == 7
    api.mla_clear_device_error(err)
    lens = torch.tensor([0, 512], dtype=torch.int32, device="cuda")
    api.mla_decode_absorb(cfg.dims, qt, x["q_pe_d"], x["c_kv_d"], x["k_r_d"], lens, cfg.scale, dev_err=err)
    assert api.mla_get_device_error(err) == 7
