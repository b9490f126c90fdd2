"""The C-ABI library builds, loads and exports every entry point include/mla_api.h declares;
host-side validation answers without touching a GPU (no call here reaches a kernel launch)."""

import ctypes
import os
import re

import pytest

from head_latent_attention_absorb_b200 import _capi
from head_latent_attention_absorb_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]

DS = _capi.MLADims(128, 512, 64, 128, 128)
FAKE = 0x10000  # an aligned non-NULL address; every call below fails validation before using it


@pytest.fixture(scope="module")
def L():
    build(quiet=True)
    return _capi.lib()


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(mla_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 11, names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
        assert n in _capi.SIGNATURES, f"{n} has no ctypes signature"


def test_abi_and_status_strings(L):
    assert L.mla_abi_version() == _capi.ABI_VERSION
    for code, name in _capi.STATUS.items():
        assert L.mla_status_string(code).decode().startswith(name)
    assert L.mla_status_string(99) == b"unknown mla_status"


def test_workspace_sizes(L):
    assert L.mla_prefill_workspace_size(DS, _capi.MLA_BF16, 2, 2048) == 2 * 2048 * 128 * 256 * 2
    assert L.mla_prefill_workspace_size(_capi.MLADims(4, 64, 16, 32, 32), _capi.MLA_F32, 1, 9) == 9 * 4 * 64 * 4
    assert L.mla_decode_workspace_size(DS, _capi.MLA_BF16, 32, 4096, 0) > 0
    assert L.mla_decode_workspace_size(DS, _capi.MLA_BF16, 0, 4096, 0) == 0
    assert L.mla_decode_workspace_size(_capi.MLADims(4, 64, 16, 32, 32), _capi.MLA_BF16, 1, 64, 0) == 0


def test_host_validation_codes(L):
    bf, f32 = _capi.MLA_BF16, _capi.MLA_F32
    tiny = _capi.MLADims(4, 64, 16, 32, 32)
    # bf16 outside the DeepSeek dimensions has no kernel
    assert L.mla_absorb_q(tiny, bf, 1, FAKE, 32, FAKE, FAKE, None) == 2
    # NULL pointers, bad sizes, misalignment
    assert L.mla_absorb_q(DS, bf, 1, None, 128, FAKE, FAKE, None) == 1
    assert L.mla_absorb_q(DS, bf, 0, FAKE, 128, FAKE, FAKE, None) == 1
    assert L.mla_absorb_q(DS, bf, 1, FAKE + 2, 128, FAKE, FAKE, None) == 1
    assert L.mla_absorb_q(DS, bf, 1, FAKE, 100, FAKE, FAKE, None) == 1
    assert b"ldq" in L.mla_last_error_message() or b"multiple" in L.mla_last_error_message()
    assert L.mla_out_up(DS, bf, 1, FAKE, None, FAKE, None) == 1
    assert L.mla_absorb_q(_capi.MLADims(0, 64, 16, 32, 32), f32, 1, FAKE, 32, FAKE, FAKE, None) == 1
    assert L.mla_absorb_q(tiny, 7, 1, FAKE, 32, FAKE, FAKE, None) == 1

    def dec(**kw):
        a = dict(dims=DS, dt=bf, B=2, qt=FAKE, ldqt=512, qp=FAKE, ldqp=64, ckv=FAKE, cb=4096 * 576, cr=576,
                 kr=FAKE, kb=4096 * 576, krr=576, n_max=4096, lengths=FAKE, topk=None, k=0, scale=0.07,
                 ctx=FAKE, lse=None, ws=FAKE, wsb=1 << 40, err=None)
        a.update(kw)
        return L.mla_decode_absorb(*a.values(), None)

    assert dec(ws=None) == 6
    assert dec(wsb=16) == 6
    assert dec(lengths=None) == 1
    assert dec(cr=500) == 1                 # row stride below d_c
    assert dec(cr=577) == 1                 # not a multiple of 8 elements
    assert dec(topk=FAKE, k=0) == 1         # top-k with an empty set
    assert dec(topk=FAKE, k=4097) == 1      # top-k larger than the cache
    assert dec(scale=0.0) == 1
    assert dec(scale=float("nan")) == 1
    assert dec(ldqt=256) == 1
    assert dec(B=0) == 1
    # prefill
    assert L.mla_prefill_naive(DS, bf, 1, 16, FAKE, FAKE, 576, FAKE, 576, FAKE, 0.07, 1, FAKE, None, 0, None) == 6
    assert L.mla_prefill_naive(DS, bf, 1, 0, FAKE, FAKE, 576, FAKE, 576, FAKE, 0.07, 1, FAKE, FAKE, 1 << 30, None) == 1
    # cache append
    def app(**kw):
        a = dict(dims=DS, dt=bf, B=2, kv=FAKE, lda=576, gain=None, eps=1e-6, base=10000.0, pos=FAKE, n_max=64,
                 ckv=FAKE, cb=64 * 576, cr=576, kr=FAKE, kb=64 * 576, krr=576, err=None)
        a.update(kw)
        return L.mla_cache_append(*a.values(), None)

    assert app(pos=None) == 1
    assert app(B=0) == 1
    assert app(lda=500) == 1                # narrower than d_c + d_r
    assert app(cr=577) == 1                 # not a multiple of 8 elements
    assert app(cb=63 * 576) == 1            # batch stride below n_max rows
    assert app(eps=-1.0) == 1
    assert app(base=0.0) == 1
    assert app(kv=FAKE + 2) == 1            # misaligned bf16 row
    assert L.mla_cache_append(_capi.MLADims(4, 64, 15, 32, 32), f32, 1, FAKE, 79, None, 1e-6, 1e4, FAKE, 8,
                              FAKE, 8 * 64, 64, FAKE, 8 * 15, 15, None, None) == 1   # odd rotary width
    assert L.mla_cache_append(tiny, bf, 1, FAKE, 80, None, 1e-6, 1e4, FAKE, 8,
                              FAKE, 8 * 64, 64, FAKE, 8 * 16, 16, None, None) == 2   # bf16 outside DeepSeek dims
    # sparse prefill and FP8 projections
    assert L.mla_prefill_sparse(DS, f32, 1, 16, FAKE, FAKE, 576, FAKE, 576, FAKE, 0.07, FAKE, 8, FAKE, FAKE,
                                1 << 30, None, None) == 2                     # bf16 only
    assert L.mla_prefill_sparse(DS, bf, 1, 16, FAKE, FAKE, 576, FAKE, 576, FAKE, 0.07, None, 8, FAKE, FAKE,
                                1 << 30, None, None) == 1                     # no top-k array
    assert L.mla_prefill_sparse(DS, bf, 1, 16, FAKE, FAKE, 576, FAKE, 576, FAKE, 0.07, FAKE, 8, FAKE, None,
                                0, None, None) == 6                           # no workspace
    assert L.mla_prefill_sparse_workspace_size(DS, bf, 2, 2048) > L.mla_prefill_workspace_size(DS, bf, 2, 2048)
    assert L.mla_prefill_sparse_workspace_size(DS, f32, 2, 2048) == 0
    assert L.mla_absorb_q_fp8(DS, 1, FAKE, 128, FAKE, None, FAKE, None, None) == 1   # no scales
    assert L.mla_absorb_q_fp8(DS, 1, FAKE, 100, FAKE, FAKE, FAKE, None, None) == 1   # ldq below d_h
    assert L.mla_absorb_q_fp8(tiny, 1, FAKE, 32, FAKE, FAKE, FAKE, None, None) == 2  # not the DeepSeek dims
    assert L.mla_out_up_fp8(DS, 0, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert L.mla_out_up_fp8(DS, 1, FAKE, FAKE + 8, FAKE, FAKE, None, None) == 1     # misaligned weight
    # top-k validation
    assert L.mla_check_topk(0, FAKE, 8, None, 64, FAKE, None) == 1
    assert L.mla_check_topk(2, None, 8, None, 64, FAKE, None) == 1
    assert L.mla_check_topk(2, FAKE, 8, None, 64, None, None) == 1
    assert L.mla_check_topk(2, FAKE, 8, None, 2_000_000, FAKE, None) == 2   # bitmap beyond shared memory
    assert L.mla_clear_device_error(None, None) == 1
    out = ctypes.c_int32(0)
    assert L.mla_get_device_error(None, ctypes.byref(out)) == 1


def test_host_validation_codes_newer_entry_points(L):
    """The FP8-cache decode, the multi-token decode (with and without per-token top-k sets), the
    static-scratch decode and the wait self-test refuse bad arguments on the host (before any
    launch)."""
    tiny = _capi.MLADims(4, 64, 16, 32, 32)

    def fp8(**kw):
        a = dict(dims=DS, B=2, qt=FAKE, ldqt=512, qp=FAKE, ldqp=64, c8=FAKE, c8b=4096 * 656, c8r=656,
                 sc=FAKE, scb=4096 * 164, scr=164, kr=FAKE, krb=4096 * 328, krr=328, n_max=4096, lengths=FAKE,
                 scale=0.07, ctx=FAKE, lse=None, ws=FAKE, wsb=1 << 40, err=None)
        a.update(kw)
        return L.mla_decode_absorb_fp8kv(*a.values(), None)

    assert fp8(dims=tiny) == 2              # bf16 DeepSeek dimensions only
    assert fp8(B=0) == 1
    assert fp8(n_max=0) == 1
    assert fp8(sc=None) == 1                # no scales
    assert fp8(lengths=None) == 1
    assert fp8(c8r=520) == 1                # code rows not a multiple of 16 bytes
    assert fp8(c8b=4096 * 656 + 8) == 1     # batch stride not a multiple of 16 bytes
    assert fp8(c8r=500) == 1                # narrower than d_c codes
    assert fp8(scr=3) == 1                  # fewer than d_c / 128 scales per row
    assert fp8(scr=166) == 1                # scale rows not a multiple of 4 floats
    assert fp8(krr=330) == 1                # rotary rows not a multiple of 8 elements
    assert fp8(ldqt=256) == 1
    assert fp8(scale=0.0) == 1
    assert fp8(scale=float("nan")) == 1
    assert fp8(c8=FAKE + 8) == 1            # misaligned code rows
    assert fp8(ws=None) == 6
    assert fp8(wsb=16) == 6
    assert fp8(ws=FAKE + 8) == 1            # misaligned workspace

    def multi(**kw):
        a = dict(dims=DS, dt=_capi.MLA_BF16, B=2, T=2, qt=FAKE, ldqt=512, qp=FAKE, ldqp=64, ckv=FAKE,
                 cb=4096 * 576, cr=576, kr=FAKE, kb=4096 * 576, krr=576, n_max=4096, lengths=FAKE, scale=0.07,
                 ctx=FAKE, lse=None, ws=FAKE, wsb=1 << 40, err=None)
        a.update(kw)
        return L.mla_decode_absorb_multi(*a.values(), None)

    assert multi(dt=_capi.MLA_F32) == 2     # several tokens per sequence: bf16 only
    assert multi(T=0) == 1
    assert multi(T=4097) == 1               # more new tokens than cache rows
    assert multi(B=0) == 1
    assert multi(qt=None) == 1
    assert multi(cr=577) == 1
    assert multi(scale=-1.0) == 1
    assert multi(ws=None) == 6
    assert multi(T=1, ws=None) == 6         # T = 1 is the one-token decode and validates as such

    def static(**kw):
        a = dict(dims=DS, dt=_capi.MLA_BF16, B=2, qt=FAKE, ldqt=512, qp=FAKE, ldqp=64, ckv=FAKE,
                 cb=4096 * 576, cr=576, kr=FAKE, kb=4096 * 576, krr=576, n_max=4096, lengths=FAKE, scale=0.07,
                 ctx=FAKE, lse=None, err=None)
        a.update(kw)
        return L.mla_decode_absorb_static(*a.values(), None)

    assert static(dt=_capi.MLA_F32) == 2
    assert static(B=0) == 1
    assert static(B=100_000, n_max=65536) == 6   # more split-KV scratch than the built-in array holds
    def multi_topk(**kw):
        a = dict(dims=DS, dt=_capi.MLA_BF16, B=2, T=2, qt=FAKE, ldqt=512, qp=FAKE, ldqp=64, ckv=FAKE,
                 cb=4096 * 576, cr=576, kr=FAKE, kb=4096 * 576, krr=576, n_max=4096, lengths=FAKE, tk=FAKE,
                 k=64, scale=0.07, ctx=FAKE, lse=None, ws=FAKE, wsb=1 << 40, err=None)
        a.update(kw)
        return L.mla_decode_absorb_multi_topk(*a.values(), None)

    assert multi_topk(tk=None) == 1          # the sets are the point of this call
    assert multi_topk(dims=tiny) == 2        # bf16 needs the DeepSeek dimensions
    assert multi_topk(T=0) == 1
    assert multi_topk(T=4097) == 1
    assert multi_topk(k=0) == 1
    assert multi_topk(k=4097) == 1           # more selected rows than cache rows
    assert multi_topk(B=40000) == 2          # more query groups than one grid dimension holds
    assert multi_topk(lengths=None) == 1
    assert multi_topk(cr=500) == 1
    assert multi_topk(scale=float("nan")) == 1
    assert multi_topk(qt=FAKE + 2) == 1      # misaligned bf16 rows
    assert multi_topk(ws=None) == 6
    assert multi_topk(wsb=16) == 6
    assert multi_topk(T=1, ws=None) == 6     # T = 1 is the one-token top-k decode
    assert L.mla_selftest_wait_timeout(1_000_000, None, None) == 1
    assert L.mla_selftest_wait_timeout(10, FAKE, None) == 1            # below 1 us
    assert L.mla_selftest_wait_timeout(2_000_000_000, FAKE, None) == 1  # above 1 s
