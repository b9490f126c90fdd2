"""The Python binding's argument marshalling on the host: tensors that the C ABI cannot take are
refused with a Python error before any call reaches the library's kernels (no GPU needed)."""

import pytest
import torch

from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.build import build

DIMS = (128, 512, 64, 128, 128)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build(quiet=True)


def _decode_args(B=2, n_max=64, dtype=torch.bfloat16):
    q_tilde = torch.zeros((B, 128, 512), dtype=dtype)
    q_pe = torch.zeros((B, 128, 64), dtype=dtype)
    cache = torch.zeros((B, n_max, 576), dtype=dtype)
    lengths = torch.full((B,), n_max, dtype=torch.int32)
    return q_tilde, q_pe, cache[..., :512], cache[..., 512:], lengths


def test_host_tensors_are_refused():
    q_tilde, q_pe, c_kv, k_r, lengths = _decode_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.mla_decode_absorb(DIMS, q_tilde, q_pe, c_kv, k_r, lengths, 0.072)


def test_layout_checks():
    q_tilde, q_pe, c_kv, k_r, lengths = _decode_args()
    # query rows must be evenly strided [B, n_h, width] with a contiguous last axis
    with pytest.raises(ValueError, match="contiguous"):
        api.mla_decode_absorb(DIMS, q_tilde.transpose(1, 2).contiguous().transpose(1, 2), q_pe, c_kv, k_r, lengths,
                              0.072)
    head_major = torch.zeros((128, 2, 512), dtype=torch.bfloat16).transpose(0, 1)  # (b, h) rows not b-major
    with pytest.raises(ValueError, match="n_h, width"):
        api.mla_decode_absorb(DIMS, head_major, q_pe, c_kv, k_r, lengths, 0.072)
    with pytest.raises(ValueError, match="contiguous"):
        api.mla_decode_absorb(DIMS, q_tilde, q_pe, c_kv.transpose(1, 2), k_r, lengths, 0.072)


def test_dtype_checks():
    q_tilde, q_pe, c_kv, k_r, lengths = _decode_args()
    with pytest.raises(TypeError, match="int32"):
        api.mla_decode_absorb(DIMS, q_tilde, q_pe, c_kv, k_r, lengths.long(), 0.072)
    with pytest.raises(TypeError, match="unsupported dtype"):
        api.mla_decode_workspace_size(DIMS, torch.float16, 2, 64)
    with pytest.raises(TypeError, match="unsupported dtype"):
        api.mla_prefill_workspace_size(DIMS, torch.float16, 1, 16)
    h = _decode_args(dtype=torch.float16)
    with pytest.raises(TypeError, match="unsupported dtype"):
        api.mla_decode_absorb(DIMS, *h, 0.072)
    q8 = torch.zeros((2, 64, 512), dtype=torch.float16)
    with pytest.raises(TypeError):
        api.mla_decode_absorb_fp8kv(DIMS, *_decode_args()[:2], q8, torch.zeros((2, 64, 4)), _decode_args()[3],
                                    _decode_args()[4], 0.072)


def test_size_queries_answer_on_the_host():
    assert api.mla_decode_workspace_size(DIMS, torch.bfloat16, 32, 4096) > 0
    assert api.mla_decode_num_launches(DIMS, torch.bfloat16, 32, 4096) == 1
    assert api.mla_prefill_workspace_size(DIMS, torch.bfloat16, 2, 2048) == 2 * 2048 * 128 * 256 * 2
