"""Device validation of top-k index arrays (range and distinctness per sequence) through the C ABI.
The flag must say exactly what a host scan of the same array says."""

import numpy as np
import pytest
import torch

from head_latent_attention_absorb_b200 import api
from head_latent_attention_absorb_b200.configs import SPARSE_V32
from head_latent_attention_absorb_b200.inputs import make_decode_inputs

pytestmark = pytest.mark.gpu

MLA_ERR_INDEX, MLA_ERR_LENGTH = 4, 7


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch.device("cuda")


def host_verdict(idx: np.ndarray, lengths, n_max: int) -> int:
    """What the flag must hold: 0, or the first error class a scan of the rows finds (the kernel
    raises every error it sees, the first to land wins, so the test cases carry one class each)."""
    for b, row in enumerate(idx):
        L = n_max if lengths is None else int(lengths[b])
        if not 1 <= L <= n_max:
            return MLA_ERR_LENGTH
        if (row < 0).any() or (row >= L).any() or len(set(row.tolist())) != len(row):
            return MLA_ERR_INDEX
    return 0


def device_verdict(idx: np.ndarray, lengths, n_max: int) -> int:
    t = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
    ln = None if lengths is None else torch.as_tensor(np.asarray(lengths, dtype=np.int32)).cuda()
    err = api.mla_check_topk(t, n_max, ln)
    return api.mla_get_device_error(err)


def test_sparse_workload_indices_are_valid(dev):
    cfg = SPARSE_V32
    x = make_decode_inputs(cfg)
    idx, lengths = x["topk"].numpy(), x["lengths"].numpy()
    assert host_verdict(idx, lengths, cfg.n_max) == 0
    assert device_verdict(idx, lengths, cfg.n_max) == 0


@pytest.mark.parametrize("case", ["duplicate", "too_large", "negative", "zero_length", "no_lengths_ok"])
def test_each_error_class(dev, case):
    rng = np.random.default_rng(8)
    B, k, n_max = 6, 300, 5000
    lengths = rng.integers(k, n_max + 1, B)
    idx = np.stack([rng.choice(L, k, replace=False) for L in lengths])
    if case == "duplicate":
        idx[3, 7] = idx[3, 200]
    elif case == "too_large":
        idx[1, 0] = lengths[1]
    elif case == "negative":
        idx[5, 299] = -1
    elif case == "zero_length":
        lengths[2] = 0
    elif case == "no_lengths_ok":
        lengths = None
    want = host_verdict(idx, lengths, n_max)
    assert want == {"duplicate": MLA_ERR_INDEX, "too_large": MLA_ERR_INDEX, "negative": MLA_ERR_INDEX,
                    "zero_length": MLA_ERR_LENGTH, "no_lengths_ok": 0}[case]
    assert device_verdict(idx, lengths, n_max) == want


def test_long_cache_bitmap(dev):
    # a million positions: a 122 KB bitmap, past the default 48 KB of shared memory
    rng = np.random.default_rng(9)
    n_max, k = 1_000_000, 2048
    idx = np.stack([rng.choice(n_max, k, replace=False) for _ in range(3)])
    assert device_verdict(idx, None, n_max) == 0
    idx[2, 1000] = idx[2, 5]
    assert device_verdict(idx, None, n_max) == MLA_ERR_INDEX
