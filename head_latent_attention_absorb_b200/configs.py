"""Named workloads for multi-head latent attention (MLA) decode and prefill.

DeepSeek-V3 dimensions ("DeepSeek-V3.2-Exp - Key-value latent", MLA-init excerpt, and
"KV Reconstruction", "How it works"): 128 heads, a 512-wide latent c^KV, a 64-wide shared
rotary key k^R, 128-wide content keys and 128-wide values; the fused up-projection wkv_b is
(128 * 256) x 512.  The softmax scale is (d_h + d_r)^-0.5.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class MLAConfig:
    name: str
    kind: str                 # "decode" | "sparse" | "prefill"
    dtype: str                # "bf16" | "f32"
    B: int
    n_h: int = 128
    d_c: int = 512
    d_r: int = 64
    d_h: int = 128
    d_v: int = 128
    n_max: int = 4096         # cache capacity per sequence (decode) / sequence length (prefill)
    lengths: Optional[Tuple[int, int]] = None   # ragged: lengths ~ U[lo, hi] (inclusive)
    topk: int = 0             # sparse decode: indices per sequence
    w_std: float = 0.02
    seed: int = 0
    rope_base: float = 10000.0
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_h + self.d_r)

    @property
    def dims(self) -> Tuple[int, int, int, int, int]:
        return (self.n_h, self.d_c, self.d_r, self.d_h, self.d_v)

    def with_(self, **kw) -> "MLAConfig":
        return replace(self, **kw)


TINY_F32 = MLAConfig(
    name="tiny_decode_f32", kind="decode", dtype="f32", B=1, n_h=4, d_c=64, d_r=16, d_h=32, d_v=32,
    n_max=64, w_std=0.05, seed=1,
    note="B=1, n_h=4, d_c=64, d_R=16, d_h=d_v=32, N=64, fp32; scale 1/sqrt(48)")

V3_DECODE = MLAConfig(
    name="v3_decode_b32_n4096", kind="decode", dtype="bf16", B=32, n_max=4096, seed=2,
    note="DeepSeek-V3 absorbed decode: B=32, 128 heads, d_c=512, d_R=64, N=4096, bf16 in / fp32 accum")

RAGGED_LONG = MLAConfig(
    name="ragged_b8_len1k_64k", kind="decode", dtype="bf16", B=8, n_max=65536, lengths=(1024, 65536), seed=3,
    note="B=8, DeepSeek-V3 dims, lengths ~ U[1024, 65536] by seed")

SPARSE_V32 = MLAConfig(
    name="sparse_b16_n32768_k2048", kind="sparse", dtype="bf16", B=16, n_max=32768, topk=2048, seed=4,
    note="DeepSeek-V3.2 sparse decode: B=16, N=32768, 2048 distinct top-k indices per sequence")

PREFILL = MLAConfig(
    name="prefill_b2_s2048", kind="prefill", dtype="bf16", B=2, n_max=2048, seed=5,
    note="naive-path causal prefill: B=2, S=2048, 128 heads, 192-wide keys")

CONFIGS = {c.name: c for c in (TINY_F32, V3_DECODE, RAGGED_LONG, SPARSE_V32, PREFILL)}
