"""Seeded synthetic inputs shaped like DeepSeek-V3 / V3.2 MLA decode and prefill.

This module only draws and shapes data; it holds none of the attention arithmetic.  The
same arrays feed the CUDA path and the CPU oracle.

Recipe (all draws from numpy's PCG64 generator seeded by the workload's seed, in float32):
* c^KV rows: N(0, 1), then RMSNorm over the latent (gain 1, eps 1e-6, in float32), as the
  latent is normalised before it is cached ("Key-value latent", RMSNorm excerpt).
* k^R rows and the query's rotary part: N(0, 1), then rotary embedding, base 10000, on
  interleaved pairs (x[2i], x[2i+1]) by angle pos * base^(-2i/d_r); cache row t has pos = t,
  the decode query has pos = length - 1, prefill query row s has pos = s.
* q_nope: N(0, 1).  wkv_b: N(0, w_std^2).
* Ragged lengths: integers uniform on [lo, hi]; top-k: distinct indices drawn without
  replacement from [0, length) per sequence.
* Finally every tensor is rounded to the workload dtype (bf16 round-to-nearest-even).
Cache rows past a sequence's length are zero.
"""

from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from .configs import MLAConfig

_TORCH_DTYPE = {"bf16": torch.bfloat16, "f32": torch.float32}


def torch_dtype(cfg: MLAConfig) -> torch.dtype:
    return _TORCH_DTYPE[cfg.dtype]


def _rmsnorm_rows(x: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    x = x.float()
    return x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + eps)


def _rope_interleaved(x: torch.Tensor, pos: torch.Tensor, base: float) -> torch.Tensor:
    """Rotate interleaved pairs of the last axis by pos * base^(-2i/d)."""
    d = x.shape[-1]
    inv = base ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)            # [d/2]
    ang = pos.to(torch.float64)[..., None] * inv                                 # [..., d/2]
    cos, sin = torch.cos(ang).float(), torch.sin(ang).float()
    while cos.dim() < x.dim():
        cos, sin = cos.unsqueeze(-2), sin.unsqueeze(-2)
    xe, xo = x[..., 0::2].float(), x[..., 1::2].float()
    out = torch.empty_like(x, dtype=torch.float32)
    out[..., 0::2] = xe * cos - xo * sin
    out[..., 1::2] = xe * sin + xo * cos
    return out


def _normal(rng: np.random.Generator, shape, std: float = 1.0) -> torch.Tensor:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return torch.from_numpy(a)


def make_weights(cfg: MLAConfig, rng: np.random.Generator) -> torch.Tensor:
    return _normal(rng, (cfg.n_h * (cfg.d_h + cfg.d_v), cfg.d_c), cfg.w_std).to(torch_dtype(cfg))


def draw_lengths(cfg: MLAConfig, rng: np.random.Generator) -> torch.Tensor:
    if cfg.lengths is None:
        return torch.full((cfg.B,), cfg.n_max, dtype=torch.int32)
    lo, hi = cfg.lengths
    return torch.from_numpy(rng.integers(lo, hi, size=cfg.B, endpoint=True).astype(np.int32))


def draw_topk(rng: np.random.Generator, lengths: torch.Tensor, k: int) -> torch.Tensor:
    rows = [rng.choice(int(L), size=k, replace=False).astype(np.int32) for L in lengths.tolist()]
    return torch.from_numpy(np.stack(rows))


def make_decode_inputs(cfg: MLAConfig, seed: Optional[int] = None,
                       lengths: Optional[torch.Tensor] = None) -> Dict[str, object]:
    """Inputs of one decode step: a packed cache [B, n_max, d_c + d_r] (c^KV then k^R per row)
    with ``c_kv`` / ``k_r`` as strided views into it, queries, wkv_b, lengths and top-k."""
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    dt = torch_dtype(cfg)
    B, N = cfg.B, cfg.n_max
    w = make_weights(cfg, rng)
    if lengths is None:
        lengths = draw_lengths(cfg, rng)
    lengths = lengths.to(torch.int32)
    cache = torch.zeros((B, N, cfg.d_c + cfg.d_r), dtype=dt)
    for b in range(B):
        L = int(lengths[b])
        c = _rmsnorm_rows(_normal(rng, (L, cfg.d_c)))
        kr = _rope_interleaved(_normal(rng, (L, cfg.d_r)), torch.arange(L), cfg.rope_base)
        cache[b, :L, :cfg.d_c] = c.to(dt)
        cache[b, :L, cfg.d_c:] = kr.to(dt)
    q_nope = _normal(rng, (B, cfg.n_h, cfg.d_h)).to(dt)
    q_pe = _rope_interleaved(_normal(rng, (B, cfg.n_h, cfg.d_r)), (lengths - 1).long(),
                             cfg.rope_base).to(dt)
    topk = draw_topk(rng, lengths, cfg.topk) if cfg.topk > 0 else None
    return {
        "cfg": cfg, "w_kv_b": w, "cache": cache,
        "c_kv": cache[..., :cfg.d_c], "k_r": cache[..., cfg.d_c:],
        "q_nope": q_nope, "q_pe": q_pe, "lengths": lengths, "topk": topk, "scale": cfg.scale,
    }


def make_prefill_inputs(cfg: MLAConfig, seed: Optional[int] = None) -> Dict[str, object]:
    """Inputs of one naive-path prefill: q [B, S, n_h, d_h + d_r] (rotary part last),
    c_kv [B, S, d_c], k_r [B, S, d_r] and wkv_b."""
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    dt = torch_dtype(cfg)
    B, S = cfg.B, cfg.n_max
    w = make_weights(cfg, rng)
    pos = torch.arange(S)
    c_kv = _rmsnorm_rows(_normal(rng, (B, S, cfg.d_c))).to(dt)
    k_r = _rope_interleaved(_normal(rng, (B, S, cfg.d_r)), pos[None, :].expand(B, S), cfg.rope_base).to(dt)
    q = _normal(rng, (B, S, cfg.n_h, cfg.d_h + cfg.d_r))
    q[..., cfg.d_h:] = _rope_interleaved(q[..., cfg.d_h:], pos[None, :].expand(B, S), cfg.rope_base)
    return {"cfg": cfg, "w_kv_b": w, "q": q.to(dt), "c_kv": c_kv, "k_r": k_r, "scale": cfg.scale}


def quantize_latent_fp8(c_kv: torch.Tensor, block: int = 128):
    """Encodes a bf16/fp32 latent cache [..., d_c] as an FP8 cache: one fp32 scale per row and
    128-feature block (block max / 448, 1 for an all-zero block) and E4M3 codes of c / scale
    (torch's float8_e4m3fn cast, round to nearest even).  Returns (c8 uint8 [..., d_c],
    kv_scale float32 [..., d_c / block])."""
    x = c_kv.float()
    shp = x.shape
    blocks = x.reshape(*shp[:-1], shp[-1] // block, block)
    scale = blocks.abs().amax(dim=-1) / 448.0
    scale = torch.where(scale > 0, scale, torch.ones_like(scale)).to(torch.float32)
    c8 = (blocks / scale[..., None]).reshape(shp).to(torch.float8_e4m3fn).view(torch.uint8)
    return c8, scale


def pack_fp8_cache(c8: torch.Tensor, kv_scale: torch.Tensor, k_r: torch.Tensor) -> torch.Tensor:
    """One 656-byte row per cached token: 512 E4M3 codes, 4 fp32 scales, 64 bf16 rotary features."""
    rows = torch.cat([c8.contiguous().view(torch.uint8), kv_scale.contiguous().view(torch.uint8),
                      k_r.to(torch.bfloat16).contiguous().view(torch.uint8)], dim=-1)
    return rows.contiguous()
