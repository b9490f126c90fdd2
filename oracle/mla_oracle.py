"""Plain fp64 CPU statement of multi-head latent attention (MLA), naive and absorbed.

Test infrastructure only: the product path never imports this module (see the package
docstring).  Every array is upcast to float64 on entry, so bf16 or fp32 inputs are used
at exactly the values the GPU receives; nothing is rounded in between.

Sources (page title, then section / equation):

* "KV Reconstruction" (DeepSeek-V3 note), "How it works": eqs. (2) and (5),
  k^C_t = W^UK c^KV_t and v^C_t = W^UV c^KV_t, with W^UK, W^UV in R^{n_h d_h x d_c};
  the key used by attention is k_{t,i} = [k^C_{t,i}; k^R_t] (192 wide for DeepSeek-V3).
  Same page, "Naive path": expand, split, concatenate k^R, run ordinary attention.
  Same page, "Absorb path (default)": the content score equals ((W^UK_i)^T q^C_i)^T c^KV_j
  and the value mix equals W^UV_i sum_j alpha_j c^KV_j; rotary scores are added separately.
  Same page, "Official code": the fused wkv_b holds, per head, the d_h key rows first and
  the d_v value rows after them.
* "DeepSeek-V3.2-Exp - Absorb key weights", the MQA-decode code excerpt: the query is folded
  through the first qk_nope_head_dim rows of each head of wkv_b; scores over the cached latent
  plus scores over the rotary cache, times the softmax scale; an optional -inf mask with 0
  scattered at the top-k indices; softmax over positions; weighted sum of the cached latent;
  then the last v_head_dim rows of each head map it back up.
* "Value up-projection", the MHA-prefill excerpt: wkv_b expansion viewed as
  [B, S, heads, d_h + d_v], split into k_nope and v, k = [k_nope; k_pe broadcast over heads],
  scaled scores, additive mask (causal), softmax, weighted sum of v.
* "DeepSeek-V3.2-Exp - Key-value latent", the MLA-init excerpt: softmax_scale is
  qk_head_dim^-0.5 with qk_head_dim = qk_nope_head_dim + qk_rope_head_dim.
* "Value up-projection", "Parameters": 8,388,608 parameters per value up-projection.
* "DeepSeek V3" (rainlin-net), "Decoupled RoPE": MLA cache = B N (d_c + d_R) s bytes,
  against 2 B N h_q d_h s for standard MHA.
* "DeepSeek-V3.2-Exp - Key-value down-projection", the mla-kv excerpt: the joint down-projection
  is split into the latent (kv_lora_rank) and the rotary key (qk_rope_head_dim); the latent goes
  through kv_norm, the key through the rotary embedding.  "Key-value latent RMSNorm": float32,
  x rsqrt(mean(x^2) + eps), then one gain per feature.

Readings where the pages are silent (each listed in the design notes):
* Mask semantics: a scatter of 0 into a -inf row is a set, so a repeated index counts once.
* Causal prefill: query position s attends keys t <= s.
* One query token per sequence in decode; the query is the last cached position.
* Rotary embedding: interleaved pairs rotated by pos base^(-2i/d) (the rotation is not shown);
  the new token's rows are written at cache row = its position.
"""

from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    """Upcast a numpy array or a CPU torch tensor (any float dtype) to float64."""
    if hasattr(x, "detach"):  # torch tensor: go through float32 (exact for bf16/fp32)
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------------------
# Weights
# ----------------------------------------------------------------------------------------

def split_wkv_b(w_kv_b, n_h: int, d_h: int, d_v: int):
    """Split the fused up-projection into W^UK and W^UV per head.

    "KV Reconstruction", "Official code": wkv_b has shape (n_h (d_h + d_v), d_c), is viewed as
    (n_h, d_h + d_v, d_c); rows [0, d_h) of each head are W^UK_i and rows [d_h, d_h + d_v) are
    W^UV_i ("Value up-projection", "Explanation": output features 128-255 of each head's 256).

    Returns (w_uk [n_h, d_h, d_c], w_uv [n_h, d_v, d_c]) as float64.
    """
    w = _f64(w_kv_b)
    d_c = w.shape[-1]
    assert w.shape == (n_h * (d_h + d_v), d_c), w.shape
    w = w.reshape(n_h, d_h + d_v, d_c)
    return w[:, :d_h, :], w[:, d_h:, :]


def value_up_params(n_h: int, d_v: int, d_c: int) -> int:
    """Parameter count of W^UV ("Value up-projection", "Parameters": n_h d_v x d_c)."""
    return n_h * d_v * d_c


def mla_cache_bytes(B: int, N: int, d_c: int, d_r: int, s: int) -> int:
    """MLA cache size B N (d_c + d_R) s ("DeepSeek V3", "Decoupled RoPE")."""
    return B * N * (d_c + d_r) * s


def mha_cache_bytes(B: int, N: int, h_q: int, d_h: int, s: int) -> int:
    """Standard MHA cache size 2 B N h_q d_h s, the page's comparison ("Decoupled RoPE")."""
    return 2 * B * N * h_q * d_h * s


# ----------------------------------------------------------------------------------------
# Softmax and masks
# ----------------------------------------------------------------------------------------

def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    """Row softmax, max-subtracted, in float64.  -inf entries get weight 0; every row must
    hold at least one finite entry."""
    s = np.asarray(s, dtype=np.float64)
    m = np.max(s, axis=axis, keepdims=True)
    assert np.all(np.isfinite(m)), "a softmax row has no finite score"
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def _logsumexp(s: np.ndarray, axis: int = -1) -> np.ndarray:
    m = np.max(s, axis=axis, keepdims=True)
    return (m + np.log(np.sum(np.exp(s - m), axis=axis, keepdims=True))).squeeze(axis)


def index_mask(length: int, topk) -> np.ndarray:
    """The sparse-attention mask of the V3.2 decode excerpt ("Absorb key weights"): a row of
    -inf of the cache length with 0 written at every top-k index.  A repeated index writes the
    same 0 twice, so the selected positions form a set."""
    mask = np.full((length,), -np.inf, dtype=np.float64)
    idx = np.asarray(topk, dtype=np.int64).reshape(-1)
    assert idx.size == 0 or (idx.min() >= 0 and idx.max() < length), "top-k index out of range"
    mask[idx] = 0.0
    return mask


# ----------------------------------------------------------------------------------------
# Naive path (the literal equations): the definition everything else is checked against
# ----------------------------------------------------------------------------------------

def naive_decode(q_nope, q_pe, c_kv, k_r, w_kv_b, scale: float, topk=None, heads=None):
    """Naive MLA decode for ONE sequence and one query token.

    q_nope [n_h, d_h], q_pe [n_h, d_r], c_kv [L, d_c] and k_r [L, d_r] hold the L cached
    positions (already cut to the sequence length), w_kv_b [n_h (d_h + d_v), d_c].
    ``heads`` optionally restricts the evaluation to a subset of heads (heads are independent).

    Steps ("KV Reconstruction", "How it works" and "Naive path"):
      1. k^C_t = W^UK c_t and v^C_t = W^UV c_t, split into heads       (eqs. 2 and 5)
      2. k_{t,i} = [k^C_{t,i}; k^R_t]                                  (key assembly)
      3. q_i = [q^C_i; q^R_i]
      4. s_{t,i} = scale * q_i . k_{t,i}
      5. sparse variant: s = -inf outside the top-k set                ("Absorb key weights")
      6. alpha = softmax over t
      7. o_i = sum_t alpha_{t,i} v^C_{t,i}
    Returns (o [n_heads, d_v], alpha [n_heads, L]).
    """
    q_nope, q_pe, c_kv, k_r = map(_f64, (q_nope, q_pe, c_kv, k_r))
    n_h, d_h = q_nope.shape
    L, d_c = c_kv.shape
    w = _f64(w_kv_b)
    d_v = w.shape[0] // n_h - d_h
    w_uk, w_uv = split_wkv_b(w, n_h, d_h, d_v)
    hs = np.arange(n_h) if heads is None else np.asarray(heads)
    # 1. reconstruction: W^UK c_t for every cached t (a plain matmul per head set)
    k_c = np.einsum("hdc,tc->thd", w_uk[hs], c_kv)           # [L, nh', d_h]
    v_c = np.einsum("hdc,tc->thd", w_uv[hs], c_kv)           # [L, nh', d_v]
    # 2. k = [k^C ; k^R] (k^R shared by all heads)
    k = np.concatenate([k_c, np.broadcast_to(k_r[:, None, :], (L, len(hs), k_r.shape[1]))], axis=-1)
    # 3. q = [q^C ; q^R]
    q = np.concatenate([q_nope[hs], q_pe[hs]], axis=-1)       # [nh', d_h + d_r]
    # 4. scores
    s = scale * np.einsum("hd,thd->ht", q, k)                # [nh', L]
    # 5. sparse mask
    if topk is not None:
        s = s + index_mask(L, topk)[None, :]
    # 6. softmax over positions
    alpha = softmax(s, axis=-1)
    # 7. weighted sum of the reconstructed values
    o = np.einsum("ht,thd->hd", alpha, v_c)
    return o, alpha


def naive_prefill(q, c_kv, k_r, w_kv_b, scale: float, n_h: int, d_h: int, d_v: int,
                  causal: bool = True, rows=None, heads=None, topk=None):
    """Naive MLA prefill for ONE sequence ("Value up-projection", MHA-prefill excerpt).

    q [S, n_h, d_h + d_r] (content part first, rotary part last), c_kv [S, d_c], k_r [S, d_r].
    ``rows`` / ``heads`` optionally restrict which query positions / heads are evaluated; each
    output row is its own softmax, so this is a subset of the same definition.

    Steps: kv = W_kv_b c (viewed [S, n_h, d_h + d_v]) -> k_nope, v; k = [k_nope; k_pe broadcast];
    scores = q . k * scale; causal additive mask (t <= s kept); softmax over t; out = sum alpha v.
    Sparse variant (the V3.2 MHA-prefill excerpt): ``topk`` [S, k] holds each query row's selected
    positions; a -inf row with 0 scattered at them is added to the causal mask and then to the
    scores, so row s attends its selected positions t <= s (a set: repeats count once).  Every
    row's set must hold at least one t <= s.
    Returns out [len(rows), len(heads), d_v].
    """
    q, c_kv, k_r = map(_f64, (q, c_kv, k_r))
    S = c_kv.shape[0]
    w = _f64(w_kv_b)
    rs = np.arange(S) if rows is None else np.asarray(rows)
    hs = np.arange(n_h) if heads is None else np.asarray(heads)
    kv = (c_kv @ w.T).reshape(S, n_h, d_h + d_v)[:, hs, :]     # wkv_b(kv), view as heads
    k_nope, v = kv[..., :d_h], kv[..., d_h:]
    k = np.concatenate([k_nope, np.broadcast_to(k_r[:, None, :], (S, len(hs), k_r.shape[1]))], axis=-1)
    qs = q[rs][:, hs, :]                                       # [R, nh', d_h + d_r]
    scores = np.einsum("rhd,thd->rht", qs, k) * scale          # [R, nh', S]
    mask = np.zeros((len(rs), S))
    if topk is not None:
        tk = np.asarray(topk)
        mask = np.stack([index_mask(S, tk[r]) for r in rs])   # the index mask of each query row
    if causal:
        t = np.arange(S)[None, :]
        mask = mask + np.where(t <= rs[:, None], 0.0, -np.inf)  # [R, S]
    scores = scores + mask[:, None, :]
    alpha = softmax(scores, axis=-1)
    return np.einsum("rht,thd->rhd", alpha, v)


# ----------------------------------------------------------------------------------------
# Absorbed path, step by step (the three entry points of the decode pipeline)
# ----------------------------------------------------------------------------------------

def absorb_q(q_nope, w_kv_b, n_h: int, d_h: int, d_v: int) -> np.ndarray:
    """q~_i = (W^UK_i)^T q^C_i: d_h content features become d_c latent features
    ("Absorb key weights", first einsum of the decode excerpt).  q_nope [..., n_h, d_h]."""
    w_uk, _ = split_wkv_b(w_kv_b, n_h, d_h, d_v)
    return np.einsum("...hd,hdc->...hc", _f64(q_nope), w_uk)


def latent_attention(q_tilde, q_pe, c_kv, k_r, scale: float, topk=None):
    """Attention taken directly over the cached latent for ONE sequence and one query token.

    q_tilde [n_h, d_c], q_pe [n_h, d_r], c_kv [L, d_c], k_r [L, d_r] (cut to the length).
    s = scale (q~ . c_t + q_pe . k^R_t); optional top-k -inf mask; alpha = softmax over t;
    ctx = sum_t alpha_t c_t  ("Absorb key weights" decode excerpt; "KV Reconstruction",
    "Absorb path").  Returns (ctx [n_h, d_c], lse [n_h], alpha [n_h, L]) where lse is the natural
    log of sum_t exp(s_t) over the kept positions (s already scaled).
    """
    q_tilde, q_pe, c_kv, k_r = map(_f64, (q_tilde, q_pe, c_kv, k_r))
    s = scale * (q_tilde @ c_kv.T + q_pe @ k_r.T)
    if topk is not None:
        s = s + index_mask(c_kv.shape[0], topk)[None, :]
    alpha = softmax(s, axis=-1)
    return alpha @ c_kv, _logsumexp(s, axis=-1), alpha


def out_up(ctx, w_kv_b, n_h: int, d_h: int, d_v: int) -> np.ndarray:
    """o_i = W^UV_i ctx_i: map the latent context back to d_v value features per head
    ("Absorb key weights", last einsum of the decode excerpt).  ctx [..., n_h, d_c]."""
    _, w_uv = split_wkv_b(w_kv_b, n_h, d_h, d_v)
    return np.einsum("...hc,hdc->...hd", _f64(ctx), w_uv)


def absorbed_decode(q_nope, q_pe, c_kv, k_r, w_kv_b, scale: float, d_v: int, topk=None):
    """The whole absorbed decode for ONE sequence: absorb_q -> latent_attention -> out_up.
    Returns a dict with q_tilde, ctx, lse, alpha and o (all float64, no intermediate rounding)."""
    n_h, d_h = np.shape(q_nope)
    qt = absorb_q(q_nope, w_kv_b, n_h, d_h, d_v)
    ctx, lse, alpha = latent_attention(qt, q_pe, c_kv, k_r, scale, topk)
    return {"q_tilde": qt, "ctx": ctx, "lse": lse, "alpha": alpha,
            "o": out_up(ctx, w_kv_b, n_h, d_h, d_v)}


def softmax_scale(d_h: int, d_r: int) -> float:
    """qk_head_dim^-0.5 with qk_head_dim = d_h + d_r ("Key-value latent", MLA-init excerpt)."""
    return 1.0 / math.sqrt(d_h + d_r)


# ----------------------------------------------------------------------------------------
# The step before the path: the new token's latent and rotary key into the caches
# ----------------------------------------------------------------------------------------

def rms_norm(x, gain=None, eps: float = 1e-6) -> np.ndarray:
    """"Key-value latent RMSNorm": each row divided by the square root of (the mean of its
    squares + eps), then multiplied by one gain per feature (ones when ``gain`` is None)."""
    x = _f64(x)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if gain is None else y * _f64(gain)


def rope_interleaved(y, positions, base: float = 10000.0) -> np.ndarray:
    """Rotary embedding of the shared key ("Key-value down-projection", mla-kv excerpt; the
    rotation itself is not shown on the pages).  Reading taken: pair i = (y[2i], y[2i+1]) is the
    complex number y[2i] + j y[2i+1], multiplied by exp(j pos base^(-2i/d)), pos = the row's
    position.  ``y`` [rows, d], ``positions`` [rows]."""
    y = _f64(y)
    d = y.shape[-1]
    pos = np.asarray(positions, dtype=np.float64)
    freq = base ** (-np.arange(0, d, 2, dtype=np.float64) / d)       # [d/2]
    z = (y[..., 0::2] + 1j * y[..., 1::2]) * np.exp(1j * pos[:, None] * freq[None, :])
    out = np.empty_like(y)
    out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


def cache_append(kv_a, positions, d_c: int, d_r: int, gain=None, eps: float = 1e-6,
                 base: float = 10000.0):
    """The new token's cache rows ("Key-value down-projection", mla-kv excerpt): split the joint
    down-projection row into the d_c latent and the d_r rotary key, RMSNorm the latent, rotate
    the key.  Returns (latent rows [B, d_c], rotary rows [B, d_r]); row b belongs at cache row
    positions[b] (the decode reads row t as position t)."""
    x = _f64(kv_a)
    return rms_norm(x[:, :d_c], gain, eps), rope_interleaved(x[:, d_c:d_c + d_r], positions, base)


# ----------------------------------------------------------------------------------------
# Rows ranked next: several new tokens per decode, FP8 block-scaled wkv_b
# ----------------------------------------------------------------------------------------

def multi_token_decode(q_nope, q_pe, c_kv, k_r, w_kv_b, scale: float, d_v: int, topk=None):
    """Absorbed decode of several new tokens of ONE sequence (the decode excerpt's "bshd" queries
    with s > 1, e.g. speculative tokens).

    q_nope [T, n_h, d_h], q_pe [T, n_h, d_r]; c_kv [L, d_c], k_r [L, d_r] hold the L cached rows,
    the T new tokens being the last T of them (positions L - T .. L - 1).  The decode excerpt adds
    no mask over s; the reading taken is the prefill excerpt's causal rule: query s attends rows
    t <= L - T + s.  So T = 1 is the one-token decode, and the T results equal the last T rows of a
    prefill over the same L rows.  ``topk`` [T, k] optionally holds each query's selected positions
    (set semantics, then the causal rule), as in the sparse prefill.
    Steps: q~ = absorb_q; s = scale (q~ . c_t + q_pe . k^R_t) + masks; alpha = softmax over t;
    ctx = sum_t alpha c_t; o = out_up(ctx).  Returns a dict with q_tilde, ctx, lse and o, each
    with the leading T axis.
    """
    q_nope, q_pe, c_kv, k_r = map(_f64, (q_nope, q_pe, c_kv, k_r))
    T, n_h, d_h = q_nope.shape
    L = c_kv.shape[0]
    qt = absorb_q(q_nope, w_kv_b, n_h, d_h, d_v)                               # [T, n_h, d_c]
    s = scale * (np.einsum("shc,tc->sht", qt, c_kv) + np.einsum("shr,tr->sht", q_pe, k_r))
    pos = L - T + np.arange(T)                                                 # each query's position
    mask = np.where(np.arange(L)[None, :] <= pos[:, None], 0.0, -np.inf)       # [T, L]
    if topk is not None:
        tk = np.asarray(topk)
        mask = mask + np.stack([index_mask(L, tk[i]) for i in range(T)])
    s = s + mask[:, None, :]
    alpha = softmax(s, axis=-1)
    ctx = np.einsum("sht,tc->shc", alpha, c_kv)
    return {"q_tilde": qt, "ctx": ctx, "lse": _logsumexp(s, axis=-1),
            "o": out_up(ctx, w_kv_b, n_h, d_h, d_v)}


def fp8_block_scale_shape(out_features: int, in_features: int, block: int = 128):
    """Scale grid of an FP8 weight ("Key-value down-projection", linear excerpt): one float32 scale
    per block x block tile, ceil(out/block) x ceil(in/block)."""
    return (out_features + block - 1) // block, (in_features + block - 1) // block


def weight_dequant(w_q, scale, block: int = 128) -> np.ndarray:
    """Dequantise an FP8 weight with one scale per 128 x 128 tile (linear excerpt: the scales are
    quantisation metadata; "Value up-projection": the decode dequantises wkv_b once and uses it
    unquantised): w[i, j] = w_q[i, j] * scale[i // block, j // block].  ``w_q`` may be a torch
    float8 tensor (its values are read exactly)."""
    w = _f64(w_q)
    s = _f64(scale)
    assert s.shape == fp8_block_scale_shape(w.shape[0], w.shape[1], block), "scale grid shape"
    return w * s[np.arange(w.shape[0]) // block][:, np.arange(w.shape[1]) // block]


# ----------------------------------------------------------------------------------------
# FP8 latent cache (a reading: the weights' FP8 format applied to the cached latent rows)
# ----------------------------------------------------------------------------------------

def e4m3_value(code) -> np.ndarray:
    """Value of FP8 E4M3 codes (uint8): sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
    exponent field 0 holds the subnormals m/8 * 2^-6; the one all-ones pattern S.1111.111 is NaN
    and there is no infinity (the finite "fn" variant the pages' float8 weights use, "Key-value
    down-projection", linear excerpt).  Written out from that definition, code by code."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = sign * val
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


def latent_cache_dequant(c8, kv_scale, block: int = 128) -> np.ndarray:
    """The FP8 latent cache read back: c_kv[t, f] = e4m3(c8[t, f]) * kv_scale[t, f // block].  One
    float32 scale per cached row and 128-feature block, the 128-wide blocks of the FP8 weights
    ("Key-value down-projection", linear excerpt: one float32 scale per 128 x 128 block) applied to
    each cached token's latent row, since rows are written one token at a time (a reading; the
    pages keep the cache in bf16).  c8 [..., d_c] uint8 codes, kv_scale [..., d_c / block]."""
    v = e4m3_value(c8)
    s = _f64(kv_scale)
    d_c = v.shape[-1]
    assert s.shape[-1] == (d_c + block - 1) // block and s.shape[:-1] == v.shape[:-1], "scale grid shape"
    return v * s[..., np.arange(d_c) // block]
