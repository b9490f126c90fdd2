"""Shared helpers of the GPU parity tests: tolerances and oracle drivers.

Tolerances (bf16 storage, fp32 accumulation): max |err| <= 2e-2 and
||err||_F / ||ref||_F <= 1e-2; fp32: both <= 1e-4.  Index work is compared bit for bit."""

import numpy as np
import torch

import oracle as O

TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-4)}


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_close(got, want, dtype, what=""):
    g = to_np(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    w = np.asarray(want, dtype=np.float64)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = g - w
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(w), 1e-300)) if err.size else 0.0
    tol_abs, tol_rel = TOL[dtype]
    assert max_abs <= tol_abs and rel <= tol_rel, f"{what}: max|err|={max_abs:.3e} rel_F={rel:.3e}"
    return max_abs, rel


def oracle_latent(q_tilde, q_pe, c_kv, k_r, lengths, scale, topk=None, batches=None):
    """Per-sequence oracle latent attention: returns ctx [nb, n_h, d_c], lse [nb, n_h]."""
    bs = range(q_tilde.shape[0]) if batches is None else batches
    ctxs, lses = [], []
    for b in bs:
        L = int(lengths[b])
        tk = None if topk is None else topk[b].numpy()
        ctx, lse, _ = O.latent_attention(q_tilde[b], q_pe[b], c_kv[b, :L], k_r[b, :L], scale, tk)
        ctxs.append(ctx)
        lses.append(lse)
    return np.stack(ctxs), np.stack(lses)
