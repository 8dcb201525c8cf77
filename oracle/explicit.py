"""Explicit (non-absorbed) MLRA attention in numpy fp64.

TEST INFRASTRUCTURE ONLY (tests and smoke check); never called by the product
path.  This is the second, independent statement of what the decode path
computes, used to pin the C oracle (check "absorbed form equals explicit
form").

It follows "MLRA: Breaking the Sharding Bottleneck in Latent Attention"
(wispaper.ai blog), section "The Core Insight: Sum of Branches, Not Sum of
Keys": every latent block (branch) b is up-projected into its own per-head
keys and values, standard softmax attention runs on each branch
independently, and the branch outputs are summed; the final calibration factor
of section "Mathematical Calibration: Scaling the Latents" multiplies the sum.
Per-head keys carry a shared decoupled RoPE part (one RoPE key per token, one
RoPE query per head).

Nothing here is absorbed: keys k[t,h,b] = [W_UK[b,h] c_b[t] ; k_r[t]] and
values v[t,h,b] = W_UV[b,h] c_b[t] are materialised, then
    y[h] = out_scale * sum_b softmax_t(scale * q[h,b] . k[t,h,b]) @ v[., h, b]
with q[h,b] = [qC[h] ; q_rope[h]].
"""
from __future__ import annotations

import numpy as np


def _softmax(s):
    s = s - s.max()
    e = np.exp(s)
    return e / e.sum()


def explicit_decode(q_c, q_rope, w_uk, w_uv, latents, ropes, scale, out_scale):
    """Explicit attention for N sequences.

    q_c     [N, H, d_h]     no-RoPE query per head
    q_rope  [N, H, d_r]     RoPE query per head (already rotated)
    w_uk    [B, H, d_h, d_c] key up-projection of branch b for head h
    w_uv    [B, d_c, H*d_h]  value up-projection (column block h belongs to head h)
    latents list of N arrays [L_n, B, d_c] (logical token order)
    ropes   list of N arrays [L_n, d_r]
    returns y [N, H*d_h] float64
    """
    q_c = np.asarray(q_c, dtype=np.float64)
    q_rope = np.asarray(q_rope, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    N, H, d_h = q_c.shape
    B = w_uk.shape[0]
    y = np.zeros((N, H * d_h), dtype=np.float64)
    for n in range(N):
        c = np.asarray(latents[n], dtype=np.float64)
        kr = np.asarray(ropes[n], dtype=np.float64)
        for h in range(H):
            acc = np.zeros(d_h)
            for b in range(B):
                keys = np.concatenate([c[:, b, :] @ w_uk[b, h].T, kr], axis=1)  # [L, d_h + d_r]
                vals = c[:, b, :] @ w_uv[b][:, h * d_h:(h + 1) * d_h]          # [L, d_h]
                q = np.concatenate([q_c[n, h], q_rope[n, h]])
                p = _softmax(scale * (keys @ q))
                acc += p @ vals
            y[n, h * d_h:(h + 1) * d_h] = out_scale * acc
    return y


def absorb_queries(q_c, w_uk):
    """q_lat[n,h,b] = W_UK[b,h]^T qC[n,h]  ->  [N, H, B, d_c] (fp64)."""
    q_c = np.asarray(q_c, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    return np.einsum("nhd,bhdk->nhbk", q_c, w_uk)
