"""Test helpers: build paged caches FROM logical token sequences.

The oracle and the kernels gather token t of a sequence through the block
table.  These helpers do the inverse, page by page (copy logical page j of
sequence n into a randomly chosen physical page and record that page in the
block table), so a test can compare paged results with attention computed on
the logical sequences directly.
"""
from __future__ import annotations

import numpy as np
import torch


def bf16_exact(shape, rng, std=1.0):
    """float64 array whose values are exactly representable in bf16."""
    x = torch.from_numpy(rng.standard_normal(shape) * std).to(torch.bfloat16)
    return x.to(torch.float64).numpy()


def paged_from_logical(latents, ropes, page_size, rng, slack_pages=0, max_pages_per_seq=None,
                       fill=np.nan):
    """latents: list of [L_n, B, d_c]; ropes: list of [L_n, d_r].

    Returns (latent_pool [pages, P, B, d_c], rope_pool [pages, P, d_r],
    block_table int32 [N, max_pages], seqlens int32 [N]).  Pool slots that
    belong to no token hold ``fill`` (NaN by default).
    """
    n_seq = len(latents)
    B, d_c = latents[0].shape[1:]
    d_r = ropes[0].shape[1]
    counts = [-(-len(c) // page_size) for c in latents]
    total = sum(counts) + slack_pages
    if max_pages_per_seq is None:
        max_pages_per_seq = max(max(counts), 1)
    perm = rng.permutation(total)
    lat_pool = np.full((total, page_size, B, d_c), fill, dtype=np.float64)
    rope_pool = np.full((total, page_size, d_r), fill, dtype=np.float64)
    table = np.full((n_seq, max_pages_per_seq), -1, dtype=np.int32)
    k = 0
    for n in range(n_seq):
        for j in range(counts[n]):
            phys = int(perm[k])
            k += 1
            piece = latents[n][j * page_size:(j + 1) * page_size]
            lat_pool[phys, :len(piece)] = piece
            rope_pool[phys, :len(piece)] = ropes[n][j * page_size:(j + 1) * page_size]
            table[n, j] = phys
    seqlens = np.array([len(c) for c in latents], dtype=np.int32)
    return lat_pool, rope_pool, table, seqlens
