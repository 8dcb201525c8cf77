"""Seeded synthetic decode workloads, shared by the tests, the smoke check and
the benchmark.

This module only draws and lays out inputs: it holds none of the attention
arithmetic.  Values follow the workload recipe: every float tensor is drawn
N(0, 1) / sqrt(last dimension) in fp32 and rounded to bf16 (round to nearest
even); W_UV is drawn N(0, 1) / sqrt(branches * d_c) (its fan-in).  Draw order
from one ``torch.Generator`` seeded with ``seed``: seqlens (ragged workloads
only), q_lat, q_rope, latent pool, RoPE pool, W_UV, page permutation.

Paging: sequence n owns ceil(L_n / P) pages.  The physical pool holds exactly
those pages (plus ``slack_pages`` unused ones).  With ``page_order="identity"``
sequence n's pages are consecutive; with ``"permuted"`` they come from a seeded
random permutation of the pool.  Unused block-table slots hold -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    """Shape of one decode step over a paged MLRA latent cache."""

    name: str
    batch: int
    heads: int
    branches: int
    d_c: int
    d_r: int
    page_size: int
    seqlen: Optional[int] = None                 # uniform context length
    seqlen_range: Optional[Tuple[int, int]] = None  # ragged: inclusive range
    d_h: int = 128                               # W_UV output width per head
    page_order: str = "identity"                 # or "permuted"
    out_scale: Optional[float] = None            # default 1/sqrt(branches)
    seed: int = 0

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(d_c + d_r)."""
        return 1.0 / math.sqrt(self.d_c + self.d_r)

    @property
    def output_scale(self) -> float:
        return self.out_scale if self.out_scale is not None else 1.0 / math.sqrt(self.branches)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five decode workloads (the fifth has three shapes) and the variant sweep.
WORKLOADS = {
    "tiny": Workload("tiny", batch=1, heads=8, branches=4, d_c=64, d_r=32, page_size=64,
                     seqlen=256, d_h=64),
    "decode_2p9b": Workload("decode_2p9b", batch=16, heads=16, branches=4, d_c=128, d_r=64,
                            page_size=64, seqlen=8192),
    "long_context": Workload("long_context", batch=4, heads=16, branches=4, d_c=128, d_r=64,
                             page_size=64, seqlen=131072, page_order="permuted"),
    "ragged": Workload("ragged", batch=64, heads=16, branches=4, d_c=128, d_r=64, page_size=64,
                       seqlen_range=(1024, 32768), page_order="permuted"),
    "mla_equal_bytes": Workload("mla_equal_bytes", batch=32, heads=16, branches=1, d_c=512,
                                d_r=64, page_size=64, seqlen=16384),
    "mlra4_equal_bytes": Workload("mlra4_equal_bytes", batch=32, heads=16, branches=4, d_c=128,
                                  d_r=64, page_size=64, seqlen=16384),
    # One tensor-parallel rank's share of MLRA-4: one branch of 128 plus the
    # replicated RoPE key; the calibration factor of the 4-branch model stays.
    "tp_shard": Workload("tp_shard", batch=32, heads=16, branches=1, d_c=128, d_r=64,
                         page_size=64, seqlen=16384, out_scale=0.5),
    # Variant sweep: the two-branch model at the same cache bytes per token
    # (2 x 256 + 64), and one sequence at the longest context the pages
    # measure (2M tokens, 2.4 GB of cache).
    "mlra2_equal_bytes": Workload("mlra2_equal_bytes", batch=32, heads=16, branches=2, d_c=256,
                                  d_r=64, page_size=64, seqlen=16384),
    "context_2m": Workload("context_2m", batch=1, heads=16, branches=4, d_c=128, d_r=64,
                           page_size=64, seqlen=2097152, page_order="permuted"),
    # Many query heads on one latent cache (every head reads the same
    # latents, as in MLA's large models): the 2.9B cache read by 64 heads.
    "heads_64": Workload("heads_64", batch=16, heads=64, branches=4, d_c=128, d_r=64,
                         page_size=64, seqlen=8192, d_h=64),
}


@dataclass
class DecodeInputs:
    workload: Workload
    q_lat: torch.Tensor        # bf16 [N, H, B, d_c]
    q_rope: torch.Tensor       # bf16 [N, H, d_r]
    latent_cache: torch.Tensor  # bf16 [num_pages, P, B, d_c]
    rope_cache: torch.Tensor   # bf16 [num_pages, P, d_r]
    block_table: torch.Tensor  # int32 [N, max_pages_per_seq]
    seqlens: torch.Tensor      # int32 [N]
    w_uv: Optional[torch.Tensor]  # bf16 [B, d_c, H * d_h]
    scale: float
    out_scale: float

    @property
    def kv_bytes(self) -> int:
        """Algorithmic KV bytes of one decode step: each token's latent row and
        RoPE row read once (bf16)."""
        w = self.workload
        return int(self.seqlens.to(torch.int64).sum()) * (w.branches * w.d_c + w.d_r) * 2

    def to(self, device) -> "DecodeInputs":
        mv = lambda t: None if t is None else t.to(device)  # noqa: E731
        return DecodeInputs(self.workload, mv(self.q_lat), mv(self.q_rope), mv(self.latent_cache),
                            mv(self.rope_cache), mv(self.block_table), mv(self.seqlens),
                            mv(self.w_uv), self.scale, self.out_scale)


def _draw(shape, dim, gen, device, gain=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return (x * (gain / math.sqrt(dim))).to(torch.bfloat16)


def draw_seqlens(w: Workload, gen: torch.Generator) -> torch.Tensor:
    if w.seqlen_range is not None:
        lo, hi = w.seqlen_range
        return torch.randint(lo, hi + 1, (w.batch,), generator=gen, dtype=torch.int64).to(torch.int32)
    return torch.full((w.batch,), int(w.seqlen), dtype=torch.int32)


def make_inputs(w: Workload, seed: Optional[int] = None, device: str = "cpu",
                with_w_uv: bool = True, q_gain: float = 1.0, slack_pages: int = 0,
                nan_fill_unused: bool = False, seqlens: Optional[torch.Tensor] = None,
                max_pages_per_seq: Optional[int] = None) -> DecodeInputs:
    """Draw one decode step's inputs.

    ``q_gain`` multiplies both queries before rounding (peaked-softmax
    variants).  ``slack_pages`` adds unused pool pages; with
    ``nan_fill_unused`` those pages and every slot past the end of a
    sequence's last page are NaN, which a correct kernel never reads.
    ``seqlens`` (int32 [N]) overrides the workload's lengths.
    Random draws happen on ``device`` (a CUDA generator gives other values
    than the CPU one for the same seed; each run is still deterministic).
    """
    seed = w.seed if seed is None else seed
    cpu_gen = torch.Generator(device="cpu").manual_seed(seed)
    # On the CPU one generator serves every draw, in the documented order.
    gen = cpu_gen if torch.device(device).type == "cpu" else \
        torch.Generator(device=device).manual_seed(seed)
    if seqlens is None:
        seqlens = draw_seqlens(w, cpu_gen)
    seqlens = seqlens.to(torch.int32).cpu()
    N, H, B, d_c, d_r, P = w.batch, w.heads, w.branches, w.d_c, w.d_r, w.page_size
    if seqlens.numel() != N:
        raise ValueError("seqlens must have one entry per sequence")
    pages_per_seq = [(max(int(L), 0) + P - 1) // P for L in seqlens.tolist()]
    used_pages = sum(pages_per_seq)
    num_pages = max(used_pages + slack_pages, 1)
    if max_pages_per_seq is None:
        max_pages_per_seq = max(max(pages_per_seq), 1)

    q_lat = _draw((N, H, B, d_c), d_c, gen, device, q_gain)
    q_rope = _draw((N, H, d_r), d_r, gen, device, q_gain)
    latent = _draw((num_pages, P, B, d_c), d_c, gen, device)
    rope = _draw((num_pages, P, d_r), d_r, gen, device)
    w_uv = _draw((B, d_c, H * w.d_h), B * d_c, gen, device) if with_w_uv else None

    if w.page_order == "permuted":
        order = torch.randperm(num_pages, generator=cpu_gen)
    elif w.page_order == "identity":
        order = torch.arange(num_pages)
    else:
        raise ValueError(f"unknown page_order {w.page_order!r}")
    block_table = torch.full((N, max_pages_per_seq), -1, dtype=torch.int32)
    cursor = 0
    for n, cnt in enumerate(pages_per_seq):
        block_table[n, :cnt] = order[cursor:cursor + cnt].to(torch.int32)
        cursor += cnt

    if nan_fill_unused:
        used = torch.zeros(num_pages, dtype=torch.bool)
        for n, cnt in enumerate(pages_per_seq):
            if cnt == 0:
                continue
            pages = block_table[n, :cnt].long()
            used[pages] = True
            tail = int(seqlens[n]) - (cnt - 1) * P   # valid slots in the last page
            last = int(pages[-1])
            latent[last, tail:] = float("nan")
            rope[last, tail:] = float("nan")
        free = (~used).nonzero().flatten().to(latent.device)
        latent[free] = float("nan")
        rope[free] = float("nan")

    return DecodeInputs(w, q_lat, q_rope, latent, rope, block_table.to(device),
                        seqlens.to(device), w_uv, w.scale, w.output_scale)
