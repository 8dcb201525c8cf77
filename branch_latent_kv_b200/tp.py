"""Branch-sharded tensor parallelism for the MLRA decode step.

MLRA's branches are independent until the up-projection sums them ("The Core
Insight: Sum of Branches, Not Sum of Keys" on the wispaper.ai MLRA blog page),
so a tensor-parallel group can split them: rank r of `world` ranks keeps
branches [r*B/world, (r+1)*B/world) of the latent cache, of the absorbed
queries and of W_UV, plus a full copy of the RoPE cache and the RoPE queries.
Under 4-way tensor parallelism with MLRA-4 that is one branch per GPU, which
is how each GPU's cache read drops to 1.5 d_h per token against 4.5 d_h for
MLA (same section).  Each rank decodes its branches with ``mlra_decode``
(global out_scale); ``mlra_up_proj_allreduce`` then multiplies them by the
rank's W_UV slice and adds all ranks' products inside the kernel, through
exchange regions that every rank maps, so every rank ends with the full y.

This module is host plumbing only: the process group (``torch.distributed``)
exchanges the regions' IPC handles once; every step runs in the library's
kernels.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import binding


def branch_range(branches: int, world: int, rank: int) -> Tuple[int, int]:
    """The contiguous branch range [b0, b1) that `rank` holds."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a group of {world}")
    if branches % world != 0:
        raise ValueError(f"{branches} branches do not split evenly over {world} ranks")
    per = branches // world
    return rank * per, (rank + 1) * per


def shard(t: torch.Tensor, dim: int, branches: int, world: int, rank: int) -> torch.Tensor:
    """This rank's branches of `t` along its branch dimension `dim`, contiguous."""
    if t.shape[dim] != branches:
        raise ValueError(f"dimension {dim} of shape {tuple(t.shape)} is not the branch dimension ({branches})")
    b0, b1 = branch_range(branches, world, rank)
    return t.narrow(dim, b0, b1 - b0).contiguous()


def shard_latent_cache(latent_cache: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """[pages, P, B, d_c] -> [pages, P, B/world, d_c] (this rank's branches)."""
    return shard(latent_cache, 2, latent_cache.shape[2], world, rank)


def shard_q_lat(q_lat: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """[N, H, B, d_c] -> [N, H, B/world, d_c]."""
    return shard(q_lat, 2, q_lat.shape[2], world, rank)


def shard_w_uv(w_uv: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """[B, d_c, H*d_h] -> [B/world, d_c, H*d_h]."""
    return shard(w_uv, 0, w_uv.shape[0], world, rank)


class ExchangeGroup:
    """One exchange region per rank of a process group, mapped by every rank.

    Collective: every rank of `group` constructs it with the same sizes
    (`branches` = branches per rank).  Each rank allocates and zeroes its own
    region, the handles travel through one all_gather_object (which no rank
    leaves before every region is zeroed), and each rank maps the others'.
    ``regions`` is the int64 device tensor of pointers that
    ``mlra_up_proj_allreduce`` takes.
    """

    def __init__(self, batch: int, heads: int, branches: int, d_c: int, d_h: int,
                 group: Optional[dist.ProcessGroup] = None, device: Optional[torch.device] = None,
                 backend=binding):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.backend = backend
        self.device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.nbytes = backend.mlra_exchange_bytes(batch, heads, branches, d_c, d_h, self.world)
        self.own, handle = backend.mlra_exchange_alloc(self.nbytes, with_handle=self.world > 1)
        handles = [None] * self.world
        dist.all_gather_object(handles, handle, group=group)
        ptrs, self._opened = [], []
        try:
            for r, h in enumerate(handles):
                if r == self.rank:
                    ptrs.append(self.own)
                else:
                    p = backend.mlra_exchange_open(h)
                    self._opened.append(p)
                    ptrs.append(p)
        except Exception:
            self._release()
            raise
        self.regions = torch.tensor(ptrs, dtype=torch.int64, device=self.device)

    def reset(self) -> None:
        """Collective, after a timeout: once every rank's kernels have ended
        (no peer can still write into a region), each rank zeroes its own
        region, and the group meets again before the next call."""
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)
        self.backend.mlra_exchange_reset(self.own, self.nbytes, device=self.device)
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)

    def close(self) -> None:
        """Collective: no rank frees its region while another may still write it."""
        if self.own is None:
            return
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)
        self._release()

    def _release(self) -> None:
        for p in self._opened:
            self.backend.mlra_exchange_close(p)
        self._opened = []
        if self.own is not None:
            self.backend.mlra_exchange_free(self.own)
            self.own = None


class BranchShardedDecode:
    """The decode step of one rank of a branch-sharded group: decode over the
    rank's branches, then the up-projection with the cross-rank branch sum.

    Inputs are this rank's shards (see ``shard_*``): q_lat [N,H,B_r,d_c],
    latent_cache [pages,P,B_r,d_c], w_uv [B_r,d_c,H*d_h]; q_rope, rope_cache,
    block_table, seqlens and gate are the full tensors, the same on every
    rank.  out_scale is the model's (it is applied before the branch sum).
    Returns y bf16 [N, H*d_h], identical on every rank.
    """

    def __init__(self, exchange: ExchangeGroup, wait_limit_ns: int = 2_000_000_000, backend=binding):
        self.ex = exchange
        self.wait_limit_ns = int(wait_limit_ns)
        self.backend = backend

    def __call__(self, q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale, out_scale,
                 w_uv, gate=None, device_status=None) -> torch.Tensor:
        out = self.backend.mlra_decode(q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens,
                                       scale, out_scale)
        return self.backend.mlra_up_proj_allreduce(out, w_uv, self.ex.regions, self.ex.rank, gate=gate,
                                                   device_status=device_status,
                                                   wait_limit_ns=self.wait_limit_ns)
