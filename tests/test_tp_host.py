"""Host logic of branch-sharded tensor parallelism, on the CPU (gloo ranks).

The kernels need a GPU; here a stand-in backend puts the oracle where the
library's decode and fused up-projection would run, and a gloo all-reduce
where the in-kernel exchange would add the ranks' products.  What is
checked is the part that runs on the host: which branches each rank holds,
how the caches, queries and W_UV are cut, that every rank maps every other
rank's exchange region and frees what it owns, and that the ranks' shards add
up to the unsharded step (the identity the sharding rests on: the branch sum
of the up-projection splits over any partition of the branches).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from branch_latent_kv_b200 import tp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_branch_range_partitions_the_branches():
    for branches, world in [(4, 1), (4, 2), (4, 4), (8, 4), (2, 2)]:
        got = [tp.branch_range(branches, world, r) for r in range(world)]
        assert got[0][0] == 0 and got[-1][1] == branches
        assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
        assert len({b1 - b0 for b0, b1 in got}) == 1
    with pytest.raises(ValueError):
        tp.branch_range(4, 3, 0)
    with pytest.raises(ValueError):
        tp.branch_range(4, 2, 2)


def test_shards_cut_the_branch_dimension():
    lat = torch.arange(3 * 2 * 4 * 5).reshape(3, 2, 4, 5)
    w = torch.arange(4 * 5 * 6).reshape(4, 5, 6)
    assert torch.equal(tp.shard_latent_cache(lat, 2, 1), lat[:, :, 2:4])
    assert torch.equal(tp.shard_q_lat(lat, 4, 3), lat[:, :, 3:4])
    assert torch.equal(tp.shard_w_uv(w, 2, 0), w[0:2])
    assert tp.shard_latent_cache(lat, 2, 1).is_contiguous()
    with pytest.raises(ValueError):
        tp.shard(lat, 1, 4, 2, 0)  # dimension 1 is not the branch dimension


class _OracleBackend:
    """The library's entry points as the sharded step calls them, with the
    oracle computing and gloo adding the ranks' partial products."""

    def __init__(self, rank, d_h):
        from oracle import oracle
        self.oracle = oracle
        self.rank = rank
        self.d_h = d_h
        self.calls = []

    def mlra_exchange_bytes(self, batch, heads, branches, d_c, d_h, world):
        return 4096

    def mlra_exchange_alloc(self, nbytes, with_handle=True):
        self.calls.append(("alloc", nbytes))
        return 1000 + self.rank, (bytes([self.rank]) * 64 if with_handle else None)

    def mlra_exchange_open(self, handle):
        assert len(handle) == 64 and len(set(handle)) == 1
        self.calls.append(("open", handle[0]))
        return 1000 + handle[0]

    def mlra_exchange_close(self, ptr):
        self.calls.append(("close", ptr))

    def mlra_exchange_free(self, ptr):
        self.calls.append(("free", ptr))

    def mlra_exchange_reset(self, ptr, nbytes, device=None):
        self.calls.append(("reset", ptr, nbytes))

    def mlra_decode(self, q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale, out_scale):
        out, _, st = self.oracle.decode(q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens,
                                        scale, out_scale)
        assert st == 0
        return torch.from_numpy(out)

    def mlra_up_proj_allreduce(self, out, w_uv, regions, rank, gate=None, device_status=None,
                               wait_limit_ns=None):
        assert rank == self.rank and regions.dtype == torch.int64
        y = torch.from_numpy(self.oracle.up_proj(out, w_uv, self.d_h))
        dist.all_reduce(y)
        if gate is not None:
            y = torch.from_numpy(self.oracle.gate(y.numpy(), gate))
        return y


def _sharded_worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    from branch_latent_kv_b200.inputs import WORKLOADS, make_inputs
    from oracle import oracle
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        w = WORKLOADS["tiny"].with_(batch=3, seqlen=None, page_order="permuted")
        x = make_inputs(w, seed=11, seqlens=torch.tensor([1, 200, 77], dtype=torch.int32))
        g = torch.Generator().manual_seed(12)
        gate = torch.randn((w.batch, w.heads * w.d_h), generator=g).to(torch.bfloat16)
        be = _OracleBackend(rank, w.d_h)
        ex = tp.ExchangeGroup(w.batch, w.heads, w.branches // world, w.d_c, w.d_h, device=torch.device("cpu"),
                              backend=be)
        step = tp.BranchShardedDecode(ex, backend=be)
        y = step(tp.shard_q_lat(x.q_lat, world, rank), x.q_rope, tp.shard_latent_cache(x.latent_cache, world, rank),
                 x.rope_cache, x.block_table, x.seqlens, x.scale, x.out_scale,
                 tp.shard_w_uv(x.w_uv, world, rank), gate=gate)
        regions = ex.regions.tolist()
        ex.close()
        # the unsharded step by the oracle, on every rank
        out, _, st = oracle.decode(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, x.seqlens,
                                   x.scale, x.out_scale)
        assert st == 0
        full = oracle.gate(oracle.up_proj(out, x.w_uv, w.d_h), gate)
        results[rank] = (y.numpy(), full, regions, be.calls)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_branch_shards_add_up_to_the_unsharded_step(oracle_lib, world):
    with mp.Manager() as manager:
        results = manager.dict()
        mp.spawn(_sharded_worker, args=(world, _free_port(), results), nprocs=world, join=True)
        got = dict(results)
    assert sorted(got) == list(range(world))
    for rank, (y, full, regions, calls) in got.items():
        np.testing.assert_allclose(y, full, rtol=1e-11, atol=1e-14)
        assert np.array_equal(y, got[0][0])  # one all-reduce: the same y on every rank
        assert regions == [1000 + r for r in range(world)]
        opened = sorted(c[1] for c in calls if c[0] == "open")
        assert opened == [r for r in range(world) if r != rank]
        assert sorted(c[1] for c in calls if c[0] == "close") == [1000 + r for r in opened]
        assert [c for c in calls if c[0] == "free"] == [("free", 1000 + rank)]
    # a partition that drops or repeats a branch would not reach the full step
    assert np.abs(got[0][1]).max() > 0


def _mutant_worker(rank, world, port, results):
    """Planted mistake: every rank takes rank 0's W_UV slice with its own
    latents -- the up-projection then pairs a branch's output with another
    branch's matrix, and the sum must miss the unsharded step."""
    sys.path.insert(0, ROOT)
    from branch_latent_kv_b200.inputs import WORKLOADS, make_inputs
    from oracle import oracle
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        w = WORKLOADS["tiny"].with_(batch=2)
        x = make_inputs(w, seed=13)
        be = _OracleBackend(rank, w.d_h)
        ex = tp.ExchangeGroup(w.batch, w.heads, w.branches // world, w.d_c, w.d_h, device=torch.device("cpu"),
                              backend=be)
        step = tp.BranchShardedDecode(ex, backend=be)
        wrong_w = x.w_uv[0:w.branches // world].contiguous()  # rank 0's slice on every rank
        y = step(tp.shard_q_lat(x.q_lat, world, rank), x.q_rope, tp.shard_latent_cache(x.latent_cache, world, rank),
                 x.rope_cache, x.block_table, x.seqlens, x.scale, x.out_scale, wrong_w)
        ex.close()
        out, _, _ = oracle.decode(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, x.seqlens,
                                  x.scale, x.out_scale)
        full = oracle.up_proj(out, x.w_uv, w.d_h)
        results[rank] = float(np.abs(y.numpy() - full).max() / np.abs(full).max())
    finally:
        dist.destroy_process_group()


def test_a_misassigned_w_uv_shard_is_caught(oracle_lib):
    with mp.Manager() as manager:
        results = manager.dict()
        mp.spawn(_mutant_worker, args=(2, _free_port(), results), nprocs=2, join=True)
        got = dict(results)
    assert min(got.values()) > 1e-2


def _reset_worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        be = _OracleBackend(rank, 64)
        ex = tp.ExchangeGroup(4, 8, 2, 64, 64, device=torch.device("cpu"), backend=be)
        ex.reset()   # after a timeout: each rank zeroes only its own region, then the group meets
        ex.close()
        ex.close()   # a second close does nothing
        results[rank] = be.calls
    finally:
        dist.destroy_process_group()


def test_reset_zeroes_only_the_own_region_and_close_is_idempotent():
    with mp.Manager() as manager:
        results = manager.dict()
        mp.spawn(_reset_worker, args=(2, _free_port(), results), nprocs=2, join=True)
        got = dict(results)
    for rank, calls in got.items():
        assert [c for c in calls if c[0] == "reset"] == [("reset", 1000 + rank, 4096)]
        assert [c for c in calls if c[0] == "free"] == [("free", 1000 + rank)]
        assert [c for c in calls if c[0] == "close"] == [("close", 1000 + (1 - rank))]
