"""Branch-sharded up-projection with the in-kernel cross-rank sum, on one GPU.

One device stands in for the group: all ranks' operands are stacked and one
launch computes every rank (ranks_in_launch = world), so the tiles that wait
for one another belong to one grid that is resident at once.  Each rank's
exchange region is a separate allocation on this device.  Checked: every
rank's y equals the oracle's unsharded up-projection (and the oracle's gated
one), all ranks' y are bit-identical, repeated calls and graph replays (the
call counter lives on the device) stay correct, a rank whose partner never
arrives gives up within its bound with MLRA_ERR_DEVICE_TIMEOUT, and the
whole sharded step (per-rank decode of its branches, then the fused sum)
matches the oracle's unsharded step.
"""
import numpy as np
import pytest
import torch

from branch_latent_kv_b200 import binding as b
from branch_latent_kv_b200 import tp
from branch_latent_kv_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 5e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.fixture
def regions():
    made = []

    def make(world, nbytes):
        ptrs = [b.mlra_exchange_alloc(nbytes, with_handle=False)[0] for _ in range(world)]
        made.extend(ptrs)
        return torch.tensor(ptrs, dtype=torch.int64, device="cuda")
    yield make
    torch.cuda.synchronize()
    for p in made:
        b.mlra_exchange_free(p)


def _close(gpu, ref, what):
    g = gpu.detach().float().cpu().double().numpy()
    diff = g - ref
    max_abs = float(np.abs(diff).max())
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"


def _draw(N, H, B, d_c, d_h, seed):
    g = torch.Generator().manual_seed(seed)
    out = (torch.randn((N, H, B, d_c), generator=g) / 8).to(torch.bfloat16)
    w = (torch.randn((B, d_c, H * d_h), generator=g) / np.sqrt(B * d_c)).to(torch.bfloat16)
    return out, w


def _stack(out, w, world):
    """[world, ...] per-rank shards of out_lat and W_UV, on the GPU."""
    return (torch.stack([tp.shard_q_lat(out, world, r) for r in range(world)]).cuda(),
            torch.stack([tp.shard_w_uv(w, world, r) for r in range(world)]).cuda())


@pytest.mark.parametrize("world,N,H,B,d_c,d_h", [
    (2, 16, 16, 4, 128, 128),   # the 2.9B shape over 2 ranks (2 branches each)
    (4, 16, 16, 4, 128, 128),   # one branch per rank
    (4, 5, 8, 4, 64, 64),       # ragged batch, narrow latents and heads
    (2, 80, 4, 2, 256, 128),    # two sequence tiles per head
    (1, 16, 16, 4, 128, 128),   # a group of one
])
def test_allreduce_matches_the_unsharded_oracle(oracle_lib, regions, world, N, H, B, d_c, d_h):
    nbytes = b.mlra_exchange_bytes(N, H, B // world, d_c, d_h, world)
    reg = regions(world, nbytes)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(3):  # both buffers, then the first again
        out, w = _draw(N, H, B, d_c, d_h, seed=100 + call)
        o_s, w_s = _stack(out, w, world)
        if world == 1:  # one rank: plain (unstacked) operands
            y = b.mlra_up_proj_allreduce(o_s[0], w_s[0], reg, 0, device_status=status).unsqueeze(0)
        else:
            y = b.mlra_up_proj_allreduce(o_s, w_s, reg, 0, ranks_in_launch=world, device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = oracle_lib.up_proj(out, w, d_h)
        for r in range(world):
            assert torch.equal(y[r], y[0]), f"rank {r} differs from rank 0 (call {call})"
        _close(y[0], ref, f"world {world} call {call}")


def test_allreduce_with_gate(oracle_lib, regions):
    world, N, H, B, d_c, d_h = 4, 16, 16, 4, 128, 128
    reg = regions(world, b.mlra_exchange_bytes(N, H, 1, d_c, d_h, world))
    out, w = _draw(N, H, B, d_c, d_h, seed=7)
    gate = (torch.randn((N, H * d_h), generator=torch.Generator().manual_seed(8)) * 2).to(torch.bfloat16)
    o_s, w_s = _stack(out, w, world)
    y = b.mlra_up_proj_allreduce(o_s, w_s, reg, 0, gate=gate.cuda(), ranks_in_launch=world)
    torch.cuda.synchronize()
    ref = oracle_lib.gate(oracle_lib.up_proj(out, w, d_h), gate)
    for r in range(world):
        _close(y[r], ref, f"gated rank {r}")


def test_allreduce_replays_from_a_graph(oracle_lib, regions):
    world, N, H, B, d_c, d_h = 4, 16, 16, 4, 128, 128
    reg = regions(world, b.mlra_exchange_bytes(N, H, 1, d_c, d_h, world))
    out, w = _draw(N, H, B, d_c, d_h, seed=20)
    o_s, w_s = _stack(out, w, world)
    y = torch.empty((world, N, H * d_h), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b.mlra_up_proj_allreduce(o_s, w_s, reg, 0, y=y, ranks_in_launch=world)  # eager call 0
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        b.mlra_up_proj_allreduce(o_s, w_s, reg, 0, y=y, ranks_in_launch=world)
    for call in range(4):
        out, w = _draw(N, H, B, d_c, d_h, seed=21 + call)
        a, c = _stack(out, w, world)
        o_s.copy_(a)
        w_s.copy_(c)
        g.replay()
        torch.cuda.synchronize()
        ref = oracle_lib.up_proj(out, w, d_h)
        for r in range(world):
            _close(y[r], ref, f"replay {call} rank {r}")


def test_missing_rank_times_out_with_a_status(regions):
    """Rank 0 of a group of 2 runs alone: rank 1's slice never arrives, the
    bounded wait gives up, the status says so and y is zero."""
    world, N, H, B, d_c, d_h = 2, 16, 4, 2, 128, 128
    reg = regions(world, b.mlra_exchange_bytes(N, H, B // world, d_c, d_h, world))
    out, w = _draw(N, H, B, d_c, d_h, seed=30)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = b.mlra_up_proj_allreduce(tp.shard_q_lat(out, world, 0).cuda(), tp.shard_w_uv(w, world, 0).cuda(), reg, 0,
                                 device_status=status, wait_limit_ns=5_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) == b.MLRA_ERR_DEVICE_TIMEOUT
    assert int(torch.count_nonzero(y).item()) == 0


def test_allreduce_rejects_bad_groups(regions):
    N, H, d_c, d_h = 16, 4, 128, 128
    reg = regions(2, b.mlra_exchange_bytes(N, H, 1, d_c, d_h, 2))
    out, w = _draw(N, H, 1, d_c, d_h, seed=40)
    o, ww = out.cuda(), w.cuda()
    for rank, k in [(2, 1), (-1, 1), (1, 2)]:
        with pytest.raises(b.MlraError) as e:
            b.mlra_up_proj_allreduce(torch.stack([o] * k) if k > 1 else o, torch.stack([ww] * k) if k > 1 else ww,
                                     reg, rank, ranks_in_launch=k)
        assert e.value.status == b.MLRA_ERR_INVALID_ARG
    with pytest.raises(b.MlraError):
        b.mlra_up_proj_allreduce(o, ww, reg, 0, wait_limit_ns=0)


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_decode_step_matches_the_unsharded_oracle(oracle_lib, regions, world):
    """Each rank decodes its own branches from its slice of the latent cache
    (plus the shared RoPE cache), then one launch adds all ranks' up-projected
    outputs: the result is the oracle's unsharded decode + up-projection."""
    w = WORKLOADS["decode_2p9b"].with_(batch=6, seqlen=None, page_order="permuted")
    seqlens = torch.tensor([1, 700, 129, 4000, 64, 2500], dtype=torch.int32)
    x = make_inputs(w, seed=50, seqlens=seqlens)
    dev = "cuda"
    outs = []
    for r in range(world):
        outs.append(b.mlra_decode(tp.shard_q_lat(x.q_lat, world, r).to(dev), x.q_rope.to(dev),
                                  tp.shard_latent_cache(x.latent_cache, world, r).to(dev), x.rope_cache.to(dev),
                                  x.block_table.to(dev), x.seqlens.to(dev), x.scale, x.out_scale))
    w_s = torch.stack([tp.shard_w_uv(x.w_uv, world, r) for r in range(world)]).to(dev)
    reg = regions(world, b.mlra_exchange_bytes(w.batch, w.heads, w.branches // world, w.d_c, w.d_h, world))
    y = b.mlra_up_proj_allreduce(torch.stack(outs), w_s, reg, 0, ranks_in_launch=world)
    torch.cuda.synchronize()
    out, _, st = oracle_lib.decode(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, x.seqlens,
                                   x.scale, x.out_scale)
    assert st == 0
    ref = oracle_lib.up_proj(out, x.w_uv, w.d_h)
    for r in range(world):
        assert torch.equal(y[r], y[0])
        _close(y[r], ref, f"sharded step rank {r}")
