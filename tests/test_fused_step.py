"""The whole decode step in one launch (mlra_decode_up_proj), needs a B200.

Its latent output must be the same bits as mlra_decode's (the same kernel
path), and y must match the fp64 oracle's decode followed by its
up-projection within the parity tolerance (max-abs 2e-2, rel-L2 5e-3), on
every workload shape the fused path covers, over consecutive calls (the
launch's grid-wide counter returns to zero each time).
"""
import math

import numpy as np
import pytest
import torch

from branch_latent_kv_b200 import binding as b
from branch_latent_kv_b200.inputs import Workload, WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 5e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _args(x):
    return (x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, x.seqlens, x.scale, x.out_scale)


def _close(gpu, ref):
    g = gpu.float().cpu().double().numpy()
    d = g - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(ref))


@pytest.mark.parametrize("name", ["decode_2p9b", "tiny", "tp_shard", "mla_equal_bytes", "mlra2_equal_bytes",
                                  "mlra4_equal_bytes"])
def test_fused_step_matches_oracle_and_mlra_decode(oracle_lib, name):
    w = WORKLOADS[name]
    x = make_inputs(w, device="cuda")
    out_ref = b.mlra_decode(*_args(x))
    ws = torch.zeros(b.mlra_decode_workspace_bytes(b.decode_dims(x.q_lat, x.q_rope, x.latent_cache,
                                                                  x.block_table)), dtype=torch.uint8, device="cuda")
    for _ in range(3):  # consecutive calls on one workspace
        out, y = b.mlra_decode_up_proj(*_args(x), x.w_uv, workspace=ws)
        assert torch.equal(out, out_ref)
        assert b.mlra_read_device_error(ws) == b.MLRA_OK
    lat, _, st = oracle_lib.decode(x.q_lat.cpu(), x.q_rope.cpu(), x.latent_cache.cpu(), x.rope_cache.cpu(),
                                   x.block_table.cpu(), x.seqlens.cpu(), x.scale, x.out_scale)
    assert st == 0
    y_ref = oracle_lib.up_proj(lat, x.w_uv.cpu(), w.d_h)
    max_abs, rel = _close(y, y_ref)
    assert max_abs <= MAX_ABS and rel <= REL_L2, (name, max_abs, rel)
    # the same product as the separate up-projection of the same latent output
    y2 = b.mlra_up_proj(out, x.w_uv)
    assert _close(y, y2.float().cpu().double().numpy())[1] <= 1e-2


@pytest.mark.parametrize("batch", [1, 5, 16, 33, 64])
@pytest.mark.parametrize("d_h", [64, 128])
def test_fused_step_batches_and_head_widths(oracle_lib, batch, d_h):
    """Every sequence padding of the warp MMA (1 to 4 row tiles) and both
    head widths, on ragged lengths with splits."""
    w = Workload("fused", batch=batch, heads=16, branches=4, d_c=128, d_r=64, page_size=64, d_h=d_h,
                 page_order="permuted")
    g = torch.Generator().manual_seed(batch)
    seqlens = torch.randint(1, 3000, (batch,), generator=g, dtype=torch.int32)
    x = make_inputs(w, seed=batch, seqlens=seqlens, device="cuda")
    out, y = b.mlra_decode_up_proj(*_args(x), x.w_uv)
    lat, _, st = oracle_lib.decode(x.q_lat.cpu(), x.q_rope.cpu(), x.latent_cache.cpu(), x.rope_cache.cpu(),
                                   x.block_table.cpu(), x.seqlens.cpu(), x.scale, x.out_scale)
    y_ref = oracle_lib.up_proj(lat, x.w_uv.cpu(), d_h)
    max_abs, rel = _close(y, y_ref)
    assert max_abs <= MAX_ABS and rel <= REL_L2, (batch, d_h, max_abs, rel)
    assert b.mlra_read_device_error() == b.MLRA_OK


def test_fused_step_writes_a_pinned_host_y(oracle_lib):
    x = make_inputs(WORKLOADS["decode_2p9b"].with_(seqlen=700), seed=3, device="cuda")
    h_y = torch.empty((16, 16 * 128), dtype=torch.bfloat16).pin_memory()
    _, y = b.mlra_decode_up_proj(*_args(x), x.w_uv, y=h_y)
    torch.cuda.synchronize()
    assert y is h_y
    _, y_dev = b.mlra_decode_up_proj(*_args(x), x.w_uv)
    assert torch.equal(h_y, y_dev.cpu())


def test_fused_step_rejects_what_it_does_not_cover():
    w = WORKLOADS["decode_2p9b"].with_(batch=65, seqlen=128)
    x = make_inputs(w, seed=1, device="cuda")
    with pytest.raises(b.MlraError) as e:
        b.mlra_decode_up_proj(*_args(x), x.w_uv)
    assert e.value.status == b.MLRA_ERR_UNSUPPORTED


@pytest.mark.parametrize("heads,d_h", [(32, 128), (48, 64), (128, 128)])
def test_fused_step_head_groups(oracle_lib, heads, d_h):
    """Groups of 16 heads in the attention, and in the up-projection more
    16-column blocks than CTAs (32 x 128 / 16 = 256, 128 x 128 / 16 = 1024
    blocks on 148 CTAs): each CTA takes blocks c, c + grid, ...  Two calls on
    one workspace: the grid-wide counter returns to zero."""
    w = Workload("fused_groups", batch=8, heads=heads, branches=4, d_c=128, d_r=64, page_size=64, d_h=d_h,
                 page_order="permuted")
    g = torch.Generator().manual_seed(heads)
    seqlens = torch.randint(1, 3000, (8,), generator=g, dtype=torch.int32)
    x = make_inputs(w, seed=heads, seqlens=seqlens, device="cuda")
    out_ref = b.mlra_decode(*_args(x))
    ws = torch.zeros(b.mlra_decode_workspace_bytes(b.decode_dims(x.q_lat, x.q_rope, x.latent_cache,
                                                                  x.block_table)), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        out, y = b.mlra_decode_up_proj(*_args(x), x.w_uv, workspace=ws)
        assert torch.equal(out, out_ref)
        assert b.mlra_read_device_error(ws) == b.MLRA_OK
    lat, _, st = oracle_lib.decode(x.q_lat.cpu(), x.q_rope.cpu(), x.latent_cache.cpu(), x.rope_cache.cpu(),
                                   x.block_table.cpu(), x.seqlens.cpu(), x.scale, x.out_scale)
    assert st == 0
    y_ref = oracle_lib.up_proj(lat, x.w_uv.cpu(), d_h)
    max_abs, rel = _close(y, y_ref)
    assert max_abs <= MAX_ABS and rel <= REL_L2, (heads, d_h, max_abs, rel)
