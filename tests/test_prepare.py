"""The decode pre-step on the GPU against the oracle: absorbed queries,
rotated RoPE queries, the appended cache rows (latents bit for bit, the
rotated key within tolerance), every other cache row untouched, the error
codes of bad sequences, and the pre-step feeding mlra_decode."""
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


def _close(gpu, ref, what):
    g = gpu.detach().float().cpu().double().numpy()
    diff = g - ref
    max_abs = float(np.abs(diff).max())
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"


def _pre_inputs(x, d_h, seed):
    """q_c, q_r, w_uk, c_new, kr_new drawn like the workload's own tensors:
    N(0,1)/sqrt(last dim), W_UK with fan-in d_h, rounded to bf16."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    N, H, B, d_c = x.q_lat.shape
    d_r = x.q_rope.shape[2]

    def draw(shape, fan):
        return (torch.randn(shape, generator=g) / math.sqrt(fan)).to(torch.bfloat16)
    return (draw((N, H, d_h), d_h), draw((N, H, d_r), d_r), draw((B, H, d_h, d_c), d_h),
            draw((N, B, d_c), d_c), draw((N, d_r), d_r))


@pytest.mark.parametrize("name,seqlens", [
    ("decode_2p9b", None), ("tiny", None), ("mla_equal_bytes", [1, 64, 65, 16384] * 8),
    ("ragged", None), ("odd", None), ("far", [2_000_001, 3]),
])
def test_prepare_matches_oracle(oracle_lib, name, seqlens):
    """The workloads' shapes, plus one ("odd") whose head dimension is not a
    multiple of the MMA's K = 16 (d_h = 24: zero-padded), whose d_c = 96
    leaves a half column block, and whose 70 sequences take two chunks of
    the absorption's 64 (the second a partial 16-row tile), and one ("far")
    whose new token sits at position 2,000,000."""
    w = WORKLOADS.get(name)
    if name == "odd":
        w = Workload("odd", batch=70, heads=3, branches=2, d_c=96, d_r=32, page_size=16, seqlen=100, d_h=24,
                     page_order="permuted")
    if name == "far":  # a position of two million: the angle's reduction to a fraction of a turn
        w = Workload("far", batch=2, heads=4, branches=1, d_c=8, d_r=64, page_size=128, d_h=64)
    if name == "decode_2p9b":
        w = w.with_(seqlen=3000)
    if name == "ragged":
        w = w.with_(batch=12, seqlen_range=(1, 40000))
    sl = torch.tensor(seqlens, dtype=torch.int32) if seqlens else None
    x = make_inputs(w, seed=4, seqlens=sl, with_w_uv=False)
    d_h = w.d_h
    q_c, q_r, w_uk, c_new, kr_new = _pre_inputs(x, d_h, seed=5)
    dev = "cuda"
    lat, rope = x.latent_cache.to(dev), x.rope_cache.to(dev)
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    q_lat, q_rope = b.mlra_prepare(q_c.to(dev), q_r.to(dev), w_uk.to(dev), c_new.to(dev), kr_new.to(dev),
                                   x.seqlens.to(dev), x.block_table.to(dev), lat, rope,
                                   device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_lat, ref_rope, kr_rot, dest, st = oracle_lib.prepare(q_c, q_r, w_uk, kr_new, x.seqlens,
                                                             x.block_table, x.latent_cache.shape[0],
                                                             w.page_size)
    assert st == 0
    _close(q_lat, ref_lat, "q_lat")
    _close(q_rope, ref_rope, "q_rope")
    lat_c, rope_c = lat.cpu(), rope.cpu()
    written = np.zeros(lat_c.shape[:2], dtype=bool)
    for n in range(x.q_lat.shape[0]):
        page, slot = (int(v) for v in dest[n])
        assert torch.equal(lat_c[page, slot], c_new[n])  # the latents are copied bit for bit
        written[page, slot] = True
    rows = torch.from_numpy(written)
    _close(rope_c[rows], kr_rot[np.lexsort((dest[:, 1], dest[:, 0]))], "rotated key")
    # every other row untouched
    assert torch.equal(lat_c[~rows], x.latent_cache[~rows])
    assert torch.equal(rope_c[~rows], x.rope_cache[~rows])


def test_prepare_reports_bad_sequences_and_skips_their_rows():
    w = WORKLOADS["decode_2p9b"].with_(batch=4, seqlen=200)
    x = make_inputs(w, seed=6, with_w_uv=False)
    q_c, q_r, w_uk, c_new, kr_new = _pre_inputs(x, w.d_h, seed=7)
    dev = "cuda"
    args = [t.to(dev) for t in (q_c, q_r, w_uk, c_new, kr_new)]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for seqlens, table_fix, code in [([200, 0, 200, 200], None, b.MLRA_ERR_DEVICE_BAD_SEQLEN),
                                     ([200, 200, 200, 4096], None, b.MLRA_ERR_DEVICE_BAD_SEQLEN),
                                     ([200, 200, 200, 200], (2, 3), b.MLRA_ERR_DEVICE_BAD_INDEX)]:
        lat, rope = x.latent_cache.to(dev), x.rope_cache.to(dev)
        table = x.block_table.clone()
        if table_fix is not None:
            table[table_fix] = x.latent_cache.shape[0]  # outside the pool
        b.mlra_prepare(*args, torch.tensor(seqlens, dtype=torch.int32, device=dev), table.to(dev), lat, rope,
                       device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == code
        bad = [i for i, L in enumerate(seqlens) if L < 1 or L > table.shape[1] * w.page_size]
        if table_fix is not None:
            bad.append(table_fix[0])
        good_rows = 0
        for n in range(4):
            p = seqlens[n] - 1
            if n in bad:
                continue
            page = int(table[n, p // w.page_size])
            assert torch.equal(lat[page, p % w.page_size].cpu(), c_new[n])
            good_rows += 1
        changed = (lat.cpu() != x.latent_cache).any(dim=-1).any(dim=-1).sum().item()
        assert changed == good_rows  # nothing written for the bad sequences


def test_prepare_then_decode_matches_oracle(oracle_lib):
    """The pre-step's outputs feed mlra_decode: the GPU chain equals the
    oracle chain (oracle prepare, append by its targets, oracle decode)."""
    w = WORKLOADS["decode_2p9b"].with_(batch=6, seqlen=None, page_order="permuted")
    seqlens = torch.tensor([1, 700, 129, 4000, 64, 2500], dtype=torch.int32)
    x = make_inputs(w, seed=8, seqlens=seqlens, with_w_uv=False)
    q_c, q_r, w_uk, c_new, kr_new = _pre_inputs(x, w.d_h, seed=9)
    dev = "cuda"
    lat, rope = x.latent_cache.to(dev), x.rope_cache.to(dev)
    q_lat, q_rope = b.mlra_prepare(q_c.to(dev), q_r.to(dev), w_uk.to(dev), c_new.to(dev), kr_new.to(dev),
                                   x.seqlens.to(dev), x.block_table.to(dev), lat, rope)
    out = b.mlra_decode(q_lat, q_rope, lat, rope, x.block_table.to(dev), x.seqlens.to(dev), x.scale,
                        x.out_scale)
    torch.cuda.synchronize()
    ref_lat, ref_rope, kr_rot, dest, st = oracle_lib.prepare(q_c, q_r, w_uk, kr_new, x.seqlens,
                                                             x.block_table, x.latent_cache.shape[0],
                                                             w.page_size)
    assert st == 0
    pool = x.latent_cache.double().numpy().copy()
    rpool = x.rope_cache.double().numpy().copy()
    for n in range(6):
        pool[dest[n, 0], dest[n, 1]] = c_new[n].double().numpy()
        rpool[dest[n, 0], dest[n, 1]] = kr_rot[n]
    ref, _, st = oracle_lib.decode(ref_lat, ref_rope, pool, rpool, x.block_table, x.seqlens, x.scale,
                                   x.out_scale)
    assert st == 0
    _close(out, ref, "prepare -> decode")
