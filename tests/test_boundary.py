"""The C ABI without a GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any CUDA work.
Also checks the host-side plan statement's invariants."""
import ctypes
import os
import re

import pytest

from branch_latent_kv_b200 import binding as b
from tests import plan_model

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"MLRA_API[^;{(]*?\b(mlra_\w+)\s*\(", text, flags=re.S))
    return names


def test_library_exports_every_declared_symbol():
    lib = b.library()
    declared = _declared_symbols()
    assert {"mlra_decode", "mlra_up_proj", "mlra_decode_workspace_bytes",
            "mlra_read_device_error", "mlra_status_string", "mlra_decode_plan"} <= declared
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings():
    for code in range(8):
        s = b.mlra_status_string(code)
        assert s.startswith("MLRA_")
    assert "unknown" in b.mlra_status_string(99)


def _dims(**kw):
    base = dict(batch=16, heads=16, branches=4, d_c=128, d_r=64, page_size=64,
                max_pages_per_seq=128, num_pages=2048)
    base.update(kw)
    return b.mlra_dims(*[base[k] for k, _ in b.mlra_dims._fields_])


def test_workspace_bytes_layout():
    d = _dims()
    n = b.mlra_decode_workspace_bytes(d, 148)
    slots = 148 + 16

    def a256(x):
        return (x + 255) // 256 * 256
    cnt_off = 256                           # after the error word: split counters
    lse_off = a256(cnt_off + 4 * 65536)     # sized for the largest batch
    o_off = a256(lse_off + 4 * slots * 4 * 16)
    assert n == a256(o_off + 4 * slots * 4 * 128 * 16)  # partial rows padded to 16 heads
    # 40 heads, d_c 128: two tiles of 32 heads, rows padded to 64 heads
    n40 = b.mlra_decode_workspace_bytes(_dims(heads=40), 148)
    o40 = a256(lse_off + 4 * slots * 4 * 64)
    assert n40 == a256(o40 + 4 * slots * 4 * 128 * 64)
    # 40 heads, d_c 64 (two branches per step): three tiles of 16, rows of 48
    n40s = b.mlra_decode_workspace_bytes(_dims(heads=40, d_c=64), 148)
    o40s = a256(lse_off + 4 * slots * 4 * 48)
    assert n40s == a256(o40s + 4 * slots * 4 * 64 * 48)
    assert b.library().mlra_decode_workspace_bytes(ctypes.byref(_dims(batch=0)), 148) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), b.MLRA_ERR_INVALID_ARG),
    (dict(heads=0), b.MLRA_ERR_INVALID_ARG),
    (dict(num_pages=0), b.MLRA_ERR_INVALID_ARG),
    (dict(num_pages=2 ** 30), b.MLRA_ERR_INVALID_ARG),
    (dict(heads=129), b.MLRA_ERR_UNSUPPORTED),
    (dict(heads=128, batch=16384), b.MLRA_ERR_UNSUPPORTED),  # 4 tiles x 16384 split counters
    (dict(d_c=96), b.MLRA_ERR_UNSUPPORTED),
    (dict(d_c=256, branches=4), b.MLRA_ERR_UNSUPPORTED),
    (dict(d_r=48), b.MLRA_ERR_UNSUPPORTED),
    (dict(page_size=8), b.MLRA_ERR_UNSUPPORTED),
    (dict(page_size=256), b.MLRA_ERR_UNSUPPORTED),
])
def test_decode_rejects_bad_dims_before_any_cuda_call(kw, code):
    lib = b.library()
    fake = 1 << 20  # never dereferenced: validation fails first
    st = lib.mlra_decode(ctypes.byref(_dims(**kw)), fake, fake, fake, fake, fake, fake, 0.1, 0.5,
                         fake, fake, 1 << 30, None)
    assert st == code


def test_decode_rejects_misaligned_or_null_pointers():
    lib = b.library()
    ok = 1 << 20
    args = [ok] * 6
    for i in range(6):
        bad = list(args)
        bad[i] = ok + 2
        st = lib.mlra_decode(ctypes.byref(_dims()), *bad, 0.1, 0.5, ok, ok, 1 << 30, None)
        assert st == b.MLRA_ERR_INVALID_ARG
    st = lib.mlra_decode(ctypes.byref(_dims()), *args, 0.1, 0.5, None, ok, 1 << 30, None)
    assert st == b.MLRA_ERR_INVALID_ARG
    st = lib.mlra_decode(ctypes.byref(_dims()), *args, float("nan"), 0.5, ok, ok, 1 << 30, None)
    assert st == b.MLRA_ERR_INVALID_ARG
    st = lib.mlra_decode(ctypes.byref(_dims()), *args, 0.1, 0.5, ok, None, 1 << 30, None)
    assert st == b.MLRA_ERR_WORKSPACE
    st = lib.mlra_decode(ctypes.byref(_dims()), *args, 0.1, 0.5, ok, ok + 16, 1 << 30, None)
    assert st == b.MLRA_ERR_WORKSPACE


def test_up_proj_rejects_bad_arguments():
    lib = b.library()
    ok = 1 << 20
    assert lib.mlra_up_proj(0, 16, 4, 128, 128, ok, ok, ok, None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_up_proj(16, 16, 4, 128, 128, ok + 8, ok, ok, None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_up_proj(16, 16, 4, 128, 96, ok, ok, ok, None) == b.MLRA_ERR_UNSUPPORTED
    assert lib.mlra_up_proj(16, 16, 3, 20, 128, ok, ok, ok, None) == b.MLRA_ERR_UNSUPPORTED


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        b.mlra_decode(x, x[0], x, x[0], x[0, 0].int(), x[0, 0, 0].int(), 0.1, 0.5)


@pytest.mark.parametrize("seqlens,ctas", [
    ([8192] * 16, 148), ([1, 127, 128, 129, 0, 300], 7), ([131072] * 4, 148),
    ([5], 148), ([0, 0], 4), (list(range(1, 2000, 37)), 148), ([128 * 1000 + 1, 3], 3),
    ([128] * 300, 148), ([1, 1, 4096, 1, 1], 148), ([8192] * 16 + [0], 5),
])
def test_plan_model_covers_every_tile_once(seqlens, ctas):
    P, maxp = 64, 4096
    flat = plan_model.plan(seqlens, P, maxp, ctas)
    tiles = [plan_model.seq_tiles(L, P, maxp) for L in seqlens]
    total = sum(tiles)
    covered = []
    for c in range(ctas):
        g0, g1, n0, n1 = flat[4 * c:4 * c + 4]
        covered += list(range(g0, g1))
        if g0 < g1:
            assert 0 <= n0 <= n1 < len(seqlens)
        else:
            assert (g0, g1, n0, n1) == (0, 0, -1, -1)
    assert covered == list(range(total))
    # a CTA's tiles plus the per-sequence charge of each sequence it enters
    # fit within one chunk of cost, up to one sequence charge; the chunk is a
    # whole number of tiles, so no CTA holds more than chunk / TILE_COST tiles
    total_cost = sum(plan_model.TILE_COST * t + plan_model.SEQ_COST for t in tiles if t)
    per = max(-(-total_cost // (ctas * plan_model.TILE_COST)), 1)
    chunk = plan_model.TILE_COST * per
    for c in range(ctas):
        g0, g1, n0, n1 = flat[4 * c:4 * c + 4]
        if g0 < g1:
            cost = plan_model.TILE_COST * (g1 - g0) + plan_model.SEQ_COST * (n1 - n0)
            assert cost <= chunk + plan_model.SEQ_COST
            assert g1 - g0 <= per
    for n, t in enumerate(tiles):
        splits, first = flat[4 * ctas + 2 * n:4 * ctas + 2 * n + 2]
        if t == 0:
            assert (splits, first) == (0, -1)
        else:
            owners = [c for c in range(ctas)
                      if flat[4 * c] < flat[4 * c + 1] and flat[4 * c + 2] <= n <= flat[4 * c + 3]]
            assert owners == list(range(first, first + splits))


def test_plan_model_bounds_the_slowest_cta():
    # 16 sequences of 64 tiles over 148 CTAs: 1024 tiles need 7 per CTA at
    # least, and no CTA gets more, whether or not its range crosses into a
    # second sequence
    flat = plan_model.plan([8192] * 16, 64, 128, 148)
    counts = [flat[4 * c + 1] - flat[4 * c] for c in range(148)]
    assert max(counts) == 7 and sum(counts) == 16 * 64


def _up_grid_tiles(batch, heads, branches, d_c):
    """Output tiles of the up-projection grid: K = branches * d_c split over a
    cluster of ks CTAs (4, else 2, else 1 dividing K / 64), up to 64 sequences
    (a multiple of 16) per CTA."""
    nchunk = branches * d_c // 64
    ks = 4 if nchunk % 4 == 0 else (2 if nchunk % 2 == 0 else 1)
    nt = 64 if batch >= 64 else -(-batch // 16) * 16
    return heads * ks * -(-batch // nt)


@pytest.mark.parametrize("batch,heads,branches,d_c,d_h,world", [
    (16, 16, 1, 128, 128, 4), (80, 4, 2, 256, 128, 2), (5, 8, 2, 64, 64, 2), (16, 16, 4, 128, 128, 1),
])
def test_exchange_bytes_follow_the_documented_layout(batch, heads, branches, d_c, d_h, world):
    """epoch [tiles] u32, then data [2][world][batch][heads*d_h] u64, each
    section rounded up to 256 bytes."""
    up256 = lambda v: (v + 255) // 256 * 256
    tiles = _up_grid_tiles(batch, heads, branches, d_c)
    want = up256(tiles * 4) + up256(2 * world * batch * heads * d_h * 8)
    assert b.mlra_exchange_bytes(batch, heads, branches, d_c, d_h, world) == want


def test_exchange_and_allreduce_reject_bad_arguments_on_the_host():
    lib = b.library()
    assert lib.mlra_exchange_bytes(16, 16, 1, 128, 128, 0) == 0
    assert lib.mlra_exchange_bytes(16, 16, 1, 128, 128, 9) == 0
    assert lib.mlra_exchange_bytes(0, 16, 1, 128, 128, 2) == 0
    assert lib.mlra_exchange_bytes(16, 16, 1, 96, 128, 2) == 0  # K not a multiple of 64
    p = ctypes.c_void_p()
    assert lib.mlra_exchange_alloc(0, ctypes.byref(p), None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_exchange_alloc(4096, None, None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_exchange_open(None, ctypes.byref(p)) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_exchange_close(None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_exchange_free(None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_exchange_reset(None, 4096, None) == b.MLRA_ERR_INVALID_ARG
    ok = 1 << 20

    def allreduce(batch=16, heads=16, branches=1, d_c=128, d_h=128, out=ok, w=ok, gate=None, y=ok,
                  regions=ok, world=4, rank=0, k=1, status=None, limit=10**9):
        return lib.mlra_up_proj_allreduce(batch, heads, branches, d_c, d_h, out, w, gate, y, regions, world,
                                          rank, k, status, limit, None)
    for kw in [dict(world=0), dict(world=9), dict(rank=4), dict(rank=-1), dict(rank=3, k=2), dict(k=0),
               dict(out=ok + 8), dict(regions=None), dict(gate=ok + 1), dict(status=ok + 2), dict(limit=0),
               dict(batch=0)]:
        assert allreduce(**kw) == b.MLRA_ERR_INVALID_ARG, kw
    assert allreduce(d_c=96) == b.MLRA_ERR_UNSUPPORTED      # K = 96
    assert allreduce(d_h=96) == b.MLRA_ERR_UNSUPPORTED


def test_copy_ranges_rejects_bad_arguments_on_the_host():
    lib = b.library()
    ok = 1 << 20
    arr = lambda *v: (ctypes.c_void_p * len(v))(*v)
    sizes = lambda *v: (ctypes.c_uint64 * len(v))(*v)
    assert lib.mlra_copy_ranges(0, arr(ok), arr(ok + 4096), sizes(16), None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_copy_ranges(9, arr(*[ok] * 9), arr(*[ok] * 9), sizes(*[16] * 9), None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_copy_ranges(1, None, arr(ok), sizes(16), None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_copy_ranges(1, arr(ok + 4), arr(ok + 4096), sizes(16), None) == b.MLRA_ERR_INVALID_ARG
    assert lib.mlra_copy_ranges(1, arr(ok), arr(ok + 4104), sizes(16), None) == b.MLRA_ERR_INVALID_ARG
