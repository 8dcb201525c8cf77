"""mlra_decode_static_scratch: the decode entry point for callers that
cannot allocate device memory (plugins barred from the host application's
memory pools, runtimes whose device memory is all owned by their own
allocator, serving loops that forbid allocation after start-up).

It is called here through the C ABI directly and must match mlra_decode
(which uses a caller-provided workspace), and the fp64 oracle, within the
parity tolerance on two calls in a row with different inputs, since every
call reuses the same static scratch array.  This file runs last so that a
failure here never hides the other GPU tests, and it needs nothing from them.
"""
import ctypes

import numpy as np
import pytest
import torch

from branch_latent_kv_b200 import binding as b
from branch_latent_kv_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 5e-3
STATIC_SCRATCH_BYTES = 8 << 20


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = b.library()
    vp = ctypes.c_void_p
    lib.mlra_decode_static_scratch.argtypes = [ctypes.POINTER(b.mlra_dims), vp, vp, vp, vp, vp, vp,
                                               ctypes.c_float, ctypes.c_float, vp, vp, vp]
    lib.mlra_decode_static_scratch.restype = ctypes.c_int
    return lib


def _static_decode(lib, x, out, status):
    dims = b.decode_dims(x.q_lat, x.q_rope, x.latent_cache, x.block_table)
    stream = torch.cuda.current_stream().cuda_stream
    return lib.mlra_decode_static_scratch(
        ctypes.byref(dims), x.q_lat.data_ptr(), x.q_rope.data_ptr(), x.latent_cache.data_ptr(),
        x.rope_cache.data_ptr(), x.block_table.data_ptr(), x.seqlens.data_ptr(), x.scale,
        x.out_scale, out.data_ptr(), status.data_ptr() if status is not None else None, stream)


def _close(a, ref):
    a = a.float().cpu().double().numpy()
    r = ref.float().cpu().double().numpy()
    d = a - r
    return float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(r))


def test_two_calls_in_a_row_match_mlra_decode(lib, oracle_lib):
    cases = [
        make_inputs(WORKLOADS["decode_2p9b"].with_(batch=6, seqlen=None), seed=21, device="cuda",
                    seqlens=torch.tensor([5000, 1, 777, 128, 4097, 2500], dtype=torch.int32)),
        make_inputs(WORKLOADS["ragged"], seed=22, device="cuda"),
        # 40 heads on one 128-wide branch: two head tiles, two blocks of split
        # counters cleared before the launch
        make_inputs(WORKLOADS["tp_shard"].with_(heads=40, batch=4, seqlen=None), seed=24, device="cuda",
                    seqlens=torch.tensor([9000, 3, 2100, 640], dtype=torch.int32)),
    ]
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for x in cases:
        ref = b.mlra_decode(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table,
                            x.seqlens, x.scale, x.out_scale)
        out = torch.full_like(x.q_lat, float("nan"))
        st = _static_decode(lib, x, out, status)
        assert st == b.MLRA_OK, b.mlra_status_string(st)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        max_abs, rel = _close(out, ref)
        assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)
        want, _, st_o = oracle_lib.decode(x.q_lat.cpu(), x.q_rope.cpu(), x.latent_cache.cpu(),
                                          x.rope_cache.cpu(), x.block_table.cpu(), x.seqlens.cpu(),
                                          x.scale, x.out_scale)
        assert st_o == 0
        d = out.float().cpu().double().numpy() - want
        max_abs, rel = float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(want))
        assert max_abs <= MAX_ABS and rel <= REL_L2, ("against the oracle", max_abs, rel)


def test_device_errors_are_reported_and_cleared(lib):
    x = make_inputs(WORKLOADS["decode_2p9b"].with_(batch=3, seqlen=None), seed=23, device="cuda",
                    seqlens=torch.tensor([300, 900, 50], dtype=torch.int32))
    bad = x.seqlens.clone()
    bad[1] = 0
    x_bad = type(x)(x.workload, x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table,
                    bad, x.w_uv, x.scale, x.out_scale)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(x.q_lat)
    assert _static_decode(lib, x_bad, out, status) == b.MLRA_OK
    torch.cuda.synchronize()
    assert int(status.item()) == b.MLRA_ERR_DEVICE_BAD_SEQLEN
    assert (out[1].float() == 0).all()
    # the next call starts from a cleared error word
    assert _static_decode(lib, x, out, status) == b.MLRA_OK
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_steps_beyond_the_static_scratch_are_rejected(lib):
    dims = b.mlra_dims(1024, 16, 4, 128, 64, 64, 4, 4096)
    assert b.mlra_decode_workspace_bytes(dims) > STATIC_SCRATCH_BYTES
    ok = 1 << 20  # never dereferenced: the size check comes first
    st = lib.mlra_decode_static_scratch(ctypes.byref(dims), ok, ok, ok, ok, ok, ok, 0.1, 0.5, ok,
                                        None, None)
    assert st == b.MLRA_ERR_WORKSPACE
