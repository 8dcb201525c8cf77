"""GPU path against the fp64 oracle, through the C ABI (needs a B200).

Tolerance (bf16 inputs, fp32 accumulation, bf16 output): max-abs error
<= 2e-2 and relative L2 error <= 5e-3 against the oracle.  Paging and index
bookkeeping are bit-exact: page permutations give identical bits, length-1
sequences return out_scale * c_b[0] exactly, the plan matches its CPU
statement exactly.
"""
import math

import numpy as np
import pytest
import torch

from branch_latent_kv_b200 import binding as b
from branch_latent_kv_b200.inputs import Workload, WORKLOADS, make_inputs
from tests import plan_model

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 5e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def _errors(gpu, ref, seq_ids=None):
    g = gpu.detach().float().cpu().double().numpy()
    if seq_ids is not None:
        g, ref = g[seq_ids], ref[seq_ids]
    diff = g - ref
    return float(np.abs(diff).max()), float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))


def _assert_close(gpu, ref, seq_ids=None, what=""):
    max_abs, rel = _errors(gpu, ref, seq_ids)
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


IMPLS = {"tc": b.mlra_decode, "simt": b.mlra_decode_simt}


def _run(x, impl="tc", **kw):
    return IMPLS[impl](x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, x.seqlens,
                       x.scale, x.out_scale, **kw)


def _oracle(oracle_lib, x, seq_ids=None):
    out, lse, status = oracle_lib.decode(x.q_lat.cpu(), x.q_rope.cpu(), x.latent_cache.cpu(),
                                         x.rope_cache.cpu(), x.block_table.cpu(), x.seqlens.cpu(),
                                         x.scale, x.out_scale, seq_ids=seq_ids)
    return out, status


def _score_gain(w, target_std):
    """Query gain that makes the score standard deviation about target_std."""
    return target_std / (w.scale * math.sqrt(1.0 / w.d_c + 1.0 / w.d_r))


RAGGED = torch.tensor([1, 200, 777, 128, 129, 64, 1000, 255], dtype=torch.int32)


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("name", sorted(WORKLOADS))
@pytest.mark.parametrize("peaked", [False, True])
def test_small_cases_match_oracle(oracle_lib, name, peaked, impl):
    """Every workload's model shape on short ragged sequences (several tiles,
    partial pages, NaN in every unused pool slot)."""
    w = WORKLOADS[name]
    if impl == "simt" and w.heads * w.branches * w.d_c > 16384:
        pytest.skip("queries and outputs exceed the CUDA-core kernel's shared memory")
    n = min(w.batch, 4)
    w = w.with_(batch=n, seqlen=None, seqlen_range=None, page_order="permuted")
    seqlens = RAGGED[:n].clone()
    if name == "tiny":
        seqlens = torch.tensor([256], dtype=torch.int32)
    gain = _score_gain(w, 4.0) if peaked else 1.0
    x = make_inputs(w, seed=3, q_gain=gain, slack_pages=5, nan_fill_unused=True,
                    seqlens=seqlens).to("cuda")
    out = _run(x, impl)
    ref, status = _oracle(oracle_lib, x)
    assert status == 0
    assert torch.isfinite(out.float()).all()
    _assert_close(out, ref, what=f"{name} peaked={peaked} {impl}")


SHAPES = [(2, 64), (4, 64), (1, 128), (2, 128), (4, 128), (1, 256), (2, 256), (1, 512)]


@pytest.mark.parametrize("branches,d_c", SHAPES)
@pytest.mark.parametrize("d_r", [32, 64])
@pytest.mark.parametrize("page_size", [16, 64, 128])
def test_every_supported_shape_matches_oracle(oracle_lib, branches, d_c, d_r, page_size):
    """Every (branches, d_c) the tensor-core kernel implements, both RoPE
    widths and three page sizes (the kernel's ring depths and slot counts
    differ per shape): short ragged sequences across several tiles, splits
    and a partial last page, 12 heads (padding to the MMA's 16), scores
    peaked enough to take the lazy-rescale path."""
    w = Workload("shape", batch=5, heads=12, branches=branches, d_c=d_c, d_r=d_r,
                 page_size=page_size, page_order="permuted")
    seqlens = torch.tensor([1000, 1, 640, 129, 2047], dtype=torch.int32)
    x = make_inputs(w, seed=11, q_gain=_score_gain(w, 4.0), slack_pages=3, nan_fill_unused=True,
                    seqlens=seqlens).to("cuda")
    out = _run(x)
    ref, status = _oracle(oracle_lib, x)
    assert status == 0
    assert torch.isfinite(out.float()).all()
    _assert_close(out, ref, what=f"B={branches} d_c={d_c} d_r={d_r} P={page_size}")


@pytest.mark.parametrize("branches,d_c", SHAPES)
@pytest.mark.parametrize("d_r", [32, 64])
def test_every_supported_shape_with_40_heads(oracle_lib, branches, d_c, d_r):
    """Every (branches, d_c) at 40 heads: two tiles of 32 heads (the second
    with 8) for d_c >= 128, three groups of 16 (the third with 8) for
    d_c = 64; ragged lengths with splits in every group, peaked scores."""
    import os
    oracle_lib.set_num_threads(len(os.sched_getaffinity(0)))
    w = Workload("shape40", batch=5, heads=40, branches=branches, d_c=d_c, d_r=d_r, page_size=64,
                 page_order="permuted")
    seqlens = torch.tensor([3000, 1, 640, 129, 2047], dtype=torch.int32)
    x = make_inputs(w, seed=13, q_gain=_score_gain(w, 4.0), slack_pages=3, nan_fill_unused=True,
                    seqlens=seqlens).to("cuda")
    out = _run(x)
    ref, status = _oracle(oracle_lib, x)
    assert status == 0
    assert torch.isfinite(out.float()).all()
    _assert_close(out, ref, what=f"H=40 B={branches} d_c={d_c} d_r={d_r}")


@pytest.mark.parametrize("heads", [1, 5, 16, 17, 32, 64, 128])
@pytest.mark.parametrize("page_size", [32, 128])
def test_head_counts_and_page_sizes(oracle_lib, heads, page_size):
    """Head counts below the MMA's 16 (queries padded by the TMA's zero
    fill), above it (groups of 16 heads, the last one partial for 17), and
    the page sizes the other tests leave out, on the 2.9B shape."""
    w = Workload("heads", batch=3, heads=heads, branches=4, d_c=128, d_r=64, page_size=page_size,
                 page_order="permuted")
    seqlens = torch.tensor([513, 33, 4097], dtype=torch.int32)
    x = make_inputs(w, seed=12, q_gain=_score_gain(w, 3.0), slack_pages=2, nan_fill_unused=True,
                    seqlens=seqlens).to("cuda")
    out = _run(x)
    ref, status = _oracle(oracle_lib, x)
    assert status == 0
    _assert_close(out, ref, what=f"H={heads} P={page_size}")


@pytest.mark.parametrize("impl", sorted(IMPLS))
def test_tiny_workload_exact_recipe(oracle_lib, impl):
    x = make_inputs(WORKLOADS["tiny"]).to("cuda")
    out = _run(x, impl)
    ref, status = _oracle(oracle_lib, x)
    assert status == 0
    _assert_close(out, ref, what="tiny")


FULL_SIZE = ["decode_2p9b", "long_context", "ragged", "mla_equal_bytes", "mlra4_equal_bytes",
             "tp_shard", "mlra2_equal_bytes", "context_2m", "heads_64"]


@pytest.mark.parametrize("name", FULL_SIZE)
def test_full_size_whole_outputs(oracle_lib, parity_report, name):
    """Every full-size workload in the launch configuration the benchmark
    times (one CTA per SM, the in-kernel split merge), compared with the
    oracle on EVERY sequence, head, branch and latent column.  The oracle runs
    on all host cores; its inputs are the GPU's own bf16 tensors copied back."""
    import os
    oracle_lib.set_num_threads(len(os.sched_getaffinity(0)))
    w = WORKLOADS[name]
    x = make_inputs(w, device="cuda")
    out = _run(x)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    ref, status = _oracle(oracle_lib, x)
    assert status == 0
    assert np.isfinite(ref).all()
    max_abs, rel = _errors(out, ref)
    parity_report.append((name, x.q_lat.shape[0], max_abs, rel, max_abs / float(np.abs(ref).max())))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{name}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("name", ["decode_2p9b", "tiny", "mla_equal_bytes"])
def test_length_one_is_bit_exact(impl, name):
    w = WORKLOADS[name].with_(batch=6, seqlen=1, page_order="permuted")
    x = make_inputs(w, seed=5, q_gain=40.0, slack_pages=3, nan_fill_unused=True).to("cuda")
    out = _run(x, impl)
    pages = x.block_table[:, 0].long()
    want = (x.latent_cache[pages, 0].float() * x.out_scale).to(torch.bfloat16)  # [N, B, d_c]
    assert torch.equal(out, want[:, None].expand_as(out))


def test_page_permutation_gives_identical_bits():
    w = WORKLOADS["decode_2p9b"].with_(batch=5, seqlen=None)
    seqlens = torch.tensor([3000, 1, 640, 129, 2049], dtype=torch.int32)
    x = make_inputs(w, seed=9, seqlens=seqlens, slack_pages=7).to("cuda")
    perm = torch.randperm(x.latent_cache.shape[0], generator=torch.Generator().manual_seed(1)).cuda()
    lat2 = torch.empty_like(x.latent_cache)
    rope2 = torch.empty_like(x.rope_cache)
    lat2[perm] = x.latent_cache
    rope2[perm] = x.rope_cache
    bt2 = torch.where(x.block_table >= 0, perm[x.block_table.long().clamp(min=0)].int(), x.block_table)
    out1 = _run(x)
    out2 = b.mlra_decode(x.q_lat, x.q_rope, lat2, rope2, bt2.contiguous(), x.seqlens, x.scale,
                         x.out_scale)
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("name", ["decode_2p9b", "ragged", "mla_equal_bytes", "tp_shard"])
def test_tensor_core_and_cuda_core_paths_agree(name):
    """Two independent GPU statements of the kernel agree within the tolerance."""
    w = WORKLOADS[name].with_(batch=6, seqlen=None, seqlen_range=None)
    seqlens = torch.tensor([5000, 1, 777, 128, 4097, 2500], dtype=torch.int32)
    x = make_inputs(w, seed=12, seqlens=seqlens, device="cuda")
    a, c = _run(x, "tc"), _run(x, "simt")
    ref = c.double().cpu().numpy()
    _assert_close(a, ref, what=f"tc vs simt {name}")


def test_repeat_calls_are_deterministic():
    x = make_inputs(WORKLOADS["ragged"].with_(batch=8), seed=2, device="cuda")
    a = _run(x).clone()
    for _ in range(3):
        assert torch.equal(_run(x), a)


def _split_counters(ws, dims):
    """The per-sequence split counters: int32 from byte 256 of the workspace
    (after the error word), one per sequence and head tile (16 heads, or 32
    when there are more and d_c >= 128)."""
    tile = 16 if dims.heads <= 16 or dims.d_c < 128 else 32
    groups = (dims.heads + tile - 1) // tile
    return ws[256:256 + 4 * dims.batch * groups].view(torch.int32)


@pytest.mark.parametrize("seqlens", [[131072], [9000, 1, 300, 130000, 128, 129], [64] * 300])
def test_split_merge_leaves_counters_at_zero(oracle_lib, seqlens):
    w = WORKLOADS["decode_2p9b"].with_(batch=len(seqlens), seqlen=None)
    x = make_inputs(w, seed=7, seqlens=torch.tensor(seqlens, dtype=torch.int32),
                    max_pages_per_seq=max(seqlens) // w.page_size + 1).to("cuda")
    dims = b.decode_dims(x.q_lat, x.q_rope, x.latent_cache, x.block_table)
    ws = torch.zeros(b.mlra_decode_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    first = _run(x, workspace=ws).clone()
    assert (_split_counters(ws, dims) == 0).all()
    assert torch.equal(_run(x, workspace=ws), first)
    assert b.mlra_read_device_error(ws) == b.MLRA_OK
    ref, _ = _oracle(oracle_lib, x)
    _assert_close(first, ref, what=f"merge {seqlens[:4]}")


@pytest.mark.parametrize("heads", [40, 48, 128])
def test_head_groups_split_and_merge(oracle_lib, heads):
    """More heads than the MMA's 16: groups of 16 heads on equal parts of the
    grid, each with its own splits, partial slots and split counters (the last
    group partial for 40).  Ragged lengths long enough that sequences split
    over several CTAs of every group; a second call on the same workspace
    gives the same bits, and every counter is back at zero."""
    import os
    oracle_lib.set_num_threads(len(os.sched_getaffinity(0)))
    w = Workload("groups", batch=20, heads=heads, branches=2, d_c=128, d_r=64, page_size=64,
                 page_order="permuted")
    g = torch.Generator().manual_seed(heads)
    seqlens = torch.randint(1, 9000, (20,), generator=g, dtype=torch.int32)
    x = make_inputs(w, seed=heads, q_gain=_score_gain(w, 3.0), seqlens=seqlens, slack_pages=3,
                    nan_fill_unused=True).to("cuda")
    dims = b.decode_dims(x.q_lat, x.q_rope, x.latent_cache, x.block_table)
    ws = torch.zeros(b.mlra_decode_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    first = _run(x, workspace=ws).clone()
    assert (_split_counters(ws, dims) == 0).all()
    assert torch.equal(_run(x, workspace=ws), first)
    assert b.mlra_read_device_error(ws) == b.MLRA_OK
    ref, status = _oracle(oracle_lib, x)
    assert status == 0
    _assert_close(first, ref, what=f"H={heads}")


def test_reading_a_timeout_clears_the_split_counters(oracle_lib):
    """A kernel that gives up on a bounded wait may leave split counters set.
    Planted on the host (no GPU wait is made to expire): the error word holds
    MLRA_ERR_DEVICE_TIMEOUT and every counter a stale count.  Reading the
    error reports the timeout and clears the counters, and the next call on
    the same workspace matches the oracle."""
    w = WORKLOADS["decode_2p9b"].with_(batch=6, seqlen=None)
    x = make_inputs(w, seed=31, seqlens=torch.tensor([9000, 130, 4000, 1, 20000, 700], dtype=torch.int32),
                    device="cuda")
    dims = b.decode_dims(x.q_lat, x.q_rope, x.latent_cache, x.block_table)
    ws = torch.zeros(b.mlra_decode_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    ws[:4].view(torch.int32)[0] = b.MLRA_ERR_DEVICE_TIMEOUT
    _split_counters(ws, dims).fill_(3)
    ws[256 + 4 * 65535:256 + 4 * 65536].view(torch.int32)[0] = 9  # the region's last word
    assert b.mlra_read_device_error(ws) == b.MLRA_ERR_DEVICE_TIMEOUT
    assert (ws[:256 + 4 * 65536] == 0).all()
    out = _run(x, workspace=ws)
    assert b.mlra_read_device_error(ws) == b.MLRA_OK
    ref, _ = _oracle(oracle_lib, x)
    _assert_close(out, ref, what="after a cleared timeout")


def test_invalid_sequences_are_zeroed_and_reported(oracle_lib):
    w = WORKLOADS["decode_2p9b"].with_(batch=4, seqlen=None)
    seqlens = torch.tensor([500, 700, 900, 300], dtype=torch.int32)
    x = make_inputs(w, seed=4, seqlens=seqlens).to("cuda")
    ws = torch.zeros(b.mlra_decode_workspace_bytes(b.decode_dims(x.q_lat, x.q_rope, x.latent_cache,
                                                                 x.block_table)),
                     dtype=torch.uint8, device="cuda")
    ref, _ = _oracle(oracle_lib, x)
    bad_len = x.seqlens.clone()
    bad_len[1] = 0
    out = b.mlra_decode(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, bad_len,
                        x.scale, x.out_scale, workspace=ws)
    assert b.mlra_read_device_error(ws) == b.MLRA_ERR_DEVICE_BAD_SEQLEN
    assert (out[1].float() == 0).all()
    _assert_close(out, ref, seq_ids=[0, 2, 3], what="others unaffected")
    assert b.mlra_read_device_error(ws) == b.MLRA_OK  # reading cleared it

    bad_page = x.block_table.clone()
    bad_page[2, 3] = x.latent_cache.shape[0]
    out = b.mlra_decode(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, bad_page, x.seqlens,
                        x.scale, x.out_scale, workspace=ws)
    assert b.mlra_read_device_error(ws) == b.MLRA_ERR_DEVICE_BAD_INDEX
    assert (out[2].float() == 0).all()
    _assert_close(out, ref, seq_ids=[0, 1, 3], what="others unaffected")

    too_long = x.seqlens.clone()
    too_long[3] = x.block_table.shape[1] * w.page_size + 1
    b.mlra_decode(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, too_long,
                  x.scale, x.out_scale, workspace=ws)
    assert b.mlra_read_device_error(ws) == b.MLRA_ERR_DEVICE_BAD_SEQLEN


@pytest.mark.parametrize("seqlens,ctas", [
    ([8192] * 16, 148), ([1, 127, 128, 129, 0, 300], 7), ([131072] * 4, 148), ([5], 148),
    (list(range(1, 5000, 97)), 148), ([0, 3, 0], 2),
])
def test_plan_is_bit_exact(seqlens, ctas):
    P, maxp = 64, 2048
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    got = b.mlra_decode_plan(sl, P, maxp, ctas).cpu().tolist()
    assert got == plan_model.plan(seqlens, P, maxp, ctas)


def test_up_proj_matches_oracle(oracle_lib):
    w = WORKLOADS["decode_2p9b"]
    x = make_inputs(w.with_(seqlen=300), seed=6).to("cuda")
    out_lat = _run(x)
    y = b.mlra_up_proj(out_lat, x.w_uv)
    y_ref = oracle_lib.up_proj(out_lat.cpu(), x.w_uv.cpu(), w.d_h)
    g = y.float().cpu().double().numpy()
    assert np.abs(g - y_ref).max() <= MAX_ABS
    assert np.linalg.norm(g - y_ref) / np.linalg.norm(y_ref) <= REL_L2
    # end to end: fp64 decode -> fp64 up-projection
    ref_lat, _ = _oracle(oracle_lib, x)
    y_ref2 = oracle_lib.up_proj(ref_lat, x.w_uv.cpu(), w.d_h)
    assert np.linalg.norm(g - y_ref2) / np.linalg.norm(y_ref2) <= REL_L2


@pytest.mark.parametrize("name", ["decode_2p9b", "mlra2_equal_bytes", "tiny"])
def test_gated_up_proj_matches_oracle(oracle_lib, name):
    """The fused output gate: y = sigmoid(gate) * up-projection, against the
    oracle's up-projection followed by its gate."""
    w = WORKLOADS[name]
    x = make_inputs(w.with_(batch=min(w.batch, 16), seqlen=300, seqlen_range=None), seed=8).to("cuda")
    out_lat = _run(x)
    gen = torch.Generator(device="cpu").manual_seed(9)
    gate = (torch.randn((x.q_lat.shape[0], x.q_lat.shape[1] * w.d_h), generator=gen) * 3).to(torch.bfloat16)
    y = b.mlra_up_proj_gated(out_lat, x.w_uv, gate.to("cuda"))
    ref = oracle_lib.gate(oracle_lib.up_proj(out_lat.cpu(), x.w_uv.cpu(), w.d_h), gate)
    g = y.float().cpu().double().numpy()
    assert np.abs(g - ref).max() <= MAX_ABS
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= REL_L2
    # gate logits of zero halve the ungated result exactly
    y0 = b.mlra_up_proj_gated(out_lat, x.w_uv, torch.zeros_like(gate, device="cuda"))
    y1 = b.mlra_up_proj(out_lat, x.w_uv)
    assert torch.equal(y0.float(), (y1.float() / 2).to(torch.bfloat16).float()) or \
        (y0.float() - y1.float() / 2).abs().max() <= 2 ** -8 * y1.float().abs().max()


@pytest.mark.parametrize("batch", [1, 5, 16, 33, 300])
def test_up_proj_batches(oracle_lib, batch):
    torch.manual_seed(batch)
    H, B, d_c, d_h = 16, 4, 128, 128
    out_lat = (torch.randn(batch, H, B, d_c) / 10).to(torch.bfloat16).cuda()
    w_uv = (torch.randn(B, d_c, H * d_h) / math.sqrt(B * d_c)).to(torch.bfloat16).cuda()
    y = b.mlra_up_proj(out_lat, w_uv)
    y_ref = oracle_lib.up_proj(out_lat.cpu(), w_uv.cpu(), d_h)
    g = y.float().cpu().double().numpy()
    assert np.linalg.norm(g - y_ref) / np.linalg.norm(y_ref) <= REL_L2
