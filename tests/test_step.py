"""DecodeStep: a decode step bound to fixed buffers and replayed from a CUDA
graph gives the same bits as the eager calls it stands for (the fused
decode + up-projection launch for batches up to 64), including its host
copies."""
import pytest
import torch

from branch_latent_kv_b200 import binding as b
from branch_latent_kv_b200.inputs import WORKLOADS, make_inputs
from branch_latent_kv_b200.step import DecodeStep

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _eager(x, q_lat=None):
    """The eager step: the fused launch (the batches here are <= 64)."""
    return b.mlra_decode_up_proj(q_lat if q_lat is not None else x.q_lat, x.q_rope, x.latent_cache,
                                 x.rope_cache, x.block_table, x.seqlens, x.scale, x.out_scale, x.w_uv)


def test_replay_matches_eager_calls():
    x = make_inputs(WORKLOADS["ragged"].with_(batch=6), seed=5).to("cuda")
    out_ref, y_ref = _eager(x)
    step = DecodeStep(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, x.seqlens,
                      x.scale, x.out_scale, w_uv=x.w_uv)
    for _ in range(3):
        y = step()
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref)
        assert torch.equal(step.out, out_ref)
    # the same latent output as mlra_decode, and the same up-projection as
    # mlra_up_proj of it within the parity tolerance
    assert torch.equal(out_ref, b.mlra_decode(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table,
                                              x.seqlens, x.scale, x.out_scale))
    y2 = b.mlra_up_proj(out_ref, x.w_uv).float()
    assert ((y.float() - y2).norm() / y2.norm()).item() <= 5e-3


def test_host_copies_follow_the_pinned_buffers():
    x = make_inputs(WORKLOADS["decode_2p9b"].with_(batch=4, seqlen=2000), seed=6).to("cuda")
    h_in = {"q_lat": x.q_lat.cpu().pin_memory(), "seqlens": x.seqlens.cpu().pin_memory()}
    d_q, d_sl = torch.empty_like(x.q_lat), x.seqlens.clone()
    h_out = torch.empty((4, x.q_lat.shape[1] * x.workload.d_h), dtype=torch.bfloat16).pin_memory()
    step = DecodeStep(d_q, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, d_sl, x.scale,
                      x.out_scale, w_uv=x.w_uv, host_inputs=h_in, host_output=h_out)
    assert step.h2d_bytes() == x.q_lat.numel() * 2 + 4 * 4
    assert step.d2h_bytes() == h_out.numel() * 2
    step()
    torch.cuda.synchronize()
    _, y_ref = _eager(x)
    assert torch.equal(h_out, y_ref.cpu())
    # new queries written into the pinned buffer reach the next step
    q2 = (x.q_lat.float() * -1.5).to(torch.bfloat16)
    h_in["q_lat"].copy_(q2.cpu())
    step()
    torch.cuda.synchronize()
    _, y2 = _eager(x, q_lat=q2)
    assert torch.equal(h_out, y2.cpu())


def test_rejects_unpinned_host_buffers():
    x = make_inputs(WORKLOADS["tiny"]).to("cuda")
    with pytest.raises(ValueError):
        DecodeStep(x.q_lat, x.q_rope, x.latent_cache, x.rope_cache, x.block_table, x.seqlens,
                   x.scale, x.out_scale, host_inputs={"q_lat": x.q_lat.cpu()})


def test_host_output_without_up_projection():
    """Decode only: the latent output is copied to the pinned host buffer."""
    x = make_inputs(WORKLOADS["decode_2p9b"].with_(batch=3, seqlen=700), seed=7).to("cuda")
    h_in = {"q_lat": x.q_lat.cpu().pin_memory(), "q_rope": x.q_rope.cpu().pin_memory(),
            "block_table": x.block_table.cpu().pin_memory(), "seqlens": x.seqlens.cpu().pin_memory()}
    d_in = {k: torch.empty_like(v, device="cuda") for k, v in h_in.items()}
    h_out = torch.empty(x.q_lat.shape, dtype=torch.bfloat16).pin_memory()
    step = DecodeStep(d_in["q_lat"], d_in["q_rope"], x.latent_cache, x.rope_cache, d_in["block_table"],
                      d_in["seqlens"], x.scale, x.out_scale, host_inputs=h_in, host_output=h_out)
    step()
    torch.cuda.synchronize()
    out_ref, _ = _eager(x)
    assert torch.equal(h_out, out_ref.cpu())
