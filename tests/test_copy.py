"""mlra_copy_ranges (one launch of SM loads and stores over several byte
ranges, host or device) and the up-projection writing its result straight
into pinned host memory: bit for bit against the same data moved by torch."""
import pytest
import torch

from branch_latent_kv_b200 import binding as b

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _bytes(n, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, 256, (n,), generator=g, dtype=torch.uint8)


@pytest.mark.parametrize("sizes", [
    [262144, 32768, 8192, 64],   # the 2.9B step's inputs
    [20, 16, 48, 1_000_000],     # byte tails and a large range
    [0, 5 * 4],                  # an empty range and lengths of a batch of 5
])
def test_host_to_device_ranges_are_exact(sizes):
    srcs = [_bytes(n, i).pin_memory() for i, n in enumerate(sizes)]
    dsts = [torch.full((n,), 7, dtype=torch.uint8, device="cuda") for n in sizes]
    b.mlra_copy_ranges(list(zip(srcs, dsts)))
    torch.cuda.synchronize()
    for s, d in zip(srcs, dsts):
        assert torch.equal(s, d.cpu())


def test_device_to_host_and_device_to_device():
    a = _bytes(4096 + 8, 1).cuda()
    c = _bytes(123456, 2).cuda()
    h = torch.zeros(4096 + 8, dtype=torch.uint8).pin_memory()
    d = torch.zeros(123456, dtype=torch.uint8, device="cuda")
    b.mlra_copy_ranges([(a, h), (c, d)])
    torch.cuda.synchronize()
    assert torch.equal(h, a.cpu()) and torch.equal(d, c)


def test_copy_rejects_pageable_misaligned_and_overlapping():
    dev = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        b.mlra_copy_ranges([(torch.zeros(64, dtype=torch.uint8), dev)])  # pageable: refused by the binding
    lib = b.library()
    import ctypes
    page = ctypes.create_string_buffer(128)  # pageable host memory, straight to the ABI
    src = (ctypes.c_void_p * 1)(ctypes.addressof(page) + (-ctypes.addressof(page)) % 16)
    dst = (ctypes.c_void_p * 1)(dev.data_ptr())
    nb = (ctypes.c_uint64 * 1)(64)
    assert lib.mlra_copy_ranges(1, src, dst, nb, None) == b.MLRA_ERR_INVALID_ARG
    big = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(b.MlraError):
        b.mlra_copy_ranges([(big[16:80], big[48:112])])  # destination overlaps the source
    with pytest.raises(b.MlraError):
        b.mlra_copy_ranges([(big[0:32], big[128:160]), (big[32:64], big[144:176])])  # destinations overlap
    with pytest.raises(b.MlraError):
        b.mlra_copy_ranges([(big[1:17], big[64:80])])  # misaligned


def test_up_proj_writes_a_pinned_host_result_bit_for_bit():
    g = torch.Generator().manual_seed(3)
    N, H, B, d_c, d_h = 16, 16, 4, 128, 128
    out = (torch.randn((N, H, B, d_c), generator=g) / 8).to(torch.bfloat16).cuda()
    w = (torch.randn((B, d_c, H * d_h), generator=g) / 16).to(torch.bfloat16).cuda()
    y_dev = b.mlra_up_proj(out, w)
    y_host = torch.zeros((N, H * d_h), dtype=torch.bfloat16).pin_memory()
    b.mlra_up_proj(out, w, y=y_host)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_dev.cpu())
    with pytest.raises(ValueError):
        b.mlra_up_proj(out, w, y=torch.zeros((N, H * d_h), dtype=torch.bfloat16))  # pageable
