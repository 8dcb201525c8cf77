"""Python binding of the C ABI in ``include/mlra.h`` (ctypes, argument
marshalling only).

Every function here checks tensor types, shapes and devices, passes raw
device pointers and the current CUDA stream to ``libmlra.so`` and raises
``MlraError`` on a non-OK status.  All arithmetic happens in the library's
CUDA kernels; there is no fallback.  If ``libmlra.so`` has not been built the
first call raises immediately.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmlra.so")

MLRA_OK = 0
MLRA_ERR_INVALID_ARG = 1
MLRA_ERR_UNSUPPORTED = 2
MLRA_ERR_WORKSPACE = 3
MLRA_ERR_CUDA = 4
MLRA_ERR_DEVICE_BAD_INDEX = 5
MLRA_ERR_DEVICE_BAD_SEQLEN = 6
MLRA_ERR_DEVICE_TIMEOUT = 7


class MlraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {mlra_status_string(status)}")


class mlra_dims(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in
                ("batch", "heads", "branches", "d_c", "d_r", "page_size", "max_pages_per_seq",
                 "num_pages")]


_lib = None
_lib_lock = threading.Lock()


def library() -> ctypes.CDLL:
    """Load libmlra.so (raises if it is missing: build it first)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lib_lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                                   "`python -m branch_latent_kv_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
            dp = ctypes.POINTER(mlra_dims)
            lib.mlra_decode_workspace_bytes.argtypes = [dp, i32]
            lib.mlra_decode_workspace_bytes.restype = sz
            lib.mlra_decode.argtypes = [dp, vp, vp, vp, vp, vp, vp, ctypes.c_float, ctypes.c_float,
                                        vp, vp, sz, vp]
            lib.mlra_decode.restype = ctypes.c_int
            lib.mlra_decode_up_proj.argtypes = [dp, vp, vp, vp, vp, vp, vp, ctypes.c_float, ctypes.c_float,
                                                vp, vp, i32, vp, vp, sz, vp]
            lib.mlra_decode_up_proj.restype = ctypes.c_int
            lib.mlra_decode_simt.argtypes = lib.mlra_decode.argtypes
            lib.mlra_decode_simt.restype = ctypes.c_int
            lib.mlra_up_proj.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp]
            lib.mlra_up_proj.restype = ctypes.c_int
            lib.mlra_up_proj_gated.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]
            lib.mlra_up_proj_gated.restype = ctypes.c_int
            lib.mlra_prepare.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, vp,
                                         vp, vp]
            lib.mlra_prepare.restype = ctypes.c_int
            lib.mlra_exchange_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
            lib.mlra_exchange_bytes.restype = sz
            lib.mlra_exchange_alloc.argtypes = [sz, ctypes.POINTER(vp), vp]
            lib.mlra_exchange_alloc.restype = ctypes.c_int
            lib.mlra_exchange_open.argtypes = [vp, ctypes.POINTER(vp)]
            lib.mlra_exchange_open.restype = ctypes.c_int
            lib.mlra_exchange_close.argtypes = [vp]
            lib.mlra_exchange_close.restype = ctypes.c_int
            lib.mlra_exchange_free.argtypes = [vp]
            lib.mlra_exchange_free.restype = ctypes.c_int
            lib.mlra_exchange_reset.argtypes = [vp, sz, vp]
            lib.mlra_exchange_reset.restype = ctypes.c_int
            lib.mlra_up_proj_allreduce.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32, i32, i32,
                                                   vp, ctypes.c_uint64, vp]
            lib.mlra_up_proj_allreduce.restype = ctypes.c_int
            lib.mlra_copy_ranges.argtypes = [i32, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                             ctypes.POINTER(ctypes.c_uint64), vp]
            lib.mlra_copy_ranges.restype = ctypes.c_int
            lib.mlra_read_device_error.argtypes = [vp, vp]
            lib.mlra_read_device_error.restype = ctypes.c_int
            lib.mlra_status_string.argtypes = [ctypes.c_int]
            lib.mlra_status_string.restype = ctypes.c_char_p
            lib.mlra_decode_plan.argtypes = [i32, i32, i32, vp, i32, vp, vp]
            lib.mlra_decode_plan.restype = ctypes.c_int
            _lib = lib
    return _lib


def mlra_status_string(status: int) -> str:
    return library().mlra_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MLRA_OK:
        raise MlraError(status, where)


def _stream_ptr(stream: Optional[torch.cuda.Stream], device: torch.device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return int(s.cuda_stream)


def _ptr(t: torch.Tensor) -> int:
    return int(t.data_ptr())


def _require(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int, device: torch.device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def decode_dims(q_lat, q_rope, latent_cache, block_table) -> mlra_dims:
    N, H, B, d_c = q_lat.shape
    num_pages, P = latent_cache.shape[:2]
    return mlra_dims(N, H, B, d_c, q_rope.shape[2], P, block_table.shape[1], num_pages)


def mlra_decode_workspace_bytes(dims: mlra_dims, num_ctas: int = 0) -> int:
    n = library().mlra_decode_workspace_bytes(ctypes.byref(dims), int(num_ctas))
    if n == 0:
        raise MlraError(MLRA_ERR_INVALID_ARG, "mlra_decode_workspace_bytes")
    return int(n)


_ws_cache = {}


def workspace_for(dims: mlra_dims, device: torch.device) -> torch.Tensor:
    """A zeroed workspace of the required size, cached per device and grown
    on demand.  Calls sharing it must not overlap on the GPU."""
    need = mlra_decode_workspace_bytes(dims)
    key = device.index if device.index is not None else torch.cuda.current_device()
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def _decode(entry, q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale, out_scale,
            out=None, workspace=None, stream=None) -> torch.Tensor:
    return _decode_call(lambda dims, *args: getattr(library(), entry)(dims, *args), entry, q_lat, q_rope,
                        latent_cache, rope_cache, block_table, seqlens, scale, out_scale, out, workspace, stream)


def _decode_call(call, name, q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale, out_scale,
                 out=None, workspace=None, stream=None) -> torch.Tensor:
    dev = q_lat.device
    if dev.type != "cuda":
        raise ValueError("mlra_decode runs on CUDA tensors only")
    _require(q_lat, "q_lat", torch.bfloat16, 4, dev)
    _require(q_rope, "q_rope", torch.bfloat16, 3, dev)
    _require(latent_cache, "latent_cache", torch.bfloat16, 4, dev)
    _require(rope_cache, "rope_cache", torch.bfloat16, 3, dev)
    _require(block_table, "block_table", torch.int32, 2, dev)
    _require(seqlens, "seqlens", torch.int32, 1, dev)
    N, H, B, d_c = q_lat.shape
    if (tuple(q_rope.shape[:2]) != (N, H) or tuple(latent_cache.shape[2:]) != (B, d_c)
            or tuple(rope_cache.shape) != (latent_cache.shape[0], latent_cache.shape[1], q_rope.shape[2])
            or block_table.shape[0] != N or seqlens.shape[0] != N):
        raise ValueError("inconsistent mlra_decode shapes")
    dims = decode_dims(q_lat, q_rope, latent_cache, block_table)
    if out is None:
        out = torch.empty_like(q_lat)
    else:
        _require(out, "out", torch.bfloat16, 4, dev)
        if out.shape != q_lat.shape:
            raise ValueError("out must have the shape of q_lat")
    if workspace is None:
        workspace = workspace_for(dims, dev)
    st = call(ctypes.byref(dims), _ptr(q_lat), _ptr(q_rope), _ptr(latent_cache), _ptr(rope_cache),
              _ptr(block_table), _ptr(seqlens), float(scale), float(out_scale), _ptr(out), _ptr(workspace),
              workspace.numel() * workspace.element_size(), _stream_ptr(stream, dev))
    _check(st, name)
    return out


def mlra_decode(q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale, out_scale,
                out=None, workspace=None, stream=None) -> torch.Tensor:
    """MLRA decode attention on the tensor cores (see mlra_decode in mlra.h).

    q_lat bf16 [N,H,B,d_c], q_rope bf16 [N,H,d_r], latent_cache bf16
    [pages,P,B,d_c], rope_cache bf16 [pages,P,d_r], block_table int32
    [N,max_pages], seqlens int32 [N]; returns out bf16 [N,H,B,d_c].
    """
    return _decode("mlra_decode", q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens,
                   scale, out_scale, out, workspace, stream)


def mlra_decode_up_proj(q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale, out_scale,
                        w_uv, d_h: Optional[int] = None, out=None, y=None, workspace=None, stream=None):
    """The whole step in one launch (see mlra_decode_up_proj in mlra.h):
    returns (out bf16 [N,H,B,d_c], y bf16 [N, H*d_h]).  y may be a pinned
    host tensor (the kernel then writes it over PCIe)."""
    dev = q_lat.device
    if dev.type != "cuda":
        raise ValueError("mlra_decode_up_proj runs on CUDA tensors only")
    _require(w_uv, "w_uv", torch.bfloat16, 3, dev)
    N, H, B, d_c = q_lat.shape
    if w_uv.shape[0] != B or w_uv.shape[1] != d_c or w_uv.shape[2] % H != 0:
        raise ValueError("w_uv must be [branches, d_c, heads*d_h]")
    if d_h is None:
        d_h = w_uv.shape[2] // H
    if w_uv.shape[2] != H * d_h:
        raise ValueError("w_uv last dimension must be heads*d_h")
    if y is None:
        y = torch.empty((N, H * d_h), dtype=torch.bfloat16, device=dev)
    else:
        _require(y, "y", torch.bfloat16, 2, y.device if y.device.type == "cpu" else dev)
        if y.device.type == "cpu" and not y.is_pinned():
            raise ValueError("a host y must be pinned memory")
        if tuple(y.shape) != (N, H * d_h):
            raise ValueError("y must be [N, heads*d_h]")
    def entry(dims, *args):
        # mlra_decode's arguments up to out, then w_uv, d_h, y, workspace, bytes, stream
        head, tail = args[:9], args[9:]
        return library().mlra_decode_up_proj(dims, *head, _ptr(w_uv), int(d_h), _ptr(y), *tail)

    out = _decode_call(entry, "mlra_decode_up_proj", q_lat, q_rope, latent_cache, rope_cache, block_table,
                       seqlens, scale, out_scale, out, workspace, stream)
    return out, y


def mlra_decode_simt(q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale,
                     out_scale, out=None, workspace=None, stream=None) -> torch.Tensor:
    """The same operation on the CUDA cores (see mlra_decode_simt in mlra.h)."""
    return _decode("mlra_decode_simt", q_lat, q_rope, latent_cache, rope_cache, block_table,
                   seqlens, scale, out_scale, out, workspace, stream)


def mlra_up_proj(out_lat, w_uv, d_h: Optional[int] = None, y=None, stream=None) -> torch.Tensor:
    """y bf16 [N, H*d_h] = per-branch W_UV up-projection summed over branches."""
    return _up_proj(out_lat, w_uv, None, d_h, y, stream)


def mlra_up_proj_gated(out_lat, w_uv, gate, d_h: Optional[int] = None, y=None,
                       stream=None) -> torch.Tensor:
    """mlra_up_proj times sigmoid(gate) elementwise; gate bf16 [N, H*d_h]."""
    if gate is None:
        raise ValueError("mlra_up_proj_gated needs a gate tensor")
    return _up_proj(out_lat, w_uv, gate, d_h, y, stream)


def _up_proj(out_lat, w_uv, gate, d_h, y, stream) -> torch.Tensor:
    dev = out_lat.device
    if dev.type != "cuda":
        raise ValueError("mlra_up_proj runs on CUDA tensors only")
    _require(out_lat, "out_lat", torch.bfloat16, 4, dev)
    _require(w_uv, "w_uv", torch.bfloat16, 3, dev)
    N, H, B, d_c = out_lat.shape
    if w_uv.shape[0] != B or w_uv.shape[1] != d_c or w_uv.shape[2] % H != 0:
        raise ValueError("w_uv must be [branches, d_c, heads*d_h]")
    if d_h is None:
        d_h = w_uv.shape[2] // H
    if w_uv.shape[2] != H * d_h:
        raise ValueError("w_uv last dimension must be heads*d_h")
    if y is None:
        y = torch.empty((N, H * d_h), dtype=torch.bfloat16, device=dev)
    else:
        # y may be pinned host memory: the kernel then writes it over PCIe
        _require(y, "y", torch.bfloat16, 2, y.device if y.device.type == "cpu" else dev)
        if y.device.type == "cpu" and not y.is_pinned():
            raise ValueError("a host y must be pinned memory")
        if tuple(y.shape) != (N, H * d_h):
            raise ValueError("y must be [N, heads*d_h]")
    if gate is None:
        st = library().mlra_up_proj(N, H, B, d_c, d_h, _ptr(out_lat), _ptr(w_uv), _ptr(y),
                                    _stream_ptr(stream, dev))
        _check(st, "mlra_up_proj")
    else:
        _require(gate, "gate", torch.bfloat16, 2, dev)
        if tuple(gate.shape) != (N, H * d_h):
            raise ValueError("gate must be [N, heads*d_h]")
        st = library().mlra_up_proj_gated(N, H, B, d_c, d_h, _ptr(out_lat), _ptr(w_uv), _ptr(gate),
                                          _ptr(y), _stream_ptr(stream, dev))
        _check(st, "mlra_up_proj_gated")
    return y


def default_workspace(device: Optional[torch.device] = None) -> Optional[torch.Tensor]:
    """The cached workspace that decode calls without an explicit workspace
    use on `device` (None if none has been made yet)."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    return _ws_cache.get(key)


def mlra_read_device_error(workspace: Optional[torch.Tensor] = None, stream=None) -> int:
    """Synchronise the stream; return and clear the device error code of
    `workspace` (default: the cached workspace of the current device).  A
    reported MLRA_ERR_DEVICE_TIMEOUT also clears the workspace's split
    counters, so the workspace serves the next call."""
    if workspace is None:
        workspace = default_workspace()
        if workspace is None:
            return MLRA_OK
    return int(library().mlra_read_device_error(_ptr(workspace),
                                                _stream_ptr(stream, workspace.device)))


def mlra_decode_plan(seqlens: torch.Tensor, page_size: int, max_pages_per_seq: int,
                     num_ctas: int, stream=None) -> torch.Tensor:
    """The split-KV work partition as int32 [num_ctas*4 + N*2] (see mlra.h)."""
    dev = seqlens.device
    _require(seqlens, "seqlens", torch.int32, 1, dev)
    out = torch.empty(num_ctas * 4 + seqlens.numel() * 2, dtype=torch.int32, device=dev)
    st = library().mlra_decode_plan(seqlens.numel(), page_size, max_pages_per_seq, _ptr(seqlens),
                                    num_ctas, _ptr(out), _stream_ptr(stream, dev))
    _check(st, "mlra_decode_plan")
    return out


def mlra_prepare(q_c, q_r, w_uk, c_new, kr_new, seqlens, block_table, latent_cache, rope_cache,
                 rope_base: float = 10000.0, q_lat=None, q_rope=None, device_status=None,
                 stream=None):
    """The decode pre-step (see mlra_prepare in mlra.h): absorbed queries
    q_lat bf16 [N,H,B,d_c], rotated RoPE queries q_rope bf16 [N,H,d_r], and the
    new token's latents and rotated RoPE key written into the caches in place.

    q_c bf16 [N,H,d_h], q_r bf16 [N,H,d_r], w_uk bf16 [B,H,d_h,d_c], c_new bf16
    [N,B,d_c], kr_new bf16 [N,d_r], seqlens int32 [N] (including the new
    token), block_table int32 [N,max_pages]; device_status: optional int32 [1]
    device tensor receiving the first device-detected error code.
    Returns (q_lat, q_rope).
    """
    dev = q_c.device
    if dev.type != "cuda":
        raise ValueError("mlra_prepare runs on CUDA tensors only")
    _require(q_c, "q_c", torch.bfloat16, 3, dev)
    _require(q_r, "q_r", torch.bfloat16, 3, dev)
    _require(w_uk, "w_uk", torch.bfloat16, 4, dev)
    _require(c_new, "c_new", torch.bfloat16, 3, dev)
    _require(kr_new, "kr_new", torch.bfloat16, 2, dev)
    _require(seqlens, "seqlens", torch.int32, 1, dev)
    _require(block_table, "block_table", torch.int32, 2, dev)
    _require(latent_cache, "latent_cache", torch.bfloat16, 4, dev)
    _require(rope_cache, "rope_cache", torch.bfloat16, 3, dev)
    N, H, d_h = q_c.shape
    B, _, _, d_c = w_uk.shape
    d_r = q_r.shape[2]
    num_pages, P = latent_cache.shape[:2]
    if (tuple(w_uk.shape) != (B, H, d_h, d_c) or tuple(q_r.shape[:2]) != (N, H)
            or tuple(c_new.shape) != (N, B, d_c) or tuple(kr_new.shape) != (N, d_r)
            or tuple(latent_cache.shape[2:]) != (B, d_c) or tuple(rope_cache.shape) != (num_pages, P, d_r)
            or seqlens.shape[0] != N or block_table.shape[0] != N):
        raise ValueError("inconsistent mlra_prepare shapes")
    if q_lat is None:
        q_lat = torch.empty((N, H, B, d_c), dtype=torch.bfloat16, device=dev)
    else:
        _require(q_lat, "q_lat", torch.bfloat16, 4, dev)
    if q_rope is None:
        q_rope = torch.empty((N, H, d_r), dtype=torch.bfloat16, device=dev)
    else:
        _require(q_rope, "q_rope", torch.bfloat16, 3, dev)
    if device_status is not None:
        _require(device_status, "device_status", torch.int32, 1, dev)
    dims = mlra_dims(N, H, B, d_c, d_r, P, block_table.shape[1], num_pages)
    st = library().mlra_prepare(ctypes.byref(dims), d_h, _ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(c_new),
                                _ptr(kr_new), _ptr(seqlens), _ptr(block_table), float(rope_base),
                                _ptr(q_lat), _ptr(q_rope), _ptr(latent_cache), _ptr(rope_cache),
                                _ptr(device_status) if device_status is not None else None,
                                _stream_ptr(stream, dev))
    _check(st, "mlra_prepare")
    return q_lat, q_rope


# ------------------------------------------------------------------ branch sharding
MLRA_IPC_HANDLE_BYTES = 64


def mlra_exchange_bytes(batch: int, heads: int, branches: int, d_c: int, d_h: int, world: int) -> int:
    """Bytes of one rank's exchange region (branches = the rank's own count)."""
    n = library().mlra_exchange_bytes(batch, heads, branches, d_c, d_h, world)
    if n == 0:
        raise MlraError(MLRA_ERR_INVALID_ARG, "mlra_exchange_bytes")
    return int(n)


def mlra_exchange_alloc(nbytes: int, with_handle: bool = True):
    """A zeroed exchange region on the current device: (pointer, IPC handle
    bytes or None).  Release it with mlra_exchange_free."""
    p = ctypes.c_void_p()
    h = ctypes.create_string_buffer(MLRA_IPC_HANDLE_BYTES) if with_handle else None
    _check(library().mlra_exchange_alloc(int(nbytes), ctypes.byref(p), h), "mlra_exchange_alloc")
    return int(p.value), (h.raw if h is not None else None)


def mlra_exchange_open(handle: bytes) -> int:
    """Map another process's exchange region from its handle."""
    if len(handle) != MLRA_IPC_HANDLE_BYTES:
        raise ValueError("an exchange handle has 64 bytes")
    p = ctypes.c_void_p()
    _check(library().mlra_exchange_open(ctypes.create_string_buffer(handle, MLRA_IPC_HANDLE_BYTES),
                                        ctypes.byref(p)), "mlra_exchange_open")
    return int(p.value)


def mlra_exchange_close(ptr: int) -> None:
    _check(library().mlra_exchange_close(ptr), "mlra_exchange_close")


def mlra_exchange_free(ptr: int) -> None:
    _check(library().mlra_exchange_free(ptr), "mlra_exchange_free")


def mlra_exchange_reset(ptr: int, nbytes: int, device: Optional[torch.device] = None, stream=None) -> None:
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    _check(library().mlra_exchange_reset(ptr, int(nbytes), _stream_ptr(stream, dev)), "mlra_exchange_reset")


def mlra_up_proj_allreduce(out_lat, w_uv, regions: torch.Tensor, rank: int, gate=None,
                           d_h: Optional[int] = None, y=None, ranks_in_launch: int = 1,
                           device_status=None, wait_limit_ns: int = 2_000_000_000,
                           stream=None) -> torch.Tensor:
    """Branch-sharded up-projection with the cross-rank branch sum (see
    mlra_up_proj_allreduce in mlra.h).

    out_lat bf16 [N,H,B_r,d_c] and w_uv bf16 [B_r,d_c,H*d_h] hold this rank's
    B_r branches; regions is an int64 device tensor [world] of the ranks'
    exchange-region pointers; returns the full y bf16 [N,H*d_h].  With
    ranks_in_launch = k > 1 the operands carry a leading rank dimension
    ([k,N,H,B_r,d_c], [k,B_r,d_c,H*d_h] -> y [k,N,H*d_h]) for ranks rank ..
    rank+k-1, all computed in one launch on this device.
    """
    dev = out_lat.device
    if dev.type != "cuda":
        raise ValueError("mlra_up_proj_allreduce runs on CUDA tensors only")
    k = int(ranks_in_launch)
    lead = 1 if k > 1 else 0
    _require(out_lat, "out_lat", torch.bfloat16, 4 + lead, dev)
    _require(w_uv, "w_uv", torch.bfloat16, 3 + lead, dev)
    _require(regions, "regions", torch.int64, 1, dev)
    if lead and (out_lat.shape[0] != k or w_uv.shape[0] != k):
        raise ValueError("stacked operands need a leading dimension of ranks_in_launch")
    N, H, B, d_c = out_lat.shape[lead:]
    if tuple(w_uv.shape[lead:lead + 2]) != (B, d_c) or w_uv.shape[-1] % H != 0:
        raise ValueError("w_uv must be [branches, d_c, heads*d_h]")
    if d_h is None:
        d_h = w_uv.shape[-1] // H
    if w_uv.shape[-1] != H * d_h:
        raise ValueError("w_uv last dimension must be heads*d_h")
    y_shape = ((k,) if lead else ()) + (N, H * d_h)
    if y is None:
        y = torch.empty(y_shape, dtype=torch.bfloat16, device=dev)
    else:
        _require(y, "y", torch.bfloat16, 2 + lead, dev)
        if tuple(y.shape) != y_shape:
            raise ValueError(f"y must be {list(y_shape)}")
    if gate is not None:
        _require(gate, "gate", torch.bfloat16, 2, dev)
        if tuple(gate.shape) != (N, H * d_h):
            raise ValueError("gate must be [N, heads*d_h]")
    if device_status is not None:
        _require(device_status, "device_status", torch.int32, 1, dev)
    st = library().mlra_up_proj_allreduce(N, H, B, d_c, d_h, _ptr(out_lat), _ptr(w_uv),
                                          _ptr(gate) if gate is not None else None, _ptr(y), _ptr(regions),
                                          regions.numel(), int(rank), k,
                                          _ptr(device_status) if device_status is not None else None,
                                          int(wait_limit_ns), _stream_ptr(stream, dev))
    _check(st, "mlra_up_proj_allreduce")
    return y


def mlra_copy_ranges(pairs, stream=None, device: Optional[torch.device] = None) -> None:
    """Copy each (src, dst) tensor pair (same byte size; device or pinned host
    memory, 16-byte aligned, contiguous) in one launch of the SMs (see
    mlra_copy_ranges in mlra.h)."""
    pairs = list(pairs)
    if not 1 <= len(pairs) <= 8:
        raise ValueError("mlra_copy_ranges takes 1 to 8 pairs")
    for k, (s_t, d_t) in enumerate(pairs):
        if s_t.numel() * s_t.element_size() != d_t.numel() * d_t.element_size():
            raise ValueError(f"mlra_copy_ranges: pair {k} differs in size")
    pairs = [(s_t, d_t) for s_t, d_t in pairs if s_t.numel() > 0]  # empty ranges copy nothing
    if not pairs:
        return
    n = len(pairs)
    src, dst, nb = (ctypes.c_void_p * n)(), (ctypes.c_void_p * n)(), (ctypes.c_uint64 * n)()
    dev = device
    for k, (s_t, d_t) in enumerate(pairs):
        for t, what in ((s_t, "src"), (d_t, "dst")):
            if not t.is_contiguous():
                raise ValueError(f"mlra_copy_ranges: {what} {k} must be contiguous")
            if t.device.type == "cpu" and not t.is_pinned():
                raise ValueError(f"mlra_copy_ranges: host {what} {k} must be pinned memory")
            if t.device.type == "cuda" and dev is None:
                dev = t.device
        src[k], dst[k], nb[k] = _ptr(s_t), _ptr(d_t), s_t.numel() * s_t.element_size()
    if dev is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    _check(library().mlra_copy_ranges(n, src, dst, nb, _stream_ptr(stream, dev)), "mlra_copy_ranges")
