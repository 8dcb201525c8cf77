"""ctypes front of the fp64 C oracle (``mlra_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may call this module; the product path (the CUDA library and
its Python binding) never does.  It shares no code with the CUDA path.

``build()`` compiles the C file with gcc and OpenMP into ``liboracle.so`` next
to it.  ``decode``, ``up_proj`` and ``gate`` accept torch CPU tensors (bf16,
passed as their bit patterns, or float64) or numpy float64 arrays and return
float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mlra_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

BF16, F64 = 0, 1
ERR_BAD_INDEX, ERR_BAD_SEQLEN = 5, 6


def build(force: bool = False) -> str:
    """Compile the oracle (gcc -O2 -fopenmp) unless an up-to-date build exists."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC,
                    "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def open_library(path: str):
    """Load a compiled oracle and declare its C signatures."""
    lib = ctypes.CDLL(path)
    i32, vp, dbl = ctypes.c_int32, ctypes.c_void_p, ctypes.c_double
    lib.oracle_mlra_decode.restype = ctypes.c_int
    lib.oracle_mlra_decode.argtypes = [i32] * 8 + [ctypes.c_int] + [vp] * 6 + [dbl, dbl, vp, i32, vp, vp]
    lib.oracle_mlra_up_proj.restype = ctypes.c_int
    lib.oracle_mlra_up_proj.argtypes = [i32] * 5 + [ctypes.c_int, vp, vp, vp]
    lib.oracle_mlra_prepare.restype = ctypes.c_int
    lib.oracle_mlra_prepare.argtypes = [i32] * 9 + [ctypes.c_int] + [vp] * 6 + [dbl] + [vp] * 4
    lib.oracle_mlra_gate.restype = ctypes.c_int
    lib.oracle_mlra_gate.argtypes = [ctypes.c_int64, ctypes.c_int, vp, vp]
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = open_library(build())
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _as_input(x, kind_holder):
    """Return (numpy array, kind) for a torch or numpy input, without rounding."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype in (torch.int32,):
                return x.numpy(), None
            return x.to(torch.float64).numpy(), F64
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    if a.dtype == np.int32:
        return a, None
    if a.dtype == np.uint16:
        return a, BF16
    return np.ascontiguousarray(a, dtype=np.float64), F64


def decode(q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale, out_scale,
           seq_ids=None, lib=None):
    """fp64 decode attention.  Returns (out [N,H,B,d_c], lse [N,H,B], status).

    Shapes: q_lat [N,H,B,d_c], q_rope [N,H,d_r], latent_cache [pages,P,B,d_c],
    rope_cache [pages,P,d_r], block_table [N,max_pages] int32, seqlens [N]
    int32.  Float inputs must all be bf16 or all be float64.  Only the
    sequences in ``seq_ids`` are computed (the others stay NaN).
    """
    arrs = [_as_input(x, None) for x in (q_lat, q_rope, latent_cache, rope_cache)]
    kinds = {k for _, k in arrs}
    if len(kinds) != 1:
        raise TypeError("oracle inputs must share one float type (all bf16 or all float64)")
    kind = kinds.pop()
    (ql, _), (qr, _), (lc, _), (rc, _) = arrs
    bt = np.ascontiguousarray(_as_input(block_table, None)[0], dtype=np.int32)
    sl = np.ascontiguousarray(_as_input(seqlens, None)[0], dtype=np.int32)
    N, H, B, d_c = ql.shape
    d_r = qr.shape[2]
    num_pages, P = lc.shape[0], lc.shape[1]
    if lc.shape[2:] != (B, d_c) or rc.shape != (num_pages, P, d_r) or qr.shape[:2] != (N, H):
        raise ValueError("inconsistent oracle input shapes")
    max_pages = bt.shape[1]
    out = np.full((N, H, B, d_c), np.nan, dtype=np.float64)
    lse = np.full((N, H, B), np.nan, dtype=np.float64)
    ids = None
    n_ids = N
    if seq_ids is not None:
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32))
        n_ids = int(ids.size)
    lib = lib or _load()
    status = lib.oracle_mlra_decode(
        N, H, B, d_c, d_r, P, max_pages, num_pages, kind,
        ql.ctypes.data, qr.ctypes.data, lc.ctypes.data, rc.ctypes.data,
        bt.ctypes.data, sl.ctypes.data, float(scale), float(out_scale),
        ids.ctypes.data if ids is not None else None, n_ids,
        out.ctypes.data, lse.ctypes.data)
    return out, lse, int(status)


def up_proj(out_lat, w_uv, d_h, lib=None):
    """fp64 per-branch up-projection plus branch sum: y [N, H*d_h]."""
    ol, ol_kind = _as_input(out_lat, None)
    if ol_kind == BF16:  # decode bf16 bit patterns to their (exact) values
        ol = (ol.astype(np.uint32) << 16).view(np.float32)
    ol = np.ascontiguousarray(ol, dtype=np.float64)
    w, kind = _as_input(w_uv, None)
    N, H, B, d_c = ol.shape
    if w.shape != (B, d_c, H * d_h):
        raise ValueError("w_uv must be [branches, d_c, heads*d_h]")
    y = np.empty((N, H * d_h), dtype=np.float64)
    status = (lib or _load()).oracle_mlra_up_proj(N, H, B, d_c, d_h, kind, ol.ctypes.data, w.ctypes.data,
                                         y.ctypes.data)
    if status != 0:
        raise ValueError(f"oracle up_proj rejected its arguments (status {status})")
    return y


def gate(y, gate_logits, lib=None):
    """fp64 elementwise sigmoid output gate: y / (1 + exp(-gate)), same shape
    as y (the gated up-projection; see oracle_mlra_gate)."""
    yy = np.array(y, dtype=np.float64, copy=True, order="C")
    g, kind = _as_input(gate_logits, None)
    if g.shape != yy.shape:
        raise ValueError("gate must have the shape of y")
    status = (lib or _load()).oracle_mlra_gate(yy.size, kind, g.ctypes.data, yy.ctypes.data)
    if status != 0:
        raise ValueError(f"oracle gate rejected its arguments (status {status})")
    return yy


def prepare(q_c, q_r, w_uk, kr_new, seqlens, block_table, num_pages, page_size, rope_base=10000.0,
            lib=None):
    """fp64 decode pre-step (see oracle_mlra_prepare).  Returns
    (q_lat [N,H,B,d_c], q_rope [N,H,d_r], kr_rot [N,d_r], dest [N,2] int32, status).
    The new token's latents are copied, not computed, so they are not returned."""
    arrs = [_as_input(a, None) for a in (q_c, q_r, w_uk, kr_new)]
    kinds = {k for _, k in arrs}
    if len(kinds) != 1:
        raise TypeError("oracle inputs must share one float type (all bf16 or all float64)")
    kind = kinds.pop()
    (qc, _), (qr, _), (wk, _), (kr, _) = arrs
    bt = np.ascontiguousarray(_as_input(block_table, None)[0], dtype=np.int32)
    sl = np.ascontiguousarray(_as_input(seqlens, None)[0], dtype=np.int32)
    N, H, d_h = qc.shape
    B, _, _, d_c = wk.shape
    d_r = qr.shape[2]
    if wk.shape != (B, H, d_h, d_c) or qr.shape[:2] != (N, H) or kr.shape != (N, d_r):
        raise ValueError("inconsistent oracle prepare shapes")
    q_lat = np.empty((N, H, B, d_c), dtype=np.float64)
    q_rope = np.empty((N, H, d_r), dtype=np.float64)
    kr_rot = np.empty((N, d_r), dtype=np.float64)
    dest = np.empty((N, 2), dtype=np.int32)
    status = (lib or _load()).oracle_mlra_prepare(
        N, H, B, d_c, d_h, d_r, page_size, bt.shape[1], num_pages, kind,
        qc.ctypes.data, qr.ctypes.data, wk.ctypes.data, kr.ctypes.data, sl.ctypes.data, bt.ctypes.data,
        float(rope_base), q_lat.ctypes.data, q_rope.ctypes.data, kr_rot.ctypes.data, dest.ctypes.data)
    return q_lat, q_rope, kr_rot, dest, int(status)
