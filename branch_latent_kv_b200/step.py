"""A decode step bound to fixed buffers and replayed from one CUDA graph.

A serving loop calls the same decode step every token with the same buffer
shapes.  ``DecodeStep`` validates the arguments once (one eager call of
``mlra_decode`` or, when ``w_uv`` is given, ``mlra_decode_up_proj``: the
whole step in one launch; batches above 64 use ``mlra_decode`` and
``mlra_up_proj``), then captures
the step -- optionally with the host-to-device transfer of its inputs and the
device-to-host transfer of its result -- into a CUDA graph, so each step costs
one graph launch on the host.  The inputs cross PCIe in one launch of
``mlra_copy_ranges`` (SM loads from the mapped pinned pages); with ``w_uv``
the up-projection writes y straight into the pinned host output.  All arithmetic is in the library's kernels;
this module only arranges launches.

Buffers are bound at construction: write the next step's inputs into the
bound tensors (or into the pinned host tensors given as ``host_inputs``)
before calling the step.  A replay is asynchronous and its copy kernel reads
the pinned host inputs while it runs, so overwrite them only after the
previous step has finished (synchronise its stream first).  The graph keeps
the kernels' arguments, including the TMA descriptors built from the bound
pointers, so the bound tensors must stay alive and in place.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import binding as b

_INPUT_NAMES = ("q_lat", "q_rope", "block_table", "seqlens")


class DecodeStep:
    """One MLRA decode step (mlra_decode, then mlra_up_proj if ``w_uv`` is
    given) on bound device buffers.

    host_inputs: optional dict with pinned CPU tensors for any of ``q_lat``,
        ``q_rope``, ``block_table``, ``seqlens`` (same shape and dtype as the
        device tensors): each step copies them to the device first.
    host_output: optional pinned CPU tensor shaped like the step's result
        (``y`` with ``w_uv``, else ``out``): each step copies the result there.
    Calling the step replays the graph on the current stream and returns the
    result tensor (the host one when ``host_output`` is given); synchronise
    before reading host memory.
    """

    def __init__(self, q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale,
                 out_scale, *, w_uv=None, d_h: Optional[int] = None, workspace=None,
                 host_inputs: Optional[Dict[str, torch.Tensor]] = None,
                 host_output: Optional[torch.Tensor] = None):
        dev = q_lat.device
        self.device = dev
        self.inputs = dict(q_lat=q_lat, q_rope=q_rope, block_table=block_table, seqlens=seqlens)
        self.host_inputs = dict(host_inputs or {})
        for name, h in self.host_inputs.items():
            if name not in _INPUT_NAMES:
                raise ValueError(f"host_inputs: unknown input {name!r}")
            d = self.inputs[name]
            if h.device.type != "cpu" or not h.is_pinned():
                raise ValueError(f"host_inputs[{name!r}] must be pinned CPU memory")
            if h.shape != d.shape or h.dtype != d.dtype:
                raise ValueError(f"host_inputs[{name!r}] must match the device tensor's shape and dtype")
            if not h.is_contiguous() or h.data_ptr() % 16 != 0:
                raise ValueError(f"host_inputs[{name!r}] must be contiguous and 16-byte aligned")
        if len(self.host_inputs) > 8:
            raise ValueError("at most 8 host inputs")
        dims = b.decode_dims(q_lat, q_rope, latent_cache, block_table)
        self.workspace = workspace if workspace is not None else torch.zeros(
            b.mlra_decode_workspace_bytes(dims), dtype=torch.uint8, device=dev)
        self.out = torch.empty_like(q_lat)
        self.y = None
        if w_uv is not None:
            N, H = q_lat.shape[:2]
            d_h = d_h if d_h is not None else w_uv.shape[2] // H
            self.y = torch.empty((N, H * d_h), dtype=torch.bfloat16, device=dev)
        result = self.y if self.y is not None else self.out
        if host_output is not None:
            if host_output.device.type != "cpu" or not host_output.is_pinned():
                raise ValueError("host_output must be pinned CPU memory")
            if not host_output.is_contiguous() or host_output.data_ptr() % 16 != 0:
                raise ValueError("host_output must be contiguous and 16-byte aligned")
            if host_output.shape != result.shape or host_output.dtype != result.dtype:
                raise ValueError("host_output must match the result's shape and dtype")
        self.host_output = host_output
        self._args = (q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens, scale, out_scale)
        self._w_uv, self._d_h = w_uv, d_h
        # decode and up-projection in one launch where that kernel covers the
        # shape (batch <= 64), else the two launches
        self._fused = w_uv is not None and q_lat.shape[0] <= 64

        # validation: one eager pass (raises on any argument error) on the
        # step's real inputs: the host inputs, if any, are brought in first,
        # so the pass never reads uninitialised bound tensors
        stream = torch.cuda.current_stream(dev)
        with torch.cuda.stream(stream):
            for name, h in self.host_inputs.items():
                self.inputs[name].copy_(h, non_blocking=True)
        self._body(stream, copies=False)
        torch.cuda.synchronize(dev)
        # the validation pass's device findings are not a step's: reading
        # clears the error word (and the split counters after a timeout), so
        # the first replay reports only its own
        b.mlra_read_device_error(self.workspace, stream)
        # capture on a side stream, ordered after the eager pass
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=cap):
            self._body(cap, copies=True)
        torch.cuda.synchronize(dev)

    def _body(self, stream, copies: bool):
        with torch.cuda.stream(stream):
            if copies and self.host_inputs:
                # every host input crosses PCIe in one launch (SM loads from
                # the mapped pinned pages), not one DMA copy per tensor
                b.mlra_copy_ranges([(h, self.inputs[name]) for name, h in self.host_inputs.items()],
                                   stream=stream, device=self.device)
            direct = copies and self.host_output is not None and self._w_uv is not None
            y_dst = self.host_output if direct else self.y  # a host output is written straight from the kernel
            if self._w_uv is not None and self._fused:
                # the whole step in one launch
                b.mlra_decode_up_proj(*self._args, self._w_uv, d_h=self._d_h, out=self.out, y=y_dst,
                                      workspace=self.workspace, stream=stream)
            else:
                b.mlra_decode(*self._args, out=self.out, workspace=self.workspace, stream=stream)
                if self._w_uv is not None:
                    b.mlra_up_proj(self.out, self._w_uv, d_h=self._d_h, y=y_dst, stream=stream)
            if copies and self.host_output is not None and not direct:
                self.host_output.copy_(self.out, non_blocking=True)

    def __call__(self) -> torch.Tensor:
        self.graph.replay()
        if self.host_output is not None:
            return self.host_output
        return self.y if self.y is not None else self.out

    def h2d_bytes(self) -> int:
        """Bytes copied host-to-device per step."""
        return sum(h.numel() * h.element_size() for h in self.host_inputs.values())

    def d2h_bytes(self) -> int:
        """Bytes copied device-to-host per step."""
        return 0 if self.host_output is None else self.host_output.numel() * self.host_output.element_size()
