"""B200-native MLRA (Multi-Head Low-Rank Attention) decode path.

``binding`` exposes the C ABI of ``libmlra.so`` (include/mlra.h) under the
same names; ``step`` binds a decode step to fixed buffers and replays it
from a CUDA graph; ``tp`` runs the step branch-sharded over a tensor-parallel
group; ``inputs`` draws the seeded synthetic workloads.
"""
from .binding import (MlraError, mlra_decode, mlra_decode_plan, mlra_decode_simt, mlra_decode_workspace_bytes,
                      mlra_dims, mlra_prepare, mlra_read_device_error, mlra_status_string,
                      mlra_up_proj, mlra_up_proj_allreduce, mlra_up_proj_gated)
from .step import DecodeStep

__all__ = ["DecodeStep", "MlraError", "mlra_decode", "mlra_decode_plan", "mlra_decode_simt", "mlra_decode_workspace_bytes", "mlra_dims",
           "mlra_prepare", "mlra_read_device_error", "mlra_status_string", "mlra_up_proj",
           "mlra_up_proj_allreduce", "mlra_up_proj_gated"]
