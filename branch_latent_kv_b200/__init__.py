"""B200-native MLRA (Multi-Head Low-Rank Attention) decode path.

``binding`` exposes the C ABI of ``libmlra.so`` (include/mlra.h) under the
same names; ``inputs`` draws the seeded synthetic workloads.
"""
from .binding import (MlraError, mlra_decode, mlra_decode_plan, mlra_decode_simt, mlra_decode_workspace_bytes,
                      mlra_dims, mlra_read_device_error, mlra_status_string, mlra_up_proj)

__all__ = ["MlraError", "mlra_decode", "mlra_decode_plan", "mlra_decode_simt", "mlra_decode_workspace_bytes", "mlra_dims",
           "mlra_read_device_error", "mlra_status_string", "mlra_up_proj"]
