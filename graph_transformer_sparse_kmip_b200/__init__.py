"""k-MIP attention for graph transformers on NVIDIA B200 (sm_100a).

The compute lives in libkmip.so (C ABI: include/kmip.h); ``binding`` is a
ctypes layer over it and ``workloads`` holds the seeded synthetic inputs.
"""
from .binding import (KmipError, attn_bwd, attn_fwd, check_status, kmip_attn_bwd,  # noqa: F401
                      kmip_attn_fwd, kmip_error_string, kmip_get_status, kmip_version)
