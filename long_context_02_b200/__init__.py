"""long_context_02_b200: lightning attention for NVIDIA B200 (sm_100a).

The computation lives in liblightning.so (C ABI declared in include/lightning.h,
CUDA kernels in csrc/). ``binding`` is a thin ctypes layer over it; importing
this package does not load the library until a binding function is called.
"""
from .binding import (LA_BF16, LA_F32, LA_OP_BACKWARD, LA_OP_DECODE, LA_OP_PREFILL,  # noqa: F401
                      LA_OP_PREFILL_VARLEN, LightningError, backward, decode, la_backward,
                      la_decode, la_get_tuning, la_last_launch_count, la_prefill,
                      la_prefill_varlen, la_read_device_status, la_set_tuning, la_status_string,
                      la_workspace_bytes, lib, prefill, prefill_varlen, workspace)
