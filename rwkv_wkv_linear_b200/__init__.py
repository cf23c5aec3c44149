"""RWKV-4 WKV time-mix recurrence (forward over T and single-step decode) for
NVIDIA B200, as hand-written sm_100a CUDA kernels behind a C ABI
(include/wkv4.h); ``wkv4`` is its thin Python binding.  The shared library
is loaded on first use, not at import."""

from . import wkv4  # noqa: F401
from .wkv4 import (BF16, F16, F32, KERNEL_AUTO, KERNEL_SCAN, KERNEL_SCAN_LDG,  # noqa: F401
                   KERNEL_SEQ, KERNEL_STEP, decode_step, device_error, forward)
