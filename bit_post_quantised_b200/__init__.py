"""B200 (sm_100a) ternary linear layer of 1.58-bit FLUX.

The compute lives in libtern.so (CUDA kernels behind a C ABI, declared in
include/tern.h); `tern` is its thin ctypes binding and `workloads` draws the
seeded synthetic FLUX-shaped inputs.
"""
from .tern import (TernError, dequantize, device_status, library_path, linear, linear_batch,
                   packed_bytes, quantize_pack, selftest_wait_timeout, set_wait_limit_ns,
                   status_string)

__all__ = ["TernError", "dequantize", "device_status", "library_path", "linear", "linear_batch",
           "packed_bytes", "quantize_pack", "selftest_wait_timeout", "set_wait_limit_ns",
           "status_string"]
