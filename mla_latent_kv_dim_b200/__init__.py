"""B200-native MLA latent-KV decode and TPLA (Tensor-Parallel Latent Attention).

The compute lives in ``libtpla.so`` (C ABI, include/tpla.h): hand-written
CUDA kernels for sm_100a.  This package holds the ctypes binding
(``_native``), the in-tree build (``build``) and the seeded synthetic
workloads (``workloads``).
"""
from ._native import (TplaError, cache_append, decode, decode_simple,  # noqa: F401
                      decode_workspace_size,
                      device_status, error_string, hadamard_apply, latent_covariance,
                      launch_count, lse_merge, lib, prefill, rotate_apply,
                      selftest_wait_timeout, version, vup_combine)

__all__ = ["TplaError", "cache_append", "decode", "decode_simple", "decode_workspace_size", "device_status",
           "selftest_wait_timeout", "latent_covariance", "rotate_apply",
           "error_string", "hadamard_apply", "launch_count", "lse_merge", "lib", "prefill", "version",
           "vup_combine"]
