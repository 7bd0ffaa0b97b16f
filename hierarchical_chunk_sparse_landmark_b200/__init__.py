"""Hierarchical chunk-sparse landmark attention (HSA / HiLS / DHSA forward pass)
for NVIDIA B200 (sm_100a).

The computation runs in hand-written CUDA kernels behind a C ABI
(``include/hsa.h``, built into ``libhsa.so``); this package is the Python
binding (PyTorch supplies device memory and streams) plus the seeded synthetic
workloads used by the tests and the benchmark.
"""
from ._binding import (HSAError, check, decode, decode_context_parallel, decode_cp_attend,
                       decode_cp_candidates, decode_cp_combine, decode_cp_merge, decode_noalloc,
                       decode_ragged, decode_workspace_size, landmarks_append,
                       landmarks, last_call_kernels, last_call_launches, lib, path_overrides,
                       prefill, prefill_backward, prefill_backward_workspace_size,
                       prefill_varlen, prefill_varlen_workspace_size,
                       prefill_workspace_size, selftest_wait_expiry, set_stage_events,
                       status_string, workspace)

__all__ = ["HSAError", "check", "decode", "decode_context_parallel", "decode_cp_attend",
           "decode_cp_candidates", "decode_cp_combine", "decode_cp_merge", "decode_noalloc",
           "decode_ragged", "decode_workspace_size", "landmarks", "landmarks_append",
           "last_call_kernels", "last_call_launches", "lib", "path_overrides", "prefill",
           "prefill_backward", "prefill_backward_workspace_size", "prefill_varlen", "prefill_varlen_workspace_size", "prefill_workspace_size", "selftest_wait_expiry", "set_stage_events", "status_string",
           "workspace"]
