"""hsa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin inside a host program that owns all device memory, or
code that must not call cudaMalloc/cudaFree on a latency-critical path)
cannot pass hsa_decode a workspace; hsa_decode_noalloc uses the library's
fixed device array instead.  This file is collected last so that a run which
stops at the first failure has already run every other test; it also passes
on its own in a fresh process.
"""
import ctypes

import pytest
import torch

import hierarchical_chunk_sparse_landmark_b200 as hsa
from hierarchical_chunk_sparse_landmark_b200 import _binding as B
from hierarchical_chunk_sparse_landmark_b200.workloads import Workload, make_decode_inputs
from oracle.parity import ATOL


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    wl = Workload("noalloc", "decode", "bf16", B=4, L=64 * 3000, H=16, Hkv=2, d=128, topk=8,
                  seed=21)
    x = make_decode_inputs(wl, "cuda")
    O_ref, idx_ref = hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=wl.topk, idx_out=True)
    hsa.check()
    lib = hsa.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):                      # the array keeps the previous call's contents
        O = torch.full_like(x["q"], float("nan"))
        idx = torch.full((wl.B, wl.Hkv, wl.topk), -7, dtype=torch.int32, device="cuda")
        st = lib.hsa_decode_noalloc(B._ptr(x["q"]), B._ptr(x["K"]), B._ptr(x["V"]), B.HSA_BF16,
                                    B._ptr(x["lm"]), B.HSA_BF16, wl.B, wl.H, wl.Hkv, wl.L, wl.d,
                                    wl.S, wl.topk, 0.0, B._ptr(O), B._ptr(idx), stream)
        assert st == B.HSA_OK, hsa.status_string(st)
        assert lib.hsa_check(None, stream) == B.HSA_OK
        assert torch.equal(idx, idx_ref), call
        err = (O.float() - O_ref.float()).abs().max().item()
        assert err <= ATOL["bf16"], (call, err)


@pytest.mark.gpu
def test_noalloc_decode_rejects_sizes_beyond_its_array():
    cap = hsa.lib().hsa_decode_noalloc_max_scratch()
    Bsz, Hkv, topk = 1 << 14, 8, 32                      # candidate lists alone exceed 1 MiB
    need = hsa.decode_workspace_size(Bsz, 8, Hkv, 64 * 1024, 128, 64, topk)
    assert need > cap
    A = 0x10000                                        # never dereferenced: rejected first
    st = hsa.lib().hsa_decode_noalloc(A, A, A, B.HSA_BF16, A, B.HSA_BF16, Bsz, 8, Hkv,
                                      64 * 1024, 128, 64, topk, 0.0, A, None, None)
    assert st == B.HSA_ERR_WORKSPACE
