"""hsa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin inside a host program that owns all device memory, or
code that must not call cudaMalloc/cudaFree on a latency-critical path)
cannot pass hsa_decode a workspace; hsa_decode_noalloc uses the library's
fixed device array instead.  This file is collected last so that a run which
stops at the first failure has already run every other test; it also passes
on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_landmark_b200 as hsa
from hierarchical_chunk_sparse_landmark_b200 import _binding as B
from hierarchical_chunk_sparse_landmark_b200.workloads import Workload, make_decode_inputs
from oracle import gather_chunks
from oracle.parity import ATOL, ParityReport, compare_outputs, compare_selection


def _f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_on_two_calls(oracle_lib):
    wl = Workload("noalloc", "decode", "bf16", B=4, L=64 * 3000, H=16, Hkv=2, d=128, topk=8,
                  seed=21)
    x = make_decode_inputs(wl, "cuda")
    O_ref, idx_ref = hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=wl.topk, idx_out=True)
    hsa.check()
    # the oracle on the same inputs
    q, lm = _f64(x["q"]), _f64(x["lm"])
    sel = oracle_lib.decode_select(q, lm, wl.topk)
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
        # the same kernels on the same inputs: bit-identical to hsa_decode
        assert torch.equal(idx, idx_ref), call
        assert torch.equal(O, O_ref), call
        # and within the bf16 tolerance of the fp64 oracle
        rep = ParityReport(rows=wl.B)
        got = idx.cpu().numpy()
        differs = compare_selection(sel["idx"], sel["sbar"], sel["gap"], sel["smag"], got, rep)
        use = np.where(differs[:, :, None], got, sel["idx"])
        ref = oracle_lib.decode_attend(q, lm, gather_chunks(x["K"], use, wl.S),
                                       gather_chunks(x["V"], use, wl.S), use, wl.S)
        compare_outputs(ref["O"], _f64(O), ATOL["bf16"], rep)
        assert rep.ok, (call, rep.summary(), rep.failures[:3])


@pytest.mark.gpu
def test_noalloc_decode_reports_a_device_timeout_once():
    # The bounded-wait failure path aimed at the array's status word (a wait
    # that nothing completes gives up after ~1 ms; no fault, no hang):
    # hsa_check(NULL, stream) reports it exactly once, and the next call works.
    lib = hsa.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.hsa_selftest_wait_expiry(None, 0, 2_000_000, stream) == B.HSA_OK
    assert lib.hsa_check(None, stream) == B.HSA_ERR_TIMEOUT
    assert lib.hsa_check(None, stream) == B.HSA_OK
    wl = Workload("noalloc2", "decode", "bf16", B=2, L=64 * 500, H=16, Hkv=2, d=128, topk=8,
                  seed=22)
    x = make_decode_inputs(wl, "cuda")
    O_ref, idx_ref = hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=wl.topk, idx_out=True)
    O, idx = hsa.decode_noalloc(x["q"], x["K"], x["V"], x["lm"], topk=wl.topk, idx_out=True)
    assert lib.hsa_check(None, stream) == B.HSA_OK
    assert torch.equal(idx, idx_ref) and torch.equal(O, O_ref)


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
