"""Prefill backward on the GPU (hsa_prefill_backward through the C ABI) against
the fp64 restatement oracle/backward.py, element by element: dQ, dK, dV and
the landmark gradient (given landmarks) or its fold into dK (DHSA), with the
forward's selection held fixed on both sides.  Covers G = 1..16, d = 64 and
128, fp32 and bf16 inputs, bf16 and fp32 landmarks, own_chunk 0/1, a ragged
tail, a sequence shorter than one chunk, run-to-run bit reproducibility and
a selection entry that names an invisible chunk (reported by hsa_check).

Tolerances: on the CUDA-core path the GPU accumulates in fp32 (inputs are
exact in both), so every gradient is compared as max |gpu - oracle| <= 1e-4 *
max |oracle| of that tensor, well above the fp32 rounding of sums of a few
thousand terms (~1e-6 relative) and of expf.  The tensor-core path (bf16, G = 8,
d = 128) rounds P and dS to bf16 before the second products (2^-9 relative per
term, as the forward rounds P), so it is held to 1e-2 * max |oracle|: a 5x
margin over that rounding, still far below any dropped or misplaced term."""
import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_landmark_b200 as hsa
from hierarchical_chunk_sparse_landmark_b200 import _binding as B
from hierarchical_chunk_sparse_landmark_b200.workloads import (Workload, make_prefill_inputs,
                                                               storage_dtype)
from oracle import backward as obwd

pytestmark = pytest.mark.gpu
DEV = "cuda"
RTOL = 1e-4
RTOL_TC = 1e-2


def _f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def _close(name, got, ref, rtol=RTOL):
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(_f64(got) - ref).max()
    assert err <= rtol * scale, f"{name}: max abs err {err:.3e} vs {rtol:.0e} * {scale:.3e}"


def backward_parity(wl, *, lm_mode="input", own=1, lm_dtype=None):
    x = make_prefill_inputs(wl.with_(landmarks="dhsa"), DEV)
    Q, K, V = x["Q"], x["K"], x["V"]
    Bsz, L, H, d = Q.shape
    lm = None
    if lm_mode == "input":
        g = torch.Generator(device=DEV)
        g.manual_seed(wl.seed + 7)
        lm = (2.0 * torch.randn(Bsz, wl.Hkv, L // 64, d, generator=g, device=DEV)).to(
            lm_dtype or storage_dtype(wl))
    # the forward's selection (held fixed in the backward)
    _, idx, _ = hsa.prefill(Q, K, V, lm, topk=wl.topk, own_chunk=own, idx_out=True)
    g = torch.Generator(device=DEV)
    g.manual_seed(wl.seed + 11)
    dO = torch.randn(Bsz, L, H, d, generator=g, device=DEV).to(Q.dtype)
    ws = torch.zeros(hsa.prefill_backward_workspace_size(Bsz, H, wl.Hkv, L, d, 64, wl.topk,
                                                         lm is None),
                     dtype=torch.uint8, device=DEV)
    dQ, dK, dV, dlm = hsa.prefill_backward(Q, K, V, idx, dO, lm, own_chunk=own, ws=ws)
    kernels = hsa.last_call_kernels()
    hsa.check(ws)
    ref = obwd.prefill_backward(_f64(Q), _f64(K), _f64(V), _f64(lm), 64, wl.topk, own, _f64(dO),
                                idx=idx.cpu().numpy().astype(np.int64))
    tc = bool(kernels & B.K_BACKWARD_TC)
    assert tc == (Q.dtype == torch.bfloat16 and H // wl.Hkv == 8 and d == 128), hex(kernels)
    rtol = RTOL_TC if tc else RTOL
    _close("dQ", dQ, ref["dQ"], rtol)
    _close("dK", dK, ref["dK"], rtol)
    _close("dV", dV, ref["dV"], rtol)
    if lm is None:
        assert dlm is None
    else:
        _close("dlm", dlm, ref["dlm"], rtol)
    assert kernels & B.K_BACKWARD, hex(kernels)
    return (Q, K, V, idx, dO, lm, own, ws), (dQ, dK, dV, dlm)


@pytest.mark.parametrize("lm_mode", ["input", "dhsa"])
@pytest.mark.parametrize("dtype,H,Hkv,d", [("f32", 4, 1, 64), ("bf16", 16, 2, 128),
                                           ("bf16", 16, 1, 64), ("f32", 8, 8, 128)])
def test_backward_matches_oracle(dtype, H, Hkv, d, lm_mode):
    wl = Workload("bwd", "prefill", dtype, B=2, L=64 * 7 + 23, H=H, Hkv=Hkv, d=d, topk=4,
                  seed=3 + H + d + (lm_mode == "dhsa"))
    backward_parity(wl, lm_mode=lm_mode)


@pytest.mark.parametrize("lm_mode", ["input", "dhsa"])
def test_backward_without_own_chunk(lm_mode):
    wl = Workload("bwd", "prefill", "bf16", B=1, L=64 * 6 + 5, H=8, Hkv=2, d=128, topk=3, seed=21)
    backward_parity(wl, lm_mode=lm_mode, own=0)


def test_backward_fp32_landmarks_with_bf16_inputs():
    wl = Workload("bwd", "prefill", "bf16", B=1, L=64 * 5 + 40, H=16, Hkv=2, d=64, topk=2, seed=5)
    backward_parity(wl, lm_mode="input", lm_dtype=torch.float32)


def test_backward_wide_selection_many_segments():
    # topk 8 over 20 chunks with G = 16: chunk 0 is selected by most tokens, so its
    # entries span several key segments (1024 query rows each)
    wl = Workload("bwd", "prefill", "bf16", B=1, L=64 * 20, H=16, Hkv=1, d=64, topk=8, seed=8)
    backward_parity(wl, lm_mode="input")


@pytest.mark.parametrize("L", [1, 37, 64])
def test_backward_short_sequences(L):
    # no chunk before the token's own: only the own-chunk term (or nothing)
    wl = Workload("bwd", "prefill", "f32", B=2, L=L, H=4, Hkv=2, d=64, topk=2, seed=L)
    backward_parity(wl, lm_mode="dhsa")


def test_backward_is_bit_reproducible():
    wl = Workload("bwd", "prefill", "bf16", B=1, L=64 * 9 + 3, H=16, Hkv=2, d=128, topk=4, seed=31)
    (Q, K, V, idx, dO, lm, own, ws), first = backward_parity(wl, lm_mode="input")
    again = hsa.prefill_backward(Q, K, V, idx, dO, lm, own_chunk=own, ws=ws)
    for a, b in zip(first, again):
        assert torch.equal(a, b)


def test_backward_reports_an_invisible_selection():
    wl = Workload("bwd", "prefill", "bf16", B=1, L=64 * 4, H=8, Hkv=1, d=64, topk=2, seed=2)
    x = make_prefill_inputs(wl.with_(landmarks="dhsa"), DEV)
    idx = torch.full((1, wl.L, 1, 2), -1, dtype=torch.int32, device=DEV)
    idx[0, 70, 0, 0] = 1            # token 70 is in chunk 1: chunk 1 is not visible
    dO = torch.ones_like(x["Q"])
    ws = torch.zeros(hsa.prefill_backward_workspace_size(1, 8, 1, wl.L, 64, 64, 2, True),
                     dtype=torch.uint8, device=DEV)
    hsa.prefill_backward(x["Q"], x["K"], x["V"], idx, dO, None, ws=ws)
    with pytest.raises(hsa.HSAError) as e:
        hsa.check(ws)
    assert e.value.status == B.HSA_ERR_INVALID_ARG
    hsa.check(ws)


@pytest.mark.parametrize("lm_mode", ["input", "dhsa"])
@pytest.mark.parametrize("own", [0, 1])
def test_backward_tensor_core_path_agrees_with_cuda_cores(lm_mode, own):
    # the same inputs on both paths (the CUDA-core one forced by the path
    # override): they differ only by the bf16 rounding of P and dS
    wl = Workload("bwd", "prefill", "bf16", B=2, L=64 * 11 + 17, H=16, Hkv=2, d=128, topk=6,
                  seed=40 + own + 2 * (lm_mode == "dhsa"))
    x = make_prefill_inputs(wl.with_(landmarks="dhsa"), DEV)
    lm = None
    if lm_mode == "input":
        lm = 2.0 * torch.randn(2, 2, wl.L // 64, 128, device=DEV)
    _, idx, _ = hsa.prefill(x["Q"], x["K"], x["V"], lm, topk=6, own_chunk=own, idx_out=True)
    dO = torch.randn_like(x["Q"].float()).to(torch.bfloat16)
    tc = hsa.prefill_backward(x["Q"], x["K"], x["V"], idx, dO, lm, own_chunk=own)
    assert hsa.last_call_kernels() & B.K_BACKWARD_TC
    with hsa.path_overrides(B.PATH_SIMT_PREFILL):
        ref = hsa.prefill_backward(x["Q"], x["K"], x["V"], idx, dO, lm, own_chunk=own)
        assert not hsa.last_call_kernels() & B.K_BACKWARD_TC
    hsa.check()
    for name, a, r in zip(("dQ", "dK", "dV", "dlm"), tc, ref):
        if r is not None:
            _close(name, a, _f64(r), RTOL_TC)


@pytest.mark.parametrize("topk", [12, 29])
def test_backward_tensor_core_more_than_eight_slots(topk):
    # the fusion-weight kernel takes slots in groups of four and the row
    # finish loops over every slot: K above eight spans several groups
    wl = Workload("bwd", "prefill", "bf16", B=1, L=64 * 34 + 9, H=16, Hkv=2, d=128, topk=topk,
                  seed=60 + topk)
    backward_parity(wl, lm_mode="input")
    backward_parity(wl.with_(seed=61 + topk), lm_mode="dhsa")


def test_backward_tensor_core_long_chunk_lists():
    # 40 chunks, top-8, G = 8: chunk 0's entries span several segments of 8 tiles
    wl = Workload("bwd", "prefill", "bf16", B=1, L=64 * 40, H=8, Hkv=1, d=128, topk=8, seed=77)
    backward_parity(wl, lm_mode="input")


def test_backward_long_sequence_paths_agree():
    # 512 chunks, DHSA landmarks: long per-chunk entry lists (chunk 0 is selected by
    # thousands of tokens) on both paths; the CUDA-core path is the fp32 reference
    wl = Workload("bwd", "prefill", "bf16", B=1, L=32768, H=16, Hkv=2, d=128, topk=8, seed=123)
    x = make_prefill_inputs(wl.with_(landmarks="dhsa"), DEV)
    _, idx, _ = hsa.prefill(x["Q"], x["K"], x["V"], None, topk=8, idx_out=True)
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    dO = torch.randn(x["Q"].shape, generator=g, device=DEV).to(torch.bfloat16)
    tc = hsa.prefill_backward(x["Q"], x["K"], x["V"], idx, dO, None)
    assert hsa.last_call_kernels() & B.K_BACKWARD_TC
    with hsa.path_overrides(B.PATH_SIMT_PREFILL):
        ref = hsa.prefill_backward(x["Q"], x["K"], x["V"], idx, dO, None)
    hsa.check()
    for name, a, r in zip(("dQ", "dK", "dV"), tc[:3], ref[:3]):
        _close(name, a, _f64(r), RTOL_TC)
