"""Variable-length chunks on the GPU (hsa_prefill_varlen through the C ABI)
against the fp64 oracle's hsa_oracle_prefill_variant with the same boundaries,
element by element: chunks of 1 to 64 tokens, landmarks given or the DHSA
sqrt(|C|) * mean computed on the device, HiLS fusion or one softmax over the
union of the selected keys, on the tensor-core path (bf16, G = 8 and 16, one-
and multi-tile selection) and the CUDA-core path (fp32; bf16 with G = 4), plus
the degenerate boundaries (one chunk, single-token chunks, uniform 64-token
chunks, which must match the fixed-size prefill) and wrong boundaries, which
the device reports through hsa_check."""
import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_landmark_b200 as hsa
from hierarchical_chunk_sparse_landmark_b200 import _binding as B
from hierarchical_chunk_sparse_landmark_b200.workloads import (Workload, make_prefill_inputs,
                                                               make_varlen_bounds,
                                                               storage_dtype)
from oracle.parity import ATOL, W_ATOL, ParityReport, compare_outputs, compare_selection

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def varlen_lm(wl, n_chunks):
    g = torch.Generator(device=DEV)
    g.manual_seed(wl.seed + 100)
    lm = torch.randn(wl.B, wl.Hkv, n_chunks, wl.d, generator=g, device=DEV) * 2.0
    return lm.to(storage_dtype(wl))


def varlen_parity(oracle_lib, wl, bounds, *, dhsa, union, own=1, rows=None):
    x = make_prefill_inputs(wl.with_(landmarks="dhsa"), DEV)
    n = len(bounds) - 1
    lm = None if dhsa else varlen_lm(wl, n)
    Bsz, L, H, d = x["Q"].shape
    ws = torch.zeros(max(256, hsa.prefill_varlen_workspace_size(Bsz, H, wl.Hkv, L, d, n,
                                                                 wl.topk)),
                     dtype=torch.uint8, device=DEV)
    O, idx, w = hsa.prefill_varlen(x["Q"], x["K"], x["V"], bounds, lm, topk=wl.topk,
                                   own_chunk=own, union_softmax=union, idx_out=True,
                                   w_out=True, ws=ws)
    kernels = hsa.last_call_kernels()
    hsa.check(ws)
    ref = oracle_lib.prefill_variant(_f64(x["Q"]), _f64(x["K"]), _f64(x["V"]), _f64(lm), 64,
                                     wl.topk, own, union_softmax=int(union), rows=rows,
                                     bounds=bounds)
    r = ref["rows"]
    rep = ParityReport(rows=len(r))
    got_idx = idx.reshape(Bsz * L, wl.Hkv, wl.topk).cpu().numpy()[r]
    differs = compare_selection(ref["idx"], ref["sbar"], ref["gap"], ref["smag"], got_idx, rep)
    assert not differs.any(), "near-tie rows with a different set: use another seed"
    compare_outputs(ref["O"], _f64(O).reshape(Bsz * L, H, d)[r], ATOL[wl.dtype], rep)
    same = np.all(ref["idx"] == got_idx, axis=(1, 2))
    got_w = _f64(w).reshape(Bsz * L, H, wl.topk)[r]
    werr = np.abs(ref["w"][same] - got_w[same]).max() if same.any() else 0.0
    if werr > W_ATOL:
        rep.failures.append(f"w: max abs err {werr:.3e}")
    return rep, kernels, x, lm, (O, idx, w)


CASES = [(False, 0, 1), (True, 0, 1), (False, 1, 1), (True, 1, 0), (False, 0, 0)]


@pytest.mark.parametrize("dhsa,union,own", CASES)
@pytest.mark.parametrize("H,Hkv,d", [(16, 2, 128), (8, 1, 64)])
def test_varlen_tensor_core_path(oracle_lib, dhsa, union, own, H, Hkv, d):
    seed = 3 + 2 * dhsa + 5 * union + own + d
    wl = Workload("varlen", "prefill", "bf16", B=2, L=64 * 21 + 29, H=H, Hkv=Hkv, d=d, topk=5,
                  seed=seed)
    bounds = make_varlen_bounds(wl.L, seed, 1, 64)
    rep, kernels, *_ = varlen_parity(oracle_lib, wl, bounds, dhsa=dhsa, union=union, own=own)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])
    assert kernels & B.K_ATTEND_TC and kernels & B.K_SELECT_TC_ONE_TILE, hex(kernels)
    assert bool(kernels & B.K_LANDMARKS) == dhsa, hex(kernels)


@pytest.mark.parametrize("dhsa,union,own", CASES)
@pytest.mark.parametrize("dtype,H,Hkv", [("f32", 4, 1), ("bf16", 8, 2)])
def test_varlen_cuda_core_path(oracle_lib, dhsa, union, own, dtype, H, Hkv):
    seed = 17 + 2 * dhsa + 5 * union + own
    wl = Workload("varlen", "prefill", dtype, B=1, L=64 * 13 + 7, H=H, Hkv=Hkv, d=64, topk=4,
                  seed=seed)
    bounds = make_varlen_bounds(wl.L, seed, 1, 64)
    rep, kernels, *_ = varlen_parity(oracle_lib, wl, bounds, dhsa=dhsa, union=union, own=own)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])
    assert kernels & B.K_ATTEND_SIMT, hex(kernels)


@pytest.mark.parametrize("union", [0, 1])
def test_varlen_multi_tile_selection(oracle_lib, union):
    # about 190 chunks of 16..48 tokens: the multi-tile selection kernel; rows sampled
    wl = Workload("varlen", "prefill", "bf16", B=1, L=6000, H=16, Hkv=2, d=128, topk=8,
                  seed=50 + union)
    bounds = make_varlen_bounds(wl.L, wl.seed, 16, 48)
    assert len(bounds) - 1 > 128
    rows = np.unique(np.concatenate([np.arange(0, wl.L, 7), np.arange(wl.L - 300, wl.L)]))
    rep, kernels, *_ = varlen_parity(oracle_lib, wl, bounds, dhsa=True, union=union, rows=rows)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])
    assert kernels & B.K_SELECT_TC_MULTI_TILE, hex(kernels)


@pytest.mark.parametrize("dtype,H,Hkv", [("bf16", 16, 2), ("f32", 4, 1)])
@pytest.mark.parametrize("shape", ["one_chunk", "single_tokens", "ragged_tail"])
def test_varlen_degenerate_boundaries(oracle_lib, dtype, H, Hkv, shape):
    if shape == "one_chunk":            # no selection: causal attention inside one chunk
        L, bounds = 50, [0, 50]
    elif shape == "single_tokens":      # every chunk is one token
        L = 64
        bounds = list(range(L + 1))
    else:                               # 64-token chunks and a one-token tail
        L = 64 * 6 + 1
        bounds = list(range(0, L, 64)) + [L]
    wl = Workload("varlen", "prefill", dtype, B=2, L=L, H=H, Hkv=Hkv, d=64, topk=3,
                  seed=len(shape))
    rep, _, _, _, (O, idx, w) = varlen_parity(oracle_lib, wl, bounds, dhsa=True, union=0)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])
    if shape == "one_chunk":
        assert (idx == -1).all()


@pytest.mark.parametrize("dhsa", [False, True])
def test_uniform_varlen_matches_fixed_chunks(oracle_lib, dhsa):
    # L a multiple of 64 and 64-token chunks: the same method as hsa_prefill
    wl = Workload("varlen", "prefill", "bf16", B=1, L=64 * 12, H=16, Hkv=2, d=128, topk=4,
                  seed=9 + dhsa)
    bounds = list(range(0, wl.L + 1, 64))
    rep, _, x, lm, (O, idx, w) = varlen_parity(oracle_lib, wl, bounds, dhsa=dhsa, union=0)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])
    O2, idx2, w2 = hsa.prefill(x["Q"], x["K"], x["V"], lm, S=64, topk=wl.topk, idx_out=True,
                               w_out=True)
    assert torch.equal(idx, idx2)
    torch.testing.assert_close(O.float(), O2.float(), atol=ATOL[wl.dtype], rtol=0)
    torch.testing.assert_close(w, w2, atol=W_ATOL, rtol=0)


@pytest.mark.parametrize("bad", ["not_increasing", "too_long", "wrong_end", "nonzero_start"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_varlen_wrong_boundaries_are_reported(bad, dtype):
    wl = Workload("varlen", "prefill", dtype, B=1, L=300, H=16, Hkv=2, d=64, topk=3, seed=1)
    x = make_prefill_inputs(wl.with_(landmarks="dhsa"), DEV)
    bounds = make_varlen_bounds(wl.L, 5, 20, 60)
    if bad == "not_increasing":
        bounds[3] = bounds[2]
    elif bad == "too_long":
        bounds = [0, 65] + list(range(115, wl.L, 50)) + [wl.L]
    elif bad == "wrong_end":
        bounds[-1] = wl.L - 1
    else:
        bounds[0] = 1
    n = len(bounds) - 1
    ws = torch.zeros(hsa.prefill_varlen_workspace_size(1, 16, 2, wl.L, 64, n, 3),
                     dtype=torch.uint8, device=DEV)
    O, idx, _ = hsa.prefill_varlen(x["Q"], x["K"], x["V"], bounds, topk=3, ws=ws, idx_out=True)
    with pytest.raises(hsa.HSAError) as e:
        hsa.check(ws)
    assert e.value.status == B.HSA_ERR_INVALID_ARG
    hsa.check(ws)                       # the check cleared the flag
    # the call computed with the even split of the tokens into n chunks
    even = [c * wl.L // n for c in range(n + 1)]
    O2, idx2, _ = hsa.prefill_varlen(x["Q"], x["K"], x["V"], even, topk=3, ws=ws, idx_out=True)
    hsa.check(ws)
    assert torch.equal(idx, idx2) and torch.equal(O, O2)


def test_varlen_host_argument_checks():
    wl = Workload("varlen", "prefill", "bf16", B=1, L=200, H=16, Hkv=2, d=64, topk=3, seed=1)
    x = make_prefill_inputs(wl.with_(landmarks="dhsa"), DEV)
    with pytest.raises(hsa.HSAError) as e:   # 3 chunks cannot cover 200 tokens at <= 64 each
        hsa.prefill_varlen(x["Q"], x["K"], x["V"], [0, 64, 128, 200], topk=3)
    assert e.value.status == B.HSA_ERR_INVALID_ARG
    assert hsa.prefill_varlen_workspace_size(1, 16, 2, 200, 64, 3, 3) == 0
    with pytest.raises(ValueError):
        hsa.prefill_varlen(x["Q"], x["K"], x["V"], [0, 100, 200], torch.zeros(
            1, 2, 3, 64, device=DEV), topk=3)
