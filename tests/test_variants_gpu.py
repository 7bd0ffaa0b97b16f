"""Retrieval variants on the GPU (hsa_prefill_variant through the C ABI)
against the fp64 oracle's hsa_oracle_prefill_variant, element by element on
every row: one selection per block of R tokens (R = 1, 8, 64) decided by the
block's first token or by the mean of its queries (DHSA's chunk-level query at
R = S), and the HiLS fusion or one softmax over the union of the selected
keys (the DHSA form), on the tensor-core path (bf16, G = 8 and 16) and the
CUDA-core path (fp32; bf16 with G = 4)."""
import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_landmark_b200 as hsa
from hierarchical_chunk_sparse_landmark_b200 import _binding as B
from hierarchical_chunk_sparse_landmark_b200.workloads import Workload, make_prefill_inputs
from oracle.parity import ATOL, W_ATOL, ParityReport, compare_outputs, compare_selection

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def variant_parity(oracle_lib, wl, x, R, pool, union, lm_override="workload"):
    lm = x["lm"] if lm_override == "workload" else lm_override
    Bsz, L, H, d = x["Q"].shape
    ws = torch.zeros(max(256, hsa.prefill_workspace_size(Bsz, H, wl.Hkv, L, d, wl.S, wl.topk)),
                     dtype=torch.uint8, device=DEV)
    O, idx, w = hsa.prefill(x["Q"], x["K"], x["V"], lm, S=wl.S, topk=wl.topk,
                            own_chunk=wl.own_chunk, idx_out=True, w_out=True, ws=ws,
                            retrieval_interval=R, pool_mean=pool, union_softmax=union)
    kernels = hsa.last_call_kernels()
    hsa.check(ws)
    K, V = _f64(x["K"]), _f64(x["V"])
    Qh = _f64(x["Q"])
    ref = oracle_lib.prefill_variant(Qh, K, V, _f64(lm), wl.S, wl.topk, wl.own_chunk,
                                     interval=R, pool_mean=int(pool), union_softmax=int(union))
    rep = ParityReport(rows=Bsz * L)
    got_idx = idx.reshape(Bsz * L, wl.Hkv, wl.topk).cpu().numpy()
    differs = compare_selection(ref["idx"], ref["sbar"], ref["gap"], ref["smag"], got_idx, rep)
    assert not differs.any(), "near-tie rows with a different set: use another seed"
    compare_outputs(ref["O"], _f64(O).reshape(Bsz * L, H, d), ATOL[wl.dtype], rep)
    # weights slot by slot where the order matches (near-tied neighbours may swap)
    same = np.all(ref["idx"] == got_idx, axis=(1, 2))
    got_w = _f64(w).reshape(ref["w"].shape)
    werr = np.abs(ref["w"][same] - got_w[same]).max() if same.any() else 0.0
    if werr > W_ATOL:
        rep.failures.append(f"w: max abs err {werr:.3e}")
    return rep, kernels, idx


CASES = [(1, 0, 1), (8, 0, 0), (8, 0, 1), (8, 1, 0), (64, 1, 0), (64, 1, 1), (2, 1, 1)]


@pytest.mark.parametrize("R,pool,union", CASES)
@pytest.mark.parametrize("H,Hkv,d", [(16, 2, 128), (16, 1, 64)])
def test_variants_tensor_core_path(oracle_lib, R, pool, union, H, Hkv, d):
    wl = Workload("var", "prefill", "bf16", B=2, L=64 * 23 + 37, H=H, Hkv=Hkv, d=d, topk=5,
                  landmarks="input_x2", seed=R + 3 * pool + 7 * union + d)
    x = make_prefill_inputs(wl, DEV)
    rep, kernels, _ = variant_parity(oracle_lib, wl, x, R, pool, union)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])
    assert kernels & B.K_ATTEND_TC and kernels & B.K_SELECT_TC_ONE_TILE, hex(kernels)


@pytest.mark.parametrize("R,pool,union", CASES)
@pytest.mark.parametrize("dtype,H,Hkv", [("f32", 4, 1), ("bf16", 8, 2)])
def test_variants_cuda_core_path(oracle_lib, R, pool, union, dtype, H, Hkv):
    wl = Workload("var", "prefill", dtype, B=1, L=64 * 17 + 9, H=H, Hkv=Hkv, d=64, topk=4,
                  landmarks="input_x2", seed=11 + R + pool + union)
    x = make_prefill_inputs(wl, DEV)
    rep, kernels, _ = variant_parity(oracle_lib, wl, x, R, pool, union)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])
    assert kernels & B.K_ATTEND_SIMT, hex(kernels)


@pytest.mark.parametrize("union", [0, 1])
def test_variants_multi_tile_selection_and_dhsa_landmarks(oracle_lib, union):
    # 150 chunks (the multi-tile selection kernel) with device DHSA landmarks,
    # per-8-token retrieval
    wl = Workload("var", "prefill", "bf16", B=1, L=64 * 150 + 11, H=16, Hkv=2, d=128, topk=8,
                  landmarks="dhsa", seed=40 + union)
    x = make_prefill_inputs(wl, DEV)
    rep, kernels, idx = variant_parity(oracle_lib, wl, x, 8, 0, union)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])
    assert kernels & B.K_SELECT_TC_MULTI_TILE, hex(kernels)
    # every token of a block of 8 shares its selection
    i = idx[0].cpu().numpy()
    assert (i.reshape(-1, 8, 2, 8)[:-1] == i.reshape(-1, 8, 2, 8)[:-1, :1]).all() if wl.L % 8 == 0 else True


def test_variant_rejects_an_interval_that_does_not_divide_the_chunk():
    wl = Workload("var", "prefill", "bf16", B=1, L=200, H=16, Hkv=2, d=128, topk=4)
    x = make_prefill_inputs(wl, DEV)
    with pytest.raises(hsa.HSAError) as e:
        hsa.prefill(x["Q"], x["K"], x["V"], x["lm"], topk=4, retrieval_interval=3)
    assert e.value.status == B.HSA_ERR_INVALID_ARG
