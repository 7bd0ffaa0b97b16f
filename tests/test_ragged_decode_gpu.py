"""Ragged-batch decode and incremental landmarks on the GPU, through the C ABI.

hsa_decode_ragged: sequence b of the batch holds lens[b] tokens of an Lmax
cache and retrieves among its first lens[b] // S chunks.  Checked against the
fp64 oracle's decode (selection and attention + fusion) run on each
sequence's visible landmark rows alone, element by element, for lengths from
0 to Lmax, including ragged tails; equal lengths give hsa_decode's bits; a
length outside 0 .. Lmax is reported by hsa_check.

hsa_landmarks_append: after growing caches, the newly completed chunks' rows
equal the oracle's sqrt(S) * mean landmarks and no other row changes; a cache
grown one token per call ends with the landmarks of its whole prefix."""
import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_landmark_b200 as hsa
from hierarchical_chunk_sparse_landmark_b200 import _binding as B
from hierarchical_chunk_sparse_landmark_b200.workloads import Workload, make_decode_inputs
from oracle import gather_chunks
from oracle.parity import ATOL, ParityReport, compare_outputs, compare_selection

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def ragged_parity(oracle_lib, wl, x, lens):
    lens_d = torch.tensor(lens, dtype=torch.int32, device=DEV)
    ws = torch.zeros(hsa.decode_workspace_size(wl.B, wl.H, wl.Hkv, wl.L, wl.d, wl.S, wl.topk),
                     dtype=torch.uint8, device=DEV)
    O, idx = hsa.decode_ragged(x["q"], x["K"], x["V"], x["lm"], lens_d, S=wl.S, topk=wl.topk,
                               idx_out=True, ws=ws)
    hsa.check(ws)
    rep = ParityReport()
    for b, n in enumerate(lens):
        nvis = n // wl.S
        got = idx[b:b + 1].cpu().numpy()
        if nvis == 0:
            assert (got == -1).all() and torch.all(O[b] == 0)
            rep.rows += 1
            continue
        q, lm = _np(x["q"][b:b + 1]), _np(x["lm"][b:b + 1, :, :nvis])
        sel = oracle_lib.decode_select(q, lm, wl.topk)
        rep.rows += 1
        differs = compare_selection(sel["idx"], sel["sbar"], sel["gap"], sel["smag"], got, rep)
        use = np.where(differs[:, :, None], got, sel["idx"])
        Kg = gather_chunks(x["K"][b:b + 1], use, wl.S)
        Vg = gather_chunks(x["V"][b:b + 1], use, wl.S)
        ref = oracle_lib.decode_attend(q, lm, Kg, Vg, use, wl.S)
        compare_outputs(ref["O"], _np(O[b:b + 1]), ATOL[wl.dtype], rep)
    return rep, (O, idx, ws)


@pytest.mark.parametrize("dtype,d,H,Hkv,topk", [("bf16", 128, 16, 2, 8), ("f32", 64, 4, 1, 3),
                                                ("bf16", 64, 16, 1, 32)])
def test_ragged_decode_matches_oracle(oracle_lib, dtype, d, H, Hkv, topk):
    Lmax = 64 * 700
    lens = [0, 37, 64 * 5, 64 * 9 + 13, Lmax, 64 * 333 + 63, 64]
    wl = Workload("rag", "decode", dtype, B=len(lens), L=Lmax, H=H, Hkv=Hkv, d=d, topk=topk,
                  seed=d + H + topk)
    x = make_decode_inputs(wl, DEV)
    rep, (O, idx, _) = ragged_parity(oracle_lib, wl, x, lens)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    # a sequence with fewer visible chunks than topk pads with -1
    assert (idx[2, :, 5:] == -1).all() if topk > 5 else True


def test_ragged_decode_with_equal_lengths_is_hsa_decode():
    wl = Workload("rag", "decode", "bf16", B=3, L=64 * 900, H=16, Hkv=2, d=128, topk=8, seed=4)
    x = make_decode_inputs(wl, DEV)
    lens = torch.full((3,), wl.L, dtype=torch.int32, device=DEV)
    O1, i1 = hsa.decode_ragged(x["q"], x["K"], x["V"], x["lm"], lens, topk=8, idx_out=True)
    O2, i2 = hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=8, idx_out=True)
    hsa.check()
    assert torch.equal(i1, i2) and torch.equal(O1, O2)


@pytest.mark.parametrize("bad", [-1, 64 * 10 + 1])
def test_ragged_decode_reports_lengths_out_of_range(bad):
    wl = Workload("rag", "decode", "bf16", B=2, L=64 * 10, H=16, Hkv=2, d=128, topk=4, seed=1)
    x = make_decode_inputs(wl, DEV)
    ws = torch.zeros(hsa.decode_workspace_size(2, 16, 2, wl.L, 128, 64, 4), dtype=torch.uint8,
                     device=DEV)
    lens = torch.tensor([64 * 3, bad], dtype=torch.int32, device=DEV)
    hsa.decode_ragged(x["q"], x["K"], x["V"], x["lm"], lens, topk=4, ws=ws)
    with pytest.raises(hsa.HSAError) as e:
        hsa.check(ws)
    assert e.value.status == B.HSA_ERR_INVALID_ARG
    hsa.check(ws)


@pytest.mark.parametrize("k_dtype,lm_dtype", [(torch.bfloat16, torch.float32),
                                              (torch.bfloat16, torch.bfloat16),
                                              (torch.float32, torch.float32)])
@pytest.mark.parametrize("d", [64, 128])
def test_landmarks_append_writes_only_completed_chunks(oracle_lib, k_dtype, lm_dtype, d):
    B_, Hkv, Lmax = 4, 2, 64 * 40
    g = torch.Generator(device=DEV)
    g.manual_seed(d)
    K = torch.randn(B_, Hkv, Lmax, d, generator=g, device=DEV).to(k_dtype)
    sentinel = 7.0
    lm = torch.full((B_, Hkv, Lmax // 64, d), sentinel, device=DEV).to(lm_dtype)
    before = [0, 63, 64 * 7 + 5, 64 * 39]
    after = [64 * 3, 64 * 2 + 1, 64 * 30, Lmax]
    lb = torch.tensor(before, dtype=torch.int32, device=DEV)
    la = torch.tensor(after, dtype=torch.int32, device=DEV)
    hsa.landmarks_append(K, lm, lb, la, max_new_chunks=2)   # a small grid hint still covers all
    torch.cuda.synchronize()
    ref = oracle_lib.landmarks(_np(K), 64)
    got = _np(lm)
    tol = 2.0 ** -8 if lm_dtype == torch.bfloat16 else 1e-5
    for b in range(B_):
        lo, hi = before[b] // 64, after[b] // 64
        new = got[b, :, lo:hi]
        np.testing.assert_allclose(new, ref[b, :, lo:hi], rtol=tol, atol=tol)
        untouched = np.concatenate([got[b, :, :lo], got[b, :, hi:]], axis=1)
        assert (untouched == sentinel).all()


def test_landmarks_append_token_by_token_equals_full_landmarks():
    B_, Hkv, Lmax, d = 2, 2, 64 * 6, 128
    g = torch.Generator(device=DEV)
    g.manual_seed(3)
    K = torch.randn(B_, Hkv, Lmax, d, generator=g, device=DEV).to(torch.bfloat16)
    lm = torch.zeros(B_, Hkv, Lmax // 64, d, device=DEV)
    full = hsa.landmarks(K)
    for n in range(Lmax):
        lb = torch.full((B_,), n, dtype=torch.int32, device=DEV)
        la = lb + 1
        hsa.landmarks_append(K, lm, lb, la)
    torch.cuda.synchronize()
    torch.testing.assert_close(lm, full, rtol=1e-6, atol=1e-6)
