"""Context-parallel decode on the GPU: the cache cut into contiguous chunk
ranges (shards), each shard run through the C ABI's four steps in turn on one
GPU (candidates, merge, per-shard fusion state, combine), compared with the
single-GPU decode of the same inputs (selection bit-identical) and with the
fp64 oracle (selection exact modulo near-ties, O within 2e-2 / 1e-4).  The
exchanges between ranks are the stacking of the shards' outputs here; on
several GPUs they are NCCL all-gathers (decode_context_parallel)."""
import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_landmark_b200 as hsa
from hierarchical_chunk_sparse_landmark_b200 import _binding as B
from hierarchical_chunk_sparse_landmark_b200.workloads import Workload, make_decode_inputs
from oracle import gather_chunks
from oracle.context_parallel import shard_ranges
from oracle.parity import ATOL, ParityReport, compare_outputs, compare_selection

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def sharded_decode(x, wl, ranges, topk=None):
    """The four steps over `ranges` (chunk ranges [c0, c1)), one shard at a time."""
    topk = topk or wl.topk
    S = wl.S
    q, K, V, lm = x["q"], x["K"], x["V"], x["lm"]
    cand = [hsa.decode_cp_candidates(q, lm[:, :, c0:c1].contiguous(), c0, S=S, topk=topk)
            for c0, c1 in ranges]
    assert hsa.last_call_kernels() == B.K_DECODE_SCAN or ranges[-1][0] == ranges[-1][1]
    idx = hsa.decode_cp_merge(torch.stack([c[0] for c in cand]), torch.stack([c[1] for c in cand]))
    assert hsa.last_call_kernels() == B.K_DECODE_CP_MERGE
    st = [hsa.decode_cp_attend(q, K[:, :, c0 * S:c1 * S].contiguous(), V[:, :, c0 * S:c1 * S].contiguous(),
                               lm[:, :, c0:c1].contiguous(), c0, idx, S=S) for c0, c1 in ranges]
    O = hsa.decode_cp_combine(torch.stack([s[0] for s in st]), torch.stack([s[1] for s in st]),
                              torch.stack([s[2] for s in st]), dtype=q.dtype)
    assert hsa.last_call_kernels() == B.K_DECODE_CP_COMBINE
    hsa.check()
    return O, idx, cand


def oracle_check(oracle_lib, x, wl, O, idx, topk=None):
    topk = topk or wl.topk
    q, lm = _f64(x["q"]), _f64(x["lm"])
    sel = oracle_lib.decode_select(q, lm, topk)
    got = idx.cpu().numpy()
    rep = ParityReport(rows=wl.B)
    differs = compare_selection(sel["idx"], sel["sbar"], sel["gap"], sel["smag"], got, rep)
    use = np.where(differs[:, :, None], got, sel["idx"])
    ref = oracle_lib.decode_attend(q, lm, gather_chunks(x["K"], use, wl.S),
                                   gather_chunks(x["V"], use, wl.S), use, wl.S)
    compare_outputs(ref["O"], _f64(O), ATOL[wl.dtype], rep)
    return rep


@pytest.mark.parametrize("R", [1, 2, 3, 7])
@pytest.mark.parametrize("topk", [1, 4, 8])
def test_sharded_decode_matches_single_gpu_and_oracle(oracle_lib, R, topk):
    wl = Workload("cp", "decode", "bf16", B=3, L=64 * 1000, H=16, Hkv=2, d=128, topk=topk,
                  seed=R * 10 + topk)
    x = make_decode_inputs(wl, DEV)
    O, idx, _ = sharded_decode(x, wl, shard_ranges(wl.L // wl.S, R))
    O1, idx1 = hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=topk, idx_out=True)
    hsa.check()
    assert torch.equal(idx, idx1)                 # the same scores, the same total order
    rep = oracle_check(oracle_lib, x, wl, O, idx)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])
    assert (O.float() - O1.float()).abs().max().item() <= 2 * ATOL["bf16"]


@pytest.mark.parametrize("dtype,lm32,d,H,Hkv", [("f32", False, 64, 4, 1), ("bf16", True, 64, 16, 1),
                                                ("f32", True, 128, 8, 2)])
def test_sharded_decode_dtypes(oracle_lib, dtype, lm32, d, H, Hkv):
    wl = Workload("cp", "decode", dtype, B=2, L=64 * 300, H=H, Hkv=Hkv, d=d, topk=8, seed=5)
    x = make_decode_inputs(wl, DEV)
    if lm32:
        x["lm"] = x["lm"].float() * 1.3
    O, idx, _ = sharded_decode(x, wl, shard_ranges(wl.L // wl.S, 3))
    rep = oracle_check(oracle_lib, x, wl, O, idx)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:5])


def test_shards_smaller_than_topk_and_an_empty_shard(oracle_lib):
    # 20 chunks over shards of 0, 3, 2, 15 chunks with topk = 8: two shards
    # have fewer chunks than K, one has none (its candidates are all padding
    # and its state is empty)
    wl = Workload("cp", "decode", "bf16", B=2, L=64 * 20, H=16, Hkv=2, d=128, topk=8, seed=8)
    x = make_decode_inputs(wl, DEV)
    ranges = [(0, 0), (0, 3), (3, 5), (5, 20)]
    O, idx, cand = sharded_decode(x, wl, ranges)
    assert (cand[0][1] == -1).all()
    assert (cand[1][1][:, :, 3:] == -1).all() and (cand[1][1][:, :, :3] >= 0).all()
    O1, idx1 = hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=8, idx_out=True)
    hsa.check()
    assert torch.equal(idx, idx1)
    rep = oracle_check(oracle_lib, x, wl, O, idx)
    assert rep.ok, rep.summary()


def test_tie_across_shards_goes_to_the_lower_index(oracle_lib):
    # chunks 10 and 70 (shards 0 and 1 of 2) get the same landmark row, the
    # best of all; with topk = 1 the lower global index must win, with topk = 2
    # both are selected in index order
    wl = Workload("cp", "decode", "bf16", B=1, L=64 * 100, H=16, Hkv=2, d=128, topk=2, seed=12)
    x = make_decode_inputs(wl, DEV)
    G = wl.H // wl.Hkv
    qbar = x["q"].float().view(wl.B, wl.Hkv, G, wl.d).mean(2)
    row = (8.0 * wl.d ** 0.5 * qbar / (qbar * qbar).sum(-1, keepdim=True)).to(x["lm"].dtype)
    x["lm"][:, :, 10] = row
    x["lm"][:, :, 70] = row
    for topk, want in ((1, [10]), (2, [10, 70])):
        O, idx, _ = sharded_decode(x, wl, shard_ranges(100, 2), topk=topk)
        assert (idx.cpu().numpy() == np.array(want)).all(), idx
        rep = oracle_check(oracle_lib, x, wl.with_(topk=topk), O, idx, topk=topk)
        assert rep.ok, rep.summary()


def test_context_parallel_entry_without_a_process_group(oracle_lib):
    # decode_context_parallel on one rank (no process group): the shard is the
    # whole cache, and the result is the single-GPU decode's
    wl = Workload("cp", "decode", "bf16", B=2, L=64 * 200, H=16, Hkv=2, d=128, topk=8, seed=3)
    x = make_decode_inputs(wl, DEV)
    O, idx = hsa.decode_context_parallel(x["q"], x["K"], x["V"], x["lm"], 0, topk=8)
    O1, idx1 = hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=8, idx_out=True)
    hsa.check()
    assert torch.equal(idx, idx1)
    rep = oracle_check(oracle_lib, x, wl, O, idx)
    assert rep.ok, rep.summary()
