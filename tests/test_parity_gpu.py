"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases are compared element by element over every row (several 64-token
tiles and a ragged tail); the five named workloads run at full size in the
launch configuration the benchmark times and are compared on sampled rows.
Selection must match the oracle exactly except at near-ties (see
oracle/parity.py); outputs within 2e-2 (bf16) / 1e-4 (fp32) max-abs.
"""
import math

import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_landmark_b200 as hsa
from hierarchical_chunk_sparse_landmark_b200 import _binding as B
from hierarchical_chunk_sparse_landmark_b200.workloads import (WORKLOADS, Workload,
                                                               make_decode_inputs,
                                                               make_prefill_inputs)
from oracle import gather_chunks
from oracle.parity import ATOL, W_ATOL, ParityReport, compare_outputs, compare_selection

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype == torch.bfloat16 \
        else t.detach().cpu().numpy().astype(np.float64)


TC_PATH = B.K_WORK_LISTS | B.K_ATTEND_TC | B.K_FUSE


def expect_tc_path(kernels: int, tc: bool):
    """The dispatch took the tensor-core chain (tc) or the CUDA-core path."""
    if tc:
        assert kernels & TC_PATH == TC_PATH and not kernels & B.K_ATTEND_SIMT, hex(kernels)
    else:
        assert kernels & B.K_ATTEND_SIMT and not kernels & B.K_ATTEND_TC, hex(kernels)


_WORKLOAD_LM = object()


def prefill_parity(oracle_lib, wl: Workload, x: dict, rows=None, lm_override=_WORKLOAD_LM,
                   scale=0.0, report=None):
    """Run hsa.prefill on x and compare rows (flattened b*L+t; default all).
    The call gets its own zero-filled workspace, whose status word is checked;
    the kernel families it launched are returned in ``report.kernels``."""
    lm = x["lm"] if lm_override is _WORKLOAD_LM else lm_override     # None: DHSA landmarks
    B_, L_, H_, d_ = x["Q"].shape
    ws = torch.zeros(max(256, hsa.prefill_workspace_size(B_, H_, wl.Hkv, L_, d_, wl.S, wl.topk)),
                     dtype=torch.uint8, device=DEV)
    O, idx, w = hsa.prefill(x["Q"], x["K"], x["V"], lm, S=wl.S, topk=wl.topk,
                            own_chunk=wl.own_chunk, scale=scale, idx_out=True, w_out=True, ws=ws)
    kernels = hsa.last_call_kernels()
    hsa.check(ws)
    B, L, H, d = x["Q"].shape
    Hkv = wl.Hkv
    if rows is None:
        rows = np.arange(B * L, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    Qr = _np(x["Q"].reshape(B * L, H, d)[torch.as_tensor(rows, device=DEV)])
    K, V = _np(x["K"]), _np(x["V"])
    lmh = None if lm is None else _np(lm)
    ref = oracle_lib.prefill(None, K, V, lmh, wl.S, wl.topk, wl.own_chunk, scale, rows=rows,
                             Q_rows=Qr)
    rt = torch.as_tensor(rows, device=DEV)
    got_idx = idx.reshape(B * L, Hkv, wl.topk)[rt].cpu().numpy()
    got_w = w.reshape(B * L, H, wl.topk)[rt].cpu().numpy().astype(np.float64)
    got_O = _np(O.reshape(B * L, H, d)[rt])
    rep = report or ParityReport()
    rep.kernels = kernels
    rep.rows += len(rows)
    differs = compare_selection(ref["idx"], ref["sbar"], ref["gap"], ref["smag"], got_idx, rep)
    ref_O = ref["O"]
    if differs.any():   # near-ties: recompute those rows on the device's selection
        sel = np.where(differs.any(axis=1))[0]
        forced = oracle_lib.prefill(None, K, V, lmh, wl.S, wl.topk, wl.own_chunk, scale,
                                    rows=rows[sel], Q_rows=Qr[sel], forced_idx=got_idx[sel])
        ref_O = ref_O.copy()
        ref_O[sel] = forced["O"]
    compare_outputs(ref_O, got_O, ATOL[wl.dtype], rep)
    same = np.all(ref["idx"] == got_idx, axis=(1, 2))
    if same.any():
        werr = np.abs(ref["w"][same] - got_w[same]).max()
        rep.max_w_err = max(rep.max_w_err, float(werr))
        if werr > W_ATOL:
            rep.failures.append(f"w: max abs err {werr:.3e}")
    return rep, (O, idx, w)


def small(dtype, B=2, L=337, H=8, Hkv=2, d=128, topk=3, own=1, lm="input", seed=0):
    return Workload("small", "prefill", dtype, B=B, L=L, H=H, Hkv=Hkv, d=d, S=64, topk=topk,
                    own_chunk=own, landmarks=lm, seed=seed)


# ------------------------------------------------------------------ small, every row
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,Hkv", [(4, 1), (8, 2), (16, 2), (16, 1), (2, 2)])
def test_prefill_small_all_rows(oracle_lib, dtype, d, H, Hkv):
    wl = small(dtype, H=H, Hkv=Hkv, d=d, seed=H * 7 + d)
    x = make_prefill_inputs(wl, DEV)
    rep, _ = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    expect_tc_path(rep.kernels, dtype == "bf16" and H // Hkv in (8, 16))


@pytest.mark.parametrize("topk", [1, 2, 8, 17, 32])
@pytest.mark.parametrize("own", [0, 1])
@pytest.mark.parametrize("H,Hkv,d", [(8, 2, 128), (16, 2, 128), (16, 1, 64)])
def test_prefill_topk_and_own_chunk(oracle_lib, topk, own, H, Hkv, d):
    # G = 4 takes the CUDA-core path, G = 8 and 16 the tensor-core chain
    # (own_chunk = 0 there still computes the own tiles, with weight 0)
    wl = small("bf16", B=1, L=64 * 40 + 5, H=H, Hkv=Hkv, d=d, topk=topk, own=own, seed=topk)
    x = make_prefill_inputs(wl, DEV)
    rep, (O, idx, w) = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    expect_tc_path(rep.kernels, H // Hkv in (8, 16))
    if not own:   # no visible chunk and no own term: exactly zero
        assert torch.all(O[:, :64] == 0)


@pytest.mark.parametrize("lm_kind", ["dhsa", "f32"])
@pytest.mark.parametrize("H,Hkv", [(8, 2), (16, 2)])
def test_prefill_landmark_modes(oracle_lib, lm_kind, H, Hkv):
    wl = small("bf16", B=2, L=64 * 9 + 31, H=H, Hkv=Hkv,
               lm="dhsa" if lm_kind == "dhsa" else "input")
    x = make_prefill_inputs(wl, DEV)
    lm = None if lm_kind == "dhsa" else x["lm"].float()
    rep, _ = prefill_parity(oracle_lib, wl, x, lm_override=lm)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    expect_tc_path(rep.kernels, H // Hkv == 8)
    assert bool(rep.kernels & B.K_LANDMARKS) == (lm_kind == "dhsa")


@pytest.mark.parametrize("seed", [5, 11, 23])
def test_prefill_large_outputs(oracle_lib, seed):
    # Few visible chunks and doubled landmarks concentrate the attention, so |O|
    # approaches max |V| and the rounding of the chunk outputs matters most.
    wl = Workload("concentrated", "prefill", "bf16", B=1, L=64 * 6 + 9, H=16, Hkv=2, d=128,
                  S=64, topk=4, landmarks="input_x2", seed=seed)
    x = make_prefill_inputs(wl, DEV)
    rep, _ = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])


@pytest.mark.parametrize("tiles", ["one", "multi"])
@pytest.mark.parametrize("lm_kind", ["bf16", "f32", "dhsa"])
@pytest.mark.parametrize("H,Hkv", [(16, 2), (16, 1)])
@pytest.mark.parametrize("d", [64, 128])
def test_prefill_tc_selection_branches(oracle_lib, tiles, lm_kind, H, Hkv, d):
    # Every tensor-core selection kernel the dispatch can launch, element by
    # element: one score tile (up to 128 chunks; qbar built per 64-column
    # block, two blocks per SM) and the multi-tile kernel (forced here on the
    # same shape), each with bf16 landmarks (3 qbar parts), fp32 landmarks
    # split into two bf16 planes (2 x 2 parts) and the DHSA landmarks computed
    # on the device (fp32, same split), at d = 64 and 128 and G = 8 and 16.
    wl = small("bf16", B=2, L=64 * 33 + 17, H=H, Hkv=Hkv, d=d, topk=8, seed=41 + d + H // Hkv)
    x = make_prefill_inputs(wl, DEV)
    lm = {"bf16": x["lm"], "f32": x["lm"].float() * 1.25, "dhsa": None}[lm_kind]
    flags = B.PATH_MULTI_TILE_SELECT if tiles == "multi" else 0
    with hsa.path_overrides(flags):
        rep, _ = prefill_parity(oracle_lib, wl, x, lm_override=lm)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    expect_tc_path(rep.kernels, True)
    want = B.K_SELECT_TC_MULTI_TILE if tiles == "multi" else B.K_SELECT_TC_ONE_TILE
    assert rep.kernels & want, hex(rep.kernels)
    assert bool(rep.kernels & B.K_SPLIT_LANDMARKS) == (lm_kind != "bf16")


@pytest.mark.parametrize("lm_kind", ["bf16", "f32", "dhsa"])
@pytest.mark.parametrize("H,Hkv,d", [(16, 2, 128), (16, 1, 64)])
def test_prefill_tc_selection_above_one_tile(oracle_lib, lm_kind, H, Hkv, d):
    # 150 chunks: the multi-tile kernel is the dispatch's own choice; every
    # landmark mode, sampled rows including the chunks next to the tile edge.
    wl = small("bf16", B=1, L=64 * 150 + 7, H=H, Hkv=Hkv, d=d, topk=8, seed=300 + d)
    x = make_prefill_inputs(wl, DEV)
    lm = {"bf16": x["lm"], "f32": x["lm"].float(), "dhsa": None}[lm_kind]
    rng = np.random.default_rng(d)
    edges = np.concatenate([np.arange(c * 64 - 2, c * 64 + 3) for c in (1, 127, 128, 129, 149)])
    rows = np.unique(np.concatenate([rng.integers(0, wl.L, 500), edges, np.arange(wl.L - 70, wl.L)]))
    rep, _ = prefill_parity(oracle_lib, wl, x, rows=rows, lm_override=lm)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    assert rep.kernels & B.K_SELECT_TC_MULTI_TILE, hex(rep.kernels)
    expect_tc_path(rep.kernels, True)


@pytest.mark.parametrize("topk", [1, 3, 17, 32])
@pytest.mark.parametrize("tiles", ["one", "multi"])
def test_prefill_tc_selection_topk(oracle_lib, topk, tiles):
    # The tensor-core selection (G = 8) at each compiled list length (8, 16 and
    # 32 keys) in both kernels (the multi-tile kernel splits the top-K between
    # two warp groups over alternate 32-chunk column blocks and merges their
    # lists per token).
    wl = small("bf16", B=1, L=64 * 40 + 5, H=16, Hkv=2, topk=topk, seed=100 + topk)
    x = make_prefill_inputs(wl, DEV)
    with hsa.path_overrides(B.PATH_MULTI_TILE_SELECT if tiles == "multi" else 0):
        rep, _ = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    want = B.K_SELECT_TC_MULTI_TILE if tiles == "multi" else B.K_SELECT_TC_ONE_TILE
    assert rep.kernels & want, hex(rep.kernels)


@pytest.mark.parametrize("topk", [8, 32])
def test_prefill_tc_selection_many_tiles(oracle_lib, topk):
    # 300 chunks: three score tiles of 128 chunks, the last one ragged (two of
    # its four 32-column blocks), so both top-K groups see full, partial and
    # empty blocks.  Sampled rows: random ones, the first tokens of chunks next
    # to the tile edges, and the tail.
    wl = small("bf16", B=1, L=64 * 300 + 5, H=16, Hkv=2, topk=topk, seed=200 + topk)
    x = make_prefill_inputs(wl, DEV)
    rng = np.random.default_rng(topk)
    edges = np.concatenate([np.arange(c * 64 - 2, c * 64 + 3) for c in (1, 2, 33, 128, 129, 256, 257, 299)])
    rows = np.unique(np.concatenate([rng.integers(0, wl.L, 400), edges, np.arange(wl.L - 70, wl.L)]))
    rep, _ = prefill_parity(oracle_lib, wl, x, rows=rows)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])


@pytest.mark.parametrize("H,Hkv", [(8, 1), (16, 1)])
def test_prefill_several_windows(oracle_lib, H, Hkv):
    # Long sequences split the work lists into token windows (a window's query
    # rows should stay in L2); 512-token windows force that path on a small
    # shape: several windows per (b, g), ragged last one.
    wl = small("bf16", B=2, L=64 * 37 + 29, H=H, Hkv=Hkv, topk=8, seed=77)
    x = make_prefill_inputs(wl, DEV)
    with hsa.path_overrides(0, 512):
        rep, _ = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    expect_tc_path(rep.kernels, True)


def test_prefill_simt_overrides_match_oracle(oracle_lib):
    # The CUDA-core prefill and the CUDA-core selection, forced on a shape the
    # tensor cores would take: both still match the oracle.
    wl = small("bf16", B=1, L=64 * 20 + 3, H=16, Hkv=2, topk=8, seed=51)
    x = make_prefill_inputs(wl, DEV)
    with hsa.path_overrides(B.PATH_SIMT_PREFILL):
        rep, _ = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary()
    expect_tc_path(rep.kernels, False)
    with hsa.path_overrides(B.PATH_SIMT_SELECT):
        rep, _ = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary()
    assert rep.kernels & B.K_SELECT_SIMT and rep.kernels & B.K_ATTEND_TC, hex(rep.kernels)


def test_bounded_wait_expiry_is_reported_and_context_survives(oracle_lib):
    # The failure path of every bounded device wait, made to run out on
    # purpose (a wait that nothing completes, ~1 ms): the status word is
    # flagged, hsa.check reports the timeout once, and the same context then
    # runs the prefill path with parity.
    ws = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    hsa.selftest_wait_expiry(ws, budget_cycles=2_000_000)
    with pytest.raises(hsa.HSAError) as e:
        hsa.check(ws)
    assert e.value.status == B.HSA_ERR_TIMEOUT
    hsa.check(ws)                       # the flag was cleared
    wl = small("bf16", B=1, L=64 * 12 + 7, H=16, Hkv=2, topk=4, seed=9)
    x = make_prefill_inputs(wl, DEV)
    rep, _ = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary()


def test_prefill_explicit_scale(oracle_lib):
    wl = small("f32", B=1, L=300, H=4, Hkv=1, d=64)
    x = make_prefill_inputs(wl, DEV)
    rep, _ = prefill_parity(oracle_lib, wl, x, scale=0.05)
    assert rep.ok, rep.summary()


@pytest.mark.parametrize("L", [1, 37, 64, 65, 128])
def test_prefill_short_sequences(oracle_lib, L):
    wl = small("bf16", B=3, L=L, topk=8)
    x = make_prefill_inputs(wl, DEV)
    rep, _ = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary()


def test_prefill_deterministic():
    wl = small("bf16", B=2, L=64 * 20 + 3, topk=8)
    x = make_prefill_inputs(wl, DEV)
    a = hsa.prefill(x["Q"], x["K"], x["V"], x["lm"], topk=8, idx_out=True, w_out=True)
    b = hsa.prefill(x["Q"], x["K"], x["V"], x["lm"], topk=8, idx_out=True, w_out=True)
    hsa.check()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_landmarks_kernel(oracle_lib):
    for dt in (torch.bfloat16, torch.float32):
        g = torch.Generator(device=DEV).manual_seed(3)
        K = torch.randn(2, 3, 64 * 11 + 9, 128, generator=g, device=DEV).to(dt)
        lm = hsa.landmarks(K)
        hsa.check()
        ref = oracle_lib.landmarks(_np(K), 64)
        err = np.abs(lm.cpu().numpy() - ref).max()
        assert lm.shape == (2, 3, 11, 128) and err < 1e-5, err
    Kc = torch.full((1, 1, 128, 64), 0.75, device=DEV, dtype=torch.bfloat16)
    assert torch.all(hsa.landmarks(Kc) == 6.0)          # sqrt(64) * mean of a constant


# ------------------------------------------------------------------ decode
def decode_parity(oracle_lib, wl: Workload, x: dict, report=None):
    O, idx = hsa.decode(x["q"], x["K"], x["V"], x["lm"], S=wl.S, topk=wl.topk, idx_out=True)
    hsa.check()
    q, lm = _np(x["q"]), _np(x["lm"])
    sel = oracle_lib.decode_select(q, lm, wl.topk)
    got_idx = idx.cpu().numpy()
    rep = report or ParityReport()
    rep.rows += q.shape[0]
    differs = compare_selection(sel["idx"], sel["sbar"], sel["gap"], sel["smag"], got_idx, rep)
    use = np.where(differs[:, :, None], got_idx, sel["idx"])
    Kg, Vg = gather_chunks(x["K"], use, wl.S), gather_chunks(x["V"], use, wl.S)
    ref = oracle_lib.decode_attend(q, lm, Kg, Vg, use, wl.S)
    compare_outputs(ref["O"], _np(O), ATOL[wl.dtype], rep)
    return rep, (O, idx)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,Hkv,topk", [(16, 2, 8), (4, 1, 3), (16, 1, 32), (2, 2, 1)])
def test_decode_small(oracle_lib, dtype, d, H, Hkv, topk):
    wl = Workload("dec", "decode", dtype, B=3, L=64 * 777, H=H, Hkv=Hkv, d=d, topk=topk,
                  seed=d + H)
    x = make_decode_inputs(wl, DEV)
    rep, _ = decode_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])


@pytest.mark.parametrize("topk", [8, 5, 3])
def test_decode_many_sequences_smaller_clusters(oracle_lib, topk):
    # 40 sequences x 2 groups x 8 blocks exceed two waves: the attend kernel runs
    # clusters of 4 blocks, each taking two slots (one when topk <= 4)
    wl = Workload("dec", "decode", "bf16", B=40, L=64 * 120, H=16, Hkv=2, d=128, topk=topk,
                  seed=90 + topk)
    x = make_decode_inputs(wl, DEV)
    rep, _ = decode_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])


def test_decode_fewer_chunks_than_topk(oracle_lib):
    wl = Workload("dec", "decode", "bf16", B=2, L=64 * 5, H=16, Hkv=2, d=128, topk=8)
    x = make_decode_inputs(wl, DEV)
    rep, (O, idx) = decode_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary()
    assert (idx[:, :, 5:] == -1).all()


def test_decode_fp32_landmarks(oracle_lib):
    wl = Workload("dec", "decode", "bf16", B=2, L=64 * 1000, H=16, Hkv=2, d=128, topk=8)
    x = make_decode_inputs(wl, DEV)
    x["lm"] = x["lm"].float() * 1.7
    rep, _ = decode_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary()


def test_decode_empty_cache():
    q = torch.randn(2, 16, 128, device=DEV, dtype=torch.bfloat16)
    K = torch.empty(2, 2, 0, 128, device=DEV, dtype=torch.bfloat16)
    lm = torch.empty(2, 2, 0, 128, device=DEV, dtype=torch.bfloat16)
    O, idx = hsa.decode(q, K, K, lm, topk=8, idx_out=True)
    hsa.check()
    assert torch.all(O == 0) and torch.all(idx == -1)


def test_decode_deterministic_and_repeatable():
    wl = Workload("dec", "decode", "bf16", B=4, L=64 * 3000, H=16, Hkv=2, d=128, topk=8)
    x = make_decode_inputs(wl, DEV)
    outs = [hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=8, idx_out=True) for _ in range(3)]
    hsa.check()
    for o in outs[1:]:
        assert torch.equal(o[0], outs[0][0]) and torch.equal(o[1], outs[0][1])


# ------------------------------------------------------------------ the named workloads
def _sample_rows(B, L, n, seed, extra=()):
    rng = np.random.default_rng(seed)
    rows = set(rng.integers(0, B * L, n).tolist())
    for b in range(B):
        rows.update([b * L, b * L + 63, b * L + 64, b * L + 65, b * L + L - 1])
    rows.update(extra)
    return np.array(sorted(r for r in rows if 0 <= r < B * L), dtype=np.int64)


def test_workload_tiny_prefill_f32_all_rows(oracle_lib):
    wl = WORKLOADS["tiny_prefill_f32"]
    x = make_prefill_inputs(wl, DEV)
    rep, _ = prefill_parity(oracle_lib, wl, x)
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])


def test_workload_train_prefill_bf16(oracle_lib):
    wl = WORKLOADS["train_prefill_bf16"]
    x = make_prefill_inputs(wl, DEV)
    rows = _sample_rows(wl.B, wl.L, 3000, 1)
    rep, _ = prefill_parity(oracle_lib, wl, x, rows=rows)
    print(rep.summary())
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])


def test_workload_long_prefill_bf16_with_needles(oracle_lib):
    wl = WORKLOADS["long_prefill_bf16"]
    x = make_prefill_inputs(wl, DEV)
    probes = x["probe_pos"]
    rows = _sample_rows(wl.B, wl.L, 600, 2, extra=probes[::8])
    rep, (O, idx, w) = prefill_parity(oracle_lib, wl, x, rows=rows)
    print(rep.summary())
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    # every visible needle is selected by every probe (needle-retrieval check)
    idx_h = idx[0].cpu().numpy()
    for t in probes:
        vis = [c for c in x["needle_chunks"] if c < t // wl.S]
        for g in range(wl.Hkv):
            assert set(vis) <= set(idx_h[t, g].tolist()), (t, g)
    del x
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["batched_decode_bf16", "decode_32m_bf16"])
def test_workload_decode(oracle_lib, name):
    wl = WORKLOADS[name]
    x = make_decode_inputs(wl, DEV)
    rep, (O, idx) = decode_parity(oracle_lib, wl, x)
    print(rep.summary())
    assert rep.ok, rep.summary() + "\n" + "\n".join(rep.failures[:10])
    if wl.needles == "decode":
        for b, c in enumerate(x["needle_chunk"]):
            assert (idx[b, :, 0] == c).all(), (idx[b], c)
    del x
    torch.cuda.empty_cache()
