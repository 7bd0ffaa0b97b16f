"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test ties the oracle to a fact fixed by the method's definition or by
mathematics: a hand-worked example, library routines it must reduce to
(PyTorch's scaled_dot_product_attention in float64), a separately written
brute-force hierarchical sum, exhaustive subset search, closed forms and
invariants.  A dropped term, a wrong sign or index, or a transposed operand in
the oracle fails at least one of them (see test_oracle_mutants.py).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(seed, B, L, H, Hkv, d, S, lm_scale=1.0):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, L, H, d))
    K = rng.standard_normal((B, Hkv, L, d))
    V = rng.standard_normal((B, Hkv, L, d))
    lm = lm_scale * rng.standard_normal((B, Hkv, L // S, d))
    return Q, K, V, lm


def sdpa_causal(Q, K, V, G, scale=None):
    """Causal attention per head with PyTorch's SDPA in float64 (GQA by repeat)."""
    q = torch.from_numpy(Q).permute(0, 2, 1, 3)                  # [B,H,L,d]
    k = torch.from_numpy(K).repeat_interleave(G, dim=1)           # [B,H,L,d]
    v = torch.from_numpy(V).repeat_interleave(G, dim=1)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()                           # [B,L,H,d]


def sdpa_full(q, k, v, scale=None):
    """Non-causal attention of query rows q [n,d] over k,v [m,d] (float64 SDPA)."""
    o = F.scaled_dot_product_attention(torch.from_numpy(q)[None, None],
                                       torch.from_numpy(k)[None, None],
                                       torch.from_numpy(v)[None, None], scale=scale)
    return o[0, 0].numpy()


# --------------------------------------------------------------------------- hand example
def test_hand_worked_example(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    L, H, d = g["L"], g["H"], g["d"]
    Q = np.broadcast_to(np.array(g["Q_per_position"]), (1, L, H, d)).copy()
    K = np.array(g["K"])[None, None]
    V = np.array(g["V"])[None, None]
    lm = np.array(g["lm"])[None, None]
    r = oracle_lib.prefill(Q, K, V, lm, g["S"], g["topk"], g["own_chunk"], g["scale"])
    np.testing.assert_allclose(r["O"], np.array(g["expected_O"]), atol=1e-12, rtol=0)
    np.testing.assert_array_equal(r["idx"][:, 0, :], np.array(g["expected_idx"]))
    np.testing.assert_allclose(r["sbar"][:, 0, :], np.array(g["expected_sbar"]), atol=1e-12)
    np.testing.assert_allclose(r["w"], np.array(g["expected_w"]), atol=1e-12)


# --------------------------------------------------------------------------- reductions
@pytest.mark.parametrize("L,S", [(16, 16), (13, 16), (64, 64)])
@pytest.mark.parametrize("H,Hkv", [(4, 1), (4, 2), (2, 2)])
def test_single_chunk_is_causal_attention(oracle_lib, L, S, H, Hkv):
    """With one chunk (L <= S) nothing is selectable; O is textbook causal attention."""
    d = 8
    Q, K, V, _ = rand_case(1, 2, L, H, Hkv, d, S)
    lm = np.zeros((2, Hkv, L // S, d))
    r = oracle_lib.prefill(Q, K, V, lm, S, topk=3, own_chunk=1)
    ref = sdpa_causal(Q, K, V, H // Hkv)                          # default scale 1/sqrt(d)
    np.testing.assert_allclose(r["O"].reshape(ref.shape), ref, atol=1e-12, rtol=0)
    assert (r["idx"] == -1).all() and (r["w"] == 0).all()


def test_own_chunk_matches_causal_prefix_of_every_chunk(oracle_lib):
    """topk=1 with one visible chunk forced to be weight 1: the own term alone is
    the causal attention restricted to the chunk (checked with SDPA per chunk)."""
    B, L, H, Hkv, d, S = 1, 48, 2, 1, 4, 16
    Q, K, V, lm = rand_case(2, B, L, H, Hkv, d, S)
    r0 = oracle_lib.prefill(Q, K, V, lm, S, topk=2, own_chunk=0)
    r1 = oracle_lib.prefill(Q, K, V, lm, S, topk=2, own_chunk=1)
    own = (r1["O"] - r0["O"]).reshape(B, L, H, d)
    for c in range(L // S):
        sl = slice(c * S, (c + 1) * S)
        ref = sdpa_causal(Q[:, sl], K[:, :, sl], V[:, :, sl], H // Hkv)
        np.testing.assert_allclose(own[:, sl], ref, atol=1e-12)


def test_topk1_is_attention_over_argmax_chunk(oracle_lib):
    B, L, H, Hkv, d, S = 2, 96, 4, 2, 8, 16
    Q, K, V, lm = rand_case(3, B, L, H, Hkv, d, S)
    G = H // Hkv
    r = oracle_lib.prefill(Q, K, V, lm, S, topk=1, own_chunk=0)
    O = r["O"].reshape(B, L, H, d)
    scale = 1 / math.sqrt(d)
    for b in range(B):
        for t in range(L):
            nvis = t // S
            for g in range(Hkv):
                if nvis == 0:
                    assert r["idx"][b * L + t, g, 0] == -1
                    assert np.all(O[b, t, g * G:(g + 1) * G] == 0)
                    continue
                qbar = Q[b, t, g * G:(g + 1) * G].mean(axis=0)
                i = int(np.argmax(lm[b, g, :nvis] @ qbar))       # first maximum = lowest index
                assert r["idx"][b * L + t, g, 0] == i
                ref = sdpa_full(Q[b, t, g * G:(g + 1) * G], K[b, g, i * S:(i + 1) * S],
                                V[b, g, i * S:(i + 1) * S], scale)
                np.testing.assert_allclose(O[b, t, g * G:(g + 1) * G], ref, atol=1e-12)
                np.testing.assert_array_equal(r["w"][b * L + t, g * G:(g + 1) * G, 0], 1.0)


def brute_force_hierarchical(Q, K, V, lm, S, own_chunk, scale):
    """Every visible chunk fused (no selection, no sort): written independently
    of the oracle with vectorised numpy and SDPA for the in-chunk attention."""
    B, L, H, d = Q.shape
    Hkv = K.shape[1]
    G = H // Hkv
    O = np.zeros_like(Q)
    for b in range(B):
        for h in range(H):
            g = h // G
            # chunk outputs o[t, i] for all t and all complete chunks i
            Nc = L // S
            Kc = K[b, g, :Nc * S].reshape(Nc, S, d)
            Vc = V[b, g, :Nc * S].reshape(Nc, S, d)
            logits = np.einsum("td,isd->tis", Q[b, :, h], Kc) * scale       # [L,Nc,S]
            p = np.exp(logits - logits.max(axis=2, keepdims=True))
            p /= p.sum(axis=2, keepdims=True)
            o_chunks = np.einsum("tis,isd->tid", p, Vc)                       # [L,Nc,d]
            s = Q[b, :, h] @ lm[b, g].T * scale                               # [L,Nc]
            for t in range(L):
                nvis = t // S
                if nvis:
                    e = np.exp(s[t, :nvis] - s[t, :nvis].max())
                    O[b, t, h] = (e / e.sum()) @ o_chunks[t, :nvis]
        if own_chunk:
            O[b] += sdpa_chunked_causal(Q[b:b + 1], K[b:b + 1], V[b:b + 1], S, G, scale)[0]
    return O


def sdpa_chunked_causal(Q, K, V, S, G, scale):
    B, L, H, d = Q.shape
    out = np.zeros_like(Q)
    for c0 in range(0, L, S):
        sl = slice(c0, min(L, c0 + S))
        out[:, sl] = sdpa_causal(Q[:, sl], K[:, :, sl], V[:, :, sl], G, scale)
    return out


@pytest.mark.parametrize("own_chunk", [0, 1])
@pytest.mark.parametrize("L", [128, 120])
def test_topk_all_visible_matches_bruteforce_sum(oracle_lib, own_chunk, L):
    B, H, Hkv, d, S = 2, 4, 2, 8, 16
    Q, K, V, lm = rand_case(4, B, L, H, Hkv, d, S)
    scale = 0.3
    r = oracle_lib.prefill(Q, K, V, lm, S, topk=L // S, own_chunk=own_chunk, scale=scale)
    ref = brute_force_hierarchical(Q, K, V, lm, S, own_chunk, scale)
    np.testing.assert_allclose(r["O"].reshape(ref.shape), ref, atol=1e-12)


# --------------------------------------------------------------------------- invariants
def test_fusion_weights_sum_to_one(oracle_lib):
    B, L, H, Hkv, d, S = 1, 256, 8, 2, 16, 16
    Q, K, V, lm = rand_case(5, B, L, H, Hkv, d, S)
    r = oracle_lib.prefill(Q, K, V, lm, S, topk=4)
    nvis = (np.arange(L) // S)
    wsum = r["w"].sum(axis=2)
    np.testing.assert_allclose(wsum[nvis >= 1], 1.0, atol=1e-12)
    assert np.all(wsum[nvis == 0] == 0)
    assert np.all(r["w"] >= 0)
    # padded slots carry weight 0 and index -1
    pad = r["idx"] < 0
    assert np.all(r["w"].reshape(L, Hkv, H // Hkv, 4)[np.repeat(pad[:, :, None, :], H // Hkv, 2)] == 0)


def test_unselected_chunks_do_not_matter(oracle_lib):
    """Changing K/V of every chunk a query did not select leaves its output bit-identical."""
    B, L, H, Hkv, d, S, topk = 1, 256, 4, 1, 8, 16, 3
    Q, K, V, lm = rand_case(6, B, L, H, Hkv, d, S)
    r = oracle_lib.prefill(Q, K, V, lm, S, topk)
    rng = np.random.default_rng(99)
    for t in (40, 130, 255):
        sel = set(int(i) for i in r["idx"][t, 0] if i >= 0)
        K2, V2 = K.copy(), V.copy()
        c_t = t // S
        for i in range(L // S):
            if i not in sel and i != c_t:
                K2[0, 0, i * S:(i + 1) * S] = rng.standard_normal((S, d)) * 5
                V2[0, 0, i * S:(i + 1) * S] = rng.standard_normal((S, d)) * 5
        # keys after t inside the own chunk are causally masked too
        K2[0, 0, t + 1:(c_t + 1) * S] = 7.0
        V2[0, 0, t + 1:(c_t + 1) * S] = -7.0
        r2 = oracle_lib.prefill(Q, K2, V2, lm, S, topk, rows=np.array([t]))
        assert np.array_equal(r2["O"][0], r["O"][t])
        assert np.array_equal(r2["idx"][0], r["idx"][t])


def test_selection_is_best_subset_by_exhaustive_search(oracle_lib):
    """Tiny case: the selected set maximises the summed group score over all
    subsets of the visible chunks of size min(K, nvis), and ranks them in order."""
    B, L, H, Hkv, d, S, topk = 1, 256, 2, 2, 4, 16, 3
    Q, K, V, lm = rand_case(7, B, L, H, Hkv, d, S)
    r = oracle_lib.prefill(Q, K, V, lm, S, topk, scale=1.0)
    for t in range(0, L, 7):
        nvis = t // S
        for g in range(Hkv):
            qbar = Q[0, t, g:g + 1].mean(axis=0)            # G=1 here
            s = lm[0, g, :nvis] @ qbar
            m = min(topk, nvis)
            best = max(itertools.combinations(range(nvis), m), key=lambda c: sum(s[list(c)]),
                       default=())
            got = [int(i) for i in r["idx"][t, g] if i >= 0]
            assert sorted(got) == sorted(best)
            assert all(s[got[j]] >= s[got[j + 1]] for j in range(len(got) - 1))


def test_ties_go_to_lowest_index(oracle_lib):
    B, L, H, Hkv, d, S, topk = 1, 128, 2, 1, 4, 16, 2
    Q, K, V, _ = rand_case(8, B, L, H, Hkv, d, S)
    lm = np.zeros((1, 1, L // S, d))
    lm[0, 0, :] = np.array([1.0, 0.5, -0.25, 2.0])   # all chunks tie exactly
    lm[0, 0, 5] *= 2.0                                 # chunk 5 strictly best when qbar.l0 > 0
    r = oracle_lib.prefill(Q, K, V, lm, S, topk)
    for t in range(S, L):
        nvis = t // S
        qbar = Q[0, t].mean(axis=0)
        s0 = float(lm[0, 0, 0] @ qbar)
        got = [int(i) for i in r["idx"][t, 0] if i >= 0]
        if nvis <= 5 or s0 == 0:
            assert got == list(range(min(topk, nvis)))
        elif s0 > 0:
            assert got == [5, 0]
        else:  # chunk 5 is the unique worst; lowest-index ties fill the set
            assert got == [0, 1]


# --------------------------------------------------------------------------- landmarks
def test_dhsa_landmark_closed_form(oracle_lib):
    S, d = 64, 8
    K = np.zeros((1, 1, 3 * S + 5, d))
    # dyadic constants: every partial sum is exact, so the closed form holds bit for bit
    consts = [np.arange(d) * 0.5 - 1, np.full(d, 3.25), np.arange(d) * -0.375 + 1.125]
    for i, c in enumerate(consts):
        K[0, 0, i * S:(i + 1) * S] = c
    lm = oracle_lib.landmarks(K, S)
    assert lm.shape == (1, 1, 3, d)          # the partial tail chunk has no landmark
    for i, c in enumerate(consts):
        np.testing.assert_array_equal(lm[0, 0, i], 8.0 * c)   # sqrt(64) * mean of a constant


def test_dhsa_landmark_matches_numpy_mean(oracle_lib):
    rng = np.random.default_rng(10)
    S = 16
    K = rng.standard_normal((2, 3, 5 * S + 3, 8))
    lm = oracle_lib.landmarks(K, S)
    ref = math.sqrt(S) * K[:, :, :5 * S].reshape(2, 3, 5, S, 8).mean(axis=3)
    np.testing.assert_allclose(lm, ref, atol=1e-13)


def test_dhsa_mode_equals_explicit_landmarks(oracle_lib):
    B, L, H, Hkv, d, S = 1, 160, 4, 2, 8, 16
    Q, K, V, _ = rand_case(11, B, L, H, Hkv, d, S)
    lm = math.sqrt(S) * K[:, :, :(L // S) * S].reshape(B, Hkv, L // S, S, d).mean(axis=3)
    r1 = oracle_lib.prefill(Q, K, V, None, S, 3)
    r2 = oracle_lib.prefill(Q, K, V, lm, S, 3)
    np.testing.assert_array_equal(r1["idx"], r2["idx"])
    np.testing.assert_allclose(r1["O"], r2["O"], atol=1e-12)


# --------------------------------------------------------------------------- GQA
def test_duplicated_heads_match_single_head_group(oracle_lib):
    """G identical query heads select what one head selects, and each head's
    output equals the G=1 output."""
    B, L, d, S, topk = 1, 192, 8, 16, 4
    Q1, K, V, lm = rand_case(12, B, L, 1, 1, d, S)
    r1 = oracle_lib.prefill(Q1, K, V, lm, S, topk)
    Q4 = np.repeat(Q1, 4, axis=2)
    r4 = oracle_lib.prefill(Q4, K, V, lm, S, topk)
    np.testing.assert_array_equal(r1["idx"], r4["idx"])
    for h in range(4):
        np.testing.assert_allclose(r4["O"][:, h], r1["O"][:, 0], atol=1e-13)


def test_group_selection_uses_mean_of_heads(oracle_lib):
    """Group score = mean over heads: a group whose heads disagree picks the
    chunks best for the average, checked against a direct per-head sum."""
    B, L, H, Hkv, d, S, topk = 1, 256, 4, 1, 8, 16, 2
    Q, K, V, lm = rand_case(13, B, L, H, Hkv, d, S)
    r = oracle_lib.prefill(Q, K, V, lm, S, topk)
    for t in range(S, L, 11):
        nvis = t // S
        per_head = np.stack([lm[0, 0, :nvis] @ Q[0, t, h] for h in range(H)])   # [H,nvis]
        total = per_head.sum(axis=0)
        order = sorted(range(nvis), key=lambda i: (-total[i], i))[:topk]
        assert [int(i) for i in r["idx"][t, 0] if i >= 0] == order
        np.testing.assert_allclose(r["sbar"][t, 0, :len(order)],
                                   total[order] / H / math.sqrt(d), atol=1e-12)


# --------------------------------------------------------------------------- needles
def test_planted_needles_rank_first(oracle_lib):
    from hierarchical_chunk_sparse_landmark_b200.workloads import WORKLOADS, make_prefill_inputs
    wl = WORKLOADS["long_prefill_bf16"].with_(L=4096, B=1)
    x = make_prefill_inputs(wl, "cpu")
    probes = np.array(x["probe_pos"][:64])
    r = oracle_lib.prefill(x["Q"], x["K"], x["V"], None, wl.S, wl.topk, rows=probes)
    needles = x["needle_chunks"]
    for n, t in enumerate(probes):
        vis = [c for c in needles if c < t // wl.S]
        assert vis
        for g in range(wl.Hkv):
            top = [int(i) for i in r["idx"][n, g][:len(vis)]]
            assert sorted(top) == sorted(vis), (t, g, top, vis)


# --------------------------------------------------------------------------- decode
def test_decode_equals_prefill_row_at_position_Lc(oracle_lib):
    """Decode's query at position Lc sees all Lc/S chunks and has no own term:
    it equals the prefill row t = Lc of a sequence one token longer with
    own_chunk = 0."""
    B, H, Hkv, d, S, topk = 2, 4, 2, 8, 16, 3
    Lc = 8 * S
    rng = np.random.default_rng(14)
    q = rng.standard_normal((B, H, d))
    K = rng.standard_normal((B, Hkv, Lc, d))
    V = rng.standard_normal((B, Hkv, Lc, d))
    lm = rng.standard_normal((B, Hkv, Lc // S, d))
    dec = oracle_lib.decode(q, K, V, lm, S, topk)
    Lp = Lc + 1
    Kp = np.concatenate([K, rng.standard_normal((B, Hkv, 1, d))], axis=2)
    Vp = np.concatenate([V, rng.standard_normal((B, Hkv, 1, d))], axis=2)
    Qp = np.zeros((B, Lp, H, d))
    Qp[:, Lc] = q
    rows = np.array([b * Lp + Lc for b in range(B)])
    pre = oracle_lib.prefill(Qp, Kp, Vp, lm, S, topk, own_chunk=0, rows=rows)
    np.testing.assert_array_equal(dec["idx"], pre["idx"])
    np.testing.assert_allclose(dec["O"], pre["O"], atol=1e-13)


def test_decode_bruteforce(oracle_lib):
    B, H, Hkv, d, S, topk = 3, 8, 2, 16, 16, 4
    Lc = 12 * S
    rng = np.random.default_rng(15)
    q = rng.standard_normal((B, H, d))
    K = rng.standard_normal((B, Hkv, Lc, d))
    V = rng.standard_normal((B, Hkv, Lc, d))
    lm = rng.standard_normal((B, Hkv, Lc // S, d))
    dec = oracle_lib.decode(q, K, V, lm, S, topk)
    G = H // Hkv
    scale = 1 / math.sqrt(d)
    for b in range(B):
        for g in range(Hkv):
            s = lm[b, g] @ q[b, g * G:(g + 1) * G].mean(axis=0)
            order = np.lexsort((np.arange(len(s)), -s))[:topk]
            np.testing.assert_array_equal(dec["idx"][b, g], order)
            for h in range(g * G, (g + 1) * G):
                logit = lm[b, g, order] @ q[b, h] * scale
                wgt = np.exp(logit - logit.max())
                wgt /= wgt.sum()
                o = sum(wgt[j] * sdpa_full(q[b, h][None], K[b, g, i * S:(i + 1) * S],
                                           V[b, g, i * S:(i + 1) * S], scale)[0]
                        for j, i in enumerate(order))
                np.testing.assert_allclose(dec["O"][b, h], o, atol=1e-12)


def test_decode_fewer_chunks_than_topk(oracle_lib):
    B, H, Hkv, d, S, topk = 1, 2, 1, 4, 16, 8
    rng = np.random.default_rng(16)
    q = rng.standard_normal((B, H, d))
    K = rng.standard_normal((B, Hkv, 3 * S, d))
    V = rng.standard_normal((B, Hkv, 3 * S, d))
    lm = rng.standard_normal((B, Hkv, 3, d))
    dec = oracle_lib.decode(q, K, V, lm, S, topk)
    assert sorted(dec["idx"][0, 0, :3].tolist()) == [0, 1, 2]
    assert (dec["idx"][0, 0, 3:] == -1).all()
    assert np.isinf(dec["gap"][0, 0])
    np.testing.assert_allclose(dec["w"].sum(-1), 1.0, atol=1e-12)


# --------------------------------------------------------------------------- forced selection
def _hand_inputs(g):
    L, H, d = g["L"], g["H"], g["d"]
    Q = np.broadcast_to(np.array(g["Q_per_position"]), (1, L, H, d)).copy()
    return Q, np.array(g["K"])[None, None], np.array(g["V"])[None, None], np.array(g["lm"])[None, None]


def test_forced_selection_hand_rows(oracle_lib):
    """Rows recomputed on a given selection (the entry point the GPU parity
    tests use on near-tie rows), worked by hand on the 6-token example:
    a reordered set keeps O and reorders w; pads and chunks that are not
    visible from the row (its own chunk or later ones) are dropped."""
    base = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    g = json.load(open(os.path.join(GOLDEN, "forced_and_gap.json")))["forced"]
    Q, K, V, lm = _hand_inputs(base)
    rows = np.array(g["rows"], dtype=np.int64)
    forced = np.array(g["forced_idx"], dtype=np.int32)[:, None, :]
    r = oracle_lib.prefill(Q, K, V, lm, base["S"], base["topk"], base["own_chunk"],
                           base["scale"], rows=rows, forced_idx=forced)
    np.testing.assert_array_equal(r["idx"][:, 0, :], np.array(g["expected_idx"]))
    np.testing.assert_allclose(r["O"], np.array(g["expected_O"]), atol=1e-12, rtol=0)
    np.testing.assert_allclose(r["w"], np.array(g["expected_w"]), atol=1e-12, rtol=0)


@pytest.mark.parametrize("own_chunk", [0, 1])
def test_forced_selection_equal_to_own_is_bit_identical(oracle_lib, own_chunk):
    """Forcing the oracle's own selection reproduces its outputs bit for bit."""
    B, L, H, Hkv, d, S, topk = 2, 200, 4, 2, 8, 16, 3
    Q, K, V, lm = rand_case(17, B, L, H, Hkv, d, S)
    r = oracle_lib.prefill(Q, K, V, lm, S, topk, own_chunk)
    f = oracle_lib.prefill(Q, K, V, lm, S, topk, own_chunk, forced_idx=r["idx"])
    np.testing.assert_array_equal(f["idx"], r["idx"])
    np.testing.assert_array_equal(f["O"], r["O"])
    np.testing.assert_array_equal(f["w"], r["w"])
    np.testing.assert_array_equal(f["sbar"], r["sbar"])
    assert np.isnan(f["gap"]).all()


def test_forced_selection_swapped_chunk_matches_bruteforce(oracle_lib):
    """One selected chunk swapped for an unselected visible one: O equals the
    fusion, written out separately here, of attention over the forced chunks."""
    B, L, H, Hkv, d, S, topk = 1, 160, 2, 1, 4, 16, 3
    Q, K, V, lm = rand_case(18, B, L, H, Hkv, d, S)
    r = oracle_lib.prefill(Q, K, V, lm, S, topk, own_chunk=0)
    rows = np.arange(8 * S, L)
    forced = r["idx"][rows].copy()
    for n, t in enumerate(rows):
        unsel = [c for c in range(t // S) if c not in forced[n, 0]]
        forced[n, 0, 1] = unsel[n % len(unsel)]
    f = oracle_lib.prefill(Q, K, V, lm, S, topk, own_chunk=0, rows=rows, forced_idx=forced)
    scale = 1 / math.sqrt(d)
    for n, t in enumerate(rows):
        for h in range(H):
            sel = forced[n, 0]
            logit = lm[0, 0, sel] @ Q[0, t, h] * scale
            wgt = np.exp(logit - logit.max())
            wgt /= wgt.sum()
            o = sum(wgt[j] * sdpa_full(Q[0, t, h][None], K[0, 0, i * S:(i + 1) * S],
                                       V[0, 0, i * S:(i + 1) * S], scale)[0]
                    for j, i in enumerate(sel))
            np.testing.assert_allclose(f["O"][n, h], o, atol=1e-12)
            np.testing.assert_allclose(f["w"][n, h], wgt, atol=1e-14)


# --------------------------------------------------------------------------- near-tie gap
@pytest.mark.parametrize("topk", [1, 2, 3])
def test_prefill_gap_hand_scores(oracle_lib, topk):
    """gap = K-th minus (K+1)-th group score, +inf when at most K chunks are
    visible, on scores set by hand (tests/golden/forced_and_gap.json)."""
    g = json.load(open(os.path.join(GOLDEN, "forced_and_gap.json")))["gap"]
    S, L = g["S"], g["L"]
    s = np.array(g["scores"])
    lm = np.zeros((1, 1, len(s), 2))
    lm[0, 0, :, 0] = s
    Q = np.zeros((1, L, 1, 2))
    Q[..., 0] = 1.0
    K = np.zeros((1, 1, L, 2))
    r = oracle_lib.prefill(Q, K, K, lm, S, topk, scale=1.0)
    want = np.array([np.inf if v == "inf" else v for v in g["expected_gap"][str(topk)]])
    np.testing.assert_array_equal(r["gap"][:, 0], want)


def test_decode_gap_hand_scores(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "forced_and_gap.json")))["gap"]
    s = np.array(g["scores"])
    lm = np.zeros((1, 1, len(s), 2))
    lm[0, 0, :, 0] = s
    q = np.array([[[1.0, 0.0]]])
    for k, v in g["decode"]["expected_gap"].items():
        r = oracle_lib.decode_select(q, lm, int(k), scale=1.0)
        assert r["gap"][0, 0] == (np.inf if v == "inf" else v), (k, r["gap"])


def test_score_term_magnitudes_hand_case(oracle_lib):
    """smag: scale * sum_j |qbar_j l_ij| of each selected chunk in rank order,
    then of the (K+1)-th ranked chunk.  Hand case with one cancelling score:
    qbar = (1, 1); l0 = (2, -2) scores 0 from terms of magnitude 4;
    l1 = (1, 0.5) scores 1.5 (magnitude 1.5); l2 = (0.25, 0.25) scores 0.5."""
    S, d = 2, 2
    lm = np.array([[[[2.0, -2.0], [1.0, 0.5], [0.25, 0.25]]]])
    L = 8                                          # row t = 6, 7 sees all three chunks
    Q = np.ones((1, L, 1, d))
    K = np.zeros((1, 1, L, d))
    r1 = oracle_lib.prefill(Q, K, K, lm, S, 1, scale=1.0, rows=np.array([7]))
    np.testing.assert_array_equal(r1["idx"][0, 0], [1])
    np.testing.assert_array_equal(r1["smag"][0, 0], [1.5, 0.5])
    assert r1["gap"][0, 0] == 1.0
    r2 = oracle_lib.prefill(Q, K, K, lm, S, 2, scale=1.0, rows=np.array([7]))
    np.testing.assert_array_equal(r2["idx"][0, 0], [1, 2])
    np.testing.assert_array_equal(r2["smag"][0, 0], [1.5, 0.5, 4.0])
    assert r2["gap"][0, 0] == 0.5
    r3 = oracle_lib.prefill(Q, K, K, lm, S, 3, scale=0.5, rows=np.array([7]))
    np.testing.assert_array_equal(r3["smag"][0, 0], [0.75, 0.25, 2.0, 0.0])   # no 4th chunk
    dec = oracle_lib.decode_select(np.ones((1, 1, d)), lm, 2, scale=1.0)
    np.testing.assert_array_equal(dec["smag"][0, 0], [1.5, 0.5, 4.0])


# --------------------------------------------------------------------------- retrieval variants
def test_variant_interval_one_is_the_per_token_oracle(oracle_lib):
    """Retrieval every token with the HiLS fusion is hsa_oracle_prefill."""
    Q, K, V, lm = rand_case(30, 2, 70, 4, 2, 8, 8)
    for own in (0, 1):
        a = oracle_lib.prefill(Q, K, V, lm, 8, 3, own)
        for pool in (0, 1):
            b = oracle_lib.prefill_variant(Q, K, V, lm, 8, 3, own, pool_mean=pool)
            np.testing.assert_array_equal(a["idx"], b["idx"])
            np.testing.assert_allclose(a["O"], b["O"], atol=1e-13, rtol=0)
            np.testing.assert_allclose(a["w"], b["w"], atol=1e-14, rtol=0)


@pytest.mark.parametrize("interval", [2, 4, 8])
def test_variant_first_token_retrieval_reuses_the_block_start_selection(oracle_lib, interval):
    """One selection per block of `interval` tokens, decided by the block's
    first token: token t uses the per-token selection of its block start, and
    its output is the per-token oracle's output on that forced selection."""
    B, L, H, Hkv, d, S, topk = 1, 8 * 13 + 5, 4, 2, 8, 8, 3
    Q, K, V, lm = rand_case(31, B, L, H, Hkv, d, S)
    r = oracle_lib.prefill_variant(Q, K, V, lm, S, topk, 1, interval=interval)
    starts = (np.arange(L) // interval) * interval
    per_tok = oracle_lib.prefill(Q, K, V, lm, S, topk, 1)
    np.testing.assert_array_equal(r["idx"], per_tok["idx"][starts])
    forced = oracle_lib.prefill(Q, K, V, lm, S, topk, 1, forced_idx=per_tok["idx"][starts])
    np.testing.assert_allclose(r["O"], forced["O"], atol=1e-13, rtol=0)
    np.testing.assert_allclose(r["w"], forced["w"], atol=1e-14, rtol=0)


@pytest.mark.parametrize("interval", [4, 8])
def test_variant_mean_pooled_selection_is_the_top_k_of_the_block_mean(oracle_lib, interval):
    """Mean pooling (the DHSA chunk-level query at interval = S): the block's
    selection is the top-K, lower index on ties, of the landmark scores of the
    mean over its tokens and the group's heads, computed here with numpy."""
    B, L, H, Hkv, d, S, topk = 2, 8 * 11 + 3, 4, 2, 8, 8, 3
    Q, K, V, lm = rand_case(32, B, L, H, Hkv, d, S)
    r = oracle_lib.prefill_variant(Q, K, V, lm, S, topk, 1, interval=interval, pool_mean=1)
    G = H // Hkv
    for b in range(B):
        for t in range(L):
            t0 = (t // interval) * interval
            t1 = min(t0 + interval, L)
            for g in range(Hkv):
                qm = Q[b, t0:t1, g * G:(g + 1) * G].mean(axis=(0, 1))
                nvis = t // S
                s = lm[b, g, :nvis] @ qm
                want = np.lexsort((np.arange(nvis), -s))[:topk]
                got = r["idx"][b * L + t, g]
                np.testing.assert_array_equal(got[:len(want)], want)
                assert (got[len(want):] == -1).all()


def test_variant_union_softmax_matches_the_numpy_restatement(oracle_lib):
    """One softmax over the union of the selected keys (and the own chunk)
    equals oracle/variants.py's numpy restatement, which is pinned to SDPA."""
    from oracle import variants
    Q, K, V, lm = rand_case(33, 2, 53, 4, 2, 8, 8)
    for own in (0, 1):
        r = oracle_lib.prefill_variant(Q, K, V, lm, 8, 2, own, union_softmax=1)
        ref = variants.flat_union_prefill(Q, K, V, lm, 8, 2, own)
        np.testing.assert_array_equal(r["idx"].reshape(ref["idx"].shape), ref["idx"])
        np.testing.assert_allclose(r["O"].reshape(ref["O"].shape), ref["O"], atol=1e-12, rtol=0)
        assert (r["w"] == 0).all()


def test_variant_union_softmax_of_every_chunk_is_causal_attention(oracle_lib):
    """All visible chunks selected plus the own chunk: plain causal attention
    (PyTorch SDPA in float64)."""
    Q, K, V, lm = rand_case(34, 1, 48, 4, 2, 8, 8)
    for interval in (1, 8):
        r = oracle_lib.prefill_variant(Q, K, V, lm, 8, 6, 1, union_softmax=1, interval=interval)
        ref = sdpa_causal(Q, K, V, 2)
        np.testing.assert_allclose(r["O"].reshape(ref.shape), ref, atol=1e-12, rtol=0)


def test_variant_gap_and_magnitudes_are_those_of_the_block_selection(oracle_lib):
    """The near-tie gap and score-term magnitudes of a block's selection are
    those of the per-token oracle at the block's first token (first-token
    pooling), for every token of the block."""
    Q, K, V, lm = rand_case(35, 1, 8 * 9 + 5, 4, 2, 8, 8)
    L = Q.shape[1]
    r = oracle_lib.prefill_variant(Q, K, V, lm, 8, 3, 1, interval=4)
    starts = (np.arange(L) // 4) * 4
    ref = oracle_lib.prefill(Q, K, V, lm, 8, 3, 1, rows=starts)
    np.testing.assert_array_equal(r["sbar"], ref["sbar"])
    np.testing.assert_array_equal(r["gap"], ref["gap"])
    np.testing.assert_array_equal(r["smag"], ref["smag"])


# --------------------------------------------------------------------------- variable-length chunks
@pytest.mark.parametrize("own", [0, 1])
@pytest.mark.parametrize("given_lm", [False, True])
def test_varlen_chunks_match_the_numpy_restatement(oracle_lib, own, given_lm):
    """Variable-length chunks in the C oracle equal oracle/varlen.py (pinned
    to the fixed-chunk oracle, to causal attention and to the landmark closed
    form), for DHSA landmarks sqrt(|C|) * mean and for given landmarks."""
    from oracle import varlen
    rng = np.random.default_rng(40 + own + 2 * given_lm)
    B, L, H, Hkv, d = 2, 71, 4, 2, 8
    Q = rng.standard_normal((B, L, H, d))
    K = rng.standard_normal((B, Hkv, L, d))
    V = rng.standard_normal((B, Hkv, L, d))
    bounds = [0, 5, 13, 14, 30, 37, 50, 64, 71]
    n = len(bounds) - 1
    lm = rng.standard_normal((B, Hkv, n, d)) if given_lm else None
    for union in (0, 1):
        r = oracle_lib.prefill_variant(Q, K, V, lm, 16, 3, own, bounds=bounds, union_softmax=union)
        if union:
            continue
        ref = varlen.varlen_prefill(Q, K, V, bounds, 3, own, lm=lm)
        np.testing.assert_array_equal(r["idx"], ref["idx"].reshape(B * L, Hkv, 3))
        np.testing.assert_allclose(r["O"], ref["O"].reshape(B * L, H, d), atol=1e-12, rtol=0)


def test_varlen_union_softmax_of_every_chunk_is_causal_attention(oracle_lib):
    """Variable chunks, every visible chunk selected and the own chunk: one
    softmax over all keys up to t, i.e. causal attention (float64 SDPA)."""
    Q, K, V, _ = rand_case(41, 1, 40, 4, 2, 8, 8)
    bounds = [0, 3, 11, 12, 25, 33, 40]
    r = oracle_lib.prefill_variant(Q, K, V, None, 8, 6, 1, bounds=bounds, union_softmax=1)
    ref = sdpa_causal(Q, K, V, 2)
    np.testing.assert_allclose(r["O"].reshape(ref.shape), ref, atol=1e-12, rtol=0)


def test_varlen_uniform_bounds_equal_fixed_chunks(oracle_lib):
    """Boundaries every S tokens (the last chunk partial and, unlike the fixed
    form, holding a landmark of its own): selection over the complete chunks
    is unchanged only where the partial chunk is not visible, i.e. everywhere
    when L is a multiple of S; then the outputs equal the fixed-chunk oracle."""
    Q, K, V, lm = rand_case(42, 2, 64, 4, 2, 8, 8)
    bounds = list(range(0, 65, 8))
    for own in (0, 1):
        r = oracle_lib.prefill_variant(Q, K, V, lm, 8, 3, own, bounds=bounds)
        ref = oracle_lib.prefill(Q, K, V, lm, 8, 3, own)
        np.testing.assert_array_equal(r["idx"], ref["idx"])
        np.testing.assert_allclose(r["O"], ref["O"], atol=1e-13, rtol=0)
