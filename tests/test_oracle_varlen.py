"""Pins for the variable-length-chunk restatement (oracle/varlen.py): with
uniform boundaries it equals the C oracle's fixed-chunk prefill (input and
DHSA landmarks), one chunk is causal attention, the landmark of a chunk of
constant keys is sqrt(|C|) times the key, and the selection only ever names
chunks that end before the query's own chunk."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import varlen


def case(seed, B=2, L=45, H=4, Hkv=2, d=8, S=8):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, L, H, d)), rng.standard_normal((B, Hkv, L, d)),
            rng.standard_normal((B, Hkv, L, d)), rng.standard_normal((B, Hkv, L // S, d)))


@pytest.mark.parametrize("own", [0, 1])
@pytest.mark.parametrize("dhsa", [False, True])
def test_uniform_boundaries_equal_fixed_chunks(oracle_lib, own, dhsa):
    Q, K, V, lm = case(1 + own + 2 * dhsa)
    S, L = 8, Q.shape[1]
    bounds = list(range(0, L, S)) + [L]               # the tail chunk is partial
    nfull = L // S
    lm_v = None if dhsa else np.concatenate([lm, np.zeros((2, 2, 1, 8))], axis=2)[:, :, :len(bounds) - 1]
    r = varlen.varlen_prefill(Q, K, V, bounds, 3, own, lm=lm_v)
    ref = oracle_lib.prefill(Q, K, V, None if dhsa else lm, S, 3, own_chunk=own)
    B, L, H, d = Q.shape
    np.testing.assert_array_equal(r["idx"].reshape(B * L, -1, 3), ref["idx"])
    np.testing.assert_allclose(r["O"].reshape(B * L, H, d), ref["O"], atol=1e-12)
    assert nfull == len(bounds) - 2                    # the partial tail is never selectable


def test_single_chunk_is_causal_attention():
    Q, K, V, _ = case(2)
    B, L, H, d = Q.shape
    G = H // K.shape[1]
    r = varlen.varlen_prefill(Q, K, V, [0, L], 4, 1)
    q = torch.tensor(Q).permute(0, 2, 1, 3)
    k = torch.tensor(K).repeat_interleave(G, dim=1)
    v = torch.tensor(V).repeat_interleave(G, dim=1)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(r["O"], ref, atol=1e-12)
    assert (r["idx"] == -1).all()


def test_landmark_of_constant_keys():
    rng = np.random.default_rng(3)
    bounds = [0, 3, 10, 11, 20]
    K = np.zeros((1, 2, 20, 4))
    consts = rng.standard_normal((2, 4, 4))
    for i in range(4):
        K[0, :, bounds[i]:bounds[i + 1]] = consts[:, i][:, None, :]
    lm = varlen.varlen_landmarks(K, bounds)
    for i in range(4):
        np.testing.assert_allclose(lm[0, :, i], np.sqrt(bounds[i + 1] - bounds[i]) * consts[:, i],
                                   atol=1e-14)


def test_selection_names_only_finished_chunks():
    Q, K, V, _ = case(4, L=60)
    rng = np.random.default_rng(4)
    cuts = np.sort(rng.choice(np.arange(1, 60), size=9, replace=False))
    bounds = np.concatenate([[0], cuts, [60]])
    r = varlen.varlen_prefill(Q, K, V, bounds, 3, 1)
    for t in range(60):
        own = int(np.searchsorted(bounds, t, side="right")) - 1
        sel = r["idx"][:, t]
        assert ((sel == -1) | (sel < own)).all()
        assert ((sel >= 0).sum(axis=-1) == min(3, own)).all()
