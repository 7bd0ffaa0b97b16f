"""Pins for the union-softmax retrieval variant (oracle/variants.py): it reduces
to causal attention when every visible chunk is selected (checked against
PyTorch's scaled_dot_product_attention in float64), to attention over the
argmax chunk at K = 1 without the own term, it does not depend on the order of
the selected chunks, it shares the selection of the C oracle, and it equals the
chunk outputs fused with their own softmax normalisers as weights."""
import numpy as np
import torch
import torch.nn.functional as F

from oracle import variants


def case(seed, B=2, L=53, H=4, Hkv=2, d=8, S=8):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, L, H, d)), rng.standard_normal((B, Hkv, L, d)),
            rng.standard_normal((B, Hkv, L, d)), rng.standard_normal((B, Hkv, L // S, d)))


def test_all_chunks_selected_is_causal_attention():
    Q, K, V, lm = case(1)
    B, L, H, d = Q.shape
    G = H // K.shape[1]
    r = variants.flat_union_prefill(Q, K, V, lm, 8, topk=L, own_chunk=1)
    q = torch.tensor(Q).permute(0, 2, 1, 3)                       # [B, H, L, d]
    k = torch.tensor(K).repeat_interleave(G, dim=1)
    v = torch.tensor(V).repeat_interleave(G, dim=1)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(r["O"], ref, atol=1e-12)


def test_top1_without_own_term_is_attention_over_the_argmax_chunk():
    Q, K, V, lm = case(2)
    S, G = 8, 2
    r = variants.flat_union_prefill(Q, K, V, lm, S, topk=1, own_chunk=0)
    scale = 1 / np.sqrt(Q.shape[-1])
    for b in range(Q.shape[0]):
        for t in range(Q.shape[1]):
            for h in range(Q.shape[2]):
                g = h // G
                i = r["idx"][b, t, g, 0]
                if i < 0:
                    assert (r["O"][b, t, h] == 0).all()
                    continue
                lg = scale * (K[b, g, i * S:(i + 1) * S] @ Q[b, t, h])
                p = np.exp(lg - lg.max())
                np.testing.assert_allclose(r["O"][b, t, h], (p / p.sum()) @ V[b, g, i * S:(i + 1) * S],
                                           atol=1e-12)


def test_order_of_the_selected_chunks_does_not_matter():
    Q, K, V, lm = case(3)
    r = variants.flat_union_prefill(Q, K, V, lm, 8, topk=3, own_chunk=1)
    rev = r["idx"].copy()
    for row in rev.reshape(-1, 3):
        n = int((row >= 0).sum())
        row[:n] = row[:n][::-1]
    r2 = variants.flat_union_prefill(Q, K, V, lm, 8, topk=3, own_chunk=1, idx=rev)
    np.testing.assert_allclose(r2["O"], r["O"], atol=1e-12)


def test_selection_is_the_c_oracles(oracle_lib):
    Q, K, V, lm = case(4)
    r = variants.flat_union_prefill(Q, K, V, lm, 8, topk=3, own_chunk=1)
    ref = oracle_lib.prefill(Q, K, V, lm, 8, 3, own_chunk=1)
    B, L = Q.shape[:2]
    np.testing.assert_array_equal(r["idx"].reshape(B * L, -1, 3), ref["idx"])


def test_equals_chunk_outputs_fused_by_their_normalisers():
    Q, K, V, lm = case(5)
    S, G, topk = 8, 2, 3
    r = variants.flat_union_prefill(Q, K, V, lm, S, topk=topk, own_chunk=0)
    scale = 1 / np.sqrt(Q.shape[-1])
    b, t = 1, Q.shape[1] - 1
    for h in range(Q.shape[2]):
        g = h // G
        Zs, os_ = [], []
        for i in r["idx"][b, t, g]:
            e = np.exp(scale * (K[b, g, i * S:(i + 1) * S] @ Q[b, t, h]))
            Zs.append(e.sum())
            os_.append((e / e.sum()) @ V[b, g, i * S:(i + 1) * S])
        Zs = np.array(Zs)
        np.testing.assert_allclose(r["O"][b, t, h], (Zs / Zs.sum()) @ np.array(os_), atol=1e-12)
