"""fp64 restatement of a retrieval variant: one softmax over the union of the
selected chunks (DHSA form) instead of a softmax per chunk fused by the
retrieval scores (HiLS form).

TEST INFRASTRUCTURE ONLY: the reference for a future kernel of this variant.
Nothing in the library imports it.

Dynamic Hierarchical Sparse Attention ("What carries the argument") attends,
after the top-K chunk selection, with a single softmax over the keys of all
selected chunks together with the local keys; the landmark scores only choose
the chunks.  Per query row (t, h) of KV group g with selected chunks
i_1 .. i_K (the same selection as the HiLS form: group score, top-K, lower
index on ties):

    keys  = the S keys of every selected chunk, plus keys c_t*S .. t when the
            own chunk is attended
    O     = softmax(scale * q_h . keys) . values

Written as a fusion of chunk outputs this is sum_k Z_k o_k / sum_k Z_k with
Z_k the chunk's own softmax normaliser: the weights come from the keys, not
from the landmarks.  Plain numpy, float64.
"""
from __future__ import annotations

import numpy as np

from oracle.backward import dhsa_landmarks, select


def flat_union_prefill(Q, K, V, lm, S: int, topk: int, own_chunk: int, scale: float = 0.0,
                       idx=None):
    """Q [B,L,H,d], K/V [B,Hkv,L,d], lm [B,Hkv,L//S,d] or None (DHSA landmarks
    from K) -> dict O [B,L,H,d], idx [B,L,Hkv,topk]."""
    Q, K, V = (np.asarray(a, dtype=np.float64) for a in (Q, K, V))
    B, L, H, d = Q.shape
    Hkv = K.shape[1]
    G = H // Hkv
    scale = scale if scale else 1.0 / np.sqrt(d)
    lmv = dhsa_landmarks(K, S) if lm is None else np.asarray(lm, dtype=np.float64)
    if idx is None:
        idx = select(Q, lmv, S, topk, scale)
    O = np.zeros_like(Q)
    for b in range(B):
        for t in range(L):
            c = t // S
            for g in range(Hkv):
                rows = [np.arange(i * S, (i + 1) * S) for i in idx[b, t, g] if i >= 0]
                if own_chunk:
                    rows.append(np.arange(c * S, t + 1))
                if not rows:
                    continue
                r = np.concatenate(rows)
                for h in range(g * G, (g + 1) * G):
                    logits = scale * (K[b, g, r] @ Q[b, t, h])
                    p = np.exp(logits - logits.max())
                    O[b, t, h] = (p / p.sum()) @ V[b, g, r]
    return {"O": O, "idx": idx}
