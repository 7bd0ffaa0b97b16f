"""fp64 restatement of prefill with variable-length chunks.

TEST INFRASTRUCTURE ONLY: the reference for a future variable-chunk kernel.
Nothing in the library imports it.

Dynamic Hierarchical Sparse Attention ("What carries the argument") cuts the
sequence into chunks of varying size and represents chunk C by sqrt(|C|)
times the mean of its keys, so that landmark scores of chunks of different
sizes stay comparable.  Everything else is the HiLS form the oracle computes
for fixed chunks (HiLS Attention abstract; HSA "Methodology in Plain
English"): per (t, g) the top-K chunks that end before the chunk holding t,
by group score (desc) then index (asc); softmax attention inside each; fusion
by the softmax of scale * q_h . l_k; plus causal attention over the start of
t's own chunk up to t.

Chunks are given by boundaries 0 = c_0 < c_1 < ... < c_n = L, shared by the
batch; chunk i holds tokens c_i .. c_{i+1} - 1.  Plain numpy, float64.
"""
from __future__ import annotations

import numpy as np


def varlen_landmarks(K, bounds) -> np.ndarray:
    """sqrt(|C_i|) * mean of chunk i's keys, [B, Hkv, n, d]."""
    K = np.asarray(K, dtype=np.float64)
    b = np.asarray(bounds)
    return np.stack([np.sqrt(b[i + 1] - b[i]) * K[:, :, b[i]:b[i + 1]].mean(axis=2)
                     for i in range(len(b) - 1)], axis=2)


def varlen_prefill(Q, K, V, bounds, topk: int, own_chunk: int, lm=None, scale: float = 0.0):
    """Q [B,L,H,d], K/V [B,Hkv,L,d], bounds [n+1], lm [B,Hkv,n,d] or None
    (sqrt(|C|) * mean form) -> dict O [B,L,H,d], idx [B,L,Hkv,topk] (-1 padding)."""
    Q, K, V = (np.asarray(a, dtype=np.float64) for a in (Q, K, V))
    B, L, H, d = Q.shape
    Hkv = K.shape[1]
    G = H // Hkv
    bnd = np.asarray(bounds, dtype=np.int64)
    assert bnd[0] == 0 and bnd[-1] == L and np.all(np.diff(bnd) > 0)
    scale = scale if scale else 1.0 / np.sqrt(d)
    lmv = varlen_landmarks(K, bnd) if lm is None else np.asarray(lm, dtype=np.float64)
    O = np.zeros_like(Q)
    idx = np.full((B, L, Hkv, topk), -1, dtype=np.int64)

    def attend(b, g, lo, hi, q):
        lg = scale * (K[b, g, lo:hi] @ q)
        p = np.exp(lg - lg.max())
        return (p / p.sum()) @ V[b, g, lo:hi]

    for b in range(B):
        for t in range(L):
            own = int(np.searchsorted(bnd, t, side="right")) - 1     # chunk holding t
            nvis = own                                              # chunks 0 .. own-1 end before it
            for g in range(Hkv):
                qbar = Q[b, t, g * G:(g + 1) * G].mean(axis=0)
                s = scale * (lmv[b, g, :nvis] @ qbar)
                sel = np.lexsort((np.arange(nvis), -s))[:topk]
                idx[b, t, g, :len(sel)] = sel
                for h in range(g * G, (g + 1) * G):
                    q = Q[b, t, h]
                    o = np.zeros(d)
                    if len(sel):
                        z = scale * (lmv[b, g, sel] @ q)
                        w = np.exp(z - z.max())
                        w /= w.sum()
                        for wk, i in zip(w, sel):
                            o += wk * attend(b, g, bnd[i], bnd[i + 1], q)
                    if own_chunk:
                        o += attend(b, g, bnd[own], t + 1, q)
                    O[b, t, h] = o
    return {"O": O, "idx": idx}
