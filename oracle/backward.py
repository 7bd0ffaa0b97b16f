"""fp64 restatement of the prefill backward pass (gradients of O).

TEST INFRASTRUCTURE ONLY: the reference for a future backward kernel.  Nothing
in the library imports it.

The forward is the one the oracle computes (HiLS Attention abstract: attention
inside each retrieved chunk, outputs fused by weights from the retrieval
scores; HSA "Methodology in Plain English": per-token top-K over chunk
landmarks; DHSA "What carries the argument": landmark sqrt(S) * chunk mean).
For query row (t, h) of KV group g with selected chunks i_1 .. i_K:

    z_k = scale * q_h . l_{i_k},   w = softmax(z)
    a_kj = scale * q_h . k_j (j in chunk i_k),  p_k = softmax(a_k),  o_k = p_k V
    own: the same attention over keys c_t*S .. t, weight 1
    O = sum_k w_k o_k + own

The selection itself is a hard top-K: it takes no gradient, and the indices
are held fixed (those of the forward).  Reverse-mode steps, per row:

    dw_k = dO . o_k,   dz = w * (dw - sum_k w_k dw_k)
    do_k = w_k dO      (own: dO)
    dV_j += p_kj do_k, dp_kj = do_k . v_j, da_k = p_k * (dp_k - p_k . dp_k)
    dq_h += scale * (sum_j da_kj k_j + sum_k dz_k l_{i_k})
    dk_j += scale * da_kj q_h,   dl_{i_k} += scale * dz_k q_h

With DHSA landmarks (computed from K), dl flows back into K: every key of
chunk i gets sqrt(S) / S * dl_i.  Plain numpy, float64, loops over rows.
"""
from __future__ import annotations

import numpy as np


def _softmax(x):
    e = np.exp(x - x.max())
    return e / e.sum()


def select(Q, lm, S: int, topk: int, scale: float) -> np.ndarray:
    """Forward selection, [B, L, Hkv, topk] (-1 padding): per (b, t, g) the
    top-K visible chunks by group score (desc), then index (asc)."""
    B, L, H, d = Q.shape
    Hkv = lm.shape[1]
    G = H // Hkv
    idx = np.full((B, L, Hkv, topk), -1, dtype=np.int64)
    for b in range(B):
        for t in range(L):
            nvis = min(t // S, lm.shape[2])
            for g in range(Hkv):
                qbar = Q[b, t, g * G:(g + 1) * G].mean(axis=0)
                s = scale * (lm[b, g, :nvis] @ qbar)
                order = np.lexsort((np.arange(nvis), -s))[:topk]
                idx[b, t, g, :len(order)] = order
    return idx


def dhsa_landmarks(K, S: int) -> np.ndarray:
    """sqrt(S) * mean of each complete chunk's keys, [B, Hkv, L // S, d]."""
    B, Hkv, L, d = K.shape
    Nc = L // S
    return np.sqrt(S) * K[:, :, :Nc * S].reshape(B, Hkv, Nc, S, d).mean(axis=3)


def prefill_backward(Q, K, V, lm, S: int, topk: int, own_chunk: int, dO, scale: float = 0.0,
                     idx=None):
    """Gradients of sum(dO * O) for the oracle's prefill forward.

    Q [B,L,H,d], K/V [B,Hkv,L,d], lm [B,Hkv,L//S,d] or None (DHSA from K),
    dO [B,L,H,d].  Returns dict O (the forward output), dQ, dK, dV, dlm (None
    in DHSA mode, whose landmark gradient is folded into dK) and idx."""
    Q, K, V, dO = (np.asarray(a, dtype=np.float64) for a in (Q, K, V, dO))
    B, L, H, d = Q.shape
    Hkv = K.shape[1]
    G = H // Hkv
    scale = scale if scale else 1.0 / np.sqrt(d)
    dhsa = lm is None
    lmv = dhsa_landmarks(K, S) if dhsa else np.asarray(lm, dtype=np.float64)
    if idx is None:
        idx = select(Q, lmv, S, topk, scale)
    O = np.zeros_like(Q)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    dlm = np.zeros_like(lmv)

    def attend(b, g, lo, hi, q):
        """softmax attention of q over keys lo .. hi-1 -> (p, o)."""
        p = _softmax(scale * (K[b, g, lo:hi] @ q))
        return p, p @ V[b, g, lo:hi]

    def attend_back(b, g, lo, hi, q, p, do, dq):
        dV[b, g, lo:hi] += np.outer(p, do)
        dp = V[b, g, lo:hi] @ do
        da = p * (dp - p @ dp)
        dq += scale * (da @ K[b, g, lo:hi])
        dK[b, g, lo:hi] += scale * np.outer(da, q)

    for b in range(B):
        for t in range(L):
            c = t // S
            for h in range(H):
                g = h // G
                q = Q[b, t, h]
                sel = [int(i) for i in idx[b, t, g] if i >= 0]
                dq = np.zeros(d)
                if sel:
                    z = scale * (lmv[b, g, sel] @ q)
                    w = _softmax(z)
                    po = [attend(b, g, i * S, (i + 1) * S, q) for i in sel]
                    O[b, t, h] += sum(wk * o for wk, (_, o) in zip(w, po))
                    dw = np.array([dO[b, t, h] @ o for _, o in po])
                    dz = w * (dw - w @ dw)
                    for k, i in enumerate(sel):
                        attend_back(b, g, i * S, (i + 1) * S, q, po[k][0], w[k] * dO[b, t, h], dq)
                        dq += scale * dz[k] * lmv[b, g, i]
                        dlm[b, g, i] += scale * dz[k] * q
                if own_chunk:
                    p, o = attend(b, g, c * S, t + 1, q)
                    O[b, t, h] += o
                    attend_back(b, g, c * S, t + 1, q, p, dO[b, t, h], dq)
                dQ[b, t, h] = dq
    if dhsa:
        Nc = lmv.shape[2]
        dK[:, :, :Nc * S] += np.repeat(dlm * (np.sqrt(S) / S), S, axis=2)
        dlm_out = None
    else:
        dlm_out = dlm
    return {"O": O, "dQ": dQ, "dK": dK, "dV": dV, "dlm": dlm_out, "idx": idx}
