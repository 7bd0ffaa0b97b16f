"""fp64 restatement of decode split over sequence shards (context parallel).

TEST INFRASTRUCTURE ONLY: the reference for a multi-GPU decode whose KV cache
and landmarks are cut into contiguous chunk ranges, one per rank.  Nothing in
the library imports it.

The method (HSA "Methodology in Plain English": per-token top-K retrieval over
chunk landmarks; HiLS Attention abstract: attention inside each retrieved
chunk, outputs fused by the retrieval scores) is unchanged; only where each
step runs moves:

1. every shard scores its own chunks with the group's mean query and keeps its
   local top-K candidates (score, global chunk index);
2. exchange: all candidates are gathered and the global top-K is taken in the
   same total order as the single-GPU selection (larger score first, lower
   chunk index on ties);
3. every shard attends inside the selected chunks it holds and folds them into
   a per-head fusion state (m = largest fusion logit, Z = sum of exp(z - m),
   acc = sum of exp(z - m) * o);
4. exchange: the states are gathered and combined in shard order,
   O = sum_r exp(m_r - M) acc_r / sum_r exp(m_r - M) Z_r with M = max_r m_r.

A global top-K element is within its own shard's top K, so step 2 sees every
chunk it needs, and step 4 is the softmax over the selection written as a sum
over shards; the result equals the single-GPU decode.  Plain numpy, float64.
"""
from __future__ import annotations

import numpy as np


def shard_ranges(Nc: int, n_shards: int) -> list[tuple[int, int]]:
    """Contiguous chunk ranges [c0, c1) of nearly equal size, in order."""
    base, extra = divmod(Nc, n_shards)
    out, c = [], 0
    for r in range(n_shards):
        n = base + (1 if r < extra else 0)
        out.append((c, c + n))
        c += n
    return out


def _order(scores: np.ndarray, idx: np.ndarray, topk: int) -> np.ndarray:
    """Positions of the topk best (score desc, index asc) entries."""
    return np.lexsort((idx, -scores))[:topk]


def local_candidates(q, lm_shard, c0: int, topk: int, scale: float):
    """Step 1 on one shard: q [B,H,d], lm_shard [B,Hkv,n,d] holding chunks
    c0 .. c0+n-1.  Returns scores, global indices [B,Hkv,topk] (padding: -inf, -1)."""
    q = np.asarray(q, dtype=np.float64)
    lm = np.asarray(lm_shard, dtype=np.float64)
    B, H, d = q.shape
    _, Hkv, n, _ = lm.shape
    G = H // Hkv
    sc = np.full((B, Hkv, topk), -np.inf)
    ix = np.full((B, Hkv, topk), -1, dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            qbar = q[b, g * G:(g + 1) * G].mean(axis=0)
            s = scale * (lm[b, g] @ qbar)
            gi = np.arange(c0, c0 + n, dtype=np.int64)
            sel = _order(s, gi, topk)
            sc[b, g, :len(sel)] = s[sel]
            ix[b, g, :len(sel)] = gi[sel]
    return sc, ix


def merge_candidates(scores: list, indices: list, topk: int) -> np.ndarray:
    """Step 2: the global top-K over all shards' candidates -> idx [B,Hkv,topk]."""
    sc = np.concatenate(scores, axis=2)
    ix = np.concatenate(indices, axis=2)
    B, Hkv, _ = sc.shape
    out = np.full((B, Hkv, topk), -1, dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            valid = ix[b, g] >= 0
            s, i = sc[b, g][valid], ix[b, g][valid]
            sel = _order(s, i, topk)
            out[b, g, :len(sel)] = i[sel]
    return out


def local_state(q, K_shard, V_shard, lm_shard, c0: int, idx, S: int, scale: float):
    """Step 3 on one shard: the fusion state of the selected chunks it holds.
    K_shard, V_shard [B,Hkv,n*S,d], lm_shard [B,Hkv,n,d].  Returns m, Z [B,H]
    and acc [B,H,d] (m = -inf, Z = 0, acc = 0 where the shard holds none)."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K_shard, dtype=np.float64)
    V = np.asarray(V_shard, dtype=np.float64)
    lm = np.asarray(lm_shard, dtype=np.float64)
    B, H, d = q.shape
    _, Hkv, n, _ = lm.shape
    G = H // Hkv
    m = np.full((B, H), -np.inf)
    Z = np.zeros((B, H))
    acc = np.zeros((B, H, d))
    for b in range(B):
        for h in range(H):
            g = h // G
            zs, os_ = [], []
            for i in idx[b, g]:
                if i < c0 or i >= c0 + n:
                    continue                     # padding or another shard's chunk
                li = int(i) - c0
                zs.append(scale * float(q[b, h] @ lm[b, g, li]))
                Kc, Vc = K[b, g, li * S:(li + 1) * S], V[b, g, li * S:(li + 1) * S]
                logits = scale * (Kc @ q[b, h])
                p = np.exp(logits - logits.max())
                os_.append((p / p.sum()) @ Vc)
            if zs:
                z = np.array(zs)
                m[b, h] = z.max()
                e = np.exp(z - m[b, h])
                Z[b, h] = e.sum()
                acc[b, h] = e @ np.array(os_)
    return m, Z, acc


def combine_states(ms: list, Zs: list, accs: list) -> np.ndarray:
    """Step 4: O [B,H,d] from the shards' states, combined in shard order."""
    m = np.stack(ms)                                    # [R,B,H]
    M = m.max(axis=0)
    w = np.where(np.isfinite(m), np.exp(m - np.where(np.isfinite(M), M, 0.0)), 0.0)
    Z = (w * np.stack(Zs)).sum(axis=0)
    acc = (w[..., None] * np.stack(accs)).sum(axis=0)
    return np.where(Z[..., None] > 0, acc / np.where(Z > 0, Z, 1.0)[..., None], 0.0)


def decode(q, K, V, lm, S: int, topk: int, n_shards: int, scale: float = 0.0):
    """The whole split decode in one process: q [B,H,d], K/V [B,Hkv,Lc,d],
    lm [B,Hkv,Lc/S,d] -> dict O [B,H,d], idx [B,Hkv,topk]."""
    d = np.asarray(q).shape[-1]
    scale = scale if scale else 1.0 / np.sqrt(d)
    Nc = np.asarray(lm).shape[2]
    ranges = shard_ranges(Nc, n_shards)
    cand = [local_candidates(q, lm[:, :, c0:c1], c0, topk, scale) for c0, c1 in ranges]
    idx = merge_candidates([c[0] for c in cand], [c[1] for c in cand], topk)
    st = [local_state(q, K[:, :, c0 * S:c1 * S], V[:, :, c0 * S:c1 * S], lm[:, :, c0:c1], c0, idx,
                      S, scale) for c0, c1 in ranges]
    O = combine_states([s[0] for s in st], [s[1] for s in st], [s[2] for s in st])
    return {"O": O, "idx": idx}
