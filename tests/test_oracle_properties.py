"""Properties of the fp64 oracle over randomly drawn small shapes (hypothesis):
what the method's definition fixes for every shape, not only for the fixed
cases of test_oracle.py.

- selection: distinct visible chunks (i < t // S), ordered by group score
  (desc) then index (asc), exactly min(K, t // S) of them, -1 after;
- fusion weights: sum to 1 over the selected slots, 0 on padding;
- no visible chunk and no own term: O = 0; with the own term alone (K = 0
  visible): O is causal attention over the token's own chunk;
- decode split over any number of sequence shards equals single-GPU decode.
"""
import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import context_parallel as cp

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)


@st.composite
def prefill_case(draw):
    S = draw(st.sampled_from([4, 8, 16]))
    G = draw(st.sampled_from([1, 2, 4]))
    Hkv = draw(st.integers(1, 2))
    L = draw(st.integers(1, 9 * S + S - 1))
    topk = draw(st.integers(1, 6))
    own = draw(st.integers(0, 1))
    d = draw(st.sampled_from([4, 8]))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    return S, G, Hkv, L, topk, own, d, seed


@SETTINGS
@given(prefill_case())
def test_prefill_invariants(oracle_lib, case):
    S, G, Hkv, L, topk, own, d, seed = case
    H, B = G * Hkv, 1
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, L, H, d))
    K = rng.standard_normal((B, Hkv, L, d))
    V = rng.standard_normal((B, Hkv, L, d))
    lm = rng.standard_normal((B, Hkv, L // S, d))
    r = oracle_lib.prefill(Q, K, V, lm, S, topk, own_chunk=own)
    scale = 1.0 / math.sqrt(d)
    for t in range(L):
        nvis = t // S
        keff = min(topk, nvis)
        for g in range(Hkv):
            sel = r["idx"][t, g]
            assert (sel[keff:] == -1).all() and (sel[:keff] >= 0).all()
            chosen = sel[:keff]
            assert len(set(chosen.tolist())) == keff and (chosen < nvis).all()
            # rank order: group score desc, then index asc, and nothing better left out
            qbar = Q[0, t, g * G:(g + 1) * G].mean(axis=0)
            s = scale * (lm[0, g, :nvis] @ qbar)
            best = np.lexsort((np.arange(nvis), -s))[:keff]
            np.testing.assert_array_equal(chosen, best)
        w = r["w"][t]
        if keff:
            np.testing.assert_allclose(w[:, :keff].sum(axis=1), 1.0, atol=1e-12)
        assert (w[:, keff:] == 0).all()
        if keff == 0 and not own:
            assert (r["O"][t] == 0).all()
        if keff == 0 and own:
            # causal attention over keys c*S .. t of the token's own chunk
            c0 = (t // S) * S
            for h in range(H):
                g = h // G
                lg = scale * (K[0, g, c0:t + 1] @ Q[0, t, h])
                p = np.exp(lg - lg.max())
                np.testing.assert_allclose(r["O"][t, h], (p / p.sum()) @ V[0, g, c0:t + 1], atol=1e-12)


@SETTINGS
@given(st.integers(1, 40), st.integers(1, 9), st.integers(1, 6), st.integers(0, 2 ** 31 - 1))
def test_split_decode_equals_decode_for_any_shard_count(oracle_lib, Nc, topk, n_shards, seed):
    S, d, H, Hkv, B = 8, 8, 4, 2, 1
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, d))
    K = rng.standard_normal((B, Hkv, Nc * S, d))
    V = rng.standard_normal((B, Hkv, Nc * S, d))
    lm = rng.standard_normal((B, Hkv, Nc, d))
    ref = oracle_lib.decode(q, K, V, lm, S, topk)
    got = cp.decode(q, K, V, lm, S, topk, n_shards)
    np.testing.assert_array_equal(got["idx"], ref["idx"])
    np.testing.assert_allclose(got["O"], ref["O"], atol=1e-12)
