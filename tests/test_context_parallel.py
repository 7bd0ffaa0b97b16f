"""Decode split over sequence shards (the multi-GPU form with an exchange
step): the fp64 restatement in oracle/context_parallel.py against the pinned
single-GPU oracle decode, and the two exchanges (candidate gather, fusion-state
gather) run between two gloo ranks on CPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import context_parallel as cp


def case(seed, B=2, H=8, Hkv=2, d=16, S=16, Nc=37):
    rng = np.random.default_rng(seed)
    Lc = Nc * S
    return (rng.standard_normal((B, H, d)), rng.standard_normal((B, Hkv, Lc, d)),
            rng.standard_normal((B, Hkv, Lc, d)), rng.standard_normal((B, Hkv, Nc, d)))


def test_shard_ranges_cover_the_chunks_in_order():
    for Nc, R in [(37, 1), (37, 2), (37, 7), (5, 8), (0, 3)]:
        rg = cp.shard_ranges(Nc, R)
        assert len(rg) == R and rg[0][0] == 0 and rg[-1][1] == Nc
        assert all(a[1] == b[0] for a, b in zip(rg, rg[1:]))
        assert max(c1 - c0 for c0, c1 in rg) - min(c1 - c0 for c0, c1 in rg) <= 1


@pytest.mark.parametrize("n_shards", [1, 2, 3, 7])
@pytest.mark.parametrize("topk", [1, 4, 9])
def test_split_decode_equals_single_gpu_decode(oracle_lib, n_shards, topk):
    q, K, V, lm = case(40 + n_shards + 10 * topk)
    ref = oracle_lib.decode(q, K, V, lm, 16, topk)
    got = cp.decode(q, K, V, lm, 16, topk, n_shards)
    np.testing.assert_array_equal(got["idx"], ref["idx"])
    np.testing.assert_allclose(got["O"], ref["O"], atol=1e-12)


def test_fewer_chunks_than_topk_and_shards_smaller_than_topk(oracle_lib):
    q, K, V, lm = case(7, Nc=5)
    ref = oracle_lib.decode(q, K, V, lm, 16, 8)
    got = cp.decode(q, K, V, lm, 16, 8, n_shards=3)
    np.testing.assert_array_equal(got["idx"], ref["idx"])
    np.testing.assert_allclose(got["O"], ref["O"], atol=1e-12)


def test_selection_concentrated_in_one_shard(oracle_lib):
    # the best chunks all lie in the last shard: the other shards' states are
    # empty and must drop out of the combination
    q, K, V, lm = case(8, Nc=24)
    G = q.shape[1] // lm.shape[1]
    for g in range(lm.shape[1]):
        qbar = q[:, g * G:(g + 1) * G].mean(axis=1)            # [B, d]
        lm[:, g, 18:] += 6.0 * qbar[:, None, :] / np.linalg.norm(qbar, axis=1)[:, None, None]
    ref = oracle_lib.decode(q, K, V, lm, 16, 4)
    assert (ref["idx"] >= 18).all()
    got = cp.decode(q, K, V, lm, 16, 4, n_shards=4)
    np.testing.assert_array_equal(got["idx"], ref["idx"])
    np.testing.assert_allclose(got["O"], ref["O"], atol=1e-12)


def test_equal_scores_across_shards_go_to_the_lower_index(oracle_lib):
    # chunks 3 and 30 (different shards) carry the same landmark: a tie that the
    # merge must break by the lower global index, as the single-GPU selection does
    q, K, V, lm = case(9, Nc=40)
    lm[:, :, 30] = lm[:, :, 3]
    G = q.shape[1] // lm.shape[1]
    for g in range(lm.shape[1]):
        qbar = q[:, g * G:(g + 1) * G].mean(axis=1)
        lm[:, g, 3] += 20.0 * qbar / np.linalg.norm(qbar, axis=1)[:, None]
        lm[:, g, 30] = lm[:, g, 3]
    ref = oracle_lib.decode(q, K, V, lm, 16, 1)
    assert (ref["idx"] == 3).all()
    got = cp.decode(q, K, V, lm, 16, 1, n_shards=2)
    np.testing.assert_array_equal(got["idx"], ref["idx"])


# ---------------------------------------------------------------- two gloo ranks
def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, topk, q_):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, K, V, lm = case(11)
        S = 16
        d = q.shape[-1]
        scale = 1.0 / np.sqrt(d)
        c0, c1 = cp.shard_ranges(lm.shape[2], world)[rank]
        # this rank holds only its slice of the cache and landmarks
        Ks, Vs, lms = K[:, :, c0 * S:c1 * S], V[:, :, c0 * S:c1 * S], lm[:, :, c0:c1]
        sc, ix = cp.local_candidates(q, lms, c0, topk, scale)
        # exchange 1: every rank gathers all candidates
        scs = [torch.empty(sc.shape, dtype=torch.float64) for _ in range(world)]
        ixs = [torch.empty(ix.shape, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(scs, torch.from_numpy(sc))
        dist.all_gather(ixs, torch.from_numpy(ix))
        idx = cp.merge_candidates([t.numpy() for t in scs], [t.numpy() for t in ixs], topk)
        m, Z, acc = cp.local_state(q, Ks, Vs, lms, c0, idx, S, scale)
        # exchange 2: every rank gathers all fusion states, combined in rank order
        gathered = []
        for a in (m, Z, acc):
            parts = [torch.empty(a.shape, dtype=torch.float64) for _ in range(world)]
            dist.all_gather(parts, torch.from_numpy(np.ascontiguousarray(a)))
            gathered.append([p.numpy() for p in parts])
        O = cp.combine_states(*gathered)
        q_.put((rank, idx, O))
    finally:
        dist.destroy_process_group()


def test_two_rank_exchange_matches_single_gpu_decode(oracle_lib):
    world, topk = 2, 5
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, topk, q_)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q_.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, K, V, lm = case(11)
    ref = oracle_lib.decode(q, K, V, lm, 16, topk)
    for rank, idx, O in res:
        np.testing.assert_array_equal(idx, ref["idx"])
        np.testing.assert_allclose(O, ref["O"], atol=1e-12)
