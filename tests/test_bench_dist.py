"""bench.py's multi-GPU host logic on CPU: two gloo ranks check that the
whole-job throughput is the work summed over ranks divided by the slowest
rank's time, and that every rank draws an independent batch (weak scaling)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from hierarchical_chunk_sparse_landmark_b200.workloads import WORKLOADS, make_prefill_inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_env()
        assert (ws, r, local) == (world, rank, rank)
        # rank r processed (r+1) units in (r+1)*0.5 s
        units, secs = bench.aggregate(dist, float(rank + 1), 0.5 * (rank + 1), "cpu")
        wl = WORKLOADS["train_prefill_bf16"].with_(B=1, L=256)
        x = make_prefill_inputs(wl.with_(seed=wl.seed + rank), "cpu")
        q_sum = torch.tensor([float(x["Q"].float().sum())])
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, q_sum)
        q.put((rank, units, secs, [float(g) for g in gathered]))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_and_independent_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, units, secs, sums in res:
        assert units == pytest.approx(3.0)        # 1 + 2 units over both ranks
        assert secs == pytest.approx(1.0)         # max over ranks, not the sum
        assert sums[0] != sums[1]                 # per-rank seeds give different batches


def test_single_process_aggregation_is_identity():
    assert bench.aggregate(None, 5.0, 2.0) == (5.0, 2.0)


def test_flop_and_byte_counts_match_definitions():
    wl = WORKLOADS["train_prefill_bf16"]
    f = bench.prefill_flops(wl)
    # hand count for one batch element, token by token
    tot = 0
    for t in range(wl.L):
        nvis = t // wl.S
        keff = min(wl.topk, nvis)
        own = t - wl.S * nvis + 1
        tot += (wl.Hkv * 2 * wl.d * nvis + wl.H * 2 * wl.d * keff + wl.H * 4 * wl.d * wl.S * keff
                + wl.H * 4 * wl.d * own)
    assert f["total"] == pytest.approx(wl.B * tot)
    d5 = WORKLOADS["decode_32m_bf16"]
    nc = d5.L // d5.S
    assert bench.decode_bytes(d5) == d5.B * (d5.Hkv * nc * d5.d * 2 + d5.Hkv * 8 * 64 * d5.d * 2 * 2
                                             + 2 * d5.H * d5.d * 2)


def test_work_counts_of_the_long_and_decode_workloads():
    # the published per-step counts of the long prefill and the two decode
    # workloads (algorithmic work only, dense work avoided not counted)
    lp = WORKLOADS["long_prefill_bf16"]
    f = bench.prefill_flops(lp)
    assert f["selection"] == pytest.approx(6.87e10, rel=2e-3)
    assert f["fusion"] == pytest.approx(4.29e9, rel=2e-3)
    assert f["in_chunk"] == pytest.approx(5.485e11, rel=2e-3)
    assert f["own_chunk"] == pytest.approx(3.49e10, rel=2e-3)
    # DHSA landmark pass: 1 x 2 x 131072 x 128 bf16 keys read, 2048 fp32 landmarks per head written
    assert bench.landmark_bytes(lp) == 2 * (131072 * 128 * 2 + 2048 * 128 * 4)
    assert bench.decode_bytes(WORKLOADS["decode_32m_bf16"]) == 268_967_936
    assert bench.decode_bytes(WORKLOADS["batched_decode_bf16"]) == 285_474_816


def test_traffic_record_is_tied_to_its_workload():
    # the committed ncu DRAM figure of the attention kernel was taken on one
    # workload; other workloads must not report it
    files = ["hierarchical_chunk_sparse_landmark_b200/csrc/attend_tc.cu"]
    t = bench.measured_traffic("attend_tc", files, workload="train_prefill_bf16")
    if t is None:
        pytest.skip("traffic record predates the current attend_tc.cu")
    assert t > 0
    assert bench.measured_traffic("attend_tc", files, workload="long_prefill_bf16") is None
    assert bench.measured_traffic("attend_tc", files, "dram_write_bytes_per_launch",
                                  workload="long_prefill_bf16") is None


def test_launch_ranks_starts_a_whole_job(capfd):
    # bench.launch_ranks (what `bench.py --gpus N` does without torchrun) on a
    # CPU stand-in for the device step: two ranks join one gloo group, the
    # line reports n_gpus = 2 and the work summed over both ranks.
    import json
    import sys
    standin = os.path.join(os.path.dirname(__file__), "_bench_rank_standin.py")
    rc = bench.launch_ranks(2, [sys.executable, standin], timeout_s=120)
    assert rc == 0
    out = capfd.readouterr().out.strip().splitlines()
    line = json.loads(out[-1])
    assert line["n_gpus"] == 2 and line["units"] == pytest.approx(3.0)
    assert line["seconds"] >= 0.1                   # the slower rank's time
    assert line["value"] == pytest.approx(line["units"] / line["seconds"])


def test_bench_main_self_launches_without_a_launcher(monkeypatch):
    calls = []
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench, "launch_ranks", lambda n, cmd, **kw: calls.append((n, cmd)) or 0)
    assert bench.main(["--gpus", "4", "--steps", "3", "--warmup", "3"]) == 0
    n, cmd = calls[0]
    assert n == 4 and cmd[1].endswith("bench.py") and cmd[2:] == ["--gpus", "4", "--steps", "3",
                                                                  "--warmup", "3"]
