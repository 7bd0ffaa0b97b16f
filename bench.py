"""Benchmark: hierarchical chunk-sparse landmark attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-decode] [--no-e2e] [--no-cpu-baseline]
                    [--no-extra] [--decode-workload NAME]

One step = one full hsa_prefill call (DHSA landmarks, selection, work lists,
in-chunk attention, fusion, own-chunk term) over one batch of the workload,
inputs resident in HBM.  The main line is the largest single-GPU prefill
workload (L = 131072, DHSA landmarks computed on the device, planted needle
chunks).  ``value`` is algorithmic TFLOP/s summed over ranks / max-over-ranks
device time (weak scaling: every rank runs its own independent batch, seeded
by rank; no collective on the data path).

The same JSON line carries: the roofline of the dominant kernel timed live
with CUDA events on the launching stream; the landmark kernel's HBM roofline;
an end-to-end figure through host buffers; the SM clocks sampled during the
timed region; the fp64 CPU oracle timed on a bounded sample of the same
workload, whose rows double as a parity sample of the GPU's outputs (near-ties
counted); the train-shape bf16 and the fp32 prefill workloads, each with its
roofline (tensor-core bf16 peak, resp. the FP32 CUDA-core peak); and the
32M-context and batched decode lines (tokens/s, HBM roofline, parity of every
sequence against the oracle).

``--gpus N`` without a launcher starts N ranks itself (one process per GPU).
``--impl reference`` times the fp64 CPU oracle (the only reference for this
method) on the host cores, each step a bounded sample of the workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0, "source": "fallback"}
L2_FLUSH_BYTES = 256 << 20          # > 126 MB L2
SM_COUNT = 148


# ----------------------------------------------------------------------------- work counts
def prefill_token_counts(wl):
    t = np.arange(wl.L, dtype=np.int64)
    nvis = t // wl.S
    keff = np.minimum(wl.topk, nvis)
    own = (t - wl.S * nvis + 1) if wl.own_chunk else np.zeros_like(t)
    return nvis, keff, own


def prefill_flops(wl) -> dict:
    """Algorithmic FLOPs of one prefill call (what the method must compute):
    selection once per KV group, fusion logits, in-chunk QK^T and PV, own-chunk
    causal attention.  Softmax exponentials and dense work avoided are not counted."""
    nvis, keff, own = prefill_token_counts(wl)
    d, H, Hkv, S, B = wl.d, wl.H, wl.Hkv, wl.S, wl.B
    sel = B * float((Hkv * 2 * d * nvis).sum())
    fuse = B * float((H * 2 * d * keff).sum())
    chunk = B * float((H * 4 * d * S * keff).sum())
    ownf = B * float((H * 4 * d * own).sum())
    return {"selection": sel, "fusion": fuse, "in_chunk": chunk, "own_chunk": ownf,
            "total": sel + fuse + chunk + ownf,
            # the tensor-core kernel computes the fusion logits in its S tiles
            "attention_kernel": chunk + ownf + fuse}


def backward_flops(wl) -> float:
    """Algorithmic FLOPs of one prefill backward (selection held fixed): per
    (token, head, selected chunk) the five 64 x d products of attention's
    backward -- scores recomputed, dO.V^T, dV, dQ, dK (2.5x the forward's two)
    -- plus the fusion logit, its dq and dl terms (3 x 2d); the own chunk the
    same five products over its causal keys."""
    _, keff, own = prefill_token_counts(wl)
    d, H, S, B = wl.d, wl.H, wl.S, wl.B
    chunk = B * float((H * 10 * d * S * keff).sum())
    fuse = B * float((H * 6 * d * keff).sum())
    ownf = B * float((H * 10 * d * own).sum())
    return chunk + fuse + ownf


def chunk_output_bytes(wl) -> float:
    """Bytes of fp16 chunk outputs the tensor-core attention writes (and the
    fusion reads back): one G*d block per selected (token, group, chunk) and
    one own-chunk block per (token, group).  Design traffic of the chunk-
    bucketed schedule, not algorithmic work: with random selections a token's
    chunks are processed on different SMs, so each chunk output crosses from
    an SM to L2 once."""
    _, keff, _ = prefill_token_counts(wl)
    return float(wl.B * wl.Hkv * (keff + 1).sum() * wl.G * wl.d * 2)


def decode_bytes(wl, lm_elem_bytes=2) -> float:
    """Algorithmic HBM bytes of one decode step: every visible landmark, the K
    and V of the selected chunks, q and O.  The full cache is never read."""
    Nc = wl.L // wl.S
    el = 2 if wl.dtype == "bf16" else 4
    per_seq = (wl.Hkv * Nc * wl.d * lm_elem_bytes + wl.Hkv * min(wl.topk, Nc) * wl.S * wl.d * el * 2
               + 2 * wl.H * wl.d * el)
    return float(wl.B * per_seq)


def landmark_bytes(wl) -> float:
    """HBM bytes the DHSA landmark pass must move: the keys of every complete
    chunk read once and each chunk's fp32 landmark written."""
    el = 2 if wl.dtype == "bf16" else 4
    Nc = wl.L // wl.S
    return float(wl.B * wl.Hkv * Nc * (wl.S * wl.d * el + wl.d * 4))


# ----------------------------------------------------------------------------- environment
def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str | None):
        self.uuid = gpu_uuid
        self.proc = None
        self.lines = []

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def make_events(n):
    """CUDA events with their handles created (torch creates them lazily at
    the first record, and the library needs the handle up front)."""
    import torch
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    return evs


def kernel_source_hash(files) -> str:
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, src_files, key: str = "dram_bytes_per_launch",
                     workload: str | None = None) -> float | None:
    """Per-launch DRAM bytes (`key`: read + write, or the write part alone) of
    `kernel` on `workload` from the committed ncu summary (entry
    "kernel:workload"), if it was taken on the current source of that kernel
    (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{kernel}:{workload}")
    if not d or d.get("source_hash") != kernel_source_hash(src_files):
        return None
    return d.get(key)


# kernel families of the roofline lines: ncu kernel-name pattern, source files
TRAFFIC_FAMILIES = {
    "attend_tc": (("attend_tc_kernel",), ["attend_tc.cu"]),
    "attend_simt": (("attend_simt_kernel",), ["attend_simt.cu"]),
    "decode": (("decode_scan_kernel", "decode_attend_kernel"), ["decode.cu"]),
    "landmarks": (("landmarks_kernel",), ["landmarks.cu"]),
}


def traffic_from_ncu(csv_path: str, workload: str, families: str = "",
                     out_path: str | None = None) -> dict:
    """Per-launch DRAM bytes of each kernel family from an ncu CSV of one
    workload (metrics dram__bytes_read.sum and dram__bytes_write.sum, one row
    per launch and metric): the median launch of every kernel of the family,
    summed over the family's kernels (the decode call is its scan plus its
    attend kernel).  Merged into profiles/traffic.json under "family:workload"
    with the hash of the family's current source.  `families` (comma-separated)
    limits the families taken from this CSV (a command can run two workloads)."""
    import csv
    import statistics as st
    per = {}
    hdr = None
    for r in csv.reader(open(csv_path)):
        if r and r[0] == "ID":
            hdr = r
            continue
        if not hdr or len(r) != len(hdr):
            continue
        d = dict(zip(hdr, r))
        name = d["Kernel Name"].split("(")[0].split("<")[0].split("::")[-1].strip().split(" ")[-1]
        if d["Metric Name"] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            val = float(d["Metric Value"].replace(",", ""))
            unit = d.get("Metric Unit", "byte").lower()
            val *= {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9}.get(unit, 1)
            per.setdefault((name, d["ID"]), {})[d["Metric Name"]] = val
    out_path = out_path or os.path.join(ROOT, "profiles", "traffic.json")
    table = json.load(open(out_path)) if os.path.exists(out_path) else {}
    wanted = [f for f in families.split(",") if f] or list(TRAFFIC_FAMILIES)
    for fam, (kernels, files) in TRAFFIC_FAMILIES.items():
        if fam not in wanted or not all(any(k == n for (n, _) in per) for k in kernels):
            continue
        rd = wr = 0.0
        for k in kernels:
            launches = [v for (n, _), v in per.items() if n == k]
            rd += st.median(v.get("dram__bytes_read.sum", 0.0) for v in launches)
            wr += st.median(v.get("dram__bytes_write.sum", 0.0) for v in launches)
        table[f"{fam}:{workload}"] = {
            "source_hash": kernel_source_hash([ATTN_SRC + f for f in files]),
            "dram_bytes_per_launch": rd + wr, "dram_write_bytes_per_launch": wr,
            "workload": workload, "kernels": list(kernels),
            "note": "dram__bytes_read.sum + dram__bytes_write.sum, median launch per kernel "
                    "(ncu --clock-control none, one pass)"}
    with open(out_path, "w") as f:
        json.dump(table, f, indent=2, sort_keys=True)
        f.write("\n")
    return table


# ----------------------------------------------------------------------------- dist
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate(dist, value_units: float, seconds: float, device=None):
    """Whole-job throughput: units summed over ranks / max-over-ranks time."""
    if dist is None:
        return value_units, seconds
    import torch
    t = torch.tensor([value_units, seconds], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    u = t[:1].clone()
    s = t[1:].clone()
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    dist.all_reduce(s, op=dist.ReduceOp.MAX)
    return float(u.item()), float(s.item())


# ----------------------------------------------------------------------------- GPU arm
METRIC = "HSA prefill TFLOP/s + 32M-ctx decode tokens/s (% of B200 roofline)"
ATTN_SRC = "hierarchical_chunk_sparse_landmark_b200/csrc/"


def fp32_simt_peak_tflops(peaks) -> float:
    """FP32 CUDA-core peak: 148 SMs x 128 FP32 lanes x 2 flop (FMA) x the
    maximum SM clock (1965 MHz on these GPUs) = 74.4 TFLOP/s."""
    return SM_COUNT * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12


def bench_prefill(args, name, dev, peaks, rank, dist, steps, warmup, keep_inputs=False):
    """Time hsa_prefill on one workload: `steps` timed calls after `warmup`,
    L2 flushed between calls (outside the events).  Returns the line's figures
    (and the device inputs and one call's outputs when keep_inputs)."""
    import torch

    import hierarchical_chunk_sparse_landmark_b200 as hsa
    from hierarchical_chunk_sparse_landmark_b200.workloads import WORKLOADS, make_prefill_inputs
    wl = WORKLOADS[name].with_(seed=WORKLOADS[name].seed + rank)
    x = make_prefill_inputs(wl, dev)
    flops = prefill_flops(wl)
    out = torch.empty_like(x["Q"])
    ws = hsa.workspace(hsa.prefill_workspace_size(wl.B, wl.H, wl.Hkv, wl.L, wl.d, wl.S,
                                                  wl.topk), dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    # timed steps record only the events the roofline needs (call start, both
    # sides of the attention kernel, call end): an event between two kernels
    # ends their programmatic launch overlap.  The stage breakdown comes from a
    # few extra calls with an event at every stage boundary.
    timed_ev = [make_events(4) for _ in range(steps)]
    n_brk = min(3, steps)
    stage_ev = [make_events(6) for _ in range(n_brk)]

    def step():
        hsa.prefill(x["Q"], x["K"], x["V"], x["lm"], S=wl.S, topk=wl.topk,
                    own_chunk=wl.own_chunk, out=out, ws=ws)

    for _ in range(warmup):
        step()
        flush.fill_(1)
    hsa.check(ws)
    kernels = hsa.last_call_kernels()
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    launches = 0
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(uuid) as clk:
        for i in range(steps):
            e = timed_ev[i]
            hsa.set_stage_events([e[0], None, None, e[1], e[2], e[3]])
            step()
            launches += hsa.last_call_launches()
            hsa.set_stage_events([])
            flush.fill_(1)           # L2 flush between timed steps (outside the events)
        torch.cuda.synchronize()
    hsa.check(ws)
    if dist is not None:
        dist.barrier()
    for i in range(n_brk):           # stage breakdown (not part of the timed value)
        hsa.set_stage_events(stage_ev[i])
        step()
        hsa.set_stage_events([])
        flush.fill_(1)
    torch.cuda.synchronize()
    hsa.check(ws)
    step_ms = [e[0].elapsed_time(e[3]) for e in timed_ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in timed_ev]
    fuse_ms = [e[2].elapsed_time(e[3]) for e in timed_ev]
    total_s = sum(step_ms) / 1e3
    units, tmax = aggregate(dist, flops["total"] * steps / 1e12, total_s, dev)
    tc_path = bool(kernels & 64)                     # HSA_K_ATTEND_TC
    attn_s = statistics.mean(attn_ms) / 1e3
    kfile = "attend_tc" if tc_path else "attend_simt"
    files = [ATTN_SRC + kfile + ".cu"]
    if tc_path:
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        kflops = flops["attention_kernel"]
        roofline = {"kernel": "attend_tc_kernel", "bound": "tensor",
                    "peak_source": peaks["source"] + " bf16 burst"}
        stage = {"landmarks": round(statistics.mean(e[0].elapsed_time(e[1]) for e in stage_ev), 4),
                 "selection": round(statistics.mean(e[1].elapsed_time(e[2]) for e in stage_ev), 4),
                 "work_list": round(statistics.mean(e[2].elapsed_time(e[3]) for e in stage_ev), 4),
                 "attention": round(statistics.mean(attn_ms), 4),
                 "fusion": round(statistics.mean(fuse_ms), 4),
                 "note": "attention and fusion from the timed calls; landmarks, selection and "
                         "work lists from %d extra calls with an event at every stage "
                         "boundary" % n_brk}
    else:
        # fp32 path: selection and attention+fusion on CUDA cores; the
        # attention kernel fuses in place, so the whole call is the unit
        peak = fp32_simt_peak_tflops(peaks)
        kflops = flops["total"]
        attn_s = statistics.mean(step_ms) / 1e3
        roofline = {"kernel": "select_kernel + attend_simt_kernel (whole call)", "bound": "alu",
                    "peak_source": "FP32 CUDA-core peak: 148 SMs x 128 lanes x 2 flop x "
                                   "%.0f MHz" % peaks.get("sm_max_mhz", 1965.0)}
        stage = None
    ach = kflops / attn_s / 1e12
    roofline.update({"achieved": round(ach, 3), "peak": round(peak, 1), "unit": "TFLOP/s",
                     "frac": round(ach / peak, 5),
                     "traffic": measured_traffic(kfile, files, workload=wl.name),
                     "algorithmic_flops_per_launch": kflops,
                     "ms_per_launch": round(attn_s * 1e3, 4)})
    if tc_path:
        # what the kernel actually streams: its chunk outputs, SM -> L2 -> HBM
        cob = chunk_output_bytes(wl)
        roofline["chunk_outputs"] = {"bytes_per_launch": cob,
                                     "achieved_GBps": round(cob / attn_s / 1e9, 1),
                                     "note": "fp16 chunk outputs written by the attention kernel "
                                             "and read back by the fusion kernel"}
    res = {"workload": wl.name, "value": round(units / tmax, 4), "unit": "TFLOP/s",
           "ms_per_step": round(tmax * 1e3 / steps, 4), "steps": steps,
           "config": {"workload": wl.name, "B": wl.B, "L": wl.L, "H": wl.H, "Hkv": wl.Hkv,
                      "d": wl.d, "S": wl.S, "topk": wl.topk, "own_chunk": wl.own_chunk,
                      "landmarks": wl.landmarks, "dtype": wl.dtype},
           "roofline": roofline, "clocks": clk.summary(), "gpu_launches": launches,
           "flops_per_step": flops}
    if stage is not None:
        res["stage_ms"] = stage
    extra = None
    if keep_inputs:
        O, idx, _ = hsa.prefill(x["Q"], x["K"], x["V"], x["lm"], S=wl.S, topk=wl.topk,
                                own_chunk=wl.own_chunk, idx_out=True, ws=ws)
        hsa.check(ws)
        extra = {"wl": wl, "x": x, "O": O, "idx": idx, "ws": ws}
    else:
        del x, out
    del flush
    torch.cuda.empty_cache()
    return res, extra


def bench_backward(args, name, dev, peaks, rank, dist, steps, warmup):
    """Time hsa_prefill_backward on one workload (the forward's selection held
    fixed, computed once outside the timed region; L2 flushed between calls).
    The roofline is the bf16 tensor peak when the key pass ran on the tensor
    cores, else the FP32 CUDA-core peak."""
    import torch

    import hierarchical_chunk_sparse_landmark_b200 as hsa
    from hierarchical_chunk_sparse_landmark_b200.workloads import WORKLOADS, make_prefill_inputs
    wl = WORKLOADS[name].with_(seed=WORKLOADS[name].seed + rank)
    x = make_prefill_inputs(wl, dev)
    _, idx, _ = hsa.prefill(x["Q"], x["K"], x["V"], x["lm"], S=wl.S, topk=wl.topk,
                            own_chunk=wl.own_chunk, idx_out=True)
    g = torch.Generator(device=dev)
    g.manual_seed(wl.seed + 11)
    dO = torch.randn(x["Q"].shape, generator=g, device=dev).to(x["Q"].dtype)
    f32 = dict(dtype=torch.float32, device=dev)
    dQ = torch.empty(x["Q"].shape, **f32)
    dK = torch.empty(x["K"].shape, **f32)
    dV = torch.empty(x["V"].shape, **f32)
    dlm = None if x["lm"] is None else torch.empty(x["lm"].shape, **f32)
    ws = hsa.workspace(hsa.prefill_backward_workspace_size(wl.B, wl.H, wl.Hkv, wl.L, wl.d, wl.S,
                                                           wl.topk, x["lm"] is None), dev,
                       "backward")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = [make_events(2) for _ in range(steps)]

    def step():
        hsa.prefill_backward(x["Q"], x["K"], x["V"], idx, dO, x["lm"], S=wl.S,
                             own_chunk=wl.own_chunk, dQ=dQ, dK=dK, dV=dV, dlm=dlm, ws=ws)

    for _ in range(warmup):
        step()
        flush.fill_(1)
    hsa.check(ws)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    launches = 0
    torch.cuda.synchronize()
    with ClockSampler(uuid) as clk:
        for i in range(steps):
            hsa.set_stage_events(ev[i])
            step()
            launches += hsa.last_call_launches()
            hsa.set_stage_events([])
            flush.fill_(1)
        torch.cuda.synchronize()
    hsa.check(ws)
    ms = [e[0].elapsed_time(e[1]) for e in ev]
    flops = backward_flops(wl)
    units, tmax = aggregate(dist, flops * steps / 1e12, sum(ms) / 1e3, dev)
    tc_path = bool(hsa.last_call_kernels() & 16384)          # HSA_K_BACKWARD_TC
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) if tc_path \
        else fp32_simt_peak_tflops(peaks)
    ach = flops / (statistics.mean(ms) / 1e3) / 1e12
    res = {"workload": wl.name, "value": round(units / tmax, 4), "unit": "TFLOP/s",
           "ms_per_step": round(tmax * 1e3 / steps, 4), "steps": steps,
           "config": {"workload": wl.name, "pass": "backward (dQ, dK, dV, dlm)", "B": wl.B,
                      "L": wl.L, "H": wl.H, "Hkv": wl.Hkv, "d": wl.d, "S": wl.S,
                      "topk": wl.topk, "own_chunk": wl.own_chunk, "landmarks": wl.landmarks,
                      "dtype": wl.dtype},
           "roofline": {"kernel": ("weights + sort + bwd_key_tc (tcgen05) + row finish + dl + "
                                   "reduce (whole call)") if tc_path else
                                  "bwd_row + sort + bwd_key + reduce (whole call)",
                        "bound": "tensor" if tc_path else "alu", "achieved": round(ach, 3),
                        "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(ach / peak, 5),
                        "traffic": None, "algorithmic_flops_per_launch": flops,
                        "peak_source": (peaks["source"] + " bf16 burst") if tc_path else
                                       "FP32 CUDA-core peak: 148 SMs x 128 lanes x 2 flop x "
                                       "%.0f MHz" % peaks.get("sm_max_mhz", 1965.0)},
           "clocks": clk.summary(), "gpu_launches": launches}
    del x, dO, dQ, dK, dV, dlm, flush
    torch.cuda.empty_cache()
    return res


def run_ours(args, dist, rank, world):
    import torch

    import hierarchical_chunk_sparse_landmark_b200 as hsa
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    main, keep = bench_prefill(args, args.workload, dev, peaks, rank, dist, args.steps,
                               args.warmup, keep_inputs=True)
    wl, x = keep["wl"], keep["x"]
    res = {
        "metric": METRIC,
        "value": main["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic (seeded N(0,1), per-rank seed)",
        "config": dict(main["config"], parallelism=f"independent batches x{world}",
                       l2="flushed between timed steps (256 MiB write)"),
        "stage_ms": main.get("stage_ms"),
        "flops_per_step": main["flops_per_step"],
        "roofline": main["roofline"], "clocks": main["clocks"], "gpu_launches": main["gpu_launches"],
    }
    if wl.landmarks == "dhsa":
        res["landmarks_roofline"] = landmark_roofline(hsa, wl, x, peaks, dev)
    if args.e2e:
        res["e2e"] = e2e_prefill(args, wl, x, keep["ws"], dev, dist)
    if rank == 0 and world == 1 and args.cpu_baseline:
        cb, par = cpu_baseline_and_parity(args, keep)
        res["cpu_baseline"] = cb
        res["parity"] = par
    del keep, x
    torch.cuda.empty_cache()
    if args.extra:
        for name, key in (("train_prefill_bf16", "train_prefill"),
                          ("tiny_prefill_f32", "tiny_prefill_f32")):
            if name != args.workload:
                r, _ = bench_prefill(args, name, dev, peaks, rank, dist, max(5, args.steps // 2), 3)
                r.pop("flops_per_step", None)
                res[key] = r
    if args.extra:
        res["backward_train"] = bench_backward(args, "train_prefill_bf16", dev, peaks, rank, dist,
                                               max(3, args.steps // 4), 3)
        res["backward_long"] = bench_backward(args, "long_prefill_bf16", dev, peaks, rank, dist, 3, 3)
    if args.decode:
        names = [args.decode_workload]
        if args.extra and "batched_decode_bf16" not in names:
            names.append("batched_decode_bf16")
        for name in names:
            key = "decode_32m" if name == "decode_32m_bf16" else \
                "decode_batched" if name == "batched_decode_bf16" else "decode_" + name
            res[key] = bench_decode(args, name, dev, peaks, rank, dist,
                                    parity=(rank == 0 and world == 1 and args.cpu_baseline))
    return res


def landmark_roofline(hsa, wl, x, peaks, dev) -> dict:
    """hsa_landmarks alone: the workload's keys repeated over the batch until
    they exceed 512 MB (4x L2), so back-to-back calls stream every key from
    HBM; CUDA events around 5 calls after 3 warm-up calls.  (The landmark
    stage inside a prefill step is the first work after the L2 flush and
    shares HBM with the write-back of the flush's dirty lines.)"""
    import torch
    try:
        reps = max(1, math.ceil((512 << 20) / x["K"].nbytes))
        Kb = x["K"].repeat(reps, 1, 1, 1).contiguous()
        out = torch.empty(Kb.shape[0], wl.Hkv, wl.L // wl.S, wl.d, dtype=torch.float32, device=dev)
        for _ in range(3):
            hsa.landmarks(Kb, S=wl.S, out=out)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(5):
            hsa.landmarks(Kb, S=wl.S, out=out)
        b.record()
        torch.cuda.synchronize()
        hsa.check()
        sec = a.elapsed_time(b) / 5 / 1e3
        nb = landmark_bytes(wl) * reps
        del Kb, out
        torch.cuda.empty_cache()
    except Exception as e:                      # an auxiliary figure: report, do not abort the line
        return {"kernel": "landmarks_kernel", "error": f"{type(e).__name__}: {e}"}
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    return {"kernel": "landmarks_kernel", "bound": "hbm", "achieved": round(nb / sec / 1e9, 1),
            "peak": hbm, "unit": "GB/s", "frac": round(nb / sec / 1e9 / hbm, 4),
            "algorithmic_bytes_per_launch": nb, "ms_per_launch": round(sec * 1e3, 4),
            "batch": f"{reps} x B={wl.B}", "peak_source": peaks["source"] + " copy bandwidth",
            "l2": "no flush: keys larger than L2, calls back to back"}


def e2e_prefill(args, wl, x, ws, dev, dist):
    """Same metric through the public API with host buffers, as a serving loop
    runs it: every step copies its Q/K/V/landmarks from pinned host memory to
    the device, calls hsa_prefill and copies O back to pinned host memory.
    Two buffer slots and three streams (host->device, compute, device->host)
    let the copies of one step overlap the neighbouring steps; events keep a
    slot's buffers until the step that last used them is done.  The timed
    region runs from the first input copy to the last output copy."""
    import torch

    import hierarchical_chunk_sparse_landmark_b200 as hsa
    hQ, hK, hV = (x[k].cpu().pin_memory() for k in ("Q", "K", "V"))
    hlm = x["lm"].cpu().pin_memory() if x["lm"] is not None else None
    slots = []
    for _ in range(2):
        slots.append({
            "Q": torch.empty_like(x["Q"]), "K": torch.empty_like(x["K"]),
            "V": torch.empty_like(x["V"]),
            "lm": torch.empty_like(x["lm"]) if hlm is not None else None,
            "O": torch.empty_like(x["Q"]),
            "hO": torch.empty(x["Q"].shape, dtype=x["Q"].dtype).pin_memory(),
            "in": torch.cuda.Event(), "comp": torch.cuda.Event(), "out": torch.cuda.Event()})
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    steps = max(4, args.steps // 2)
    # one workspace per compute stream (the binding caches them per stream)
    with torch.cuda.stream(s_comp):
        ws = hsa.workspace(hsa.prefill_workspace_size(wl.B, wl.H, wl.Hkv, wl.L, wl.d, wl.S,
                                                      wl.topk), dev)

    def issue(i):
        sl = slots[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(sl["comp"])          # step i-2 no longer reads the inputs
            sl["Q"].copy_(hQ, non_blocking=True)
            sl["K"].copy_(hK, non_blocking=True)
            sl["V"].copy_(hV, non_blocking=True)
            if hlm is not None:
                sl["lm"].copy_(hlm, non_blocking=True)
            sl["in"].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(sl["in"])
            if i >= 2:
                s_comp.wait_event(sl["out"])         # step i-2's O has been copied out
            hsa.prefill(sl["Q"], sl["K"], sl["V"], sl["lm"], S=wl.S, topk=wl.topk,
                        own_chunk=wl.own_chunk, out=sl["O"], ws=ws)
            sl["comp"].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(sl["comp"])
            sl["hO"].copy_(sl["O"], non_blocking=True)
            sl["out"].record(s_out)

    for i in range(2):
        issue(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        issue(i)
    s_out.wait_event(slots[(steps - 1) % 2]["out"])
    t1.record(s_out)
    torch.cuda.synchronize()
    hsa.check(ws)
    secs = t0.elapsed_time(t1) / 1e3
    flops = prefill_flops(wl)["total"]
    units, tmax = aggregate(dist, flops * steps / 1e12, secs, dev)
    h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV) + ((hlm,) if hlm is not None else ()))
    del slots
    torch.cuda.empty_cache()
    return {"value": round(units / tmax, 4), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": int(x["Q"].numel() * x["Q"].element_size()),
            "steps": steps, "ms_per_step": round(tmax * 1e3 / steps, 4),
            "pipeline": "2 buffer slots; host->device, compute and device->host on separate streams"}


def bench_decode(args, name, dev, peaks, rank, dist, parity=False):
    import torch

    import hierarchical_chunk_sparse_landmark_b200 as hsa
    from hierarchical_chunk_sparse_landmark_b200.workloads import WORKLOADS, make_decode_inputs
    wl = WORKLOADS[name].with_(seed=rank)
    x = make_decode_inputs(wl, dev)
    out = torch.empty_like(x["q"])
    ws = hsa.workspace(hsa.decode_workspace_size(wl.B, wl.H, wl.Hkv, wl.L, wl.d, wl.S, wl.topk),
                       dev, ("decode", wl.B * wl.Hkv))
    # The landmark stream alone (B*Hkv*Nc*d bf16 = 256 MiB for both decode
    # workloads) is larger than the 126 MB L2, so calls run back to back without
    # a flush: nothing a call reads can still be in L2 from the previous one in
    # any useful amount.
    steps = max(5, args.steps)
    for _ in range(3):
        hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=wl.topk, out=out, ws=ws)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = make_events(2)
    t0.record()
    for i in range(steps):
        hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=wl.topk, out=out, ws=ws)
    t1.record()
    torch.cuda.synchronize()
    hsa.check(ws)
    secs = t0.elapsed_time(t1) / 1e3
    nbytes = decode_bytes(wl)
    toks, tmax = aggregate(dist, float(wl.B * steps), secs, dev)
    per = secs / steps
    gbs = nbytes / per / 1e9
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    files = [ATTN_SRC + "decode.cu"]
    traffic = measured_traffic("decode", files, workload=wl.name)
    res = {"workload": wl.name, "value": round(toks / tmax, 2), "unit": "tokens/s",
           "ms_per_step": round(per * 1e3, 4), "steps": steps,
           "roofline": {"kernel": "decode_scan_kernel + decode_attend_kernel (whole call)",
                        "bound": "hbm", "achieved": round(gbs, 1),
                        "peak": peak, "unit": "GB/s", "frac": round(gbs / peak, 4),
                        "traffic": traffic, "algorithmic_bytes_per_launch": nbytes,
                        "peak_source": peaks["source"] + " copy bandwidth"},
           "l2": "no flush: inputs (256 MiB of landmarks) larger than L2, calls back to back"}
    if parity:
        O, idx = hsa.decode(x["q"], x["K"], x["V"], x["lm"], topk=wl.topk, idx_out=True, ws=ws)
        hsa.check(ws)
        res["parity"] = decode_parity_sample(wl, x, O, idx)
    del x, out
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample_rows(wl, n_rows, seed=0):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(wl.B * wl.L, size=min(n_rows, wl.B * wl.L), replace=False))


def sample_flops(wl, rows) -> float:
    t = rows % wl.L
    nvis = t // wl.S
    keff = np.minimum(wl.topk, nvis)
    own = (t - wl.S * nvis + 1) if wl.own_chunk else np.zeros_like(t)
    d, H, Hkv, S = wl.d, wl.H, wl.Hkv, wl.S
    return float((Hkv * 2 * d * nvis + H * 2 * d * keff + H * 4 * d * S * keff
                  + H * 4 * d * own).sum())


def _host_f64(t):
    import torch
    return None if t is None else t.detach().to("cpu").to(torch.float64).numpy()


def cpu_baseline(args, wl, budget_s: float = 12.0, x_host=None):
    """Time the fp64 oracle, as it stands, on the host cores over a bounded
    sample of rows of the same workload; throughput in the same unit.
    ``x_host`` may hold the inputs (numpy float64 K, V, lm and a torch Q on any
    device, of which only the sampled rows are copied).  Returns the figure
    and the oracle's results for the first sample (rows, outputs)."""
    import torch

    import oracle
    from hierarchical_chunk_sparse_landmark_b200.workloads import make_prefill_inputs
    orc = oracle.Oracle()
    if x_host is None:
        x = make_prefill_inputs(wl, "cpu")
        x_host = {"K": _host_f64(x["K"]), "V": _host_f64(x["V"]), "lm": _host_f64(x["lm"]),
                  "Q": x["Q"]}
    K, V, lm = x_host["K"], x_host["V"], x_host["lm"]
    Qall = x_host["Q"].reshape(wl.B * wl.L, wl.H, wl.d)
    n = 256
    total_f, total_s, total_rows, it = 0.0, 0.0, 0, 0
    first = None
    while total_s < budget_s:
        rows = oracle_sample_rows(wl, n, seed=it)
        it += 1
        Qr = _host_f64(Qall[torch.as_tensor(rows, device=Qall.device)])
        t0 = time.perf_counter()
        r = orc.prefill(None, K, V, lm, wl.S, wl.topk, wl.own_chunk, rows=rows, Q_rows=Qr)
        dt = time.perf_counter() - t0
        if first is None:
            first = (rows, Qr, r)
        total_f += sample_flops(wl, rows)
        total_s += dt
        total_rows += len(rows)
        n = min(4 * n, 8192)
    info = {"value": round(total_f / total_s / 1e12, 6), "unit": "TFLOP/s",
            "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{total_rows} random rows (all heads) of {wl.name}, fp64 C/OpenMP oracle",
            "seconds": round(total_s, 2)}
    return info, first


def cpu_baseline_and_parity(args, keep):
    """The oracle timed on the host cores (cpu_baseline) on the very inputs the
    GPU read, copied back; the rows of its first sample then double as a
    parity sample of the GPU call made outside the timed region: selection
    compared set by set (near-ties counted, their outputs recomputed on the
    GPU's selection), O within the workload dtype's tolerance."""
    import torch

    import oracle
    from oracle.parity import ATOL, ParityReport, compare_outputs, compare_selection
    wl, x = keep["wl"], keep["x"]
    xh = {"K": _host_f64(x["K"]), "V": _host_f64(x["V"]), "lm": _host_f64(x["lm"]), "Q": x["Q"]}
    info, (rows, Qr, ref) = cpu_baseline(args, wl, x_host=xh)
    rt = torch.as_tensor(rows, device=keep["O"].device)
    got_idx = keep["idx"].reshape(wl.B * wl.L, wl.Hkv, wl.topk)[rt].cpu().numpy()
    got_O = _host_f64(keep["O"].reshape(wl.B * wl.L, wl.H, wl.d)[rt])
    rep = ParityReport(rows=len(rows))
    differs = compare_selection(ref["idx"], ref["sbar"], ref["gap"], ref["smag"], got_idx, rep)
    ref_O = ref["O"]
    if differs.any():
        sel = np.where(differs.any(axis=1))[0]
        forced = oracle.Oracle().prefill(None, xh["K"], xh["V"], xh["lm"], wl.S, wl.topk,
                                         wl.own_chunk, rows=rows[sel], Q_rows=Qr[sel],
                                         forced_idx=got_idx[sel])
        ref_O = ref_O.copy()
        ref_O[sel] = forced["O"]
    compare_outputs(ref_O, got_O, ATOL[wl.dtype], rep)
    par = {"workload": wl.name, "rows": int(len(rows)), "groups": int(len(rows) * wl.Hkv),
           "near_ties": rep.near_ties, "set_mismatch": rep.set_mismatch,
           "order_mismatch": rep.order_mismatch, "max_abs_err": float(f"{rep.max_abs_err:.4g}"),
           "atol": ATOL[wl.dtype], "ok": rep.ok,
           "how": "first sample of the cpu_baseline rows, GPU call outside the timed region"}
    return info, par


def decode_parity_sample(wl, x, O, idx):
    """Every sequence of a decode workload against the oracle (the oracle
    scans all landmarks and attends over the chunks it selects)."""
    import oracle
    from oracle import gather_chunks
    from oracle.parity import ATOL, ParityReport, compare_outputs, compare_selection
    orc = oracle.Oracle()
    q, lm = _host_f64(x["q"]), _host_f64(x["lm"])
    sel = orc.decode_select(q, lm, wl.topk)
    got = idx.cpu().numpy()
    rep = ParityReport(rows=wl.B)
    differs = compare_selection(sel["idx"], sel["sbar"], sel["gap"], sel["smag"], got, rep)
    use = np.where(differs[:, :, None], got, sel["idx"])
    ref = orc.decode_attend(q, lm, gather_chunks(x["K"], use, wl.S), gather_chunks(x["V"], use, wl.S),
                            use, wl.S)
    compare_outputs(ref["O"], _host_f64(O), ATOL[wl.dtype], rep)
    return {"sequences": wl.B, "groups": wl.B * wl.Hkv, "near_ties": rep.near_ties,
            "set_mismatch": rep.set_mismatch, "order_mismatch": rep.order_mismatch,
            "max_abs_err": float(f"{rep.max_abs_err:.4g}"), "atol": ATOL[wl.dtype], "ok": rep.ok}


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on host cores (rank 0 only)."""
    from hierarchical_chunk_sparse_landmark_b200.workloads import WORKLOADS, make_prefill_inputs
    if rank != 0:
        return None
    wl = WORKLOADS[args.workload]
    x = make_prefill_inputs(wl, "cpu")
    xh = {"K": _host_f64(x["K"]), "V": _host_f64(x["V"]), "lm": _host_f64(x["lm"]), "Q": x["Q"]}
    per_step_budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(args, wl, budget_s=per_step_budget / 4, x_host=xh)
    vals, secs = [], 0.0
    info = None
    for _ in range(args.steps):
        info, _ = cpu_baseline(args, wl, budget_s=per_step_budget, x_host=xh)
        vals.append(info["value"])
        secs += info["seconds"]
    value = statistics.mean(vals)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs * 1e3 / max(1, args.steps), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "L": wl.L, "H": wl.H, "Hkv": wl.Hkv,
                       "d": wl.d, "S": wl.S, "topk": wl.topk, "own_chunk": wl.own_chunk,
                       "landmarks": wl.landmarks, "dtype": wl.dtype,
                       "parallelism": f"independent batches x{world}",
                       "l2": "not applicable (host)"},
            "cpu_baseline": {"kind": "oracle", "cores": info["cores"], "sample": info["sample"],
                             "value": value, "unit": "TFLOP/s"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- launch
def free_port() -> int:
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def launch_ranks(n: int, cmd: list, env: dict | None = None, timeout_s: float = 3600.0) -> int:
    """Start `cmd` as n ranks of one job on this node (RANK, LOCAL_RANK,
    WORLD_SIZE, MASTER_ADDR=127.0.0.1 and a free MASTER_PORT in each rank's
    environment), the way torchrun does; rank 0's output is passed through,
    the others' stdout is dropped.  Returns the worst exit code."""
    base = dict(os.environ if env is None else env)
    base.update(WORLD_SIZE=str(n), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(free_port()))
    procs = []
    for r in range(n):
        e = dict(base, RANK=str(r), LOCAL_RANK=str(r))
        procs.append(subprocess.Popen(cmd, env=e, stdout=None if r == 0 else subprocess.DEVNULL))
    deadline = time.time() + timeout_s
    rcs = []
    for p in procs:
        try:
            rcs.append(p.wait(timeout=max(1.0, deadline - time.time())))
        except subprocess.TimeoutExpired:
            p.kill()
            rcs.append(124)
    return max((abs(rc) for rc in rcs), default=0)


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_prefill_bf16",
                    help="prefill workload of the main line (long_prefill_bf16, the largest "
                         "single-GPU prefill; train_prefill_bf16; tiny_prefill_f32)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", dest="decode", action="store_false")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the prefill backward on --workload and print its line")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-extra", dest="extra", action="store_false",
                    help="leave out the lines of the other workloads (train-shape and fp32 "
                         "prefill, batched decode)")
    ap.add_argument("--traffic-from-ncu", nargs=3, metavar=("CSV", "WORKLOAD", "FAMILIES"),
                    help="write the per-launch DRAM bytes of the kernel FAMILIES (comma-"
                         "separated: attend_tc, attend_simt, decode, landmarks) in an ncu CSV "
                         "of WORKLOAD into profiles/traffic.json and exit")
    ap.add_argument("--decode-workload", default="decode_32m_bf16",
                    help="decode workload of the decode line (decode_32m_bf16, batched_decode_bf16)")
    args = ap.parse_args(argv)
    if args.traffic_from_ncu:
        traffic_from_ncu(*args.traffic_from_ncu)
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU, started here when no launcher did it
        return launch_ranks(args.gpus, [sys.executable, os.path.abspath(__file__), *argv])
    world, rank, local = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    import torch
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as td
        torch.cuda.set_device(local)
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = td
    else:
        torch.cuda.set_device(0)
    if args.backward_only:       # diagnostic: the backward line alone (profiling commands)
        res = bench_backward(args, args.workload, torch.device("cuda", torch.cuda.current_device()),
                             load_peaks(), rank, dist, args.steps, args.warmup)
    else:
        res = run_ours(args, dist, rank, world)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
