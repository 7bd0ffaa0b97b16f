"""Seeded synthetic workloads for hierarchical chunk-sparse landmark attention.

This module only *draws* inputs.  It holds none of the method's arithmetic
(no scores, no selection, no softmax): both the CUDA path and the fp64 oracle
read the tensors produced here, so keeping them free of the computation keeps
the two sides independent.

The five named workloads restate the shapes the method is described with:
chunk size 64 and top-8 retrieval (Understanding and Improving Length
Generalization in Hierarchical Sparse Attention Models, "Methodology in Plain
English"), contexts up to 32M tokens (same page, "Main Findings"), and the
DHSA landmark form sqrt(|C|) * mean of a chunk's keys (Dynamic Hierarchical
Sparse Attention review, "What carries the argument").  The pages measure on
RULER / BABILong / LongBench; seeded N(0,1) tensors with planted needle chunks
stand in for those suites here.

Value recipes
-------------
* Q, K, V, landmarks ~ N(0, 1) drawn in fp32 from a seeded generator, then
  rounded to the storage dtype (round-to-nearest-even for bf16).
* ``landmarks="input_x2"``: landmarks ~ 2 * N(0, 1) so top-K scores are well
  separated.
* ``needles="prefill"``: a second generator (seed + 1) draws one unit
  direction u_g per KV head, 8 distinct needle chunks uniform in [0, Nc-1),
  and 1024 distinct probe positions uniform in [S*(min needle + 1), L).  Every
  key of a needle chunk gets +3*u_g; every query head of group g at a probe
  position gets +3*u_g (added in fp32 before rounding).
* ``needles="decode"``: a second generator (seed + 1) draws one depth i* per
  sequence, uniform in [0, Nc).  The landmark row l[b, g, i*] is replaced by
  8*sqrt(d) * qbar / |qbar|^2, qbar being the mean of the group's query heads,
  so that the needle's group score is 8 (before bf16 rounding of the row).
* Variable-length chunks (``make_varlen_bounds``): chunk lengths drawn uniform
  in [lo, hi] from a seeded CPU generator until they cover L tokens, the last
  chunk cut to what is left; landmarks for them (when given) ~ 2 * N(0, 1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "PRIMARY_WORKLOAD",
    "make_prefill_inputs",
    "make_decode_inputs",
    "make_varlen_bounds",
    "storage_dtype",
]


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str              # "prefill" | "decode"
    dtype: str             # "f32" | "bf16"
    B: int
    L: int                 # prefill sequence length, or decode KV-cache length Lc
    H: int
    Hkv: int
    d: int
    S: int = 64
    topk: int = 8
    own_chunk: int = 1     # prefill only: add the causal own-chunk term
    landmarks: str = "input"   # "input" | "input_x2" | "dhsa"
    needles: str = "none"      # "none" | "prefill" | "decode"
    seed: int = 0
    description: str = ""

    @property
    def G(self) -> int:
        return self.H // self.Hkv

    @property
    def n_chunks(self) -> int:
        """Number of complete chunks (the selectable ones)."""
        return self.L // self.S

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_prefill_f32": Workload(
        "tiny_prefill_f32", "prefill", "f32", B=1, L=1024, H=4, Hkv=1, d=64, S=64, topk=4,
        description="B=1 L=1024, 4 query heads sharing 1 KV head, d=64, S=64 (16 chunks), "
                    "top-4, fp32, landmarks an N(0,1) input"),
    "train_prefill_bf16": Workload(
        "train_prefill_bf16", "prefill", "bf16", B=4, L=4096, H=16, Hkv=2, d=128, S=64, topk=8,
        landmarks="input_x2",
        description="B=4 L=4096, 16 query / 2 KV heads (GQA 8), d=128, S=64 (64 chunks), "
                    "top-8, bf16, landmarks an input ~2*N(0,1)"),
    "long_prefill_bf16": Workload(
        "long_prefill_bf16", "prefill", "bf16", B=1, L=131072, H=16, Hkv=2, d=128, S=64, topk=8,
        landmarks="dhsa", needles="prefill",
        description="B=1 L=131072, 16/2 heads, d=128, S=64 (2048 chunks), top-8, bf16, "
                    "DHSA landmarks computed on device, 8 planted needle chunks"),
    "batched_decode_bf16": Workload(
        "batched_decode_bf16", "decode", "bf16", B=32, L=1 << 20, H=16, Hkv=2, d=128, S=64,
        topk=8, own_chunk=0,
        description="B=32 sequences, one query each against a 1,048,576-token cache, "
                    "16/2 heads, d=128, S=64 (16384 chunks/head), top-8, bf16"),
    "decode_32m_bf16": Workload(
        "decode_32m_bf16", "decode", "bf16", B=1, L=1 << 25, H=16, Hkv=2, d=128, S=64,
        topk=8, own_chunk=0, needles="decode",
        description="B=1, one query against a 33,554,432-token cache, 16/2 heads, d=128, "
                    "S=64 (524288 chunks/head), top-8, bf16, one planted needle chunk"),
}

# The workload the prefill throughput figure is quoted on.
PRIMARY_WORKLOAD = "long_prefill_bf16"


def storage_dtype(wl: Workload) -> torch.dtype:
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


# Elements drawn per generator call when filling large device buffers slice by slice.
_SLICE = 1 << 27


def _normal_(out: torch.Tensor, gen: torch.Generator, scale: float = 1.0) -> torch.Tensor:
    """Fill ``out`` (any float dtype, contiguous) with scale*N(0,1) drawn in fp32."""
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, _SLICE):
        e = min(n, s + _SLICE)
        tmp = torch.randn(e - s, generator=gen, device=out.device, dtype=torch.float32)
        if scale != 1.0:
            tmp.mul_(scale)
        flat[s:e].copy_(tmp)
    return out


def _gen(device: torch.device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_prefill_inputs(wl: Workload, device="cpu") -> dict:
    """Draw Q [B,L,H,d], K/V [B,Hkv,L,d] and (unless DHSA) landmarks [B,Hkv,Nc,d].

    Returns a dict with keys Q, K, V, lm (None in DHSA mode) and, for planted
    needles, ``needle_chunks`` (sorted list), ``probe_pos`` (sorted list) and
    ``needle_dirs`` [Hkv, d] fp32 (host).
    """
    assert wl.kind == "prefill"
    device = torch.device(device)
    dt = storage_dtype(wl)
    g = _gen(device, wl.seed)
    B, L, H, Hkv, d, S = wl.B, wl.L, wl.H, wl.Hkv, wl.d, wl.S
    G = H // Hkv
    Nc = L // S
    out = {}
    if wl.needles == "prefill":
        # Draw in fp32 so the planted shifts are added before rounding.
        Q = _normal_(torch.empty(B, L, H, d, device=device, dtype=torch.float32), g)
        K = _normal_(torch.empty(B, Hkv, L, d, device=device, dtype=torch.float32), g)
        V = _normal_(torch.empty(B, Hkv, L, d, device=device, dtype=dt), g)
        g1 = _gen(torch.device("cpu"), wl.seed + 1)
        dirs = torch.randn(Hkv, d, generator=g1, dtype=torch.float64)
        dirs = dirs / dirs.norm(dim=1, keepdim=True)
        n_needles = min(8, max(Nc - 1, 0))
        chunks = torch.randperm(max(Nc - 1, 1), generator=g1)[:n_needles].sort().values
        lo = S * (int(chunks.min()) + 1) if n_needles else L
        n_probe = min(1024, max(L - lo, 0))
        probes = (torch.randperm(max(L - lo, 1), generator=g1)[:n_probe] + lo).sort().values
        u = (3.0 * dirs).to(torch.float32).to(device)
        for c in chunks.tolist():
            K[:, :, c * S:(c + 1) * S, :] += u[None, :, None, :]
        pr = probes.to(device)
        for gi in range(Hkv):
            Q[:, pr, gi * G:(gi + 1) * G, :] += u[gi][None, None, None, :]
        out["Q"], out["K"], out["V"] = Q.to(dt), K.to(dt), V
        del Q, K
        out["needle_chunks"] = chunks.tolist()
        out["probe_pos"] = probes.tolist()
        out["needle_dirs"] = dirs.to(torch.float32)
    else:
        out["Q"] = _normal_(torch.empty(B, L, H, d, device=device, dtype=dt), g)
        out["K"] = _normal_(torch.empty(B, Hkv, L, d, device=device, dtype=dt), g)
        out["V"] = _normal_(torch.empty(B, Hkv, L, d, device=device, dtype=dt), g)
    if wl.landmarks == "dhsa":
        out["lm"] = None
    else:
        scale = 2.0 if wl.landmarks == "input_x2" else 1.0
        out["lm"] = _normal_(torch.empty(B, Hkv, Nc, d, device=device, dtype=dt), g, scale)
    return out


def make_decode_inputs(wl: Workload, device="cpu") -> dict:
    """Draw q [B,H,d], K/V cache [B,Hkv,Lc,d] and landmarks [B,Hkv,Lc/S,d].

    With ``needles="decode"`` the dict also carries ``needle_chunk`` [B] (list).
    """
    assert wl.kind == "decode"
    device = torch.device(device)
    dt = storage_dtype(wl)
    g = _gen(device, wl.seed)
    B, Lc, H, Hkv, d, S = wl.B, wl.L, wl.H, wl.Hkv, wl.d, wl.S
    G = H // Hkv
    Nc = Lc // S
    out = {
        "q": _normal_(torch.empty(B, H, d, device=device, dtype=dt), g),
        "K": _normal_(torch.empty(B, Hkv, Lc, d, device=device, dtype=dt), g),
        "V": _normal_(torch.empty(B, Hkv, Lc, d, device=device, dtype=dt), g),
        "lm": _normal_(torch.empty(B, Hkv, Nc, d, device=device, dtype=dt), g),
    }
    if wl.needles == "decode":
        g1 = _gen(torch.device("cpu"), wl.seed + 1)
        depth = torch.randint(0, Nc, (B,), generator=g1)
        qd = out["q"].to(torch.float64).view(B, Hkv, G, d).mean(dim=2)   # [B,Hkv,d]
        row = 8.0 * math.sqrt(d) * qd / (qd * qd).sum(dim=-1, keepdim=True)
        for b in range(B):
            out["lm"][b, :, int(depth[b]), :] = row[b].to(dt)
        out["needle_chunk"] = depth.tolist()
    return out


def make_varlen_bounds(L: int, seed: int, lo: int = 1, hi: int = 64) -> list:
    """Chunk boundaries 0 = b_0 < ... < b_n = L with lengths uniform in [lo, hi]
    (the last one cut to the tokens left)."""
    assert 1 <= lo <= hi
    g = torch.Generator()
    g.manual_seed(seed)
    bounds = [0]
    while bounds[-1] < L:
        n = int(torch.randint(lo, hi + 1, (1,), generator=g))
        bounds.append(min(L, bounds[-1] + n))
    return bounds
