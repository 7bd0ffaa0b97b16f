"""fp64 CPU oracle for hierarchical chunk-sparse landmark attention.

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's CPU
baseline leg are the only callers.  The library's product path never imports
this package, and this package imports nothing from the library.

The arithmetic lives in ``hsa_oracle.c`` (plain C, double precision, OpenMP
over rows).  This module only builds it with gcc, converts arrays to float64
and marshals pointers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hsa_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libhsa_oracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-std=c99", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
             "-shared", "-fPIC", "-Wall"]


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the oracle shared library with gcc; returns the .so path."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", *GCC_FLAGS, *extra_flags, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    i64p = ctypes.POINTER(ctypes.c_int64)
    i32p = ctypes.POINTER(ctypes.c_int32)
    i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.hsa_oracle_landmarks.argtypes = [dp, i32, i32, i64, i32, i32, dp]
    lib.hsa_oracle_prefill.argtypes = [dp, i64p, i64, dp, dp, dp, i32, i32, i32, i64, i32, i32,
                                       i32, i32, dbl, i32p, dp, i32p, dp, dp, dp, dp]
    lib.hsa_oracle_decode_select.argtypes = [dp, dp, i32, i32, i32, i64, i32, i32, dbl, i32p,
                                             dp, dp, dp]
    lib.hsa_oracle_decode_attend.argtypes = [dp, dp, dp, dp, i32p, i32, i32, i32, i64, i32,
                                             i32, i32, dbl, dp, dp]
    lib.hsa_oracle_prefill_variant.argtypes = [dp, i64p, i64, dp, dp, dp, i32, i32, i32, i64, i32,
                                               i32, i32, i32, dbl, i32, i32, i32, i64p, i64, dp,
                                               i32p, dp, dp, dp, dp]
    for name in ("hsa_oracle_landmarks", "hsa_oracle_prefill", "hsa_oracle_decode_select",
                 "hsa_oracle_decode_attend", "hsa_oracle_num_threads",
                 "hsa_oracle_prefill_variant"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            stale = (not os.path.exists(_LIB_PATH)
                     or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
            if stale:
                build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):          # torch tensor
        a = a.detach().to("cpu")
        import torch
        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _dp(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed with oracle status {rc}")


class Oracle:
    """Thin marshalling wrapper around one loaded oracle library."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def num_threads(self) -> int:
        return int(self.lib.hsa_oracle_num_threads())

    def landmarks(self, K, S: int) -> np.ndarray:
        """K [B,Hkv,L,d] -> landmarks [B,Hkv,L//S,d] (sqrt(S) * chunk mean)."""
        k = _f64(K)
        B, Hkv, L, d = k.shape
        out = np.zeros((B, Hkv, L // S, d), dtype=np.float64)
        _check(self.lib.hsa_oracle_landmarks(_dp(k), B, Hkv, L, d, S, _dp(out)), "landmarks")
        return out

    def prefill(self, Q, K, V, lm, S: int, topk: int, own_chunk: int = 1, scale: float = 0.0,
                rows=None, forced_idx=None, Q_rows=None):
        """Prefill forward.

        Q [B,L,H,d] (or pass ``Q_rows`` [n,H,d] with ``rows``), K/V [B,Hkv,L,d],
        lm [B,Hkv,L//S,d] or None (DHSA landmarks from K).  ``rows`` are
        flattened positions b*L+t (default: every position).
        Returns dict O [n,H,d], idx [n,Hkv,K], w [n,H,K], sbar [n,Hkv,K], gap [n,Hkv],
        smag [n,Hkv,K+1] (magnitudes of the selected scores' terms, then of the
        (K+1)-th candidate's).
        """
        k, v = _f64(K), _f64(V)
        B, Hkv, L, d = k.shape
        if Q_rows is not None:
            q = _f64(Q_rows)
            H = q.shape[1]
            assert rows is not None
        else:
            qf = _f64(Q)
            H = qf.shape[2]
            if rows is None:
                rows = np.arange(B * L, dtype=np.int64)
            rows = np.ascontiguousarray(rows, dtype=np.int64)
            q = np.ascontiguousarray(qf.reshape(B * L, H, d)[rows])
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.shape[0]
        lmf = None if lm is None else _f64(lm)
        O = np.zeros((n, H, d), dtype=np.float64)
        idx = np.zeros((n, Hkv, topk), dtype=np.int32)
        w = np.zeros((n, H, topk), dtype=np.float64)
        sbar = np.zeros((n, Hkv, topk), dtype=np.float64)
        gap = np.zeros((n, Hkv), dtype=np.float64)
        smag = np.zeros((n, Hkv, topk + 1), dtype=np.float64)
        fi = None
        if forced_idx is not None:
            fi = np.ascontiguousarray(forced_idx, dtype=np.int32)
            assert fi.shape == (n, Hkv, topk)
        rc = self.lib.hsa_oracle_prefill(
            _dp(q), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n, _dp(k), _dp(v),
            _dp(lmf), B, H, Hkv, L, d, S, topk, int(own_chunk), float(scale),
            None if fi is None else fi.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
            _dp(O), idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), _dp(w), _dp(sbar),
            _dp(gap), _dp(smag))
        _check(rc, "prefill")
        return {"O": O, "idx": idx, "w": w, "sbar": sbar, "gap": gap, "smag": smag, "rows": rows}

    def prefill_variant(self, Q, K, V, lm, S: int, topk: int, own_chunk: int = 1,
                        scale: float = 0.0, interval: int = 1, pool_mean: int = 0,
                        union_softmax: int = 0, rows=None, bounds=None):
        """Retrieval variants (see hsa_oracle_prefill_variant): one selection
        per `interval` tokens (first token's or mean group query), HiLS fusion
        or one softmax over the union of the selected keys.  Q [B,L,H,d] (all
        tokens), K/V [B,Hkv,L,d], lm [B,Hkv,L//S,d] or None (DHSA).  ``bounds``
        (n+1 increasing token offsets from 0 to L): variable-length chunks, lm
        then [B,Hkv,n,d] or None (sqrt(|C|) * mean of each chunk's keys).
        Returns dict O [n,H,d], idx [n,Hkv,K], w [n,H,K], sbar [n,Hkv,K],
        gap [n,Hkv], smag [n,Hkv,K+1] (of the block's selection, as for prefill)."""
        qf, k, v = _f64(Q), _f64(K), _f64(V)
        B, L, H, d = qf.shape
        Hkv = k.shape[1]
        if rows is None:
            rows = np.arange(B * L, dtype=np.int64)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.shape[0]
        lmf = None if lm is None else _f64(lm)
        O = np.zeros((n, H, d), dtype=np.float64)
        idx = np.zeros((n, Hkv, topk), dtype=np.int32)
        w = np.zeros((n, H, topk), dtype=np.float64)
        sbar = np.zeros((n, Hkv, topk), dtype=np.float64)
        gap = np.zeros((n, Hkv), dtype=np.float64)
        smag = np.zeros((n, Hkv, topk + 1), dtype=np.float64)
        bnd = None if bounds is None else np.ascontiguousarray(bounds, dtype=np.int64)
        rc = self.lib.hsa_oracle_prefill_variant(
            _dp(qf), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n, _dp(k), _dp(v),
            _dp(lmf), B, H, Hkv, L, d, S, topk, int(own_chunk), float(scale), int(interval),
            int(pool_mean), int(union_softmax),
            None if bnd is None else bnd.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
            0 if bnd is None else len(bnd) - 1, _dp(O),
            idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), _dp(w), _dp(sbar), _dp(gap),
            _dp(smag))
        _check(rc, "prefill_variant")
        return {"O": O, "idx": idx, "w": w, "sbar": sbar, "gap": gap, "smag": smag, "rows": rows}

    def decode_select(self, q, lm, topk: int, scale: float = 0.0):
        """q [B,H,d], lm [B,Hkv,Nc,d] -> dict idx [B,Hkv,K], sbar, gap, smag."""
        qf, lmf = _f64(q), _f64(lm)
        B, H, d = qf.shape
        _, Hkv, Nc, _ = lmf.shape
        idx = np.zeros((B, Hkv, topk), dtype=np.int32)
        sbar = np.zeros((B, Hkv, topk), dtype=np.float64)
        gap = np.zeros((B, Hkv), dtype=np.float64)
        smag = np.zeros((B, Hkv, topk + 1), dtype=np.float64)
        rc = self.lib.hsa_oracle_decode_select(
            _dp(qf), _dp(lmf), B, H, Hkv, Nc, d, topk, float(scale),
            idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), _dp(sbar), _dp(gap), _dp(smag))
        _check(rc, "decode_select")
        return {"idx": idx, "sbar": sbar, "gap": gap, "smag": smag}

    def decode_attend(self, q, lm, Kg, Vg, idx, S: int, scale: float = 0.0):
        """Attention + fusion over gathered chunks Kg/Vg [B,Hkv,K,S,d] named by idx."""
        qf, lmf, kg, vg = _f64(q), _f64(lm), _f64(Kg), _f64(Vg)
        B, H, d = qf.shape
        _, Hkv, Nc, _ = lmf.shape
        topk = kg.shape[2]
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        O = np.zeros((B, H, d), dtype=np.float64)
        w = np.zeros((B, H, topk), dtype=np.float64)
        rc = self.lib.hsa_oracle_decode_attend(
            _dp(qf), _dp(lmf), _dp(kg), _dp(vg),
            idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), B, H, Hkv, Nc, d, S, topk,
            float(scale), _dp(O), _dp(w))
        _check(rc, "decode_attend")
        return {"O": O, "w": w}

    def decode(self, q, K, V, lm, S: int, topk: int, scale: float = 0.0):
        """Full decode for caches small enough to hold on the host."""
        sel = self.decode_select(q, lm, topk, scale)
        Kg, Vg = gather_chunks(K, sel["idx"], S), gather_chunks(V, sel["idx"], S)
        att = self.decode_attend(q, lm, Kg, Vg, sel["idx"], S, scale)
        return {**sel, **att}


def gather_chunks(KV, idx, S: int) -> np.ndarray:
    """Copy the S rows of chunk idx[b,g,k] out of KV [B,Hkv,L,d] -> [B,Hkv,K,S,d].

    Pure data movement (no arithmetic); padded slots (-1) are left zero.  Works
    on numpy arrays and on torch tensors (any device: only the selected slices
    are copied to the host).
    """
    idx = np.asarray(idx)
    B, Hkv, topk = idx.shape
    d = KV.shape[-1]
    out = np.zeros((B, Hkv, topk, S, d), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            for kk in range(topk):
                i = int(idx[b, g, kk])
                if i >= 0:
                    out[b, g, kk] = _f64(KV[b, g, i * S:(i + 1) * S])
    return out
