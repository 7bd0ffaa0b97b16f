"""ctypes binding of libhsa.so (the C ABI declared in include/hsa.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory and the current
stream.  If the shared library is missing the import of the ops fails with a
clear error; there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhsa.so")

HSA_OK, HSA_ERR_INVALID_ARG, HSA_ERR_UNSUPPORTED = 0, 1, 2
HSA_ERR_WORKSPACE, HSA_ERR_CUDA, HSA_ERR_TIMEOUT = 3, 4, 5
HSA_F32, HSA_BF16 = 0, 1

# kernel families of a call (hsa_last_call_kernels) and path overrides
K_LANDMARKS, K_SPLIT_LANDMARKS, K_SELECT_TC_ONE_TILE, K_SELECT_TC_MULTI_TILE = 1, 2, 4, 8
K_SELECT_SIMT, K_WORK_LISTS, K_ATTEND_TC, K_FUSE, K_ATTEND_SIMT = 16, 32, 64, 128, 256
K_DECODE_SCAN, K_DECODE_ATTEND, K_DECODE_CP_MERGE, K_DECODE_CP_COMBINE = 512, 1024, 2048, 4096
K_BACKWARD, K_BACKWARD_TC = 8192, 16384
PATH_SIMT_PREFILL, PATH_SIMT_SELECT, PATH_MULTI_TILE_SELECT = 1, 2, 4

EXPORTED = ("hsa_landmarks", "hsa_prefill_workspace_size", "hsa_prefill",
            "hsa_decode_workspace_size", "hsa_decode", "hsa_check", "hsa_status_string",
            "hsa_version", "hsa_set_stage_events", "hsa_last_call_launches",
            "hsa_decode_noalloc", "hsa_decode_noalloc_max_scratch", "hsa_selftest_wait_expiry",
            "hsa_last_call_kernels", "hsa_set_path_overrides", "hsa_decode_cp_candidates",
            "hsa_decode_cp_merge", "hsa_decode_cp_attend", "hsa_decode_cp_combine",
            "hsa_prefill_variant", "hsa_prefill_varlen_workspace_size", "hsa_prefill_varlen",
            "hsa_prefill_backward_workspace_size", "hsa_prefill_backward", "hsa_decode_ragged",
            "hsa_landmarks_append")


class Variant(ctypes.Structure):
    """hsa_variant_t: retrieval interval, pooling of the block's queries, fusion form."""
    _fields_ = [("retrieval_interval", ctypes.c_int), ("pool_mean", ctypes.c_int),
                ("union_softmax", ctypes.c_int)]


class HSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None
_lock = threading.Lock()


def _declare(lib):
    vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                            ctypes.c_size_t)
    lib.hsa_landmarks.argtypes = [vp, i32, vp, i32, i32, i64, i32, i32, vp]
    lib.hsa_prefill_workspace_size.argtypes = [i32, i32, i32, i64, i32, i32, i32]
    lib.hsa_prefill_workspace_size.restype = sz
    lib.hsa_prefill.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32, i64, i32, i32, i32, i32,
                                f32, vp, vp, vp, vp, sz, vp]
    lib.hsa_prefill_variant.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32, i64, i32, i32,
                                        i32, i32, f32, ctypes.POINTER(Variant), vp, vp, vp, vp,
                                        sz, vp]
    lib.hsa_prefill_varlen_workspace_size.argtypes = [i32, i32, i32, i64, i32, i64, i32]
    lib.hsa_prefill_varlen_workspace_size.restype = sz
    lib.hsa_prefill_varlen.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32, i64, i32, vp,
                                       i64, i32, i32, f32, i32, vp, vp, vp, vp, sz, vp]
    lib.hsa_prefill_backward_workspace_size.argtypes = [i32, i32, i32, i64, i32, i32, i32, i32]
    lib.hsa_prefill_backward_workspace_size.restype = sz
    lib.hsa_prefill_backward.argtypes = [vp, vp, vp, i32, vp, i32, vp, vp, i32, i32, i32, i64,
                                         i32, i32, i32, i32, f32, vp, vp, vp, vp, vp, sz, vp]
    lib.hsa_decode_workspace_size.argtypes = [i32, i32, i32, i64, i32, i32, i32]
    lib.hsa_decode_workspace_size.restype = sz
    lib.hsa_decode.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32, i64, i32, i32, i32, f32,
                               vp, vp, vp, sz, vp]
    lib.hsa_decode_ragged.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32, i64, i32, i32,
                                      i32, f32, vp, vp, vp, vp, sz, vp]
    lib.hsa_landmarks_append.argtypes = [vp, i32, vp, i32, i32, i32, i64, i32, i32, vp, vp, i32,
                                         vp]
    lib.hsa_check.argtypes = [vp, vp]
    lib.hsa_selftest_wait_expiry.argtypes = [vp, sz, i64, vp]
    lib.hsa_decode_noalloc.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32, i64, i32, i32,
                                       i32, f32, vp, vp, vp]
    lib.hsa_decode_noalloc_max_scratch.argtypes = []
    lib.hsa_decode_noalloc_max_scratch.restype = sz
    lib.hsa_set_stage_events.argtypes = [ctypes.POINTER(vp), i32]
    lib.hsa_last_call_kernels.argtypes = []
    lib.hsa_last_call_kernels.restype = ctypes.c_uint
    lib.hsa_set_path_overrides.argtypes = [i32, i64]
    lib.hsa_decode_cp_candidates.argtypes = [vp, i32, vp, i32, i32, i32, i32, i64, i32, i32, i32,
                                             f32, i64, vp, vp, vp, sz, vp]
    lib.hsa_decode_cp_merge.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp]
    lib.hsa_decode_cp_attend.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32, i64, i32, i32,
                                         i32, f32, i64, vp, vp, vp, vp, vp]
    lib.hsa_decode_cp_combine.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
    lib.hsa_status_string.argtypes = [i32]
    lib.hsa_status_string.restype = ctypes.c_char_p
    for n in ("hsa_landmarks", "hsa_prefill", "hsa_decode", "hsa_check", "hsa_version",
              "hsa_set_stage_events", "hsa_last_call_launches", "hsa_decode_noalloc",
              "hsa_selftest_wait_expiry", "hsa_set_path_overrides", "hsa_decode_cp_candidates",
              "hsa_decode_cp_merge", "hsa_decode_cp_attend", "hsa_decode_cp_combine",
              "hsa_prefill_variant", "hsa_prefill_varlen", "hsa_prefill_backward",
              "hsa_decode_ragged", "hsa_landmarks_append"):
        getattr(lib, n).restype = i32
    return lib


def lib():
    """The loaded libhsa (raises if the CUDA library was not built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise ImportError(
                        f"libhsa.so not found at {LIB_PATH}; build it with "
                        "`python -m hierarchical_chunk_sparse_landmark_b200.build`")
                _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def status_string(status: int) -> str:
    return lib().hsa_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != HSA_OK:
        raise HSAError(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return HSA_F32
    if t.dtype == torch.bfloat16:
        return HSA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _opt(t):
    """A tensor argument or None (flags such as ``idx_out=False`` mean "not wanted")."""
    return t if isinstance(t, torch.Tensor) else None


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


# Workspaces are cached per (device, stream, kind): calls on one stream are
# ordered, so reusing the buffer there is safe.  A prefill and a decode never
# share one (each relies on its own regions being left as its previous call
# left them), and decode workspaces are also keyed by B*Hkv: their
# per-(sequence, group) counters must start at zero, which a completed call
# guarantees only for the counters it used.
_ws_cache: dict = {}


def workspace(nbytes: int, device, kind: str = "prefill") -> torch.Tensor:
    """A zero-filled (on creation) device workspace of at least `nbytes`,
    cached per (device, current stream, kind); kind is "prefill" or
    ("decode", B*Hkv)."""
    device = torch.device(device)
    key = (device.index, torch.cuda.current_stream(device).cuda_stream, kind)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def landmarks(K: torch.Tensor, S: int = 64, out: torch.Tensor | None = None) -> torch.Tensor:
    """DHSA landmarks sqrt(S) * mean of each complete chunk's keys, fp32 [B,Hkv,L//S,d]."""
    _dev(K, "K")
    B, Hkv, L, d = K.shape
    if out is None:
        out = torch.empty(B, Hkv, L // S, d, dtype=torch.float32, device=K.device)
    _check(lib().hsa_landmarks(_ptr(K), _dtype_code(K), _ptr(out), B, Hkv, L, d, S,
                               _stream(K.device)), "hsa_landmarks")
    return out


def prefill_workspace_size(B, H, Hkv, L, d, S, topk) -> int:
    return int(lib().hsa_prefill_workspace_size(B, H, Hkv, L, d, S, topk))


def prefill(Q, K, V, lm=None, *, S: int = 64, topk: int = 8, own_chunk: int = 1,
            scale: float = 0.0, out=None, idx_out=None, w_out=None, ws=None,
            retrieval_interval: int = 1, pool_mean: bool = False, union_softmax: bool = False):
    """Hierarchical chunk-sparse prefill.  Returns (O, idx, w); idx/w are None
    unless buffers are given or ``idx_out=True`` / ``w_out=True``.  The
    keyword arguments after ``ws`` select a retrieval variant (hsa_variant_t):
    one selection per ``retrieval_interval`` tokens from the block's first
    token (or the mean of its queries with ``pool_mean``), and one softmax
    over the union of the selected keys with ``union_softmax``."""
    for n, t in (("Q", Q), ("K", K), ("V", V)):
        _dev(t, n)
    B, L, H, d = Q.shape
    Hkv = K.shape[1]
    if K.shape != (B, Hkv, L, d) or V.shape != K.shape:
        raise ValueError("K and V must be [B, Hkv, L, d] matching Q [B, L, H, d]")
    if lm is not None:
        _dev(lm, "lm")
        if lm.shape != (B, Hkv, L // S, d):
            raise ValueError(f"lm must be [B, Hkv, L//S, d] = {(B, Hkv, L // S, d)}")
    dev = Q.device
    if out is None:
        out = torch.empty_like(Q)
    if idx_out is True:
        idx_out = torch.empty(B, L, Hkv, topk, dtype=torch.int32, device=dev)
    if w_out is True:
        w_out = torch.empty(B, L, H, topk, dtype=torch.float32, device=dev)
    nbytes = prefill_workspace_size(B, H, Hkv, L, d, S, topk)
    if ws is None:
        ws = workspace(nbytes, dev)
    var = Variant(int(retrieval_interval), int(bool(pool_mean)), int(bool(union_softmax)))
    st = lib().hsa_prefill_variant(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(lm),
                                   _dtype_code(lm) if lm is not None else HSA_F32, B, H, Hkv, L,
                                   d, S, topk, int(own_chunk), float(scale), ctypes.byref(var),
                                   _ptr(out), _ptr(_opt(idx_out)), _ptr(_opt(w_out)), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(dev))
    _check(st, "hsa_prefill")
    return out, _opt(idx_out), _opt(w_out)


def prefill_varlen_workspace_size(B, H, Hkv, L, d, n_chunks, topk) -> int:
    return int(lib().hsa_prefill_varlen_workspace_size(B, H, Hkv, L, d, n_chunks, topk))


def prefill_varlen(Q, K, V, bounds, lm=None, *, topk: int = 8, own_chunk: int = 1,
                   scale: float = 0.0, union_softmax: bool = False, out=None, idx_out=None,
                   w_out=None, ws=None):
    """Prefill over variable-length chunks (hsa_prefill_varlen): ``bounds``
    holds the n+1 chunk boundaries 0 = b_0 < ... < b_n = L (a sequence, or an
    int32 tensor on Q's device), each chunk at most 64 tokens.  ``lm`` is
    [B, Hkv, n, d] or None (sqrt(|C|) * mean of each chunk's keys).  Returns
    (O, idx, w) as prefill does.  Wrong boundaries are found on the device:
    check(ws) then raises HSA_ERR_INVALID_ARG."""
    for n, t in (("Q", Q), ("K", K), ("V", V)):
        _dev(t, n)
    B, L, H, d = Q.shape
    Hkv = K.shape[1]
    if K.shape != (B, Hkv, L, d) or V.shape != K.shape:
        raise ValueError("K and V must be [B, Hkv, L, d] matching Q [B, L, H, d]")
    dev = Q.device
    if not isinstance(bounds, torch.Tensor):
        bounds = torch.tensor(list(bounds), dtype=torch.int32, device=dev)
    _dev(bounds, "bounds")
    if bounds.dtype != torch.int32 or bounds.dim() != 1 or bounds.numel() < 2:
        raise ValueError("bounds must be a 1-D int32 tensor of n_chunks + 1 offsets")
    n_chunks = bounds.numel() - 1
    if lm is not None:
        _dev(lm, "lm")
        if lm.shape != (B, Hkv, n_chunks, d):
            raise ValueError(f"lm must be [B, Hkv, n_chunks, d] = {(B, Hkv, n_chunks, d)}")
    if out is None:
        out = torch.empty_like(Q)
    if idx_out is True:
        idx_out = torch.empty(B, L, Hkv, topk, dtype=torch.int32, device=dev)
    if w_out is True:
        w_out = torch.empty(B, L, H, topk, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(prefill_varlen_workspace_size(B, H, Hkv, L, d, n_chunks, topk), dev)
    st = lib().hsa_prefill_varlen(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(lm),
                                  _dtype_code(lm) if lm is not None else HSA_F32, B, H, Hkv, L,
                                  d, _ptr(bounds), n_chunks, topk, int(own_chunk), float(scale),
                                  int(bool(union_softmax)), _ptr(out), _ptr(_opt(idx_out)),
                                  _ptr(_opt(w_out)), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(dev))
    _check(st, "hsa_prefill_varlen")
    return out, _opt(idx_out), _opt(w_out)


def prefill_backward_workspace_size(B, H, Hkv, L, d, S, topk, dhsa: bool) -> int:
    return int(lib().hsa_prefill_backward_workspace_size(B, H, Hkv, L, d, S, topk, int(dhsa)))


def prefill_backward(Q, K, V, idx, dO, lm=None, *, S: int = 64, own_chunk: int = 1,
                     scale: float = 0.0, dQ=None, dK=None, dV=None, dlm=None, ws=None):
    """Gradients of sum(dO * O) for the prefill with the selection ``idx``
    [B, L, Hkv, topk] (int32, the forward's) held fixed (hsa_prefill_backward).
    Returns fp32 (dQ [B,L,H,d], dK, dV [B,Hkv,L,d], dlm [B,Hkv,L//S,d] or None
    with DHSA landmarks, whose gradient is folded into dK)."""
    for n, t in (("Q", Q), ("K", K), ("V", V), ("idx", idx), ("dO", dO)):
        _dev(t, n)
    B, L, H, d = Q.shape
    Hkv = K.shape[1]
    if K.shape != (B, Hkv, L, d) or V.shape != K.shape or dO.shape != Q.shape:
        raise ValueError("K, V must be [B, Hkv, L, d] and dO like Q [B, L, H, d]")
    if idx.dtype != torch.int32 or idx.dim() != 4 or idx.shape[:3] != (B, L, Hkv):
        raise ValueError("idx must be int32 [B, L, Hkv, topk]")
    topk = idx.shape[3]
    dev = Q.device
    if lm is not None:
        _dev(lm, "lm")
        if lm.shape != (B, Hkv, L // S, d):
            raise ValueError(f"lm must be [B, Hkv, L//S, d] = {(B, Hkv, L // S, d)}")
        if dlm is None:
            dlm = torch.empty(B, Hkv, L // S, d, dtype=torch.float32, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dQ = torch.empty(B, L, H, d, **f32) if dQ is None else dQ
    dK = torch.empty(B, Hkv, L, d, **f32) if dK is None else dK
    dV = torch.empty(B, Hkv, L, d, **f32) if dV is None else dV
    nbytes = prefill_backward_workspace_size(B, H, Hkv, L, d, S, topk, lm is None)
    if ws is None:
        ws = workspace(nbytes, dev, "backward")
    st = lib().hsa_prefill_backward(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(lm),
                                    _dtype_code(lm) if lm is not None else HSA_F32, _ptr(idx),
                                    _ptr(dO), B, H, Hkv, L, d, S, topk, int(own_chunk),
                                    float(scale), _ptr(dQ), _ptr(dK), _ptr(dV),
                                    _ptr(dlm if lm is not None else None), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(dev))
    _check(st, "hsa_prefill_backward")
    return dQ, dK, dV, (dlm if lm is not None else None)


def decode_workspace_size(B, H, Hkv, Lc, d, S, topk) -> int:
    return int(lib().hsa_decode_workspace_size(B, H, Hkv, Lc, d, S, topk))


def decode(q, K, V, lm, *, S: int = 64, topk: int = 8, scale: float = 0.0, out=None,
           idx_out=None, ws=None):
    """One query per sequence at position Lc against a Lc-token cache.  Returns (O, idx)."""
    for n, t in (("q", q), ("K", K), ("V", V), ("lm", lm)):
        _dev(t, n)
    B, H, d = q.shape
    _, Hkv, Lc, _ = K.shape
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if idx_out is True:
        idx_out = torch.empty(B, Hkv, topk, dtype=torch.int32, device=dev)
    nbytes = decode_workspace_size(B, H, Hkv, Lc, d, S, topk)
    if ws is None:
        ws = workspace(nbytes, dev, ("decode", B * Hkv))
    st = lib().hsa_decode(_ptr(q), _ptr(K), _ptr(V), _dtype_code(q), _ptr(lm), _dtype_code(lm),
                          B, H, Hkv, Lc, d, S, topk, float(scale), _ptr(out),
                          _ptr(_opt(idx_out)), _ptr(ws), ws.numel() * ws.element_size(),
                          _stream(dev))
    _check(st, "hsa_decode")
    return out, _opt(idx_out)


def decode_ragged(q, K, V, lm, lens, *, S: int = 64, topk: int = 8, scale: float = 0.0,
                  out=None, idx_out=None, ws=None):
    """hsa_decode over caches of different lengths: sequence b holds lens[b]
    (int32 [B] on the device) of the Lmax = K.shape[2] allocated tokens and
    retrieves among its first lens[b] // S chunks.  Returns (O, idx)."""
    for n, t in (("q", q), ("K", K), ("V", V), ("lm", lm), ("lens", lens)):
        _dev(t, n)
    B, H, d = q.shape
    _, Hkv, Lmax, _ = K.shape
    if lens.dtype != torch.int32 or lens.shape != (B,):
        raise ValueError("lens must be int32 [B]")
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if idx_out is True:
        idx_out = torch.empty(B, Hkv, topk, dtype=torch.int32, device=dev)
    nbytes = decode_workspace_size(B, H, Hkv, Lmax, d, S, topk)
    if ws is None:
        ws = workspace(nbytes, dev, ("decode", B * Hkv))
    st = lib().hsa_decode_ragged(_ptr(q), _ptr(K), _ptr(V), _dtype_code(q), _ptr(lm),
                                 _dtype_code(lm), B, H, Hkv, Lmax, d, S, topk, float(scale),
                                 _ptr(lens), _ptr(out), _ptr(_opt(idx_out)), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(dev))
    _check(st, "hsa_decode_ragged")
    return out, _opt(idx_out)


def landmarks_append(K, lm, len_before, len_after, *, S: int = 64, max_new_chunks: int = 1):
    """Write the DHSA landmarks of the chunks completed while each cache grew
    from len_before[b] to len_after[b] tokens into lm [B, Hkv, Lmax//S, d]
    (fp32 or bf16), leaving every other row as it is."""
    for n, t in (("K", K), ("lm", lm), ("len_before", len_before), ("len_after", len_after)):
        _dev(t, n)
    B, Hkv, Lmax, d = K.shape
    if lm.shape != (B, Hkv, Lmax // S, d):
        raise ValueError(f"lm must be [B, Hkv, Lmax//S, d] = {(B, Hkv, Lmax // S, d)}")
    for t in (len_before, len_after):
        if t.dtype != torch.int32 or t.shape != (B,):
            raise ValueError("lengths must be int32 [B]")
    _check(lib().hsa_landmarks_append(_ptr(K), _dtype_code(K), _ptr(lm), _dtype_code(lm), B, Hkv,
                                      Lmax, d, S, _ptr(len_before), _ptr(len_after),
                                      int(max_new_chunks), _stream(K.device)),
           "hsa_landmarks_append")
    return lm


def decode_noalloc(q, K, V, lm, *, S: int = 64, topk: int = 8, scale: float = 0.0, out=None,
                   idx_out=None):
    """hsa_decode for callers that cannot allocate device memory: the scratch
    is the library's fixed device array (see hsa_decode_noalloc in hsa.h), so
    no workspace is passed.  ``out`` and ``idx_out`` should be preallocated by
    such callers (when omitted they are created here with torch, for tests).
    Calls must be ordered on one stream.  Returns (O, idx)."""
    for n, t in (("q", q), ("K", K), ("V", V), ("lm", lm)):
        _dev(t, n)
    B, H, d = q.shape
    _, Hkv, Lc, _ = K.shape
    if out is None:
        out = torch.empty_like(q)
    if idx_out is True:
        idx_out = torch.empty(B, Hkv, topk, dtype=torch.int32, device=q.device)
    with torch.cuda.device(q.device):      # the array is looked up on the current device
        st = lib().hsa_decode_noalloc(_ptr(q), _ptr(K), _ptr(V), _dtype_code(q), _ptr(lm),
                                      _dtype_code(lm), B, H, Hkv, Lc, d, S, topk, float(scale),
                                      _ptr(out), _ptr(_opt(idx_out)), _stream(q.device))
    _check(st, "hsa_decode_noalloc")
    return out, _opt(idx_out)


# ----------------------------------------------------------------------------- context parallel
def decode_cp_candidates(q, lm, chunk_offset: int, *, S: int = 64, topk: int = 8,
                         scale: float = 0.0, ws=None):
    """Step 1 of a context-parallel decode on one shard: lm [B,Hkv,n,d] holds
    chunks chunk_offset .. chunk_offset+n-1 of the whole cache.  Returns the
    shard's top-K candidates (scores [B,Hkv,topk] fp32, global chunk indices
    [B,Hkv,topk] int32, -1 where the shard has fewer chunks)."""
    _dev(q, "q")
    _dev(lm, "lm")
    B, H, d = q.shape
    _, Hkv, n, _ = lm.shape
    dev = q.device
    score = torch.empty(B, Hkv, topk, dtype=torch.float32, device=dev)
    cidx = torch.empty(B, Hkv, topk, dtype=torch.int32, device=dev)
    Lc = n * S
    if ws is None:
        ws = workspace(max(256, decode_workspace_size(B, H, Hkv, Lc, d, S, topk)), dev,
                       ("decode", B * Hkv))
    _check(lib().hsa_decode_cp_candidates(_ptr(q), _dtype_code(q), _ptr(lm), _dtype_code(lm), B, H,
                                          Hkv, Lc, d, S, topk, float(scale), int(chunk_offset),
                                          _ptr(score), _ptr(cidx), _ptr(ws),
                                          ws.numel() * ws.element_size(), _stream(dev)),
           "hsa_decode_cp_candidates")
    return score, cidx


def decode_cp_merge(scores, cidx):
    """Step 2: the global top-K from the gathered candidates of R shards
    (scores [R,B,Hkv,topk] fp32, cidx [R,B,Hkv,topk] int32) -> idx [B,Hkv,topk]."""
    _dev(scores, "scores")
    _dev(cidx, "cidx")
    R, B, Hkv, topk = scores.shape
    idx = torch.empty(B, Hkv, topk, dtype=torch.int32, device=scores.device)
    _check(lib().hsa_decode_cp_merge(_ptr(scores), _ptr(cidx), R, B, Hkv, topk, _ptr(idx),
                                     _stream(scores.device)), "hsa_decode_cp_merge")
    return idx


def decode_cp_attend(q, K, V, lm, chunk_offset: int, idx, *, S: int = 64, scale: float = 0.0):
    """Step 3: the shard's per-head fusion state over the selected chunks it
    holds (K/V [B,Hkv,n*S,d], lm [B,Hkv,n,d]) -> m, Z [B,H], acc [B,H,d] fp32."""
    for nm, t in (("q", q), ("K", K), ("V", V), ("lm", lm), ("idx", idx)):
        _dev(t, nm)
    B, H, d = q.shape
    _, Hkv, Lc, _ = K.shape
    topk = idx.shape[-1]
    dev = q.device
    m = torch.empty(B, H, dtype=torch.float32, device=dev)
    Z = torch.empty(B, H, dtype=torch.float32, device=dev)
    acc = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    _check(lib().hsa_decode_cp_attend(_ptr(q), _ptr(K), _ptr(V), _dtype_code(q), _ptr(lm),
                                      _dtype_code(lm), B, H, Hkv, Lc, d, S, topk, float(scale),
                                      int(chunk_offset), _ptr(idx), _ptr(m), _ptr(Z), _ptr(acc),
                                      _stream(dev)), "hsa_decode_cp_attend")
    return m, Z, acc


def decode_cp_combine(m, Z, acc, dtype=torch.bfloat16):
    """Step 4: O [B,H,d] from the gathered states of R shards (m, Z [R,B,H],
    acc [R,B,H,d])."""
    for nm, t in (("m", m), ("Z", Z), ("acc", acc)):
        _dev(t, nm)
    R, B, H, d = acc.shape
    O = torch.empty(B, H, d, dtype=dtype, device=acc.device)
    _check(lib().hsa_decode_cp_combine(_ptr(m), _ptr(Z), _ptr(acc), R, B, H, d, _dtype_code(O),
                                       _ptr(O), _stream(acc.device)), "hsa_decode_cp_combine")
    return O


def decode_context_parallel(q, K, V, lm, chunk_offset: int, *, S: int = 64, topk: int = 8,
                            scale: float = 0.0, group=None):
    """One rank's part of a decode whose cache is cut along the sequence into
    contiguous chunk ranges, one per rank of `group` (torch.distributed; NCCL
    on GPUs): this rank holds K/V [B,Hkv,n*S,d] and lm [B,Hkv,n,d], chunks
    chunk_offset .. chunk_offset+n-1; q [B,H,d] is the same on every rank.
    The two exchanges are all-gathers over the group (candidates, then fusion
    states); every rank returns the same (O, idx).  Without a process group
    (or with one rank) the shard is the whole cache."""
    import torch.distributed as dist
    world = dist.get_world_size(group) if (group is not None or dist.is_initialized()) else 1

    def gather(t):
        if world == 1:
            return t.unsqueeze(0)
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
        return out

    score, cidx = decode_cp_candidates(q, lm, chunk_offset, S=S, topk=topk, scale=scale)
    idx = decode_cp_merge(gather(score), gather(cidx))
    m, Z, acc = decode_cp_attend(q, K, V, lm, chunk_offset, idx, S=S, scale=scale)
    O = decode_cp_combine(gather(m), gather(Z), gather(acc), dtype=q.dtype)
    return O, idx


def set_stage_events(events) -> None:
    """Timing hook: record these torch.cuda.Event objects at the stage
    boundaries of this thread's next calls (see hsa_set_stage_events); None
    skips a boundary; pass an empty list to stop."""
    arr = (ctypes.c_void_p * max(1, len(events)))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else None) for e in events])
    _check(lib().hsa_set_stage_events(arr, len(events)), "hsa_set_stage_events")


def last_call_launches() -> int:
    """Kernels launched by this thread's most recent library call."""
    return int(lib().hsa_last_call_launches())


def last_call_kernels() -> int:
    """Kernel families (K_* bits) of this thread's most recent library call."""
    return int(lib().hsa_last_call_kernels())


class path_overrides:
    """Context manager: this thread's prefill calls take the paths named by
    ``flags`` (PATH_* bits) and token windows of ``window_tokens`` (0 = the
    library's choice); see hsa_set_path_overrides.  Restores the defaults."""

    def __init__(self, flags: int = 0, window_tokens: int = 0):
        self.flags, self.window = int(flags), int(window_tokens)

    def __enter__(self):
        _check(lib().hsa_set_path_overrides(self.flags, self.window), "hsa_set_path_overrides")
        return self

    def __exit__(self, *exc):
        lib().hsa_set_path_overrides(0, 0)
        return False


def selftest_wait_expiry(ws, budget_cycles: int = 2_000_000, device=None):
    """Run the library's bounded-wait failure path once: a device wait that
    nothing completes gives up after `budget_cycles` and flags the status word
    of `ws`; the following check(ws) raises HSAError with status HSA_ERR_TIMEOUT.
    ``ws=None`` aims at the status word of decode_noalloc's fixed array on
    ``device`` (reported by check(None, device))."""
    if ws is None:
        dev = torch.device(device if device is not None else "cuda")
        with torch.cuda.device(dev):
            _check(lib().hsa_selftest_wait_expiry(None, 0, int(budget_cycles), _stream(dev)),
                   "hsa_selftest_wait_expiry")
        return
    _dev(ws, "ws")
    _check(lib().hsa_selftest_wait_expiry(_ptr(ws), ws.numel() * ws.element_size(), int(budget_cycles),
                                          _stream(ws.device)), "hsa_selftest_wait_expiry")


def check(ws=None, device=None):
    """Synchronise the current stream and report device-side status flags."""
    device = device if device is not None else (ws.device if ws is not None else "cuda")
    _check(lib().hsa_check(_ptr(ws), _stream(device)), "hsa_check")
