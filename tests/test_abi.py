"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/hsa.h declares, and rejects bad arguments before launching."""
import ctypes
import os
import re

import pytest

import hierarchical_chunk_sparse_landmark_b200 as hsa
from hierarchical_chunk_sparse_landmark_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hsa.h")
A = 0x10000          # a fake, 16-byte aligned device address (never dereferenced)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hsa_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("hsa_landmarks", "hsa_prefill", "hsa_prefill_workspace_size", "hsa_decode",
              "hsa_decode_workspace_size", "hsa_check", "hsa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(B.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    assert hsa.status_string(0) == "ok"
    for s in range(1, 6):
        assert hsa.status_string(s) and hsa.status_string(s) != "unknown status"
    assert hsa.status_string(99) == "unknown status"
    assert hsa.lib().hsa_version() >= 100


def test_workspace_sizes():
    assert hsa.prefill_workspace_size(4, 16, 2, 4096, 128, 64, 8) > 0
    assert hsa.prefill_workspace_size(4, 16, 2, 4096, 128, 64, 8) >= \
        hsa.prefill_workspace_size(4, 16, 2, 1024, 128, 64, 8)
    assert hsa.decode_workspace_size(1, 16, 2, 1 << 25, 128, 64, 8) > 256
    # invalid requests report 0
    assert hsa.prefill_workspace_size(4, 15, 2, 4096, 128, 64, 8) == 0      # H % Hkv
    assert hsa.prefill_workspace_size(4, 16, 2, 4096, 96, 64, 8) == 0       # d
    assert hsa.prefill_workspace_size(4, 16, 2, 4096, 128, 32, 8) == 0      # S
    assert hsa.decode_workspace_size(1, 16, 2, 1000, 128, 64, 8) == 0       # Lc % S


def _prefill(**kw):
    a = dict(Q=A, K=A, V=A, dt=1, lm=A, lm_dt=1, B=1, H=16, Hkv=2, L=256, d=128, S=64, topk=8,
             own=1, scale=0.0, O=A, idx=None, w=None, ws=A, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return hsa.lib().hsa_prefill(a["Q"], a["K"], a["V"], a["dt"], a["lm"], a["lm_dt"], a["B"],
                                 a["H"], a["Hkv"], a["L"], a["d"], a["S"], a["topk"], a["own"],
                                 a["scale"], a["O"], a["idx"], a["w"], a["ws"], a["ws_bytes"],
                                 a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(Q=None), B.HSA_ERR_INVALID_ARG),
    (dict(K=A + 8), B.HSA_ERR_INVALID_ARG),                 # misaligned
    (dict(O=None), B.HSA_ERR_INVALID_ARG),
    (dict(ws=None), B.HSA_ERR_INVALID_ARG),
    (dict(H=15), B.HSA_ERR_INVALID_ARG),
    (dict(H=6, Hkv=2), B.HSA_ERR_UNSUPPORTED),               # G = 3
    (dict(d=96), B.HSA_ERR_UNSUPPORTED),
    (dict(S=32), B.HSA_ERR_UNSUPPORTED),
    (dict(topk=0), B.HSA_ERR_INVALID_ARG),
    (dict(topk=33), B.HSA_ERR_UNSUPPORTED),
    (dict(dt=7), B.HSA_ERR_UNSUPPORTED),
    (dict(own=2), B.HSA_ERR_INVALID_ARG),
    (dict(scale=-1.0), B.HSA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.HSA_ERR_INVALID_ARG),
    (dict(ws_bytes=16), B.HSA_ERR_WORKSPACE),
    (dict(B=0), B.HSA_ERR_INVALID_ARG),
    (dict(L=-1), B.HSA_ERR_INVALID_ARG),
])
def test_prefill_rejects_before_launch(kw, status):
    assert _prefill(**kw) == status


def test_prefill_empty_sequence_is_a_no_op():
    assert _prefill(L=0, Q=None, K=None, V=None, O=None, ws=None) == B.HSA_OK


def _decode(**kw):
    a = dict(q=A, K=A, V=A, dt=1, lm=A, lm_dt=1, B=2, H=16, Hkv=2, Lc=4096, d=128, S=64, topk=8,
             scale=0.0, O=A, idx=None, ws=A, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return hsa.lib().hsa_decode(a["q"], a["K"], a["V"], a["dt"], a["lm"], a["lm_dt"], a["B"],
                                a["H"], a["Hkv"], a["Lc"], a["d"], a["S"], a["topk"], a["scale"],
                                a["O"], a["idx"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), B.HSA_ERR_INVALID_ARG),
    (dict(lm=None), B.HSA_ERR_INVALID_ARG),
    (dict(V=A + 4), B.HSA_ERR_INVALID_ARG),
    (dict(Lc=4000), B.HSA_ERR_INVALID_ARG),                  # not a whole number of chunks
    (dict(d=32), B.HSA_ERR_UNSUPPORTED),
    (dict(topk=40), B.HSA_ERR_UNSUPPORTED),
    (dict(ws_bytes=100), B.HSA_ERR_WORKSPACE),
    (dict(idx=A + 2), B.HSA_ERR_INVALID_ARG),
])
def test_decode_rejects_before_launch(kw, status):
    assert _decode(**kw) == status


def test_landmarks_rejects_before_launch():
    lib = hsa.lib()
    assert lib.hsa_landmarks(None, 1, A, 1, 2, 4096, 128, 64, None) == B.HSA_ERR_INVALID_ARG
    assert lib.hsa_landmarks(A, 1, A, 1, 2, 4096, 100, 64, None) == B.HSA_ERR_UNSUPPORTED
    assert lib.hsa_landmarks(A, 1, A, 1, 2, 4096, 128, 16, None) == B.HSA_ERR_UNSUPPORTED
    assert lib.hsa_landmarks(A, 1, A, 1, 2, 63, 128, 64, None) == B.HSA_OK   # no complete chunk


def test_python_binding_raises_on_error_status():
    with pytest.raises(B.HSAError) as e:
        B._check(B.HSA_ERR_TIMEOUT, "x")
    assert e.value.status == B.HSA_ERR_TIMEOUT and "timed out" in str(e.value)


def test_product_path_has_no_cpu_tensors_path():
    import torch
    with pytest.raises(ValueError):
        hsa.prefill(torch.zeros(1, 64, 2, 64), torch.zeros(1, 1, 64, 64), torch.zeros(1, 1, 64, 64))


def test_path_overrides_validate_their_arguments():
    lib = B.lib()
    assert lib.hsa_set_path_overrides(8, 0) == B.HSA_ERR_INVALID_ARG        # unknown flag
    assert lib.hsa_set_path_overrides(0, 100) == B.HSA_ERR_INVALID_ARG      # window < 256
    assert lib.hsa_set_path_overrides(0, -1) == B.HSA_ERR_INVALID_ARG
    assert lib.hsa_set_path_overrides(7, 512) == B.HSA_OK
    assert lib.hsa_set_path_overrides(0, 0) == B.HSA_OK


def test_window_override_changes_the_workspace_layout():
    # the work lists of 512-token windows need more tile slots than one window
    # per sequence; the override applies to this thread's size queries too
    base = hsa.prefill_workspace_size(2, 16, 2, 64 * 37 + 29, 128, 64, 8)
    with hsa.path_overrides(0, 512):
        small = hsa.prefill_workspace_size(2, 16, 2, 64 * 37 + 29, 128, 64, 8)
    assert small != base and hsa.prefill_workspace_size(2, 16, 2, 64 * 37 + 29, 128, 64, 8) == base


def test_library_reads_no_environment_variables():
    import re
    csrc = os.path.join(ROOT, "hierarchical_chunk_sparse_landmark_b200", "csrc")
    for f in os.listdir(csrc):
        src = open(os.path.join(csrc, f)).read()
        assert not re.search(r"\bgetenv\s*\(", src), f


def test_selftest_rejects_before_launch():
    lib = B.lib()
    # NULL aims at hsa_decode_noalloc's array; a bad budget is still rejected first
    assert lib.hsa_selftest_wait_expiry(None, 0, 0, None) == B.HSA_ERR_INVALID_ARG
    assert lib.hsa_selftest_wait_expiry(ctypes.c_void_p(A), 8, 1000, None) == B.HSA_ERR_INVALID_ARG
    assert lib.hsa_selftest_wait_expiry(ctypes.c_void_p(A + 4), 4096, 1000, None) == B.HSA_ERR_INVALID_ARG
    assert lib.hsa_selftest_wait_expiry(ctypes.c_void_p(A), 4096, 0, None) == B.HSA_ERR_INVALID_ARG
    assert lib.hsa_selftest_wait_expiry(ctypes.c_void_p(A), 4096, 5_000_000_000, None) == B.HSA_ERR_INVALID_ARG


def test_header_is_plain_c_and_the_example_links(tmp_path):
    # include/hsa.h is a C header: a C99 program that drives prefill and decode
    # through it (tests/c_abi_example.c) compiles with warnings as errors and
    # links against libhsa.so and the CUDA runtime.  Running it needs a B200.
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    cuda_inc = "/usr/local/cuda/include"
    if cc is None or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime_api.h")):
        pytest.skip("no C compiler or CUDA headers")
    pkg = os.path.dirname(B.LIB_PATH)
    exe = tmp_path / "c_abi_example"
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", cuda_inc, os.path.join(ROOT, "tests", "c_abi_example.c"), "-L", pkg, "-lhsa",
           "-L", "/usr/local/cuda/lib64", "-lcudart", "-lm", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert exe.exists()
