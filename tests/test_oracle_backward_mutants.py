"""Plant plausible mistakes in copies of oracle/backward.py and check that the
autograd pin catches each: a mutant's gradients must differ from reverse-mode
differentiation of the separately written PyTorch forward on at least one of
the pin cases (retrieved chunks with and without the own term, input and DHSA
landmarks)."""
import importlib.util
import os

import numpy as np
import pytest
import torch

from test_oracle_backward import case, torch_forward

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "backward.py")

MUTANTS = {
    "no_fusion_logit_gradient": ("dq += scale * dz[k] * lmv[b, g, i]", "dq += 0.0 * dz[k] * lmv[b, g, i]"),
    "softmax_backward_sign": ("da = p * (dp - p @ dp)", "da = p * (dp + p @ dp)"),
    "fusion_softmax_not_centred": ("dz = w * (dw - w @ dw)", "dz = w * dw"),
    "dv_unweighted": ("attend_back(b, g, i * S, (i + 1) * S, q, po[k][0], w[k] * dO[b, t, h], dq)",
                      "attend_back(b, g, i * S, (i + 1) * S, q, po[k][0], dO[b, t, h], dq)"),
    "dk_missing_scale": ("dK[b, g, lo:hi] += scale * np.outer(da, q)", "dK[b, g, lo:hi] += np.outer(da, q)"),
    "dhsa_factor_sqrtS": ("np.repeat(dlm * (np.sqrt(S) / S), S, axis=2)", "np.repeat(dlm * np.sqrt(S), S, axis=2)"),
    "own_chunk_excludes_self": ("p, o = attend(b, g, c * S, t + 1, q)\n                    O[b, t, h] += o\n"
                                "                    attend_back(b, g, c * S, t + 1, q, p, dO[b, t, h], dq)",
                                "p, o = attend(b, g, c * S, t + 1, q)\n                    O[b, t, h] += o\n"
                                "                    attend_back(b, g, c * S, t, q, p[:-1], dO[b, t, h], dq)"),
}


def load(src_text, name, tmp_path):
    path = tmp_path / f"bw_{name}.py"
    path.write_text(src_text)
    spec = importlib.util.spec_from_file_location(f"bw_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def agrees(mod):
    for own, topk, dhsa, seed in [(1, 3, False, 5), (0, 2, False, 6), (1, 2, True, 7)]:
        Q, K, V, lm, dO = case(seed, L=29)
        S, scale = 8, 1.0 / np.sqrt(Q.shape[-1])
        try:
            r = mod.prefill_backward(Q, K, V, None if dhsa else lm, S, topk, own, dO)
        except Exception:
            return False
        tQ, tK, tV = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
        tl = None if dhsa else torch.tensor(lm, requires_grad=True)
        (torch_forward(tQ, tK, tV, tl, S, own, r["idx"], scale) * torch.tensor(dO)).sum().backward()
        pairs = [(r["dQ"], tQ.grad), (r["dK"], tK.grad), (r["dV"], tV.grad)]
        if not dhsa:
            pairs.append((r["dlm"], tl.grad))
        if not all(np.allclose(a, t.numpy(), atol=1e-10) for a, t in pairs):
            return False
    return True


def test_unmutated_copy_agrees(tmp_path):
    assert agrees(load(open(SRC).read(), "copy", tmp_path))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_autograd_pin_catches_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found"
    assert not agrees(load(src.replace(old, new), name, tmp_path)), f"pin missed {name}"
