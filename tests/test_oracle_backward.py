"""Pins for the fp64 backward restatement (oracle/backward.py): its forward
equals the C oracle's prefill, and its hand-derived gradients equal (1) reverse-
mode automatic differentiation of a separately written PyTorch float64 forward
with the same (fixed) selection and (2) central finite differences."""
import numpy as np
import pytest
import torch

from oracle import backward as bw


def case(seed, B=1, L=45, H=4, Hkv=2, d=8, S=8):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, L, H, d)), rng.standard_normal((B, Hkv, L, d)),
            rng.standard_normal((B, Hkv, L, d)), rng.standard_normal((B, Hkv, L // S, d)),
            rng.standard_normal((B, L, H, d)))


def torch_forward(Q, K, V, lm, S, own, idx, scale):
    """Plain PyTorch forward with the selection held fixed; lm None = DHSA."""
    B, L, H, d = Q.shape
    Hkv = K.shape[1]
    G = H // Hkv
    if lm is None:
        Nc = L // S
        lm = (S ** 0.5) * K[:, :, :Nc * S].reshape(B, Hkv, Nc, S, d).mean(dim=3)
    rows = []
    for b in range(B):
        for t in range(L):
            for h in range(H):
                g, q = h // G, Q[b, t, h]
                o = torch.zeros(d, dtype=torch.float64)
                sel = [int(i) for i in idx[b, t, g] if i >= 0]
                if sel:
                    w = torch.softmax(scale * torch.stack([lm[b, g, i] @ q for i in sel]), dim=0)
                    for k, i in enumerate(sel):
                        p = torch.softmax(scale * (K[b, g, i * S:(i + 1) * S] @ q), dim=0)
                        o = o + w[k] * (p @ V[b, g, i * S:(i + 1) * S])
                if own:
                    c0 = (t // S) * S
                    p = torch.softmax(scale * (K[b, g, c0:t + 1] @ q), dim=0)
                    o = o + p @ V[b, g, c0:t + 1]
                rows.append(o)
    return torch.stack(rows).reshape(B, L, H, d)


@pytest.mark.parametrize("own", [0, 1])
@pytest.mark.parametrize("dhsa", [False, True])
def test_forward_matches_the_c_oracle(oracle_lib, own, dhsa):
    Q, K, V, lm, dO = case(1)
    r = bw.prefill_backward(Q, K, V, None if dhsa else lm, 8, 3, own, dO)
    ref = oracle_lib.prefill(Q, K, V, None if dhsa else lm, 8, 3, own_chunk=own)
    B, L, H, d = Q.shape
    np.testing.assert_array_equal(r["idx"].reshape(B * L, -1, 3), ref["idx"])
    np.testing.assert_allclose(r["O"].reshape(B * L, H, d), ref["O"], atol=1e-12)


@pytest.mark.parametrize("own,topk", [(1, 3), (0, 2), (1, 8)])
@pytest.mark.parametrize("dhsa", [False, True])
def test_gradients_match_autograd(own, topk, dhsa):
    Q, K, V, lm, dO = case(2 + topk + 10 * own)
    S, scale = 8, 1.0 / np.sqrt(Q.shape[-1])
    r = bw.prefill_backward(Q, K, V, None if dhsa else lm, S, topk, own, dO)
    tQ, tK, tV = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
    tl = None if dhsa else torch.tensor(lm, requires_grad=True)
    O = torch_forward(tQ, tK, tV, tl, S, own, r["idx"], scale)
    np.testing.assert_allclose(O.detach().numpy(), r["O"], atol=1e-12)
    (O * torch.tensor(dO)).sum().backward()
    np.testing.assert_allclose(r["dQ"], tQ.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(r["dK"], tK.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(r["dV"], tV.grad.numpy(), atol=1e-10)
    if not dhsa:
        np.testing.assert_allclose(r["dlm"], tl.grad.numpy(), atol=1e-10)


def test_gradients_match_finite_differences():
    Q, K, V, lm, dO = case(3, L=21, H=2, Hkv=1, d=4, S=4)
    S, topk, own = 4, 2, 1
    r = bw.prefill_backward(Q, K, V, lm, S, topk, own, dO)
    idx = r["idx"]

    def loss(Qx, Kx, Vx, lmx):
        return float((bw.prefill_backward(Qx, Kx, Vx, lmx, S, topk, own, dO, idx=idx)["O"] * dO).sum())

    rng = np.random.default_rng(0)
    eps = 1e-6
    base = [Q, K, V, lm]
    for slot, grad in enumerate((r["dQ"], r["dK"], r["dV"], r["dlm"])):
        for _ in range(6):
            arr = base[slot]
            pos = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus, minus = list(base), list(base)
            plus[slot], minus[slot] = arr.copy(), arr.copy()
            plus[slot][pos] += eps
            minus[slot][pos] -= eps
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            assert fd == pytest.approx(grad[pos], rel=1e-5, abs=1e-7), (slot, pos)
