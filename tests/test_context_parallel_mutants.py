"""Plant plausible mistakes in copies of oracle/context_parallel.py and check
that the pins of test_context_parallel.py's kind catch them: each mutant,
loaded from a temporary copy, must disagree with the single-GPU oracle decode
on at least one of the pin cases (random shard splits, a selection held by one
shard, a score tie across shards)."""
import importlib.util
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "context_parallel.py")

MUTANTS = {
    "tie_to_higher_index": ("return np.lexsort((idx, -scores))[:topk]",
                            "return np.lexsort((-idx, -scores))[:topk]"),
    "local_list_too_short": ("sel = _order(s, gi, topk)", "sel = _order(s, gi, max(1, topk - 1))"),
    "local_index_not_offset": ("gi = np.arange(c0, c0 + n, dtype=np.int64)",
                               "gi = np.arange(0, n, dtype=np.int64)"),
    "states_not_rescaled": ("w = np.where(np.isfinite(m), np.exp(m - np.where(np.isfinite(M), M, 0.0)), 0.0)",
                            "w = np.where(np.isfinite(m), 1.0, 0.0)"),
    "chunk_softmax_unnormalised": ("os_.append((p / p.sum()) @ Vc)", "os_.append(p @ Vc)"),
    "fusion_logit_unscaled": ("zs.append(scale * float(q[b, h] @ lm[b, g, li]))",
                              "zs.append(float(q[b, h] @ lm[b, g, li]))"),
    "owned_range_off_by_one": ("if i < c0 or i >= c0 + n:", "if i < c0 or i > c0 + n:"),
}


def load_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found"
    path = tmp_path / f"cp_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"cp_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def pin_cases():
    """(q, K, V, lm, topk, n_shards) cases of the kinds the pins use (S = 16)."""
    out = []
    for seed, Nc, topk, R in [(1, 37, 4, 3), (2, 37, 9, 2), (3, 5, 8, 3), (4, 23, 1, 7)]:
        rng = np.random.default_rng(seed)
        out.append((rng.standard_normal((2, 8, 16)), rng.standard_normal((2, 2, Nc * 16, 16)),
                    rng.standard_normal((2, 2, Nc * 16, 16)), rng.standard_normal((2, 2, Nc, 16)),
                    topk, R))
    # selection held by the last shard
    q, K, V, lm = [a.copy() for a in out[0][:4]]
    for g in range(2):
        qbar = q[:, g * 4:(g + 1) * 4].mean(axis=1)
        lm[:, g, 30:] += 6.0 * qbar[:, None, :] / np.linalg.norm(qbar, axis=1)[:, None, None]
    out.append((q, K, V, lm, 4, 4))
    # an exact tie between chunks 3 and 30, in different shards
    q, K, V, lm = [a.copy() for a in out[1][:4]]
    for g in range(2):
        qbar = q[:, g * 4:(g + 1) * 4].mean(axis=1)
        lm[:, g, 3] += 20.0 * qbar / np.linalg.norm(qbar, axis=1)[:, None]
        lm[:, g, 30] = lm[:, g, 3]
    out.append((q, K, V, lm, 1, 2))
    return out


def agrees(mod, oracle_lib):
    for q, K, V, lm, topk, R in pin_cases():
        ref = oracle_lib.decode(q, K, V, lm, 16, topk)
        try:
            got = mod.decode(q, K, V, lm, 16, topk, R)
        except Exception:
            return False
        if not (np.array_equal(got["idx"], ref["idx"]) and np.allclose(got["O"], ref["O"], atol=1e-12)):
            return False
    return True


def test_unmutated_copy_agrees(oracle_lib, tmp_path):
    spec = importlib.util.spec_from_file_location("cp_copy", SRC)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    assert agrees(mod, oracle_lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(oracle_lib, tmp_path, name):
    assert not agrees(load_mutant(name, tmp_path), oracle_lib), f"no pin case caught {name}"
