"""Comparison of a device result with the oracle (test infrastructure only).

Index parity (exact selection, modulo near-ties): for every (row, KV group)
the selected *set* must equal the oracle's.  A difference is accepted only
where the oracle's K-th and (K+1)-th group scores differ by less than
``NEAR_TIE_REL`` relative; such rows are counted and their outputs are
compared with the oracle recomputed on the device's selection instead.  Order
inside the set must match as well, except between neighbours whose oracle
scores are near-tied in the same sense.

"Relative" is taken relative to the magnitude of the terms of the two scores,
scale * sum_j |qbar_j l_ij| (the oracle's ``smag``), the larger of the two:
a score is a dot product, and any finite-precision evaluation of it errs in
proportion to that magnitude, not to its value, which can cancel to nearly
zero (with about 2K visible chunks the K-th and (K+1)-th scores sit near the
median, close to 0).  Where the score does not cancel (qbar parallel to l) the
magnitude equals |score|.

Output parity: max-abs error against the fp64 oracle, 2e-2 for bf16 inputs
and 1e-4 for fp32 inputs.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

NEAR_TIE_REL = 1e-5
ATOL = {"bf16": 2e-2, "f32": 1e-4}
W_ATOL = 1e-5


@dataclass
class ParityReport:
    rows: int = 0
    set_mismatch: int = 0          # rows*groups whose set differs (all near-ties if ok)
    near_ties: int = 0             # rows*groups with an oracle near-tie at the K boundary
    order_mismatch: int = 0        # order differences between near-tied neighbours
    max_abs_err: float = 0.0
    max_w_err: float = 0.0
    failures: list = field(default_factory=list)

    @property
    def ok(self) -> bool:
        return not self.failures

    def summary(self) -> str:
        return (f"rows={self.rows} near_ties={self.near_ties} set_mismatch={self.set_mismatch} "
                f"order_mismatch={self.order_mismatch} max_abs_err={self.max_abs_err:.3e} "
                f"max_w_err={self.max_w_err:.3e} failures={len(self.failures)}")


def _near(a: float, b: float, ma: float, mb: float) -> bool:
    """Scores a, b (term magnitudes ma, mb) are near-tied."""
    return abs(a - b) < NEAR_TIE_REL * max(ma, mb)


def compare_selection(ref_idx, ref_sbar, ref_gap, ref_smag, got_idx, report: ParityReport):
    """Rows x groups selection check against the oracle's idx, sbar, gap and
    smag (term magnitudes of the selected scores, then of the (K+1)-th).
    Returns a bool mask [n, Hkv] of rows whose device set differs from the
    oracle's (accepted near-ties)."""
    n, Hkv, K = ref_idx.shape
    differs = np.zeros((n, Hkv), dtype=bool)
    for r in range(n):
        for g in range(Hkv):
            ri, gi = ref_idx[r, g], got_idx[r, g]
            mag = ref_smag[r, g]
            nsel = int((ri >= 0).sum())
            gap = ref_gap[r, g]
            near = bool(np.isfinite(gap) and nsel == K
                        and gap < NEAR_TIE_REL * max(mag[K - 1], mag[K]))
            report.near_ties += int(near)
            if set(ri.tolist()) != set(gi.tolist()):
                report.set_mismatch += 1
                differs[r, g] = True
                if not near:
                    report.failures.append(f"row {r} group {g}: selection {gi.tolist()} != "
                                           f"oracle {ri.tolist()} (gap {gap:.3e})")
                continue
            for k in range(nsel):
                if ri[k] != gi[k]:
                    # allowed only between oracle-near-tied neighbours
                    j = int(np.where(ri == gi[k])[0][0])
                    lo, hi = min(j, k), max(j, k)
                    if all(_near(ref_sbar[r, g, m], ref_sbar[r, g, m + 1], mag[m], mag[m + 1])
                           for m in range(lo, hi)):
                        report.order_mismatch += 1
                    else:
                        report.failures.append(f"row {r} group {g}: order {gi.tolist()} != "
                                               f"oracle {ri.tolist()}")
                    break
    return differs


def compare_outputs(ref_O, got_O, atol: float, report: ParityReport, what: str = "O"):
    err = np.abs(np.asarray(got_O, dtype=np.float64) - ref_O)
    m = float(err.max()) if err.size else 0.0
    report.max_abs_err = max(report.max_abs_err, m)
    if not np.isfinite(got_O).all():
        report.failures.append(f"{what}: non-finite values")
    if m > atol:
        where = np.unravel_index(int(err.argmax()), err.shape)
        report.failures.append(f"{what}: max abs err {m:.3e} > {atol:.1e} at {where}")
    return m
