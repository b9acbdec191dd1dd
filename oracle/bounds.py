"""Error-bound constants of FourSight §9.3 (Lemma 2, Lemma 3, Theorem 1; Eq. 6).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Lemma 2: for a normal, non-saturating block scale, each element's NVFP4 error is
at most c * a_b with c = 17/96 (half the largest E2M1 gap, 1, over the scaled
maximum 6, inflated by the UE4M3 unit roundoff 1/16: (1/6)(1 + 1/16) = 17/96).
Lemma 3 lifts it to norms with a factor sqrt(B).  Theorem 1 / Eq. 6 combine them
into E||y_S - y||^2 <= C ||W||_F^2 sum_{j not in S} m_j with
C = (sqrt(B) c_W + sqrt(B) c_A (1 + sqrt(B) c_W))^2, about 3.68 for B = 16.
"""
from __future__ import annotations

import math

C_ELEM = 17.0 / 96.0
U_E4M3 = 1.0 / 16.0
B = 16


def c_elem(max_gap: float = 2.0, max_val: float = 6.0, u: float = U_E4M3) -> float:
    """(max_gap / 2) / max_val * (1 + u): the per-element constant of Lemma 2."""
    return (max_gap / 2.0) / max_val * (1.0 + u)


def theorem1_C(cA: float = C_ELEM, cW: float = C_ELEM, block: int = B) -> float:
    r = math.sqrt(block)
    return (r * cW + r * cA * (1.0 + r * cW)) ** 2
