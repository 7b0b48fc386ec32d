"""Dense causal attention, float64 (the special case RecSA reduces to).

TEST INFRASTRUCTURE (see the package docstring).

RecSA abstract: summaries stand in only for *unselected* candidates, so when k
is at least the candidate count at every level nothing is summarised and the
shared softmax covers every token up to the query; with candidate-local RoPE
the token-level indices are then the true positions.  This module is that
textbook definition, softmax(q K^T / sqrt(d)) V over positions 0..t, used to
check the oracle's k = all case and as the oracle of the dense comparator.
"""

from __future__ import annotations

import math

import numpy as np

from .recsa import rope_rotate


def dense_causal_attention(q: np.ndarray, t: int, K: np.ndarray, V: np.ndarray,
                           rope: bool = False, rope_base: float = 1e6) -> np.ndarray:
    """softmax over keys 0..t of <q, k_j>/sqrt(d), weighted sum of v_j.

    With ``rope`` the query is rotated to position t and key j to position j.
    """
    q = np.asarray(q, dtype=np.float64)
    Kt = np.asarray(K[: t + 1], dtype=np.float64)
    Vt = np.asarray(V[: t + 1], dtype=np.float64)
    if rope:
        q = rope_rotate(q, t, rope_base)
        Kt = rope_rotate(Kt, np.arange(t + 1), rope_base)
    s = Kt @ q / math.sqrt(q.shape[0])
    p = np.exp(s - s.max())
    return (p @ Vt) / p.sum()
