"""Several reference queries per pooler (R > 1), float64.

TEST INFRASTRUCTURE (see the package docstring): imported only by the tests,
the smoke check and the CPU legs of the benchmark.

"Subquadratic Attention with a Hierarchical Tree-Structured Indexer" (ZHA),
Figure 3 caption: several reference queries are used, and the key nodes of
each are stored in parallel; a parent key is the attention-weighted sum of its
children's keys against a reference query, recursively up the levels.  So the
tree holds R key trees side by side -- reference j's keys at level l pool
reference j's keys at level l - 1 -- and one value tree (the mean-pooled
values do not depend on the reference).  Figure 4 names the reference count
as a geometry parameter; its Table II trains 16 reference queries per layer.

Reading (the pages do not say how a node's R keys give one routing score): a
node's score is the largest of q . key_j / sqrt(d) over its R keys -- the node
is as relevant as its best-matching reference summary, and each selection is
attributed to one reference query (Figure 9 counts selections per reference
query).  R > 1 is defined for the ZHA routing variant, whose attention uses no
summary key.

Pins (tests/test_oracle_pins.py): R copies of one reference give the R = 1
tree and routing; reference j's keys equal the single-reference tree built
with reference j; a hand-built two-reference level fixes max (a sum or mean of
the R scores would expand another node); p = 1 is dense attention for any R.
"""

from __future__ import annotations

from typing import List, Tuple

import numpy as np

from .recsa import LazyTree, build_tree


def build_tree_multi(K: np.ndarray, V: np.ndarray, Rq: np.ndarray, B: int, b: int
                     ) -> List[Tuple[np.ndarray, np.ndarray]]:
    """Tree with R reference queries Rq [R, d]: [(keys_l [n_l, R, d], vals_l [n_l, d])]."""
    Rq = np.atleast_2d(np.asarray(Rq, dtype=np.float64))
    per_ref = [build_tree(K, V, Rq[j], B, b) for j in range(Rq.shape[0])]
    levels = []
    for lev in range(len(per_ref[0])):
        keys = np.stack([per_ref[j][lev][0] for j in range(Rq.shape[0])], axis=1)
        levels.append((keys, per_ref[0][lev][1]))
    return levels


class MultiTree:
    """Tree source of ``build_tree_multi`` output: key(level, j) is [R, d]."""

    def __init__(self, levels):
        self.levels = levels

    def key(self, level: int, j: int) -> np.ndarray:
        return self.levels[level - 1][0][j]

    def val(self, level: int, j: int) -> np.ndarray:
        return self.levels[level - 1][1][j]


class LazyMultiTree:
    """On-demand counterpart of MultiTree for long caches: one LazyTree per
    reference query (the R key trees are independent), values from the first."""

    def __init__(self, K, V, Rq, B: int, b: int):
        Rq = np.atleast_2d(np.asarray(Rq, dtype=np.float64))
        self.trees = [LazyTree(K, V, Rq[j], B, b) for j in range(Rq.shape[0])]

    def key(self, level: int, j: int) -> np.ndarray:
        return np.stack([t.key(level, j) for t in self.trees])

    def val(self, level: int, j: int) -> np.ndarray:
        return self.trees[0].val(level, j)
