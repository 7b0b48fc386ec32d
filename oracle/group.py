"""Per-KV-group shared selection, float64, the G query heads of one KV head
at a time.

TEST INFRASTRUCTURE (see the package docstring): imported only by the tests,
the smoke check and the CPU legs of the benchmark.

The variant: the G query heads that share a KV head also share one selection,
so one stream of summary rows and exact K/V rows serves all of them.
"Subquadratic Attention with a Hierarchical Tree-Structured Indexer" (ZHA),
Table IX (the MSA roofline's variables) counts selected blocks "per KV group":
that is the convention followed here, applied to RecSA's top-down traversal
("Recursive Sparse Attention: Million-Token Length Extrapolation at
Logarithmic Cost", abstract).

Readings (the pages do not say how the heads' scores combine):
  * candidates, counts and indices are RecSA's (children of the kept nodes,
    then the orphans; c_l = b * kappa_{l+1} + o_l, kappa_l = min(k, c_l));
  * each head scores the candidates with its own RecSA logit
    <R(c) q_h, R(i) key> / sqrt(d); the group score of a candidate is the sum
    over the G heads of its softmax probability among the level's candidates
    (each head's attention share for it, so no single head's logit scale
    dominates); the top min(k, c) group scores are kept (ties -> lower index);
  * with the shared selection fixed, every head attends exactly as in RecSA:
    its own logits over the unselected summaries and the exact tokens.

Pins (tests/test_oracle_pins.py): G = 1 and G identical heads reduce to
per-head RecSA; k = keep-all is dense causal attention for every head; the
group score's rule is fixed by a hand-built case in which a sum of logits
would keep another node; the result does not depend on the order of heads.
"""

from __future__ import annotations

import math
from typing import Dict, List

import numpy as np

from .recsa import Geometry, rope_rotate, traverse_and_attend, visible_counts


def group_select(Qg: np.ndarray, t: int, tree, geo: Geometry) -> dict:
    """Shared selection of the G query heads Qg [G, d] at position t.

    Returns dict(kept{level: node ids, candidate order}, cand{level: c},
    cand_ids{level: ids in candidate order}, group{level: [group score per
    candidate]}, top, a).
    """
    Qg = np.asarray(Qg, dtype=np.float64)
    G, d = Qg.shape
    B, b, k, W = geo.leaf_block, geo.branching, geo.k, geo.window
    inv_sqrt_d = 1.0 / math.sqrt(d)

    def rot(x, p):
        return rope_rotate(x, p, geo.rope_base) if geo.rope else np.asarray(x, np.float64)

    a, v = visible_counts(t, B, b, W)
    top = len(v)
    kept: Dict[int, List[int]] = {}
    cand_count: Dict[int, int] = {}
    cand_list: Dict[int, List[int]] = {}
    group_scores: Dict[int, List[float]] = {}
    parents: List[int] = []
    for lev in range(top, 0, -1):
        v_up = v[lev] if lev < top else 0
        cand = [p * b + j for p in parents for j in range(b)] + list(range(b * v_up, v[lev - 1]))
        c = len(cand)
        keys = [rot(tree.key(lev, n), i) for i, n in enumerate(cand)]
        score = np.zeros(c)
        for h in range(G):
            qr = rot(Qg[h], c)
            logit = np.array([float(qr @ kk) * inv_sqrt_d for kk in keys])
            w = np.exp(logit - logit.max())
            score += w / w.sum()
        order = sorted(range(c), key=lambda i: (-score[i], i))
        chosen = sorted(order[:min(k, c)])
        parents = [cand[i] for i in chosen]
        kept[lev] = parents
        cand_count[lev] = c
        cand_list[lev] = cand
        group_scores[lev] = [float(x) for x in score]
    return dict(kept=kept, cand=cand_count, cand_ids=cand_list, group=group_scores, top=top,
                a=a)


def group_traverse_and_attend(Qg: np.ndarray, t: int, K, V, tree, geo: Geometry,
                              keep_override: Dict[int, List[int]] | None = None) -> dict:
    """Outputs [G, d] of the G heads under their shared selection.

    ``keep_override`` (level -> kept ids) replaces the group's selection
    (used where several selections are correct: near-equal group scores).
    Returns dict(out [G, d], kept, cand, cand_ids, group, heads [per-head
    oracle results]); cand_ids and group describe the group's own selection.
    """
    sel = group_select(Qg, t, tree, geo)
    kept = sel["kept"] if keep_override is None else keep_override
    heads = [traverse_and_attend(Qg[h], t, K, V, tree, geo, keep_override=kept)
             for h in range(np.asarray(Qg).shape[0])]
    return dict(out=np.stack([r["out"] for r in heads]), kept=kept, cand=sel["cand"],
                cand_ids=sel["cand_ids"], group=sel["group"], top=sel["top"], a=sel["a"],
                heads=heads)
