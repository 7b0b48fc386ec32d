"""ZHA routing variant of the oracle, float64, one query head at a time.

TEST INFRASTRUCTURE (see the package docstring): imported only by the tests,
the smoke check and the CPU legs of the benchmark.

"Subquadratic Attention with a Hierarchical Tree-Structured Indexer" (ZHA),
Figure 3 caption: the tree is built as in RecSA (ZHA is the close variant that
RecSA's tree follows); routing starts at the top of the tree, scores the
level's nodes against the query by dot product, selects the nodes to expand by
top-p, and descends level by level to the leaves; the union of the leaves
reached is the sparse subset of the KV cache that the main attention sees.

Readings (pages silent; stated here and in the design notes):
  * candidates of a level are the children of the expanded nodes followed by
    the orphans (visible nodes whose parent is not visible), exactly as in
    RecSA, so that every visible token stays reachable;
  * routing scores are q . key / sqrt(d) on the un-rotated query and summary
    keys: the tree pools pre-RoPE keys, and RoPE belongs to the main attention;
    with several reference queries (a tree source whose keys are [R, d], see
    multiref.py) a node scores the largest of its R dot products;
  * top-p: the smallest set of highest-scoring candidates whose softmax mass
    (over the level's candidates) reaches p, ties to the lower index, capped at
    k nodes (k = keep-all: no cap);
  * the main attention covers the tokens of the reached leaves plus the exact
    window [a*B, t] (tokens not yet summarised by a visible node), at their
    true positions with standard RoPE, and no summary enters the softmax.

Pins (tests/test_oracle_pins.py): p = 1 with no cap is dense causal RoPE
attention (torch scaled_dot_product_attention in float64); the top-p set
equals a brute-force search over all subsets on small score vectors; a tiny
p expands exactly the arg-max at every level, checked against a greedy descent
written independently.
"""

from __future__ import annotations

import math
from typing import Dict, List, Sequence

import numpy as np

from .recsa import Geometry, rope_rotate, visible_counts


def top_p_prefix(scores: Sequence[float], p: float, cap: int) -> List[int]:
    """Indices (increasing) of the top-p set of ``scores`` (already scaled).

    Candidates in decreasing score order (ties: lower index first) are taken
    until their softmax mass reaches p or ``cap`` are taken.
    """
    s = np.asarray(scores, dtype=np.float64)
    w = np.exp(s - s.max())
    w = w / w.sum()
    order = sorted(range(len(s)), key=lambda i: (-s[i], i))
    chosen, mass = [], 0.0
    for i in order:
        chosen.append(i)
        mass += w[i]
        if mass >= p or len(chosen) >= cap:
            break
    return sorted(chosen)


def zha_route_and_attend(q: np.ndarray, t: int, K, V, tree, geo: Geometry, top_p: float,
                         keep_override: Dict[int, List[int]] | None = None) -> dict:
    """Output of one query head at position t under ZHA routing.

    ``keep_override`` (level -> expanded node ids) recomputes the output for a
    given routing (used where several routings are correct: a mass within
    rounding of p, or near-equal scores).  Returns dict(out, kept{level: ids},
    cand{level: c}, cand_ids{level: ids in candidate order}, scores{level: [..]
    in candidate order}, mass{level: [cumulative masses in decreasing-score
    order]}, n_exact, top, a).
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    B, b, W = geo.leaf_block, geo.branching, geo.window
    inv_sqrt_d = 1.0 / math.sqrt(d)
    a, v = visible_counts(t, B, b, W)
    top = len(v)
    kept_nodes: Dict[int, List[int]] = {}
    cand_count: Dict[int, int] = {}
    cand_list: Dict[int, List[int]] = {}
    level_scores: Dict[int, List[float]] = {}
    level_mass: Dict[int, List[float]] = {}
    expanded: List[int] = []
    for lev in range(top, 0, -1):
        v_up = v[lev] if lev < top else 0
        children = [n * b + c for n in expanded for c in range(b)]
        orphans = list(range(b * v_up, v[lev - 1]))
        cand = children + orphans
        # a node with several reference keys [R, d] scores its best match
        scores = [float(np.max(np.atleast_2d(np.asarray(tree.key(lev, n), np.float64)) @ q))
                  * inv_sqrt_d for n in cand]
        if keep_override is not None:
            want = set(int(x) for x in keep_override[lev])
            idx = [i for i, n in enumerate(cand) if n in want]
            if len(idx) != len(want):
                raise ValueError(f"level {lev}: routed ids {sorted(want)} are not all candidates")
        else:
            idx = top_p_prefix(scores, top_p, geo.k)
        s = np.asarray(scores)
        w = np.exp(s - s.max())
        w = w / w.sum()
        order = sorted(range(len(s)), key=lambda i: (-s[i], i))
        level_mass[lev] = list(np.cumsum(w[order]))
        expanded = [cand[i] for i in idx]
        kept_nodes[lev] = expanded
        cand_count[lev] = len(cand)
        cand_list[lev] = cand
        level_scores[lev] = scores
    exact = [blk * B + o for blk in (expanded if top > 0 else []) for o in range(B)]
    exact += list(range(a * B, t + 1))
    if geo.rope:
        qr = rope_rotate(q, t, geo.rope_base)
        ks = rope_rotate(np.asarray(K[exact], np.float64), np.asarray(exact), geo.rope_base)
    else:
        qr = q
        ks = np.asarray(K[exact], np.float64)
    logits = ks @ qr * inv_sqrt_d
    pw = np.exp(logits - logits.max())
    out = (pw[:, None] * np.asarray(V[exact], np.float64)).sum(axis=0) / pw.sum()
    return dict(out=out, kept=kept_nodes, cand=cand_count, cand_ids=cand_list,
                scores=level_scores,
                mass=level_mass, n_exact=len(exact), top=top, a=a)
