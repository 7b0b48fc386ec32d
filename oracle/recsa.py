"""RecSA oracle, float64, one (sequence, KV head) tree and one query head at a time.

TEST INFRASTRUCTURE (see the package docstring): imported only by the tests,
the smoke check and the CPU-baseline leg of the benchmark.

Every step follows the pages in their order; where the pages leave a step open
the plainest reading is taken and stated beside the code ("reading: ...").

Parity pins (tests/test_oracle_pins.py):
  * tree values      -- mean of the leaf values of the node's span (closed form);
  * tree keys        -- single child, equal scores, hand-worked two-key example;
  * level counts     -- 3 / 4 / 6 summary levels for the 4K / 524K / 2M shapes;
  * traversal        -- set-based brute force on tiny trees (independent code);
  * k >= candidates  -- textbook dense causal attention, RoPE off and on;
  * entries read     -- the closed form and its O(log L) bound.
  * finite k with RoPE on: the summary-entry indices are pinned only by the
    set-based brute force written from the same reading -- "parity unpinned"
    beyond that reading (no page prints a worked value).
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Sequence, Tuple

import numpy as np

KEEP_ALL = 2**31 - 1


@dataclass(frozen=True)
class Geometry:
    """Tree geometry and attention shape (RecSA abstract; ZHA Table VIII).

    leaf_block  B: tokens summarised by one level-1 node.
    branching   b: children per node above level 1 (ZHA's chunk size C).
    k           at most k candidates kept per level (RecSA abstract).
    window      W: exact local window (reading: tokens [a*B, t] with
                a = floor(max(0, t+1-W)/B), so no partial leaf is summarised).
    """

    head_dim: int
    n_q_heads: int
    n_kv_heads: int
    leaf_block: int
    branching: int
    k: int
    window: int
    rope: bool = True
    rope_base: float = 1e6

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


# ---------------------------------------------------------------------------
# Tree shape
# ---------------------------------------------------------------------------

def level_counts(length: int, B: int, b: int) -> List[int]:
    """Complete nodes per level for a cache of ``length`` tokens.

    ZHA Table VIII: only full nodes exist, n_l = floor(T / C^l); here a
    level-l node spans B * b^(l-1) tokens.  Reading: a level exists while it
    holds at least one complete node (equivalently, level l+1 is added while
    n_l >= b), which gives 3, 4 and 6 summary levels for the 4K (B16 b16),
    524K (B64 b16) and 2M (B32 b8) shapes.
    """
    counts = []
    span = B
    while length // span >= 1:
        counts.append(length // span)
        span *= b
    return counts


def visible_counts(t: int, B: int, b: int, W: int) -> Tuple[int, List[int]]:
    """Nodes visible to the query at position t.

    Reading (pages silent): the exact window starts at a*B with
    a = floor(max(0, t+1-W) / B); a level-l node is visible iff its span ends
    at or before a*B, so v_l = floor(a / b^(l-1)).  Returns (a, [v_1, ...])
    with trailing zero levels dropped.
    """
    s = max(0, t + 1 - W)
    a = s // B
    v = []
    per = 1
    while a // per >= 1:
        v.append(a // per)
        per *= b
    return a, v


# ---------------------------------------------------------------------------
# Pooler and tree build
# ---------------------------------------------------------------------------

def pool_keys(keys: np.ndarray, r: np.ndarray) -> np.ndarray:
    """Summary key of one node from its children's keys.

    RecSA abstract: one pooler per layer, shared by all levels.  Its form
    (the workload definition): weights = softmax over children of r.k/sqrt(d),
    key = sum of weight * child key.  ZHA Figure 3: the parent key is an
    attention-weighted sum of the child keys against a reference query.
    """
    keys = np.asarray(keys, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    d = keys.shape[-1]
    s = keys @ r / math.sqrt(d)
    w = np.exp(s - s.max())
    w = w / w.sum()
    return w @ keys


def build_tree(K: np.ndarray, V: np.ndarray, r: np.ndarray, B: int, b: int
               ) -> List[Tuple[np.ndarray, np.ndarray]]:
    """All complete nodes over one KV head's cache K, V [T, d].

    Level 1 pools each leaf block of B tokens; level l > 1 pools b consecutive
    level-(l-1) summary keys (ZHA Figure 3: higher levels from the summaries of
    lower levels).  Value = mean of the children's values (RecSA abstract:
    mean-pooled value), i.e. the mean of the leaf values under the node.
    Returns [(keys_l [n_l, d], vals_l [n_l, d]) for l = 1..D].
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    counts = level_counts(K.shape[0], B, b)
    levels: List[Tuple[np.ndarray, np.ndarray]] = []
    for lev, n in enumerate(counts):
        fan = B if lev == 0 else b
        src_k = K if lev == 0 else levels[-1][0]
        src_v = V if lev == 0 else levels[-1][1]
        keys = np.empty((n, K.shape[1]))
        vals = np.empty((n, K.shape[1]))
        for j in range(n):
            keys[j] = pool_keys(src_k[j * fan:(j + 1) * fan], r)
            vals[j] = src_v[j * fan:(j + 1) * fan].mean(axis=0)
        levels.append((keys, vals))
    return levels


def node_summary(K: np.ndarray, V: np.ndarray, r: np.ndarray, B: int, b: int,
                 level: int, j: int) -> Tuple[np.ndarray, np.ndarray]:
    """(key, value) of node j at ``level`` (1-based), recomputed from its span.

    A node depends only on the tokens of its span, so it can be computed alone;
    used for sampled checks on caches too large for ``build_tree``.
    """
    if level == 1:
        ks = np.asarray(K[j * B:(j + 1) * B], dtype=np.float64)
        vs = np.asarray(V[j * B:(j + 1) * B], dtype=np.float64)
        return pool_keys(ks, r), vs.mean(axis=0)
    child = [node_summary(K, V, r, B, b, level - 1, j * b + c) for c in range(b)]
    ck = np.stack([c[0] for c in child])
    cv = np.stack([c[1] for c in child])
    return pool_keys(ck, r), cv.mean(axis=0)


class FullTree:
    """Tree source backed by ``build_tree`` output."""

    def __init__(self, levels):
        self.levels = levels

    def key(self, level: int, j: int) -> np.ndarray:
        return self.levels[level - 1][0][j]

    def val(self, level: int, j: int) -> np.ndarray:
        return self.levels[level - 1][1][j]


class LazyTree:
    """Tree source that computes nodes on demand (memoised) from K, V.

    For sampled checks on long caches: only the nodes a traversal touches are
    ever computed.
    """

    def __init__(self, K, V, r, B: int, b: int):
        self.K, self.V, self.r, self.B, self.b = K, V, np.asarray(r, np.float64), B, b
        self.cache: Dict[Tuple[int, int], Tuple[np.ndarray, np.ndarray]] = {}

    def _node(self, level: int, j: int):
        hit = self.cache.get((level, j))
        if hit is not None:
            return hit
        if level == 1:
            ks = np.asarray(self.K[j * self.B:(j + 1) * self.B], dtype=np.float64)
            vs = np.asarray(self.V[j * self.B:(j + 1) * self.B], dtype=np.float64)
            out = (pool_keys(ks, self.r), vs.mean(axis=0))
        else:
            ch = [self._node(level - 1, j * self.b + c) for c in range(self.b)]
            out = (pool_keys(np.stack([c[0] for c in ch]), self.r),
                   np.stack([c[1] for c in ch]).mean(axis=0))
        self.cache[(level, j)] = out
        return out

    def key(self, level: int, j: int) -> np.ndarray:
        return self._node(level, j)[0]

    def val(self, level: int, j: int) -> np.ndarray:
        return self._node(level, j)[1]


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def rope_cos_sin(pos, d: int, base: float):
    """cos and sin of pos * base^(-2j/d), j < d/2, in float64.

    Reading (pages silent on the layout): rotate-half pairing (dims j and
    j + d/2), the convention of the Qwen3 family the pages initialise from.
    """
    pos = np.asarray(pos, dtype=np.float64)
    j = np.arange(d // 2, dtype=np.float64)
    inv = base ** (-2.0 * j / d)
    ang = pos[..., None] * inv
    return np.cos(ang), np.sin(ang)


def rope_rotate(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate x [..., d] to position(s) ``pos`` (broadcast over leading dims)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    c, s = rope_cos_sin(pos, d, base)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ---------------------------------------------------------------------------
# Traversal and shared softmax
# ---------------------------------------------------------------------------

def _top_k_sorted(scores: Sequence[float], k: int) -> List[int]:
    """Indices of the top-min(k, n) scores; ties go to the lower index.

    Returned in increasing index order (= position order of the candidates).
    """
    order = sorted(range(len(scores)), key=lambda i: (-scores[i], i))
    return sorted(order[: min(k, len(scores))])


def traverse_and_attend(q: np.ndarray, t: int, K, V, tree, geo: Geometry,
                        keep_override: Dict[int, List[int]] | None = None) -> dict:
    """Output of one query head at position t, with its selection trace.

    RecSA abstract, step by step:
      1. Start at the highest level with a visible node; its visible nodes are
         the candidates.  At each lower level the candidates are the children
         of the kept nodes followed by the orphans (visible nodes whose parent
         is not visible), in position order, indexed 0..c-1.
      2. Each level keeps at most k candidates (top scores; ties -> lower
         index).  Reading: the selection score is the candidate's softmax
         logit <R(c) q, R(i) key>/sqrt(d) -- RoPE position of a candidate is its
         index i among the level's candidates, and the query sits one past the
         last candidate (index c).  One logit for selection and summary follows
         the digest's note that one pooler serves selection and summary keys.
      3. Unselected candidates contribute (logit, summary value) to the softmax.
      4. Kept level-1 nodes expand to their B exact tokens; with the window
         tokens [a*B, t] they form the token level, indexed 0..n0-1 in
         position order, query index n0-1 (the query is the last token).
      5. One softmax over all summary and exact entries, scale 1/sqrt(d).

    ``keep_override`` (level -> kept node ids) recomputes the output for a
    given selection (used where several selections are correct: near ties);
    the ids must be candidates of their level.  Returns dict(out, kept{level: node ids}, cand{level: c},
    scores{level: [..]}, entries, keys_read, n_exact).
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    B, b, k, W = geo.leaf_block, geo.branching, geo.k, geo.window
    base = geo.rope_base
    inv_sqrt_d = 1.0 / math.sqrt(d)

    def rot(x, p):
        return rope_rotate(x, p, base) if geo.rope else np.asarray(x, np.float64)

    a, v = visible_counts(t, B, b, W)
    top = len(v)
    logits: List[float] = []
    values: List[np.ndarray] = []
    kept_nodes: Dict[int, List[int]] = {}
    cand_count: Dict[int, int] = {}
    level_scores: Dict[int, List[float]] = {}
    keys_read = 0
    kept_parent: List[int] = []
    for lev in range(top, 0, -1):
        v_up = v[lev] if lev < top else 0       # visible nodes one level up
        children = [p * b + c for p in kept_parent for c in range(b)]
        orphans = list(range(b * v_up, v[lev - 1]))
        cand = children + orphans
        c = len(cand)
        qr = rot(q, c)
        scores = [float(qr @ rot(tree.key(lev, n), i)) * inv_sqrt_d
                  for i, n in enumerate(cand)]
        keys_read += c
        if keep_override is not None:
            want = set(int(x) for x in keep_override[lev])
            kept_idx = [i for i, n in enumerate(cand) if n in want]
            if len(kept_idx) != len(want):
                raise ValueError(f"level {lev}: kept ids {sorted(want)} are not all candidates")
        else:
            kept_idx = _top_k_sorted(scores, k)
        kept_set = set(kept_idx)
        for i, n in enumerate(cand):
            if i not in kept_set:
                logits.append(scores[i])
                values.append(np.asarray(tree.val(lev, n), np.float64))
        kept_parent = [cand[i] for i in kept_idx]
        kept_nodes[lev] = kept_parent
        cand_count[lev] = c
        level_scores[lev] = scores
    exact = [blk * B + o for blk in (kept_parent if top > 0 else []) for o in range(B)]
    exact += list(range(a * B, t + 1))
    n0 = len(exact)
    qr = rot(q, n0 - 1)
    for i, pos in enumerate(exact):
        kk = np.asarray(K[pos], dtype=np.float64)
        logits.append(float(qr @ rot(kk, i)) * inv_sqrt_d)
        values.append(np.asarray(V[pos], dtype=np.float64))
    keys_read += n0
    lg = np.array(logits)
    p = np.exp(lg - lg.max())
    out = (p[:, None] * np.stack(values)).sum(axis=0) / p.sum()
    return dict(out=out, kept=kept_nodes, cand=cand_count, scores=level_scores,
                entries=len(logits), keys_read=keys_read, n_exact=n0, a=a, top=top)


def closed_form_counts(t: int, geo: Geometry) -> dict:
    """Candidate, softmax-entry and key-read counts of one query, in closed form.

    c_top = v_top; c_l = b * kappa_{l+1} + o_l with o_l = v_l - b * v_{l+1};
    kappa_l = min(k, c_l).  Softmax entries E = sum_l (c_l - kappa_l)
    + B * kappa_1 + (t + 1 - a*B); keys read = sum_l c_l + B * kappa_1 +
    (t + 1 - a*B).  RecSA abstract: each query reads O(log L) entries; the
    bound is E <= D (b k + b - 1) + B k + W + B - 1.
    """
    B, b, k, W = geo.leaf_block, geo.branching, geo.k, geo.window
    a, v = visible_counts(t, B, b, W)
    top = len(v)
    c: Dict[int, int] = {}
    kap: Dict[int, int] = {}
    kappa_up = 0
    for lev in range(top, 0, -1):
        v_up = v[lev] if lev < top else 0
        c[lev] = b * kappa_up + (v[lev - 1] - b * v_up)
        kap[lev] = min(k, c[lev])
        kappa_up = kap[lev]
    window = t + 1 - a * B
    leaf_tokens = B * kap.get(1, 0)
    E = sum(c[l] - kap[l] for l in c) + leaf_tokens + window
    R = sum(c.values()) + leaf_tokens + window
    return dict(cand=c, kept=kap, entries=E, keys_read=R, a=a, top=top,
                n_exact=leaf_tokens + window)
