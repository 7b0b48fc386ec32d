"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against a closed form, a special case that reduces
to a library routine (torch's scaled_dot_product_attention in float64), a
hand-worked fixture under tests/golden/, or an independently written brute force
(set-based enumeration with complex-number RoPE), chosen so that a dropped term,
a wrong index or sign, or a transposed operand in the oracle fails one of them.
"""

import cmath
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import Geometry

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _rand_kv(rng, T, d, scale=1.0):
    K = rng.standard_normal((T, d)) * scale
    V = rng.standard_normal((T, d))
    return K, V


# ---------------------------------------------------------------------------
# Tree shape
# ---------------------------------------------------------------------------

def test_level_counts_match_workload_depths():
    # 3, 4 and 6 summary levels for the 4K, 524K and 2M workload shapes.
    assert oracle.level_counts(4096, 16, 16) == [256, 16, 1]
    assert oracle.level_counts(524288, 64, 16) == [8192, 512, 32, 2]
    assert oracle.level_counts(2097152, 32, 8) == [65536, 8192, 1024, 128, 16, 2]
    assert oracle.level_counts(131072, 64, 16) == [2048, 128, 8]
    assert oracle.level_counts(1048576, 64, 32) == [16384, 512, 16]
    # Only complete nodes: a ragged tail adds nothing.
    assert oracle.level_counts(4096 + 15, 16, 16) == [256, 16, 1]
    assert oracle.level_counts(15, 16, 16) == []
    assert oracle.level_counts(16, 16, 16) == [1]


def test_visible_counts_definition():
    # Brute force: node j at level l visible iff (j+1) * B * b^(l-1) <= a * B.
    B, b, W = 4, 3, 9
    for t in range(0, 300):
        a, v = oracle.visible_counts(t, B, b, W)
        assert a * B <= max(0, t + 1 - W) < a * B + B
        for lev in range(1, 8):
            span = B * b ** (lev - 1)
            brute = sum(1 for j in range(400) if (j + 1) * span <= a * B)
            got = v[lev - 1] if lev <= len(v) else 0
            assert got == brute


# ---------------------------------------------------------------------------
# Pooler and tree values
# ---------------------------------------------------------------------------

def test_pool_two_key_golden(golden_dir):
    rows = {}
    ck, cv = [], []
    with open(os.path.join(golden_dir, "pool_two_keys.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, *vals = line.split()
            vals = [float(x) for x in vals]
            if name == "child_key":
                ck.append(vals)
            elif name == "child_val":
                cv.append(vals)
            else:
                rows[name] = vals
    key = oracle.pool_keys(np.array(ck), np.array(rows["r"]))
    np.testing.assert_allclose(key, rows["expect_key"], rtol=0, atol=1e-12)
    # Through build_tree: a 2-token leaf block gives the same node.
    levels = oracle.build_tree(np.array(ck), np.array(cv), np.array(rows["r"]), 2, 2)
    np.testing.assert_allclose(levels[0][0][0], rows["expect_key"], atol=1e-12)
    np.testing.assert_allclose(levels[0][1][0], rows["expect_val"], atol=1e-12)


def test_pool_special_cases():
    rng = np.random.default_rng(3)
    keys = rng.standard_normal((7, 16))
    # One child: the summary is the child itself.
    np.testing.assert_allclose(oracle.pool_keys(keys[:1], rng.standard_normal(16)),
                               keys[0], atol=1e-12)
    # r = 0: equal scores, the summary is the plain mean.
    np.testing.assert_allclose(oracle.pool_keys(keys, np.zeros(16)), keys.mean(0),
                               atol=1e-12)
    # A reference vector far along one child's key picks that child.
    r = 1e4 * keys[3] / np.linalg.norm(keys[3])
    np.testing.assert_allclose(oracle.pool_keys(keys, r), keys[3], atol=1e-9)
    # The weights are a softmax: the summary lies in the convex hull.
    r = rng.standard_normal(16)
    key = oracle.pool_keys(keys, r)
    assert np.all(key <= keys.max(0) + 1e-12) and np.all(key >= keys.min(0) - 1e-12)


def test_node_value_is_mean_of_leaf_values():
    rng = np.random.default_rng(0)
    B, b, d = 4, 3, 8
    K, V = _rand_kv(rng, 4 * 27 + 5, d)
    r = rng.standard_normal(d) / math.sqrt(d)
    levels = oracle.build_tree(K, V, r, B, b)
    assert [len(l[0]) for l in levels] == [28, 9, 3, 1]
    for lev, (_, vals) in enumerate(levels, start=1):
        span = B * b ** (lev - 1)
        for j in range(vals.shape[0]):
            np.testing.assert_allclose(vals[j], V[j * span:(j + 1) * span].mean(0),
                                       atol=1e-12)
    # node_summary and LazyTree agree with build_tree.
    lazy = oracle.LazyTree(K, V, r, B, b)
    for lev in range(1, 5):
        for j in range(len(levels[lev - 1][0])):
            kk, vv = oracle.node_summary(K, V, r, B, b, lev, j)
            np.testing.assert_allclose(kk, levels[lev - 1][0][j], atol=1e-12)
            np.testing.assert_allclose(vv, levels[lev - 1][1][j], atol=1e-12)
            np.testing.assert_allclose(lazy.key(lev, j), kk, atol=1e-12)


def test_parent_key_pools_child_summaries_not_tokens():
    # Level-2 key = pool over the level-1 *summary keys* (recursive pooling),
    # which differs from pooling all tokens of the span at once.
    rng = np.random.default_rng(1)
    B, b, d = 4, 2, 4
    K, V = _rand_kv(rng, 8, d)
    r = rng.standard_normal(d)
    levels = oracle.build_tree(K, V, r, B, b)
    l1 = [oracle.pool_keys(K[0:4], r), oracle.pool_keys(K[4:8], r)]
    np.testing.assert_allclose(levels[1][0][0], oracle.pool_keys(np.stack(l1), r),
                               atol=1e-12)
    assert not np.allclose(levels[1][0][0], oracle.pool_keys(K, r))


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def _rope_complex(x, pos, base):
    """Independent RoPE: pair (x_j, x_{j+d/2}) as a complex number, times e^{i p w_j}."""
    d = len(x)
    h = d // 2
    out = np.empty(d)
    for j in range(h):
        w = base ** (-2.0 * j / d)
        z = complex(x[j], x[j + h]) * cmath.exp(1j * pos * w)
        out[j], out[j + h] = z.real, z.imag
    return out


def test_rope_matches_complex_rotation_and_is_relative():
    rng = np.random.default_rng(2)
    d = 16
    x, y = rng.standard_normal(d), rng.standard_normal(d)
    for pos in [0, 1, 7, 1000, 123457]:
        np.testing.assert_allclose(oracle.rope_rotate(x, pos, 1e6),
                                   _rope_complex(x, pos, 1e6), atol=1e-9)
    np.testing.assert_allclose(oracle.rope_rotate(x, 0, 1e6), x, atol=0)
    # <R(m) x, R(n) y> depends only on m - n.
    a = oracle.rope_rotate(x, 50, 1e4) @ oracle.rope_rotate(y, 20, 1e4)
    bb = oracle.rope_rotate(x, 130, 1e4) @ oracle.rope_rotate(y, 100, 1e4)
    assert abs(a - bb) < 1e-9
    # Dimension 0 turns by exactly `pos` radians (inverse frequency 1).
    c, s = oracle.rope_cos_sin(np.array([3.0]), d, 1e6)
    assert abs(c[0, 0] - math.cos(3.0)) < 1e-15 and abs(s[0, 0] - math.sin(3.0)) < 1e-15


# ---------------------------------------------------------------------------
# Traversal against an independent set-based brute force
# ---------------------------------------------------------------------------

def brute_force(q, t, K, V, levels, geo):
    """Set-based restatement: classify every visible node, then one softmax.

    Candidates at a level = visible nodes whose parent is kept or whose parent
    is not visible (all visible nodes at the top level); each is scored at its
    rank (by position) among the level's candidates with the query one past the
    last; the best k by (score desc, rank asc) are kept.
    """
    d = len(q)
    B, b, k, W = geo.leaf_block, geo.branching, geo.k, geo.window
    a = max(0, t + 1 - W) // B

    def rot(x, p):
        return _rope_complex(x, p, geo.rope_base) if geo.rope else np.asarray(x)

    vis = {}
    for lev in range(1, len(levels) + 1):
        span = B * b ** (lev - 1)
        vis[lev] = [j for j in range(len(levels[lev - 1][0])) if (j + 1) * span <= a * B]
    tops = [lev for lev in vis if vis[lev]]
    entries = []
    kept = {}
    cand_sizes = {}
    if tops:
        top = max(tops)
        for lev in range(top, 0, -1):
            up_vis = set(vis.get(lev + 1, []))
            cand = sorted(j for j in vis[lev]
                          if lev == top or (j // b) in kept[lev + 1] or (j // b) not in up_vis)
            rank = {j: i for i, j in enumerate(cand)}
            qr = rot(q, len(cand))
            score = {j: float(qr @ rot(levels[lev - 1][0][j], rank[j])) / math.sqrt(d)
                     for j in cand}
            best = sorted(cand, key=lambda j: (-score[j], rank[j]))[:k]
            kept[lev] = set(best)
            cand_sizes[lev] = len(cand)
            for j in cand:
                if j not in kept[lev]:
                    entries.append((score[j], levels[lev - 1][1][j]))
    toks = set(range(a * B, t + 1))
    for blk in kept.get(1, set()):
        toks |= set(range(blk * B, blk * B + B))
    toks = sorted(toks)
    qr = rot(q, len(toks) - 1)
    for i, pos in enumerate(toks):
        entries.append((float(qr @ rot(K[pos], i)) / math.sqrt(d), V[pos]))
    m = max(e[0] for e in entries)
    w = np.array([math.exp(e[0] - m) for e in entries])
    out = sum(wi * e[1] for wi, e in zip(w, entries)) / w.sum()
    return out, {lev: sorted(s) for lev, s in kept.items()}, cand_sizes, len(entries)


@pytest.mark.parametrize("B,b,k,W,T,d,rope", [
    (2, 2, 1, 1, 64, 8, True),
    (4, 3, 2, 9, 200, 8, True),
    (4, 3, 2, 9, 200, 8, False),
    (3, 4, 3, 5, 150, 6, True),
    (8, 2, 2, 16, 300, 4, True),
])
def test_traversal_matches_set_based_brute_force(B, b, k, W, T, d, rope):
    rng = np.random.default_rng(B * 100 + b * 10 + k)
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d) / math.sqrt(d)
    levels = oracle.build_tree(K, V, r, B, b)
    tree = oracle.FullTree(levels)
    geo = Geometry(d, 1, 1, B, b, k, W, rope=rope, rope_base=1e2)
    for t in list(range(0, T, 7)) + [T - 1]:
        q = rng.standard_normal(d) * 2.0
        res = oracle.traverse_and_attend(q, t, K, V, tree, geo)
        ref, kept, sizes, n_entries = brute_force(q, t, K, V, levels, geo)
        assert {l: sorted(v) for l, v in res["kept"].items()} == kept
        assert res["cand"] == sizes
        assert res["entries"] == n_entries
        np.testing.assert_allclose(res["out"], ref, atol=1e-10)


def test_needle_recall_above_chance():
    # Sanity, not a parity pin: with an untrained (random) pooler a planted
    # needle's leaf block is kept far more often than chance (4 of ~252 blocks).
    rng = np.random.default_rng(5)
    B, b, d, T = 16, 16, 64, 4096
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d) / math.sqrt(d)
    tree = oracle.FullTree(oracle.build_tree(K, V, r, B, b))
    geo = Geometry(d, 1, 1, B, b, 4, 64, rope=False)
    hits = 0
    for _ in range(32):
        j = int(rng.integers(0, T - 64))
        q = 4 * K[j] + rng.standard_normal(d)
        res = oracle.traverse_and_attend(q, T - 1, K, V, tree, geo)
        hits += (j // B) in res["kept"][1]
    assert hits >= 4


# ---------------------------------------------------------------------------
# k >= every candidate count: dense attention (library routine)
# ---------------------------------------------------------------------------

def _sdpa(q, K, V):
    qt = torch.tensor(q, dtype=torch.float64).view(1, 1, 1, -1)
    kt = torch.tensor(K, dtype=torch.float64).view(1, 1, K.shape[0], -1)
    vt = torch.tensor(V, dtype=torch.float64).view(1, 1, V.shape[0], -1)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).view(-1).numpy()


@pytest.mark.parametrize("rope", [False, True])
def test_keep_all_equals_dense_attention(rope):
    rng = np.random.default_rng(7)
    B, b, d, T, W = 4, 3, 8, 260, 5
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d)
    tree = oracle.FullTree(oracle.build_tree(K, V, r, B, b))
    geo = Geometry(d, 1, 1, B, b, oracle.recsa.KEEP_ALL, W, rope=rope, rope_base=1e3)
    for t in [0, 3, 4, 10, 57, 130, 259]:
        q = rng.standard_normal(d) * 3
        res = oracle.traverse_and_attend(q, t, K, V, tree, geo)
        if rope:
            qr = _rope_complex(q, t, 1e3)
            Kr = np.stack([_rope_complex(K[j], j, 1e3) for j in range(t + 1)])
        else:
            qr, Kr = q, K[: t + 1]
        ref = _sdpa(qr, Kr, V[: t + 1])
        np.testing.assert_allclose(res["out"], ref, atol=1e-12)
        np.testing.assert_allclose(
            oracle.dense_causal_attention(q, t, K, V, rope=rope, rope_base=1e3), ref,
            atol=1e-12)
        assert res["n_exact"] == t + 1 and res["entries"] == t + 1


def test_constant_values_give_constant_output():
    # Normalisation is shared by summaries and exact tokens: if every token has
    # the same value, every summary has it too and the output equals it.
    rng = np.random.default_rng(8)
    B, b, d, T = 4, 3, 8, 200
    K = rng.standard_normal((T, d))
    V = np.tile(rng.standard_normal(d), (T, 1))
    tree = oracle.FullTree(oracle.build_tree(K, V, rng.standard_normal(d), B, b))
    geo = Geometry(d, 1, 1, B, b, 2, 9)
    for t in [50, 199]:
        res = oracle.traverse_and_attend(rng.standard_normal(d), t, K, V, tree, geo)
        assert res["entries"] > res["n_exact"]        # summaries were used
        np.testing.assert_allclose(res["out"], V[0], atol=1e-12)


# ---------------------------------------------------------------------------
# Counts
# ---------------------------------------------------------------------------

def test_counts_closed_form_golden(golden_dir):
    with open(os.path.join(golden_dir, "closed_form_counts.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for L, B, b, k, W, D, E, R, cands in rows:
        L, B, b, k, W, D, E, R = map(int, (L, B, b, k, W, D, E, R))
        geo = Geometry(128, 32, 8, B, b, k, W)
        assert len(oracle.level_counts(L, B, b)) == D
        cf = oracle.closed_form_counts(L - 1, geo)
        assert cf["entries"] == E and cf["keys_read"] == R
        assert [cf["cand"][l] for l in sorted(cf["cand"])] == [int(x) for x in cands.split(",")]
        assert E <= D * (b * k + b - 1) + B * k + W + B - 1


@pytest.mark.parametrize("B,b,k,W", [(4, 3, 2, 9), (2, 2, 1, 1), (16, 16, 4, 64)])
def test_traversal_counts_equal_closed_form(B, b, k, W):
    rng = np.random.default_rng(11)
    d, T = 8, 1200
    K, V = _rand_kv(rng, T, d)
    tree = oracle.FullTree(oracle.build_tree(K, V, rng.standard_normal(d), B, b))
    geo = Geometry(d, 1, 1, B, b, k, W)
    for t in range(0, T, 37):
        res = oracle.traverse_and_attend(rng.standard_normal(d), t, K, V, tree, geo)
        cf = oracle.closed_form_counts(t, geo)
        assert res["entries"] == cf["entries"]
        assert res["keys_read"] == cf["keys_read"]
        assert res["cand"] == cf["cand"]


def test_entries_grow_logarithmically():
    geo = Geometry(128, 32, 8, 64, 16, 8, 512)
    prev = None
    for L in [2**p for p in range(12, 32)]:
        E = oracle.closed_form_counts(L - 1, geo)["entries"]
        D = len(oracle.level_counts(L, 64, 16))
        assert E <= D * (16 * 8 + 15) + 64 * 8 + 512 + 63
        prev = E
    assert prev < 2000          # 2^31 tokens: still under 2000 entries


# ---------------------------------------------------------------------------
# ZHA routing variant
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rope", [False, True])
def test_zha_full_mass_equals_dense_attention(rope):
    """p = 1 with no cap expands every candidate: the reached leaves and the
    window are every token up to t, at true positions -- dense causal RoPE
    attention."""
    rng = np.random.default_rng(11)
    B, b, d, T, W = 4, 3, 8, 200, 6
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d)
    tree = oracle.FullTree(oracle.build_tree(K, V, r, B, b))
    geo = Geometry(d, 1, 1, B, b, oracle.recsa.KEEP_ALL, W, rope=rope, rope_base=1e3)
    for t in [0, 5, 6, 23, 99, 199]:
        q = rng.standard_normal(d) * 2
        res = oracle.zha_route_and_attend(q, t, K, V, tree, geo, top_p=1.0)
        if rope:
            qr = _rope_complex(q, t, 1e3)
            Kr = np.stack([_rope_complex(K[j], j, 1e3) for j in range(t + 1)])
        else:
            qr, Kr = q, K[: t + 1]
        ref = _sdpa(qr, Kr, V[: t + 1])
        np.testing.assert_allclose(res["out"], ref, atol=1e-12)
        assert res["n_exact"] == t + 1


def test_zha_top_p_matches_subset_brute_force():
    """The top-p set is the smallest set of candidates whose softmax mass
    reaches p, and among sets of that size the heaviest (brute force over all
    subsets); a cap limits its size."""
    import itertools
    rng = np.random.default_rng(3)
    for trial in range(200):
        n = int(rng.integers(1, 8))
        s = rng.standard_normal(n) * float(rng.uniform(0.1, 4))
        p = float(rng.uniform(0.05, 1.0))
        cap = int(rng.integers(1, 9))
        w = np.exp(s - s.max())
        w = w / w.sum()
        best = None
        for m in range(1, n + 1):
            subs = [c for c in itertools.combinations(range(n), m)]
            heavy = max(subs, key=lambda c: (sum(w[list(c)]), [-x for x in c]))
            if sum(w[list(heavy)]) >= p - 1e-12 or m == min(cap, n):
                best = sorted(heavy)
                break
        got = oracle.top_p_prefix(list(s), p, cap)
        assert got == best, (trial, s, p, cap, got, best)


def test_zha_tiny_p_is_greedy_descent():
    """With a tiny p one candidate per level is expanded: the arg-max of
    q . key, descending from the top; checked against a greedy descent over
    node spans written here independently of the oracle's candidate lists."""
    rng = np.random.default_rng(5)
    B, b, d, T, W = 4, 3, 8, 300, 4
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d)
    levels = oracle.build_tree(K, V, r, B, b)
    tree = oracle.FullTree(levels)
    geo = Geometry(d, 1, 1, B, b, oracle.recsa.KEEP_ALL, W, rope=False)
    for t in [40, 101, 299]:
        q = rng.standard_normal(d)
        res = oracle.zha_route_and_attend(q, t, K, V, tree, geo, top_p=1e-9)
        a = max(0, t + 1 - W) // B
        # greedy: at each level the arg-max among the children of the previous
        # pick plus every visible node whose parent is not visible
        span = [B * b ** l for l in range(len(levels))]
        vis = [a * B // span[l] for l in range(len(levels))]
        top = max(l + 1 for l in range(len(levels)) if vis[l] > 0)
        pick = None
        for lev in range(top, 0, -1):
            nodes = set()
            if pick is not None:
                nodes |= {pick * b + c for c in range(b)}
            up = vis[lev] if lev < top else 0
            nodes |= set(range(b * up, vis[lev - 1]))
            nodes = sorted(nodes)
            sc = [q @ levels[lev - 1][0][n] for n in nodes]
            pick = nodes[int(np.argmax(sc))]
            assert res["kept"][lev] == [pick]
        exact = list(range(pick * B, pick * B + B)) + list(range(a * B, t + 1))
        lg = K[exact] @ q / math.sqrt(d)
        pw = np.exp(lg - lg.max())
        np.testing.assert_allclose(res["out"], (pw[:, None] * V[exact]).sum(0) / pw.sum(),
                                   atol=1e-12)


def test_zha_partial_routing_attends_at_true_positions():
    """With 0 < p < 1 and RoPE on, the attention is textbook RoPE attention
    over the reached leaves' tokens and the window, each rotated by its true
    position (not by its index in the exact list, which equals the position
    only when every token is reached): checked with complex-number RoPE and a
    plain softmax, given the oracle's routing (pinned separately above)."""
    rng = np.random.default_rng(13)
    B, b, d, T, W = 4, 3, 8, 240, 6
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d)
    tree = oracle.FullTree(oracle.build_tree(K, V, r, B, b))
    geo = Geometry(d, 1, 1, B, b, 3, W, rope=True, rope_base=1e3)
    gaps = 0
    for t in [50, 117, 239]:
        for trial in range(4):
            q = rng.standard_normal(d) * 2
            res = oracle.zha_route_and_attend(q, t, K, V, tree, geo, top_p=0.6)
            a = max(0, t + 1 - W) // B
            leaves = res["kept"].get(1, [])
            exact = sorted({j for n in leaves for j in range(n * B, n * B + B)} |
                           set(range(a * B, t + 1)))
            gaps += int(exact != list(range(exact[0], exact[-1] + 1)))
            assert res["n_exact"] == len(exact)
            qr = _rope_complex(q, t, 1e3)
            Kr = np.stack([_rope_complex(K[j], j, 1e3) for j in exact])
            np.testing.assert_allclose(res["out"], _sdpa(qr, Kr, V[exact]), atol=1e-12)
    assert gaps > 0     # some cases skip tokens, where index and position differ


# ---------------------------------------------------------------------------
# Per-KV-group shared selection
# ---------------------------------------------------------------------------

class _KeyTable:
    """A one-level tree given by its node keys and values (hand-built cases)."""

    def __init__(self, keys, vals):
        self.keys, self.vals = np.asarray(keys, float), np.asarray(vals, float)

    def key(self, lev, n):
        assert lev == 1
        return self.keys[n]

    def val(self, lev, n):
        assert lev == 1
        return self.vals[n]


@pytest.mark.parametrize("rope", [False, True])
def test_group_of_one_or_identical_heads_is_per_head_recsa(rope):
    """One head, or G copies of one head, select exactly as that head alone:
    its summed probability is a monotone function of its own logit."""
    rng = np.random.default_rng(21)
    B, b, d, T, W, k = 4, 3, 8, 300, 6, 2
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d)
    tree = oracle.FullTree(oracle.build_tree(K, V, r, B, b))
    geo = Geometry(d, 1, 1, B, b, k, W, rope=rope, rope_base=1e3)
    for t in [30, 131, 299]:
        q = rng.standard_normal(d) * 2
        ref = oracle.traverse_and_attend(q, t, K, V, tree, geo)
        for G in (1, 3):
            res = oracle.group_traverse_and_attend(np.stack([q] * G), t, K, V, tree, geo)
            assert res["kept"] == ref["kept"]
            for h in range(G):
                np.testing.assert_allclose(res["out"][h], ref["out"], atol=1e-13)


@pytest.mark.parametrize("rope", [False, True])
def test_group_keep_all_is_dense_for_every_head(rope):
    rng = np.random.default_rng(22)
    B, b, d, T, W = 4, 3, 8, 150, 5
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d)
    tree = oracle.FullTree(oracle.build_tree(K, V, r, B, b))
    geo = Geometry(d, 4, 1, B, b, oracle.recsa.KEEP_ALL, W, rope=rope, rope_base=1e3)
    for t in [0, 17, 149]:
        Qg = rng.standard_normal((4, d)) * 2
        res = oracle.group_traverse_and_attend(Qg, t, K, V, tree, geo)
        for h in range(4):
            if rope:
                qr = _rope_complex(Qg[h], t, 1e3)
                Kr = np.stack([_rope_complex(K[j], j, 1e3) for j in range(t + 1)])
            else:
                qr, Kr = Qg[h], K[: t + 1]
            np.testing.assert_allclose(res["out"][h], _sdpa(qr, Kr, V[: t + 1]), atol=1e-12)


def test_group_score_sums_head_probabilities():
    """Hand-built level of three nodes (B = 1, b = 4, W = 1, t = 3: the three
    visible leaves are orphans of the top level), k = 1, no RoPE, d = 2.
    Head 0's logits are (5, 0, 0) and head 1's (-10, 2, 2.1): the summed
    probabilities are about (0.987, 0.482, 0.532), so node 0 is kept; a sum
    of logits, (-5, 2, 2.1), would keep node 2."""
    s2 = math.sqrt(2.0)
    keys = [[1.0, 0.0], [0.0, 1.0], [0.0, 1.05]]
    vals = [[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]]
    tree = _KeyTable(keys, vals)
    Qg = np.array([[5 * s2, 0.0], [-10 * s2, 2 * s2]])
    K = np.array([[1.0, 0.0], [0.0, 1.0], [0.0, 1.05], [0.5, 0.5]])
    V = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [2.0, -1.0]])
    geo = Geometry(2, 2, 1, 1, 4, 1, 1, rope=False)
    sel = oracle.group_select(Qg, 3, tree, geo)
    assert sel["top"] == 1 and sel["cand"] == {1: 3}
    assert sel["kept"] == {1: [0]}
    e5 = math.exp(5.0)
    p1 = np.exp([-10.0, 2.0, 2.1])
    want = np.array([e5, 1.0, 1.0]) / (e5 + 2.0) + p1 / p1.sum()
    np.testing.assert_allclose(sel["group"][1], want, rtol=1e-12)
    # the heads then attend over node 1, node 2 (summaries) and tokens 0, 3
    res = oracle.group_traverse_and_attend(Qg, 3, K, V, tree, geo)
    for h in range(2):
        lg = np.array([Qg[h] @ keys[1], Qg[h] @ keys[2], Qg[h] @ K[0], Qg[h] @ K[3]]) / s2
        w = np.exp(lg - lg.max())
        ref = (w[:, None] * np.array([vals[1], vals[2], V[0], V[3]])).sum(0) / w.sum()
        np.testing.assert_allclose(res["out"][h], ref, atol=1e-14)


def test_group_selection_is_head_order_free_and_the_best_subset():
    """Permuting the heads permutes the outputs only; at every level the kept
    set has the largest total group score among all subsets of its size."""
    import itertools
    rng = np.random.default_rng(23)
    B, b, d, T, W, k = 2, 3, 8, 120, 3, 2
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d)
    tree = oracle.FullTree(oracle.build_tree(K, V, r, B, b))
    geo = Geometry(d, 4, 1, B, b, k, W, rope=True, rope_base=1e3)
    for t in [50, 119]:
        Qg = rng.standard_normal((4, d)) * 2
        res = oracle.group_traverse_and_attend(Qg, t, K, V, tree, geo)
        perm = [2, 0, 3, 1]
        res_p = oracle.group_traverse_and_attend(Qg[perm], t, K, V, tree, geo)
        assert res_p["kept"] == res["kept"]
        np.testing.assert_allclose(res_p["out"], res["out"][perm], atol=1e-13)
        for lev, kept in res["kept"].items():
            sc, ids = res["group"][lev], res["cand_ids"][lev]
            n = min(k, len(sc))
            assert len(kept) == n and res["heads"][0]["kept"][lev] == kept
            best = max(sum(sc[i] for i in s) for s in itertools.combinations(range(len(sc)), n))
            assert abs(sum(sc[ids.index(x)] for x in kept) - best) < 1e-12


# ---------------------------------------------------------------------------
# Several reference queries (R > 1, ZHA routing)
# ---------------------------------------------------------------------------

def test_multiref_copies_of_one_reference_are_the_single_tree():
    rng = np.random.default_rng(31)
    B, b, d, T, W, k = 4, 3, 8, 200, 6, 3
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d)
    single = oracle.build_tree(K, V, r, B, b)
    multi = oracle.build_tree_multi(K, V, np.stack([r, r, r]), B, b)
    for (k1, v1), (k3, v3) in zip(single, multi):
        assert k3.shape == (k1.shape[0], 3, d)
        for j in range(3):
            np.testing.assert_array_equal(k3[:, j], k1)
        np.testing.assert_array_equal(v3, v1)
    geo = Geometry(d, 1, 1, B, b, k, W, rope=True, rope_base=1e3)
    for t in [40, 199]:
        q = rng.standard_normal(d) * 2
        a = oracle.zha_route_and_attend(q, t, K, V, oracle.FullTree(single), geo, 0.7)
        c = oracle.zha_route_and_attend(q, t, K, V, oracle.MultiTree(multi), geo, 0.7)
        assert a["kept"] == c["kept"]
        np.testing.assert_allclose(a["out"], c["out"], atol=1e-15)


def test_multiref_reference_j_is_its_own_recursive_tree():
    """Reference j's parent keys pool reference j's child keys (not another
    reference's): checked node by node against a direct recursive pooling."""
    rng = np.random.default_rng(32)
    B, b, d, T = 2, 3, 4, 60
    K, V = _rand_kv(rng, T, d)
    Rq = rng.standard_normal((2, d)) * 2
    multi = oracle.build_tree_multi(K, V, Rq, B, b)
    for j in range(2):
        for lev in range(1, len(multi) + 1):
            for n in range(multi[lev - 1][0].shape[0]):
                key, val = oracle.node_summary(K, V, Rq[j], B, b, lev, n)
                np.testing.assert_allclose(multi[lev - 1][0][n, j], key, atol=1e-13)
                np.testing.assert_allclose(multi[lev - 1][1][n], val, atol=1e-13)
    # the two references give different keys (the test above is not vacuous)
    assert np.abs(multi[0][0][:, 0] - multi[0][0][:, 1]).max() > 1e-3


def test_multiref_node_score_is_the_best_reference():
    """Hand-built level of two nodes with two reference keys each (B = 1,
    b = 4, W = 1, t = 2: both visible leaves are top-level orphans), k = 1,
    p = 0.5, no RoPE, d = 2, q = (sqrt 2, 0).  Node 0's keys score (3, -3) and
    node 1's (2, 2): the best-reference rule expands node 0 (3 > 2), while a
    sum or a mean of the scores would expand node 1."""
    s2 = math.sqrt(2.0)
    keys = np.array([[[3.0, 0.0], [-3.0, 0.0]], [[2.0, 0.0], [2.0, 0.0]]])
    vals = np.array([[1.0, 0.0], [0.0, 1.0]])

    class Two:
        def key(self, lev, n):
            return keys[n]

        def val(self, lev, n):
            return vals[n]

    K = np.array([[1.0, 0.0], [0.0, 1.0], [0.5, 0.5]])
    V = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]])
    geo = Geometry(2, 1, 1, 1, 4, 1, 1, rope=False)
    q = np.array([s2, 0.0])
    res = oracle.zha_route_and_attend(q, 2, K, V, Two(), geo, 0.5)
    assert res["top"] == 1 and res["cand"] == {1: 2}
    np.testing.assert_allclose(res["scores"][1], [3.0, 2.0], atol=1e-15)
    assert res["kept"] == {1: [0]}
    # attention over leaf 0 (token 0) and the window [2, 2]
    lg = np.array([q @ K[0], q @ K[2]]) / s2
    w = np.exp(lg - lg.max())
    np.testing.assert_allclose(res["out"], (w[:, None] * V[[0, 2]]).sum(0) / w.sum(),
                               atol=1e-15)


@pytest.mark.parametrize("rope", [False, True])
def test_multiref_full_mass_is_dense(rope):
    rng = np.random.default_rng(33)
    B, b, d, T, W = 4, 3, 8, 120, 5
    K, V = _rand_kv(rng, T, d)
    Rq = rng.standard_normal((4, d))
    tree = oracle.MultiTree(oracle.build_tree_multi(K, V, Rq, B, b))
    geo = Geometry(d, 1, 1, B, b, oracle.recsa.KEEP_ALL, W, rope=rope, rope_base=1e3)
    for t in [0, 37, 119]:
        q = rng.standard_normal(d) * 2
        res = oracle.zha_route_and_attend(q, t, K, V, tree, geo, top_p=1.0)
        if rope:
            qr = _rope_complex(q, t, 1e3)
            Kr = np.stack([_rope_complex(K[j], j, 1e3) for j in range(t + 1)])
        else:
            qr, Kr = q, K[: t + 1]
        np.testing.assert_allclose(res["out"], _sdpa(qr, Kr, V[: t + 1]), atol=1e-12)


def test_lazy_multiref_tree_equals_full_build():
    rng = np.random.default_rng(34)
    B, b, d, T = 4, 3, 8, 150
    K, V = _rand_kv(rng, T, d)
    Rq = rng.standard_normal((3, d))
    full = oracle.MultiTree(oracle.build_tree_multi(K, V, Rq, B, b))
    lazy = oracle.LazyMultiTree(K, V, Rq, B, b)
    for lev in range(1, len(full.levels) + 1):
        for n in range(full.levels[lev - 1][0].shape[0]):
            np.testing.assert_allclose(lazy.key(lev, n), full.key(lev, n), atol=1e-13)
            np.testing.assert_allclose(lazy.val(lev, n), full.val(lev, n), atol=1e-13)


# ---------------------------------------------------------------------------
# Low-precision router keys (FP8 E4M3, one scale per row)
# ---------------------------------------------------------------------------

def test_e4m3_decode_matches_the_format_table():
    """All 256 codes: sign, exponent field 0 (subnormal: m/8 * 2^-6) or 1..15
    (normal: (1 + m/8) * 2^(e-7)), NaN only at S.1111.111; spot values."""
    vals = [oracle.e4m3_decode(c) for c in range(256)]
    nan = [c for c in range(256) if math.isnan(vals[c])]
    assert nan == [0x7F, 0xFF]
    finite = sorted(set(v for v in vals if not math.isnan(v)))
    assert len(finite) == 253                        # +-0 coincide
    assert max(finite) == 448.0 and min(finite) == -448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9     # smallest subnormal
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6     # smallest normal
    assert oracle.e4m3_decode(0x38) == 1.0
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0xC0) == -2.0


def test_e4m3_round_fixed_points_ties_and_saturation():
    vals = np.array([v for v in (oracle.e4m3_decode(c) for c in range(256))
                     if not math.isnan(v)])
    np.testing.assert_array_equal(oracle.e4m3_round(vals), vals)
    pos = np.array(sorted(set(vals[vals >= 0])))
    mids = (pos[:-1] + pos[1:]) / 2
    got = oracle.e4m3_round(mids)
    for m, lo, hi, g in zip(mids, pos[:-1], pos[1:], got):
        # ties to the neighbour whose mantissa is even
        even = lo if (int(np.round(lo / _quantum(lo))) % 2 == 0) else hi
        assert g == even, (m, lo, hi, g)
    assert oracle.e4m3_round(np.array([463.9, 464.0, 1e6, -1e6])).tolist() == [448, 448, 448, -448]


def _quantum(v):
    _, e = np.frexp(v)
    return 2.0 ** (max(e - 1, -6) - 3)


def test_e4m3_round_agrees_with_torch_inside_the_range():
    rng = np.random.default_rng(40)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    x = x[np.abs(x) < 440]
    ref = torch.tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.e4m3_round(x), ref)


def test_fp8_tree_keys_are_quantized_pools_of_quantized_children():
    rng = np.random.default_rng(41)
    B, b, d, T = 4, 3, 8, 120
    K, V = _rand_kv(rng, T, d)
    r = rng.standard_normal(d)
    levels = oracle.build_tree_fp8(K, V, r, B, b)
    for lev, (keys, vals) in enumerate(levels, start=1):
        fan = B if lev == 1 else b
        src = K if lev == 1 else levels[lev - 2][0]
        for j in range(keys.shape[0]):
            pooled = oracle.pool_keys(src[j * fan:(j + 1) * fan], r)
            amax = np.abs(pooled).max()
            # each stored element is within half a quantum of the float value
            q = 2.0 ** (np.maximum(np.frexp(np.abs(pooled) / (amax / 448))[1] - 1, -6) - 3)
            assert np.all(np.abs(keys[j] - pooled) <= 0.5 * q * (amax / 448) * (1 + 1e-12))
            # and is an E4M3 value times the row scale
            unit = keys[j] / (amax / 448)
            np.testing.assert_allclose(oracle.e4m3_round(unit), unit, rtol=1e-14)
            np.testing.assert_allclose(vals[j], (V if lev == 1 else levels[lev - 2][1])
                                       [j * fan:(j + 1) * fan].mean(0), atol=1e-14)


def test_e2m1_codes_rounding_and_saturation():
    vals = [oracle.e2m1_decode(c) for c in range(16)]
    assert vals[:8] == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert vals[8:] == [-v for v in vals[:8]]
    pos = np.array(vals[:8])
    np.testing.assert_array_equal(oracle.e2m1_round(pos), pos)
    np.testing.assert_array_equal(oracle.e2m1_round(-pos), -pos)
    # midpoints go to the neighbour with mantissa bit 0 (codes 0, 2, 4, 6 -> even)
    mids = (pos[:-1] + pos[1:]) / 2                     # 0.25 .75 1.25 1.75 2.5 3.5 5
    assert oracle.e2m1_round(mids).tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    assert oracle.e2m1_round(np.array([6.9, 7.0, 100.0, -50.0])).tolist() == [6, 6, 6, -6]


def test_nvfp4_row_is_block_scaled_e2m1():
    rng = np.random.default_rng(42)
    for trial in range(50):
        x = rng.standard_normal(64) * 10.0 ** rng.uniform(-3, 2)
        y = oracle.quantize_row_nvfp4(x)
        g = np.abs(x).max() / (6 * 448)
        for b0 in range(0, 64, 16):
            blk, qb = x[b0:b0 + 16], y[b0:b0 + 16]
            sb = float(oracle.e4m3_round(np.abs(blk).max() / (6 * g)))
            assert oracle.e4m3_round(np.array([sb]))[0] == sb and sb > 0
            unit = qb / (sb * g)
            np.testing.assert_allclose(oracle.e2m1_round(unit), unit, atol=1e-12)
            # within half an E2M1 step of the scaled input (steps 0.5, 1, 2), or saturated
            a = np.abs(blk / (sb * g))
            step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
            ok = (np.abs(unit - blk / (sb * g)) <= step / 2 + 1e-12) | (np.abs(unit) == 6.0)
            assert ok.all()
    assert not oracle.quantize_row_nvfp4(np.zeros(32)).any()


def test_nvfp4_golden_row(golden_dir):
    """The NVFP4 scale reading pinned by a hand-worked row (tests/golden/nvfp4_row.txt):
    row scale, block scales (with an E4M3 tie and a rounded scale), element codes
    (ties to even, saturation after a rounded-down block scale) and a zero block."""
    xs, codes = [], []
    with open(os.path.join(golden_dir, "nvfp4_row.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, *vals = line.split()
            if key == "x":
                xs += [float(v) for v in vals]
            elif key == "code":
                codes += [float(v) for v in vals]
            elif key == "row_scale":
                g = float(vals[0])
            elif key == "block_scale":
                sb = [float(v) for v in vals]
    x = np.array(xs)
    assert x.shape == (64,) and len(codes) == 64 and len(sb) == 4
    assert g == np.abs(x).max() / (6 * 448)
    want = np.array(codes) * np.repeat(sb, 16) * g
    np.testing.assert_array_equal(oracle.quantize_row_nvfp4(x), want)


def _f32_nvfp4(x64, rng):
    """A float32 computation of one NVFP4 row, as a GPU would do it: the
    pooled row carries float32 error, then every quotient is taken in float32."""
    amax = np.abs(x64).max()
    x32 = (x64 + rng.standard_normal(x64.shape) * 1e-7 * amax).astype(np.float32)
    g32 = np.float32(np.abs(x32).max()) / np.float32(6 * 448)
    el = np.zeros_like(x64)
    sbs = np.zeros(x64.shape[0] // 16)
    for b in range(x64.shape[0] // 16):
        blk = x32[b * 16:(b + 1) * 16]
        sb = float(oracle.e4m3_round(np.float32(np.abs(blk).max()) / (np.float32(6) * g32)))
        sbs[b] = sb
        if sb > 0:
            el[b * 16:(b + 1) * 16] = oracle.e2m1_round(blk / (np.float32(sb) * g32))
    return el, sbs, float(g32)


def test_lowprec_row_checkers_accept_float32_rounding_and_reject_planted_errors():
    """The code-level checkers of the GPU's FP8 / NVFP4 key rows
    (recsa_testlib.nvfp4_row_flips, fp8_row_flips) accept a float32 computation
    of the oracle's rounding -- including rows built to sit on rounding
    midpoints -- and reject a wrong element, a wrong block scale and a wrong
    row scale."""
    from recsa_testlib import fp8_row_flips, nvfp4_row_flips
    rng = np.random.default_rng(50)
    flips = 0
    for trial in range(300):
        x = rng.standard_normal(64) * 10.0 ** rng.uniform(-2, 2)
        if trial % 3 == 0:      # put some elements exactly on E2M1 midpoints of their block
            g = np.abs(x).max() / 2688
            for b in range(4):
                sb = float(oracle.e4m3_round(np.abs(x[b * 16:(b + 1) * 16]).max() / (6 * g)))
                x[b * 16 + 3] = 1.25 * sb * g
                x[b * 16 + 5] = -2.5 * sb * g
        el, sb, g32 = _f32_nvfp4(x, rng)
        fe, fb = nvfp4_row_flips(x, el, sb, g32)
        flips += fe + fb
        q, s = oracle.quantize_row(x)
        x32 = (x + rng.standard_normal(64) * 1e-7 * np.abs(x).max()).astype(np.float32)
        s32 = float(np.float32(np.abs(x32).max()) / np.float32(448))
        fp8_row_flips(x, oracle.e4m3_round(x32 / np.float32(s32)), s32)
    assert flips > 0        # the midpoint rows did exercise the one-step allowance
    x = rng.standard_normal(64)
    el, sb, g32 = _f32_nvfp4(x, rng)
    nvfp4_row_flips(x, el, sb, g32)
    bad = el.copy()
    i = int(np.argmin(np.abs(np.abs(bad) - 1.0)))      # an element far from any midpoint
    bad[i] = bad[i] + (2.0 if bad[i] < 4 else -2.0)
    with pytest.raises(AssertionError):
        nvfp4_row_flips(x, bad, sb, g32)
    wrong_sb = sb.copy()
    wrong_sb[1] = float(oracle.e4m3_round(np.array([sb[1] * 1.3]))[0])
    with pytest.raises(AssertionError):
        nvfp4_row_flips(x, el, wrong_sb, g32)
    with pytest.raises(AssertionError):
        nvfp4_row_flips(x, el, sb, g32 * 1.01)
    q, s = oracle.quantize_row(x)
    q_bad = q.copy()
    q_bad[7] = q_bad[7] * 1.5 if q_bad[7] != 0 else 1.0
    with pytest.raises(AssertionError):
        fp8_row_flips(x, q_bad, s)
