"""Work accounting for the benchmark: entries, key reads and algorithmic bytes.

Counting only (host side, numpy); the CUDA path computes the attention.

Per query at position t (geometry B, b, k, W): a = floor(max(0, t+1-W)/B) and
v_l = floor(a / b^(l-1)) nodes are visible at level l; the top visible level
offers its v nodes as candidates, every lower level the b children of each
kept node plus the v_l - b v_{l+1} orphans; min(k, c_l) are kept.  Softmax
entries = sum_l (c_l - kept_l) + B kept_1 + (t + 1 - aB) and keys read =
sum_l c_l + B kept_1 + (t + 1 - aB), which is what the query's dot products and
value accumulations touch ("Recursive Sparse Attention: Million-Token Length
Extrapolation at Logarithmic Cost", abstract: O(log L) entries read).
"""

from __future__ import annotations

import numpy as np

TRACE_HEAD = 4 + 2 * 16


def per_query_counts(t: np.ndarray, B: int, b: int, k: int, W: int, levels: int):
    """(entries, keys_read) int64 arrays for query positions t (vectorised)."""
    t = np.asarray(t, dtype=np.int64)
    a = np.maximum(t + 1 - W, 0) // B
    v = [a // (b ** l) for l in range(levels)]          # v[l-1] = visible at level l
    entries = np.zeros_like(t)
    keys = np.zeros_like(t)
    kappa_up = np.zeros_like(t)
    for lev in range(levels, 0, -1):
        v_l = v[lev - 1]
        v_up = v[lev] if lev < levels else np.zeros_like(t)
        c = np.where(v_l > 0, b * kappa_up + (v_l - b * v_up), 0)
        kap = np.minimum(c, k)
        entries += c - kap
        keys += c
        kappa_up = kap
    exact = B * kappa_up + (t + 1 - a * B)
    return entries + exact, keys + exact


def decode_bytes_from_trace(trace: np.ndarray, lens: np.ndarray, B: int, b: int, W: int,
                            G: int, d: int, elem: int, k: int,
                            summary_values: bool = True, keys_per_node: int = 1,
                            key_row_bytes: int = 0) -> dict:
    """Distinct bytes one decode launch must touch, from its selection trace.

    trace [batch, n_q, H_q, ints] (n_q = 1); lens [batch] after the append.
    Per (sequence, KV head): summary keys of the union over its G heads of the
    candidates scored (fp32 rows), summary values of the union of unselected
    candidates (fp32 rows; none when ``summary_values`` is False, as in the
    ZHA routing variant, whose softmax holds exact tokens only), K and V rows
    of the union of exact tokens (dtype); plus Q read and O written.  A node
    scored reads ``keys_per_node`` key rows (one per reference query) of
    ``key_row_bytes`` each (default fp32 rows: 4 d; FP8 rows: d + 4).
    """
    batch, n_q, hq, _ = trace.shape
    hkv = hq // G
    key_rows = val_rows = tok_rows = 0
    for s in range(batch):
        t = int(lens[s]) - 1
        if t < 0:
            continue
        a = max(t + 1 - W, 0) // B
        for qi in range(n_q):
            for g in range(hkv):
                recs = trace[s, qi, g * G:(g + 1) * G]
                top = int(recs[0, 0])
                kept = {}
                for lev in range(1, top + 1):
                    kap = recs[:, 4 + 16 + lev - 1]
                    base = TRACE_HEAD + (lev - 1) * k
                    kept[lev] = [set(recs[h, base:base + int(kap[h])].tolist())
                                 for h in range(G)]
                cand_u_total = unsel_total = 0
                for lev in range(top, 0, -1):
                    v_l = a // (b ** (lev - 1))
                    v_up = a // (b ** lev) if lev < top else 0
                    orph = set(range(b * v_up, v_l))
                    cu, uu = set(orph), set()
                    for h in range(G):
                        ch = set()
                        if lev < top:
                            for p in kept[lev + 1][h]:
                                ch.update(range(p * b, p * b + b))
                        cand = ch | orph
                        cu |= cand
                        uu |= cand - kept[lev][h]
                    cand_u_total += len(cu)
                    unsel_total += len(uu)
                leaves = set()
                if top > 0:
                    for h in range(G):
                        leaves |= kept[1][h]
                key_rows += cand_u_total
                val_rows += unsel_total if summary_values else 0
                tok_rows += len(leaves) * B + (t + 1 - a * B)
    qo = 2 * batch * n_q * hq * d * elem
    krb = key_row_bytes or d * 4
    tree_bytes = key_rows * keys_per_node * krb + val_rows * d * 4
    kv_bytes = tok_rows * d * elem * 2
    return dict(bytes=qo + tree_bytes + kv_bytes, qo=qo, tree=tree_bytes, kv=kv_bytes,
                key_rows=key_rows, val_rows=val_rows, tok_rows=tok_rows)
