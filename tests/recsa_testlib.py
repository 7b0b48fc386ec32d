"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare with the oracle on the same seeded inputs.

Tolerances:
  * bf16 inputs: max-abs 2e-2 and mean-abs 2e-3 on outputs and tree summaries
    against the float64 oracle fed the same bf16 values (the target bound);
    the outputs are written in bf16, so the max-abs bound applies beyond that
    final rounding (half a bf16 ulp of the value, 1/32 at magnitude 8);
  * fp32 inputs: max-abs 2e-4, mean-abs 2e-5 (fp32 dot products of length
    <= 128 and sums over <= ~2000 softmax entries: a few 1e-6 relative, with
    two orders of margin);
  * selection: kept node ids bit-exact for every (query, head) whose oracle
    scores have a gap above 1e-3 between the k-th and (k+1)-th candidate at
    every level; other queries are recomputed by the oracle with the GPU's
    selection (several selections are correct there) and compared on outputs.
"""

from __future__ import annotations

import math
from typing import Dict, List

import numpy as np
import torch

import oracle
from hierarchical_sparse_attention_recsa_b200 import recsa as R

GAP = 1e-3
TOL = {torch.bfloat16: (2e-2, 2e-3), torch.float32: (2e-4, 2e-5)}


def geometry(w, capacity: int, batch: int, k=None, rope=1, top_p=None) -> R.Geometry:
    """Library geometry of a workload; top_p given: the ZHA routing variant."""
    return R.Geometry(head_dim=w.head_dim, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                      leaf_block=w.leaf_block, branching=w.branching,
                      k=w.k if k is None else k, window=w.window, batch=batch,
                      capacity=capacity,
                      dtype=R.DTYPE_BF16 if w.dtype == torch.bfloat16 else R.DTYPE_F32,
                      rope_enabled=rope, rope_base=w.rope_base,
                      mode=R.MODE_RECSA if top_p is None else R.MODE_ZHA,
                      top_p=0.0 if top_p is None else top_p)


def oracle_geometry(g: R.Geometry) -> oracle.Geometry:
    return oracle.Geometry(g.head_dim, g.n_q_heads, g.n_kv_heads, g.leaf_block, g.branching,
                           g.k, g.window, rope=bool(g.rope_enabled), rope_base=g.rope_base)


def alloc_tree(g: R.Geometry) -> torch.Tensor:
    n = R.recsa_tree_bytes(g)
    return torch.zeros(n, dtype=torch.uint8, device="cuda")


def read_tree_level(g: R.Geometry, tree: torch.Tensor, lev: int):
    """(keys, vals) fp32 views of one level of the tree buffer: keys [batch, Hkv,
    n_l, d] ([batch, Hkv, n_l, n_ref, d] with n_ref > 1), vals [batch, Hkv, n_l, d]."""
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    kk = min(g.k, g.capacity)
    rows = min(max(g.branching * kk + g.branching, g.leaf_block * kk + g.window + g.leaf_block),
               g.capacity + g.branching + 1)
    if g.mode == R.MODE_ZHA:
        rows = max(rows, g.capacity + 1)
    off = up(256 + rows * (g.head_dim // 2) * 8)
    span = g.leaf_block
    nr = max(g.n_ref, 1)
    for l in range(1, lev + 1):
        n = g.capacity // span
        nbytes = g.batch * g.n_kv_heads * n * g.head_dim * 4
        kbytes = nbytes * nr
        if l == lev:
            shape = (g.batch, g.n_kv_heads, n, g.head_dim)
            kshape = shape if nr == 1 else (g.batch, g.n_kv_heads, n, nr, g.head_dim)
            keys = tree[off:off + kbytes].view(torch.float32).view(kshape)
            vals = tree[up(off + kbytes):up(off + kbytes) + nbytes].view(torch.float32).view(shape)
            return keys, vals
        off = up(up(off + kbytes) + nbytes)
        span *= g.branching
    raise ValueError(lev)


def parse_trace(rec: np.ndarray, k: int) -> dict:
    top = int(rec[0])
    out = dict(top=top, entries=int(rec[1]), keys_read=int(rec[2]), n_exact=int(rec[3]),
               cand={}, kept={})
    for lev in range(1, top + 1):
        c = int(rec[4 + lev - 1])
        kap = int(rec[4 + 16 + lev - 1])
        out["cand"][lev] = c
        base = 4 + 32 + (lev - 1) * k
        out["kept"][lev] = [int(x) for x in rec[base:base + kap]]
    return out


def gaps_clear(res: dict, k: int, gap: float = GAP) -> bool:
    for lev, sc in res["scores"].items():
        if len(sc) > k:
            s = sorted(sc, reverse=True)
            if s[k - 1] - s[k] <= gap:
                return False
    return True


def half_ulp_bf16(x) -> np.ndarray:
    """Half a bf16 unit in the last place at |x| (8 significant bits): the
    rounding error of writing x as bf16."""
    a = np.abs(np.asarray(x, np.float64))
    _, e = np.frexp(np.maximum(a, 2.0 ** -126))
    return np.ldexp(1.0, e - 1 - 8)


class Stats:
    """Error statistics of GPU values against oracle values.  For bf16 runs the
    GPU writes its outputs as bf16, so the max-abs bound applies to the error
    beyond that final rounding (half a bf16 ulp of the oracle value): outputs
    of magnitude 8 or more cannot be written closer than 1/32 in bf16."""

    def __init__(self):
        self.max_abs = 0.0
        self.max_excess = 0.0
        self.sum_abs = 0.0
        self.n = 0
        self.clear = 0
        self.near_tie = 0

    def add(self, a, b):
        b = np.asarray(b, np.float64)
        e = np.abs(np.asarray(a, np.float64) - b)
        self.max_abs = max(self.max_abs, float(e.max()))
        self.max_excess = max(self.max_excess, float(np.max(e - half_ulp_bf16(b))))
        self.sum_abs += float(e.sum())
        self.n += e.size

    @property
    def mean_abs(self):
        return self.sum_abs / max(self.n, 1)

    def check(self, dtype, what=""):
        mx, mn = TOL[dtype]
        worst = self.max_excess if dtype == torch.bfloat16 else self.max_abs
        print(f"{what}: max-abs {self.max_abs:.3e} (beyond bf16 output rounding "
              f"{self.max_excess:.3e}) mean-abs {self.mean_abs:.3e} "
              f"clear {self.clear} near-tie {self.near_tie}")
        assert worst <= mx, f"{what}: max-abs {worst:.3e} > {mx}"
        assert self.mean_abs <= mn, f"{what}: mean-abs {self.mean_abs:.3e} > {mn}"


def check_query(stats: Stats, gpu_out, trace_rec, q, t, K, V, tree_src, og, k_trace):
    """Compare one (query, head) of the GPU path with the oracle."""
    res = oracle.traverse_and_attend(q, t, K, V, tree_src, og)
    if trace_rec is not None:
        tr = parse_trace(trace_rec, k_trace)
        cf = oracle.closed_form_counts(t, og)
        assert tr["top"] == res["top"]
        assert tr["cand"] == res["cand"] == cf["cand"]
        assert tr["entries"] == res["entries"] == cf["entries"]
        assert tr["keys_read"] == res["keys_read"] == cf["keys_read"]
        assert tr["n_exact"] == res["n_exact"]
        if gaps_clear(res, og.k):
            stats.clear += 1
            assert tr["kept"] == {l: list(v) for l, v in res["kept"].items()}, (t, tr["kept"],
                                                                               res["kept"])
        else:
            stats.near_tie += 1
            if tr["kept"] != {l: list(v) for l, v in res["kept"].items()}:
                res = oracle.traverse_and_attend(q, t, K, V, tree_src, og,
                                                 keep_override=tr["kept"])
    stats.add(gpu_out, res["out"])
    return res


def to_np(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy().astype(np.float64)


# ---------------------------------------------------------------------------
# ZHA routing variant
# ---------------------------------------------------------------------------

MASS_EPS = 1e-3   # fp32 softmax masses vs float64: a few 1e-6; two orders of margin


def zha_level_clear(scores, mass, n: int, p: float, cap: int, gap: float = GAP) -> bool:
    """The top-p decision at one level cannot flip under fp32 rounding: the
    score gap at the cut exceeds ``gap`` and the masses before and at the cut
    are more than MASS_EPS from p (or the cap decides)."""
    s = sorted(scores, reverse=True)
    if n < len(s) and s[n - 1] - s[n] <= gap:
        return False
    if p >= 1.0:
        return True
    if n > 1 and mass[n - 2] >= p - MASS_EPS:
        return False
    if n < cap and mass[n - 1] < p + MASS_EPS:
        return False
    return True


def zha_routing_valid(res: dict, p: float, k: int, gap: float = GAP) -> None:
    """Assert that the routing in ``res`` (an oracle result, possibly for a
    given routing) is a correct top-p choice within rounding at every level:
    the expanded set is a score prefix (up to ties within ``gap``) and its size
    is where the mass crosses p (within MASS_EPS) or the cap."""
    for lev, kept in res["kept"].items():
        ids = res["cand_ids"][lev]
        sc = res["scores"][lev]
        mass = res["mass"][lev]
        n, c = len(kept), len(ids)
        cap = min(k, c)
        assert 1 <= n <= cap, (lev, n, cap)
        inside = [sc[i] for i, x in enumerate(ids) if x in set(kept)]
        outside = [sc[i] for i, x in enumerate(ids) if x not in set(kept)]
        if outside:
            assert min(inside) >= max(outside) - gap, (lev, min(inside), max(outside))
        if p >= 1.0:
            assert n == cap, (lev, n, cap)
            continue
        if n > 1:
            assert mass[n - 2] < p + MASS_EPS, (lev, n, mass[n - 2], p)
        if n < cap:
            assert mass[n - 1] >= p - MASS_EPS, (lev, n, mass[n - 1], p)


def check_query_zha(stats: Stats, gpu_out, trace_rec, q, t, K, V, tree_src, og, p: float,
                    k_trace):
    """Compare one (query, head) of the GPU's ZHA path with the oracle."""
    res = oracle.zha_route_and_attend(q, t, K, V, tree_src, og, p)
    if trace_rec is not None:
        tr = parse_trace(trace_rec, k_trace)
        assert tr["top"] == res["top"]
        gpu_kept = {l: list(v) for l, v in tr["kept"].items()}
        clear = all(zha_level_clear(res["scores"][l], res["mass"][l], len(res["kept"][l]), p,
                                    min(og.k, res["cand"][l]))
                    for l in res["kept"])
        if clear:
            stats.clear += 1
            assert gpu_kept == {l: list(v) for l, v in res["kept"].items()}, (t, gpu_kept,
                                                                              res["kept"])
        else:
            stats.near_tie += 1
            if gpu_kept != {l: list(v) for l, v in res["kept"].items()}:
                res = oracle.zha_route_and_attend(q, t, K, V, tree_src, og, p,
                                                  keep_override=gpu_kept)
                zha_routing_valid(res, p, og.k)
        assert tr["cand"] == res["cand"]
        assert tr["n_exact"] == res["n_exact"]
        assert tr["entries"] == res["n_exact"]
        assert tr["keys_read"] == res["n_exact"] + sum(res["cand"].values())
    stats.add(gpu_out, res["out"])
    return res


# ---------------------------------------------------------------------------
# Per-KV-group shared selection
# ---------------------------------------------------------------------------

GROUP_GAP = 2e-4   # group scores are sums of G probabilities; fp32 error ~1e-5 at most


def check_group(stats: Stats, gpu_out, trace_recs, Qg, t, K, V, tree_src, og, k_trace):
    """Compare the G heads of one KV group (GPU outputs [G, d], trace records
    [G, ints]) with the group-selection oracle."""
    res = oracle.group_traverse_and_attend(Qg, t, K, V, tree_src, og)
    if trace_recs is not None:
        trs = [parse_trace(rec, k_trace) for rec in trace_recs]
        kept = {l: list(v) for l, v in trs[0]["kept"].items()}
        cf = oracle.closed_form_counts(t, og)
        for tr in trs:
            assert {l: list(v) for l, v in tr["kept"].items()} == kept   # one selection
            assert tr["top"] == res["top"]
            assert tr["cand"] == res["cand"] == cf["cand"]
            assert tr["entries"] == cf["entries"] and tr["keys_read"] == cf["keys_read"]
        want = {l: list(v) for l, v in res["kept"].items()}
        clear = True
        for lev, sc in res["group"].items():
            n = min(og.k, len(sc))
            s = sorted(sc, reverse=True)
            if n < len(s) and s[n - 1] - s[n] <= GROUP_GAP:
                clear = False
        if clear:
            stats.clear += 1
            assert kept == want, (t, kept, want)
        else:
            stats.near_tie += 1
            if kept != want:
                # the first level that differs has the same candidates: the
                # GPU's set must be a top-k there within the gap
                lev = max(l for l in want if kept[l] != want[l])
                sc, ids = res["group"][lev], res["cand_ids"][lev]
                inside = [sc[ids.index(x)] for x in kept[lev]]
                outside = [sc[i] for i, x in enumerate(ids) if x not in set(kept[lev])]
                if outside:
                    assert min(inside) >= max(outside) - GROUP_GAP, (t, lev)
                res = oracle.group_traverse_and_attend(Qg, t, K, V, tree_src, og,
                                                       keep_override=kept)
    for h in range(len(gpu_out)):
        stats.add(gpu_out[h], res["out"][h])
    return res


def read_tree_level_fp8(g: R.Geometry, tree: torch.Tensor, lev: int):
    """(codes uint8 [batch, Hkv, n_l, n_ref, d], scales fp32 [batch, Hkv, n_l,
    n_ref], vals fp32 [batch, Hkv, n_l, d]) of one level of an FP8-key tree."""
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    kk = min(g.k, g.capacity)
    rows = min(max(g.branching * kk + g.branching, g.leaf_block * kk + g.window + g.leaf_block),
               g.capacity + g.branching + 1)
    if g.mode == R.MODE_ZHA:
        rows = max(rows, g.capacity + 1)
    off = up(256 + rows * (g.head_dim // 2) * 8)
    span = g.leaf_block
    nr = max(g.n_ref, 1)
    for l in range(1, lev + 1):
        n = g.capacity // span
        nrows = g.batch * g.n_kv_heads * n
        code_off, scale_off = off, up(off + nrows * nr * g.head_dim)
        val_off = up(scale_off + nrows * nr * 4)
        if l == lev:
            codes = tree[code_off:code_off + nrows * nr * g.head_dim].view(
                g.batch, g.n_kv_heads, n, nr, g.head_dim)
            scales = tree[scale_off:scale_off + nrows * nr * 4].view(torch.float32).view(
                g.batch, g.n_kv_heads, n, nr)
            vals = tree[val_off:val_off + nrows * g.head_dim * 4].view(torch.float32).view(
                g.batch, g.n_kv_heads, n, g.head_dim)
            return codes, scales, vals
        off = up(val_off + nrows * g.head_dim * 4)
        span *= g.branching
    raise ValueError(lev)


E4M3_TABLE = np.array([oracle.e4m3_decode(c) for c in range(256)])


def read_tree_level_nvfp4(g: R.Geometry, tree: torch.Tensor, lev: int):
    """(codes uint8 [batch, Hkv, n_l, n_ref, d/2], block scales uint8 [..., d/16],
    row scales fp32 [batch, Hkv, n_l, n_ref], vals fp32 [batch, Hkv, n_l, d])
    of one level of an NVFP4-key tree."""
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    kk = min(g.k, g.capacity)
    rows = min(max(g.branching * kk + g.branching, g.leaf_block * kk + g.window + g.leaf_block),
               g.capacity + g.branching + 1)
    if g.mode == R.MODE_ZHA:
        rows = max(rows, g.capacity + 1)
    off = up(256 + rows * (g.head_dim // 2) * 8)
    span = g.leaf_block
    nr = max(g.n_ref, 1)
    d = g.head_dim
    for l in range(1, lev + 1):
        n = g.capacity // span
        nrows = g.batch * g.n_kv_heads * n
        c_off = off
        b_off = up(c_off + nrows * nr * d // 2)
        s_off = up(b_off + nrows * nr * d // 16)
        v_off = up(s_off + nrows * nr * 4)
        if l == lev:
            shp = (g.batch, g.n_kv_heads, n, nr)
            codes = tree[c_off:c_off + nrows * nr * d // 2].view(*shp, d // 2)
            bsc = tree[b_off:b_off + nrows * nr * d // 16].view(*shp, d // 16)
            rsc = tree[s_off:s_off + nrows * nr * 4].view(torch.float32).view(*shp)
            vals = tree[v_off:v_off + nrows * d * 4].view(torch.float32).view(
                g.batch, g.n_kv_heads, n, d)
            return codes, bsc, rsc, vals
        off = up(v_off + nrows * d * 4)
        span *= g.branching
    raise ValueError(lev)


E2M1_TABLE = np.array([oracle.e2m1_decode(c) for c in range(16)])


def decode_nvfp4(codes: np.ndarray, bsc: np.ndarray, rsc: np.ndarray) -> np.ndarray:
    """Stored key values [..., d] from NVFP4 codes [..., d/2], block scales
    [..., d/16] and row scales [...] (numpy)."""
    c = codes.astype(np.int64)
    el = np.stack([E2M1_TABLE[c & 0xF], E2M1_TABLE[c >> 4]], axis=-1).reshape(*c.shape[:-1], -1)
    bs = np.repeat(E4M3_TABLE[bsc.astype(np.int64)], 16, axis=-1)
    return el * bs * rsc[..., None]


# ---------------------------------------------------------------------------
# Low-precision key rows: code-level comparison with the oracle's rounding
# ---------------------------------------------------------------------------

POOL_TOL = 2e-5   # float32 pooling error of a key row, relative to the row's largest element


def _e4m3_quantum(v):
    v = np.abs(np.asarray(v, np.float64))
    _, e = np.frexp(np.maximum(v, 2.0 ** -9))
    return np.ldexp(1.0, np.maximum(e - 1, -6) - 3)


def _e2m1_step(v):
    a = np.abs(np.asarray(v, np.float64))
    return np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))


def nvfp4_row_flips(x, got_el, got_sb, got_g, tol=POOL_TOL):
    """Compare one NVFP4 key row of the GPU with the oracle's rounding of the
    float64 pooled row x [d] (ZHA, Figure 16 caption; readings F1b):
    got_el [d] are the GPU's E2M1 element values, got_sb [d/16] its block
    scales (E4M3 values), got_g its row scale.  The row scale must equal
    max|x| / (6 * 448) to float32 pooling error.  A block scale may differ from
    E4M3(block max / (6 * row scale)) only by one E4M3 step, and only where
    that quotient lies within pooling error of the midpoint between the two;
    an element, given the GPU's block and row scales, may differ from the
    E2M1 rounding of x / (block scale * row scale) only by one E2M1 step, and
    only where the float32 value of x can fall on the other side of that
    midpoint.  Returns (element flips, block-scale flips)."""
    x = np.asarray(x, np.float64)
    amax = float(np.abs(x).max())
    if amax == 0.0:
        assert not np.any(got_el) and got_g == 0.0
        return 0, 0
    g_or = amax / (6 * 448)
    assert abs(got_g - g_or) <= 2 * tol * g_or, (got_g, g_or)
    fe = fb = 0
    for bi in range(x.shape[0] // 16):
        xb = x[bi * 16:(bi + 1) * 16]
        el = np.asarray(got_el[bi * 16:(bi + 1) * 16], np.float64)
        ratio = float(np.abs(xb).max()) / (6 * g_or)
        sb_or = float(oracle.e4m3_round(np.array([ratio]))[0])
        sb = float(got_sb[bi])
        if sb != sb_or:
            fb += 1
            lo = min(sb, sb_or)
            assert abs(sb - sb_or) == _e4m3_quantum(lo), (bi, sb, sb_or)
            # ratio = 448 * blockmax / amax: both from the float32 pooled row
            assert abs(ratio - (sb + sb_or) / 2) <= 448 * 2 * tol, (bi, ratio, sb, sb_or)
        if sb == 0.0:
            assert not np.any(el)
            continue
        unit = sb * float(got_g)
        u = xb / unit
        want = oracle.e2m1_round(u)
        bad = el != want
        if bad.any():
            fe += int(bad.sum())
            lo = np.minimum(np.abs(el[bad]), np.abs(want[bad]))
            assert np.all(np.abs(el[bad] - want[bad]) == _e2m1_step(lo)), (bi, el[bad], want[bad])
            mid = (el[bad] + want[bad]) / 2
            assert np.all(np.abs(u[bad] - mid) * unit <= tol * amax), (bi, u[bad], mid)
    return fe, fb


def fp8_row_flips(x, got_codes_val, got_scale, tol=POOL_TOL):
    """Compare one FP8 key row of the GPU (E4M3 values of the codes, row scale)
    with the oracle's rounding of the float64 pooled row x (readings F2): the
    scale equals max|x| / 448 to float32 pooling error; a code may differ from
    E4M3(x / scale) only by one E4M3 step, only where x / scale lies within
    pooling error (relative to the row's largest element, 448 in scaled units)
    of the midpoint.  Returns the number of differing codes."""
    x = np.asarray(x, np.float64)
    amax = float(np.abs(x).max())
    if amax == 0.0:
        assert not np.any(got_codes_val) and got_scale == 0.0
        return 0
    assert abs(got_scale - amax / 448) <= 2 * tol * amax / 448, (got_scale, amax / 448)
    u = x / float(got_scale)
    want = oracle.e4m3_round(u)
    got = np.asarray(got_codes_val, np.float64)
    bad = got != want
    if bad.any():
        lo = np.minimum(np.abs(got[bad]), np.abs(want[bad]))
        assert np.all(np.abs(got[bad] - want[bad]) == _e4m3_quantum(lo)), (got[bad], want[bad])
        assert np.all(np.abs(u[bad] - (got[bad] + want[bad]) / 2) <= 448 * tol), u[bad]
    return int(bad.sum())
