"""Parity of the ZHA routing variant (geometry mode RECSA_MODE_ZHA) with the
float64 oracle, through the C ABI.

"Subquadratic Attention with a Hierarchical Tree-Structured Indexer" (ZHA),
Figure 3 caption: top-p expansion down the tree over dot-product scores, main
attention over the tokens of the reached leaves (plus the exact window, at
true positions).  The routing check is bit-exact where no level's decision is
within rounding of its threshold or of a score tie, and a validity check plus
an output comparison under the GPU's routing elsewhere (recsa_testlib).
"""

import os

import numpy as np
import pytest
import torch

import oracle
from hierarchical_sparse_attention_recsa_b200 import build_lib, synth
from hierarchical_sparse_attention_recsa_b200 import recsa as R

from recsa_testlib import (E2M1_TABLE, E4M3_TABLE, Stats, alloc_tree, check_query_zha,
                           fp8_row_flips, geometry, nvfp4_row_flips,
                           oracle_geometry, parse_trace, read_tree_level, read_tree_level_fp8,
                           read_tree_level_nvfp4, to_np)

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny-4k"]
MODEL = synth.WORKLOADS["qwen3-4b-131k"]
ZK = 16   # tiny tree: a cap above the typical top-p set, so the mass decides


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_lib.build()
    R.lib()


@pytest.fixture(params=["kernel", "generic"])
def zha_impl(request):
    """The dedicated ZHA kernel (one CTA per query head) or the generic
    one-CTA-per-KV-head kernel."""
    old = os.environ.pop("RECSA_ZHA_GENERIC", None)
    if request.param == "generic":
        os.environ["RECSA_ZHA_GENERIC"] = "1"
    R.recsa_reload_switches()
    yield request.param
    os.environ.pop("RECSA_ZHA_GENERIC", None)
    if old is not None:
        os.environ["RECSA_ZHA_GENERIC"] = old
    R.recsa_reload_switches()


def _setup(w, lens, capacity, top_p, seed=0, k=None, rope=1):
    batch = len(lens)
    g = geometry(w, capacity, batch, k=k, rope=rope, top_p=top_p)
    K, V, r = synth.make_kv(w, capacity, seed=seed, device="cpu", batch=batch)
    Kd, Vd, rd = K.cuda(), V.cuda(), r.cuda()
    tree = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, lens, rd, 0, tree)
    torch.cuda.synchronize()
    return g, K, V, r, Kd, Vd, rd, tree


def _trees(g, K, V, r, lens):
    out = {}
    for s, L in enumerate(lens):
        for h in range(g.n_kv_heads):
            Kh, Vh = to_np(K[s, h, :L]), to_np(V[s, h, :L])
            out[(s, h)] = (Kh, Vh, oracle.FullTree(
                oracle.build_tree(Kh, Vh, r.double().numpy(), g.leaf_block, g.branching)))
    return out


@pytest.mark.parametrize("top_p", [0.3, 0.9])
def test_zha_decode_tiny(top_p, zha_impl):
    L, nq = TINY.length, TINY.n_q
    g, K, V, r, Kd, Vd, rd, tree = _setup(TINY, [L], L, top_p, seed=20, k=ZK)
    trees = _trees(g, K, V, r, [L])
    pos = torch.full((1, nq), L - 1, dtype=torch.int64)
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=21, n_needles=16)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((1, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens = torch.tensor([L], dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, src = trees[(0, 0)]
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    sizes = []
    for i in range(nq):
        for h in range(g.n_q_heads):
            res = check_query_zha(st, O_[0, i, h], tr[0, i, h], to_np(Q[0, i, h]), L - 1, Kh,
                                  Vh, src, og, top_p, g.k)
            sizes += [len(v) for v in res["kept"].values()]
    st.check(torch.float32, f"zha {zha_impl} decode tiny p={top_p}")
    assert st.clear > 0.7 * nq * g.n_q_heads
    # the mass target, not the cap, ends some levels
    assert min(sizes) < g.k


@pytest.mark.parametrize("entry", ["prefill", "prefill-workspace", "prefill-static"])
def test_zha_prefill_tiny(entry, zha_impl):
    L, top_p = TINY.length, 0.8
    g, K, V, r, Kd, Vd, rd, tree = _setup(TINY, [L], L, top_p, seed=22, k=ZK)
    trees = _trees(g, K, V, r, [L])
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=23)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((1, L, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    if entry == "prefill-static":
        R.recsa_prefill_static(g, Qd, Kd, Vd, tree, 0, L, O, trace)
    else:
        ws = None
        if entry == "prefill-workspace":
            ws = torch.empty(R.recsa_prefill_workspace_bytes(g, L), dtype=torch.uint8,
                             device="cuda")
        R.recsa_prefill(g, Qd, Kd, Vd, tree, 0, L, O, trace, workspace=ws)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, src = trees[(0, 0)]
    rng = np.random.default_rng(3)
    B, W = g.leaf_block, g.window
    sample = sorted(set([0, 1, B - 1, B, W - 1, W, W + 1, W + B - 1, W + B, 2 * W + 7, L - 2,
                         L - 1] + list(rng.integers(0, L, 40))))
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for t in sample:
        for h in range(g.n_q_heads):
            check_query_zha(st, O_[0, t, h], tr[0, t, h], to_np(Q[0, t, h]), t, Kh, Vh, src, og,
                            top_p, g.k)
    st.check(torch.float32, f"zha {zha_impl} {entry} tiny")


@pytest.mark.parametrize("top_p", [0.5, 0.95])
def test_zha_decode_model_small(top_p, zha_impl):
    lens = [20000, 13001]
    g, K, V, r, Kd, Vd, rd, tree = _setup(MODEL, lens, 20480, top_p, seed=24)
    trees = _trees(g, K, V, r, lens)
    nq = 3
    pos = torch.tensor([[L - 1] * nq for L in lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(MODEL, K, pos, seed=25, n_needles=2)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((2, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens_d, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    G = g.n_q_heads // g.n_kv_heads
    for s, L in enumerate(lens):
        for i in range(nq):
            for h in range(g.n_q_heads):
                Kh, Vh, src = trees[(s, h // G)]
                check_query_zha(st, O_[s, i, h], tr[s, i, h], to_np(Q[s, i, h]), L - 1, Kh, Vh,
                                src, og, top_p, g.k)
    st.check(torch.bfloat16, f"zha {zha_impl} decode model small p={top_p}")


@pytest.mark.parametrize("wname,rope", [("tiny-4k", 1), ("tiny-4k", 0), ("qwen3-4b-131k", 1)])
def test_zha_full_mass_keep_all_is_dense(wname, rope, zha_impl):
    """p = 1 with no cap reaches every leaf: dense causal attention."""
    w = synth.WORKLOADS[wname]
    L = 1500 if w.head_dim == 64 else 700
    g, K, V, r, Kd, Vd, rd, tree = _setup(w, [L], L, 1.0, seed=26, k=R.KEEP_ALL, rope=rope)
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(w, K, pos, seed=27)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    R.recsa_prefill(g, Qd, Kd, Vd, tree, 0, L, O)
    Od = torch.empty_like(Qd[:, :1])
    lens = torch.tensor([L], dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd[:, -1:].contiguous(), Kd, Vd, tree, lens, 1, Od)
    torch.cuda.synchronize()
    G = g.n_q_heads // g.n_kv_heads
    O_, Od_ = to_np(O), to_np(Od)
    st = Stats()
    for t in [0, 5, 63, 64, 65, 300, L - 1]:
        for h in range(0, g.n_q_heads, max(1, g.n_q_heads // 4)):
            ref = oracle.dense_causal_attention(to_np(Q[0, t, h]), t, to_np(K[0, h // G]),
                                                to_np(V[0, h // G]), rope=bool(rope),
                                                rope_base=w.rope_base)
            st.add(O_[0, t, h], ref)
            if t == L - 1:
                st.add(Od_[0, 0, h], ref)
    st.check(w.dtype, f"zha {zha_impl} full mass")


def test_zha_tiny_p_expands_one_node_per_level(zha_impl):
    """A mass target below every candidate's share expands only the arg-max."""
    L = TINY.length
    g, K, V, r, Kd, Vd, rd, tree = _setup(TINY, [L], L, 1e-6, seed=28)
    trees = _trees(g, K, V, r, [L])
    nq = 32
    pos = torch.full((1, nq), L - 1, dtype=torch.int64)
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=29)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((1, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens = torch.tensor([L], dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, src = trees[(0, 0)]
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for i in range(nq):
        for h in range(g.n_q_heads):
            t_ = parse_trace(tr[0, i, h], g.k)
            assert all(len(v) == 1 for v in t_["kept"].values())
            check_query_zha(st, O_[0, i, h], tr[0, i, h], to_np(Q[0, i, h]), L - 1, Kh, Vh, src,
                            og, 1e-6, g.k)
    st.check(torch.float32, f"zha {zha_impl} tiny p")


def test_zha_decode_step_equals_append_then_decode(zha_impl):
    """In ZHA mode the one-call step (append, then the routed decode) equals
    the two calls, across leaf completions, and matches the oracle."""
    w, top_p = MODEL, 0.9
    lens0 = [4000, 4031]
    steps = 70
    cap = 4096 + 256
    g, K, V, r, Kd, Vd, rd, tree_a = _setup(w, lens0, cap, top_p, seed=30)
    tree_b = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, lens0, rd, 0, tree_b)
    Ka, Va, Kb, Vb = Kd.clone(), Vd.clone(), Kd.clone(), Vd.clone()
    for X in (Ka, Va, Kb, Vb):
        X[0, :, 4000:] = 0
        X[1, :, 4031:] = 0
    la = torch.tensor(lens0, dtype=torch.int64, device="cuda")
    lb = la.clone()
    og = oracle_geometry(g)
    G = g.n_q_heads // g.n_kv_heads
    st = Stats()
    ti = R.recsa_trace_ints(g)
    for step in range(steps):
        kn = torch.stack([Kd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        vn = torch.stack([Vd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        lens_now = [L + step + 1 for L in lens0]
        pos = torch.tensor([[L - 1] for L in lens_now], dtype=torch.int64)
        Q, _, _ = synth.make_queries(w, K, pos, seed=200 + step)
        Qd = Q.cuda()
        Oa = torch.empty_like(Qd)
        Ob = torch.empty_like(Qd)
        trace = torch.zeros((2, 1, g.n_q_heads, ti), dtype=torch.int32, device="cuda")
        R.recsa_decode_step(g, Qd, Ka, Va, kn, vn, la, rd, 0, tree_a, 1, Oa, trace)
        R.recsa_append(g, Kb, Vb, kn, vn, lb, rd, 0, tree_b)
        R.recsa_decode(g, Qd, Kb, Vb, tree_b, lb, 1, Ob)
        torch.cuda.synchronize()
        assert torch.equal(Oa, Ob), step
        assert la.cpu().tolist() == lens_now
        if step in (31, steps - 1):
            tr = trace.cpu().numpy()
            for s in range(2):
                Kh_all = to_np(K[s, :, :lens_now[s]])
                Vh_all = to_np(V[s, :, :lens_now[s]])
                for h in range(0, g.n_q_heads, 7):
                    Kh, Vh = Kh_all[h // G], Vh_all[h // G]
                    src = oracle.LazyTree(Kh, Vh, r.double().numpy(), g.leaf_block, g.branching)
                    check_query_zha(st, to_np(Oa[s, 0, h]), tr[s, 0, h], to_np(Q[s, 0, h]),
                                    lens_now[s] - 1, Kh, Vh, src, og, top_p, g.k)
    st.check(torch.bfloat16, f"zha {zha_impl} decode step")
    assert torch.equal(Ka, Kb) and torch.equal(Va, Vb)
    assert torch.equal(tree_a[256:], tree_b[256:])


# ---------------------------------------------------------------------------
# Several reference queries per pooler (n_ref > 1)
# ---------------------------------------------------------------------------

def _refs(r, n_ref, seed):
    """n_ref reference queries: the workload's r, then n_ref - 1 more from the
    same distribution (N(0, 1/d)), seeded."""
    gen = torch.Generator().manual_seed(seed)
    d = r.shape[-1]
    extra = torch.randn((n_ref - 1, d), generator=gen, dtype=torch.float64) / d ** 0.5
    return torch.cat([r.double().reshape(1, d), extra]).float().contiguous()


def _setup_multi(w, lens, capacity, top_p, n_ref, seed, k=None, rope=1):
    batch = len(lens)
    g = geometry(w, capacity, batch, k=k, rope=rope, top_p=top_p)
    g.n_ref = n_ref
    K, V, r = synth.make_kv(w, capacity, seed=seed, device="cpu", batch=batch)
    Rq = _refs(r, n_ref, seed + 1000)
    Kd, Vd, Rd = K.cuda(), V.cuda(), Rq.cuda()
    tree = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, lens, Rd, 0, tree)
    torch.cuda.synchronize()
    return g, K, V, Rq, Kd, Vd, Rd, tree


def _multi_trees(g, K, V, Rq, lens):
    out = {}
    for s, L in enumerate(lens):
        for h in range(g.n_kv_heads):
            Kh, Vh = to_np(K[s, h, :L]), to_np(V[s, h, :L])
            out[(s, h)] = (Kh, Vh, oracle.MultiTree(oracle.build_tree_multi(
                Kh, Vh, Rq.double().numpy(), g.leaf_block, g.branching)))
    return out


def test_zha_multiref_tree_matches_oracle():
    L, Rn = TINY.length, 4
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_multi(TINY, [L], L, 0.7, Rn, seed=50)
    trees = _multi_trees(g, K, V, Rq, [L])
    _, _, src = trees[(0, 0)]
    st = Stats()
    for lev, (kk, vv) in enumerate(src.levels, start=1):
        gk, gv = read_tree_level(g, tree, lev)
        n = kk.shape[0]
        assert gk.shape[3] == Rn
        st.add(to_np(gk[0, 0, :n]), kk)
        st.add(to_np(gv[0, 0, :n]), vv)
    st.check(torch.float32, "zha multiref tree")


@pytest.mark.parametrize("Rn,top_p", [(4, 0.7), (16, 0.9)])
def test_zha_multiref_decode_tiny(Rn, top_p, zha_impl):
    L, nq = TINY.length, 64
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_multi(TINY, [L], L, top_p, Rn, seed=52, k=ZK)
    trees = _multi_trees(g, K, V, Rq, [L])
    pos = torch.full((1, nq), L - 1, dtype=torch.int64)
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=53, n_needles=8)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((1, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens = torch.tensor([L], dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, src = trees[(0, 0)]
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for i in range(nq):
        for h in range(g.n_q_heads):
            check_query_zha(st, O_[0, i, h], tr[0, i, h], to_np(Q[0, i, h]), L - 1, Kh, Vh, src,
                            og, top_p, g.k)
    st.check(torch.float32, f"zha {zha_impl} multiref R={Rn} decode tiny")
    assert st.clear > 0.6 * nq * g.n_q_heads


def test_zha_multiref_prefill_tiny(zha_impl):
    L, top_p, Rn = TINY.length, 0.8, 3
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_multi(TINY, [L], L, top_p, Rn, seed=54, k=ZK)
    trees = _multi_trees(g, K, V, Rq, [L])
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=55)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((1, L, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    R.recsa_prefill(g, Qd, Kd, Vd, tree, 0, L, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, src = trees[(0, 0)]
    rng = np.random.default_rng(7)
    sample = sorted(set([0, 15, 16, 64, 65, 200, L - 1] + list(rng.integers(0, L, 25))))
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for t in sample:
        for h in range(g.n_q_heads):
            check_query_zha(st, O_[0, t, h], tr[0, t, h], to_np(Q[0, t, h]), t, Kh, Vh, src, og,
                            top_p, g.k)
    st.check(torch.float32, f"zha {zha_impl} multiref prefill tiny")


def test_zha_multiref_decode_model_small(zha_impl):
    lens, top_p, Rn = [20000, 13001], 0.9, 3
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_multi(MODEL, lens, 20480, top_p, Rn, seed=56)
    trees = _multi_trees(g, K, V, Rq, lens)
    nq = 2
    pos = torch.tensor([[L - 1] * nq for L in lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(MODEL, K, pos, seed=57, n_needles=2)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((2, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens_d, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    G = g.n_q_heads // g.n_kv_heads
    for s, L in enumerate(lens):
        for i in range(nq):
            for h in range(g.n_q_heads):
                Kh, Vh, src = trees[(s, h // G)]
                check_query_zha(st, O_[s, i, h], tr[s, i, h], to_np(Q[s, i, h]), L - 1, Kh, Vh,
                                src, og, top_p, g.k)
    st.check(torch.bfloat16, f"zha {zha_impl} multiref decode model small")


def test_zha_multiref_append_matches_build(zha_impl):
    """Appending tokens one by one (leaf and level-2 completions) gives the
    tree a fresh build gives, for every reference query, and the decode after
    the last append matches the oracle."""
    w, top_p, Rn = MODEL, 0.9, 2
    lens0 = [4000, 4031]
    steps = 100
    cap = 4096 + 256
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_multi(w, lens0, cap, top_p, Rn, seed=58)
    Kw, Vw = Kd.clone(), Vd.clone()
    Kw[0, :, 4000:] = 0
    Vw[0, :, 4000:] = 0
    Kw[1, :, 4031:] = 0
    Vw[1, :, 4031:] = 0
    lens_d = torch.tensor(lens0, dtype=torch.int64, device="cuda")
    for step in range(steps):
        kn = torch.stack([Kd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        vn = torch.stack([Vd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        R.recsa_append(g, Kw, Vw, kn, vn, lens_d, Rd, 0, tree)
    new_lens = [L + steps for L in lens0]
    fresh = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, new_lens, Rd, 0, fresh)
    torch.cuda.synchronize()
    for lev in range(1, R.recsa_num_levels(g, max(new_lens)) + 1):
        a_k, a_v = read_tree_level(g, tree, lev)
        b_k, b_v = read_tree_level(g, fresh, lev)
        for s in range(2):
            n = new_lens[s] // (g.leaf_block * g.branching ** (lev - 1))
            torch.testing.assert_close(a_k[s, :, :n], b_k[s, :, :n], rtol=0, atol=1e-6)
            torch.testing.assert_close(a_v[s, :, :n], b_v[s, :, :n], rtol=0, atol=1e-6)
    pos = torch.tensor([[L - 1] for L in new_lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(w, K, pos, seed=59)
    O = torch.empty_like(Q).cuda()
    trace = torch.zeros((2, 1, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    R.recsa_decode(g, Q.cuda(), Kw, Vw, tree, lens_d, 1, O, trace)
    torch.cuda.synchronize()
    trees = _multi_trees(g, K, V, Rq, new_lens)
    og = oracle_geometry(g)
    G = g.n_q_heads // g.n_kv_heads
    tr = trace.cpu().numpy()
    st = Stats()
    for s in range(2):
        for h in range(0, g.n_q_heads, 5):
            Kh, Vh, src = trees[(s, h // G)]
            check_query_zha(st, to_np(O[s, 0, h]), tr[s, 0, h], to_np(Q[s, 0, h]),
                            new_lens[s] - 1, Kh, Vh, src, og, top_p, g.k)
    st.check(torch.bfloat16, f"zha {zha_impl} multiref after append")


@pytest.mark.parametrize("rope", [1, 0])
def test_zha_multiref_full_mass_is_dense(rope, zha_impl):
    w = TINY
    L = 1500
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_multi(w, [L], L, 1.0, 3, seed=60, k=R.KEEP_ALL,
                                                 rope=rope)
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(w, K, pos, seed=61)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    R.recsa_prefill(g, Qd, Kd, Vd, tree, 0, L, O)
    torch.cuda.synchronize()
    O_ = to_np(O)
    st = Stats()
    for t in [0, 63, 64, 700, L - 1]:
        for h in range(g.n_q_heads):
            ref = oracle.dense_causal_attention(to_np(Q[0, t, h]), t, to_np(K[0, 0]),
                                                to_np(V[0, 0]), rope=bool(rope),
                                                rope_base=w.rope_base)
            st.add(O_[0, t, h], ref)
    st.check(torch.float32, f"zha {zha_impl} multiref full mass")


# ---------------------------------------------------------------------------
# Low-precision router keys (FP8 E4M3 with one scale per key row)
# ---------------------------------------------------------------------------

def _setup_fp8(w, lens, capacity, top_p, n_ref, seed, k=None, rope=1, key_format=R.KEYS_FP8):
    batch = len(lens)
    g = geometry(w, capacity, batch, k=k, rope=rope, top_p=top_p)
    g.n_ref = n_ref
    g.key_format = key_format
    K, V, r = synth.make_kv(w, capacity, seed=seed, device="cpu", batch=batch)
    Rq = _refs(r, n_ref, seed + 1000) if n_ref > 1 else r.reshape(1, -1).contiguous()
    Kd, Vd, Rd = K.cuda(), V.cuda(), Rq.cuda()
    tree = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, lens, Rd, 0, tree)
    torch.cuda.synchronize()
    return g, K, V, Rq, Kd, Vd, Rd, tree


def _fp8_trees(g, K, V, Rq, lens):
    build = (oracle.build_tree_nvfp4_multi if g.key_format == R.KEYS_NVFP4
             else oracle.build_tree_fp8_multi)
    out = {}
    for s, L in enumerate(lens):
        for h in range(g.n_kv_heads):
            Kh, Vh = to_np(K[s, h, :L]), to_np(V[s, h, :L])
            levels = build(Kh, Vh, Rq.double().numpy(), g.leaf_block, g.branching)
            if Rq.shape[0] == 1:
                levels = [(kk[:, 0], vv) for kk, vv in levels]
                out[(s, h)] = (Kh, Vh, oracle.FullTree(levels))
            else:
                out[(s, h)] = (Kh, Vh, oracle.MultiTree(levels))
    return out


@pytest.mark.parametrize("n_ref", [1, 2])
def test_zha_fp8_tree_codes(n_ref):
    """Every stored code is the oracle's E4M3 rounding of key / scale, where the
    key is the float64 pooling of the node's children as the GPU stored them
    (tokens at level 1, the GPU's decoded child keys above): a code may differ
    only by one step, only where the float32 pooled value can fall on the other
    side of a rounding midpoint (recsa_testlib.fp8_row_flips)."""
    L = TINY.length
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(TINY, [L], L, 0.7, n_ref, seed=70)
    Kh, Vh = to_np(K[0, 0]), to_np(V[0, 0])
    Rn = Rq.double().numpy()
    levels = oracle.build_tree_fp8_multi(Kh, Vh, Rn, g.leaf_block, g.branching)
    prev = None
    for lev in range(1, len(levels) + 1):
        codes, scales, vals = read_tree_level_fp8(g, tree, lev)
        n = levels[lev - 1][0].shape[0]
        got = E4M3_TABLE[codes[0, 0, :n].cpu().numpy().astype(np.int64)]
        sc = scales[0, 0, :n].cpu().numpy().astype(np.float64)
        fan = g.leaf_block if lev == 1 else g.branching
        mism = 0
        for j in range(n):
            for ref in range(n_ref):
                src = Kh if lev == 1 else prev[:, ref]
                x = oracle.pool_keys(src[j * fan:(j + 1) * fan], Rn[ref])
                mism += fp8_row_flips(x, got[j, ref], sc[j, ref])
        assert mism <= max(2, 0.01 * n * n_ref * g.head_dim), (lev, mism)
        prev = got * sc[..., None]          # the GPU's stored keys feed the next level
        np.testing.assert_allclose(vals[0, 0, :n].cpu().numpy(), levels[lev - 1][1],
                                   atol=1e-5 if lev > 1 else 1e-6)


@pytest.mark.parametrize("n_ref,top_p", [(1, 0.7), (4, 0.9)])
def test_zha_fp8_decode_tiny(n_ref, top_p, zha_impl):
    L, nq = TINY.length, 64
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(TINY, [L], L, top_p, n_ref, seed=72, k=ZK)
    trees = _fp8_trees(g, K, V, Rq, [L])
    pos = torch.full((1, nq), L - 1, dtype=torch.int64)
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=73, n_needles=8)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((1, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens = torch.tensor([L], dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, src = trees[(0, 0)]
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for i in range(nq):
        for h in range(g.n_q_heads):
            check_query_zha(st, O_[0, i, h], tr[0, i, h], to_np(Q[0, i, h]), L - 1, Kh, Vh, src,
                            og, top_p, g.k)
    st.check(torch.float32, f"zha {zha_impl} fp8 R={n_ref} decode tiny")
    assert st.clear > 0.6 * nq * g.n_q_heads


def test_zha_fp8_prefill_tiny(zha_impl):
    L, top_p = TINY.length, 0.8
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(TINY, [L], L, top_p, 1, seed=74, k=ZK)
    trees = _fp8_trees(g, K, V, Rq, [L])
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=75)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((1, L, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    R.recsa_prefill(g, Qd, Kd, Vd, tree, 0, L, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, src = trees[(0, 0)]
    rng = np.random.default_rng(8)
    sample = sorted(set([0, 15, 16, 64, 65, 300, L - 1] + list(rng.integers(0, L, 25))))
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for t in sample:
        for h in range(g.n_q_heads):
            check_query_zha(st, O_[0, t, h], tr[0, t, h], to_np(Q[0, t, h]), t, Kh, Vh, src, og,
                            top_p, g.k)
    st.check(torch.float32, f"zha {zha_impl} fp8 prefill tiny")


def test_zha_fp8_decode_model_small(zha_impl):
    lens, top_p = [20000, 13001], 0.9
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(MODEL, lens, 20480, top_p, 1, seed=76)
    trees = _fp8_trees(g, K, V, Rq, lens)
    nq = 2
    pos = torch.tensor([[L - 1] * nq for L in lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(MODEL, K, pos, seed=77, n_needles=2)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((2, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens_d, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    G = g.n_q_heads // g.n_kv_heads
    for s, L in enumerate(lens):
        for i in range(nq):
            for h in range(g.n_q_heads):
                Kh, Vh, src = trees[(s, h // G)]
                check_query_zha(st, O_[s, i, h], tr[s, i, h], to_np(Q[s, i, h]), L - 1, Kh, Vh,
                                src, og, top_p, g.k)
    st.check(torch.bfloat16, f"zha {zha_impl} fp8 decode model small")


def test_zha_fp8_append_matches_build():
    w, top_p = MODEL, 0.9
    lens0 = [4000, 4031]
    steps = 100
    cap = 4096 + 256
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(w, lens0, cap, top_p, 2, seed=78)
    Kw, Vw = Kd.clone(), Vd.clone()
    Kw[0, :, 4000:] = 0
    Vw[0, :, 4000:] = 0
    Kw[1, :, 4031:] = 0
    Vw[1, :, 4031:] = 0
    lens_d = torch.tensor(lens0, dtype=torch.int64, device="cuda")
    for step in range(steps):
        kn = torch.stack([Kd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        vn = torch.stack([Vd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        R.recsa_append(g, Kw, Vw, kn, vn, lens_d, Rd, 0, tree)
    new_lens = [L + steps for L in lens0]
    fresh = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, new_lens, Rd, 0, fresh)
    torch.cuda.synchronize()
    for lev in range(1, R.recsa_num_levels(g, max(new_lens)) + 1):
        a_c, a_s, a_v = read_tree_level_fp8(g, tree, lev)
        b_c, b_s, b_v = read_tree_level_fp8(g, fresh, lev)
        for s in range(2):
            n = new_lens[s] // (g.leaf_block * g.branching ** (lev - 1))
            assert torch.equal(a_c[s, :, :n], b_c[s, :, :n]), lev
            torch.testing.assert_close(a_s[s, :, :n], b_s[s, :, :n], rtol=0, atol=0)
            torch.testing.assert_close(a_v[s, :, :n], b_v[s, :, :n], rtol=0, atol=1e-6)


def test_zha_fp8_full_mass_is_dense(zha_impl):
    w = TINY
    L = 1500
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(w, [L], L, 1.0, 1, seed=79, k=R.KEEP_ALL)
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(w, K, pos, seed=80)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    R.recsa_prefill(g, Qd, Kd, Vd, tree, 0, L, O)
    torch.cuda.synchronize()
    O_ = to_np(O)
    st = Stats()
    for t in [0, 63, 64, 700, L - 1]:
        for h in range(g.n_q_heads):
            ref = oracle.dense_causal_attention(to_np(Q[0, t, h]), t, to_np(K[0, 0]),
                                                to_np(V[0, 0]), rope=True, rope_base=w.rope_base)
            st.add(O_[0, t, h], ref)
    st.check(torch.float32, f"zha {zha_impl} fp8 full mass")


# ---------------------------------------------------------------------------
# NVFP4 router keys (E2M1 codes, E4M3 scale per 16, fp32 scale per row)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n_ref", [1, 3])
def test_zha_nvfp4_tree(n_ref):
    """Every stored NVFP4 row is the oracle's rounding (row scale, E4M3 block
    scales, E2M1 elements) of the float64 pooling of the node's children as
    the GPU stored them (tokens at level 1, the GPU's decoded child keys
    above).  A block scale or an element may differ only by one step of its
    format, only where the float32 pooled value can fall on the other side of
    that rounding midpoint (recsa_testlib.nvfp4_row_flips); block-scale flips
    and element flips are counted and bounded separately."""
    L = TINY.length
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(TINY, [L], L, 0.7, n_ref, seed=90,
                                               key_format=R.KEYS_NVFP4)
    Kh, Vh = to_np(K[0, 0]), to_np(V[0, 0])
    Rn = Rq.double().numpy()
    levels = oracle.build_tree_nvfp4_multi(Kh, Vh, Rn, g.leaf_block, g.branching)
    prev = None
    d = g.head_dim
    for lev in range(1, len(levels) + 1):
        codes, bsc, rsc, vals = read_tree_level_nvfp4(g, tree, lev)
        n = levels[lev - 1][0].shape[0]
        c = codes[0, 0, :n].cpu().numpy().astype(np.int64)
        el = np.stack([E2M1_TABLE[c & 0xF], E2M1_TABLE[c >> 4]], axis=-1).reshape(n, n_ref, d)
        sb = E4M3_TABLE[bsc[0, 0, :n].cpu().numpy().astype(np.int64)]
        rs = rsc[0, 0, :n].cpu().numpy().astype(np.float64)
        fan = g.leaf_block if lev == 1 else g.branching
        fe = fb = 0
        for j in range(n):
            for ref in range(n_ref):
                src = Kh if lev == 1 else prev[:, ref]
                x = oracle.pool_keys(src[j * fan:(j + 1) * fan], Rn[ref])
                e_, b_ = nvfp4_row_flips(x, el[j, ref], sb[j, ref], rs[j, ref])
                fe += e_
                fb += b_
        assert fe <= max(2, 0.01 * n * n_ref * d), (lev, fe)
        assert fb <= max(2, 0.01 * n * n_ref * d // 16), (lev, fb)
        prev = el * np.repeat(sb, 16, axis=-1) * rs[..., None]   # the GPU's stored keys
        np.testing.assert_allclose(vals[0, 0, :n].cpu().numpy(), levels[lev - 1][1],
                                   atol=1e-5 if lev > 1 else 1e-6)


@pytest.mark.parametrize("n_ref,top_p", [(1, 0.7), (4, 0.9)])
def test_zha_nvfp4_decode_tiny(n_ref, top_p, zha_impl):
    L, nq = TINY.length, 64
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(TINY, [L], L, top_p, n_ref, seed=92, k=ZK,
                                               key_format=R.KEYS_NVFP4)
    trees = _fp8_trees(g, K, V, Rq, [L])
    pos = torch.full((1, nq), L - 1, dtype=torch.int64)
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=93, n_needles=8)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((1, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens = torch.tensor([L], dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, src = trees[(0, 0)]
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for i in range(nq):
        for h in range(g.n_q_heads):
            check_query_zha(st, O_[0, i, h], tr[0, i, h], to_np(Q[0, i, h]), L - 1, Kh, Vh, src,
                            og, top_p, g.k)
    st.check(torch.float32, f"zha {zha_impl} nvfp4 R={n_ref} decode tiny")
    assert st.clear > 0.5 * nq * g.n_q_heads


def test_zha_nvfp4_decode_model_small(zha_impl):
    lens, top_p = [20000, 13001], 0.9
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(MODEL, lens, 20480, top_p, 1, seed=94,
                                               key_format=R.KEYS_NVFP4)
    trees = _fp8_trees(g, K, V, Rq, lens)
    nq = 2
    pos = torch.tensor([[L - 1] * nq for L in lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(MODEL, K, pos, seed=95, n_needles=2)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((2, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens_d, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    G = g.n_q_heads // g.n_kv_heads
    for s, L in enumerate(lens):
        for i in range(nq):
            for h in range(g.n_q_heads):
                Kh, Vh, src = trees[(s, h // G)]
                check_query_zha(st, O_[s, i, h], tr[s, i, h], to_np(Q[s, i, h]), L - 1, Kh, Vh,
                                src, og, top_p, g.k)
    st.check(torch.bfloat16, f"zha {zha_impl} nvfp4 decode model small")


def test_zha_nvfp4_append_matches_build():
    w, top_p = MODEL, 0.9
    lens0 = [4000, 4031]
    steps = 100
    cap = 4096 + 256
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(w, lens0, cap, top_p, 2, seed=96,
                                               key_format=R.KEYS_NVFP4)
    Kw, Vw = Kd.clone(), Vd.clone()
    Kw[0, :, 4000:] = 0
    Vw[0, :, 4000:] = 0
    Kw[1, :, 4031:] = 0
    Vw[1, :, 4031:] = 0
    lens_d = torch.tensor(lens0, dtype=torch.int64, device="cuda")
    for step in range(steps):
        kn = torch.stack([Kd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        vn = torch.stack([Vd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        R.recsa_append(g, Kw, Vw, kn, vn, lens_d, Rd, 0, tree)
    new_lens = [L + steps for L in lens0]
    fresh = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, new_lens, Rd, 0, fresh)
    torch.cuda.synchronize()
    for lev in range(1, R.recsa_num_levels(g, max(new_lens)) + 1):
        a = read_tree_level_nvfp4(g, tree, lev)
        b = read_tree_level_nvfp4(g, fresh, lev)
        for s in range(2):
            n = new_lens[s] // (g.leaf_block * g.branching ** (lev - 1))
            for x, y in zip(a, b):
                assert torch.equal(x[s, :, :n], y[s, :, :n]), lev


@pytest.mark.parametrize("workspace", [True, False])
def test_zha_prefill_model_small(workspace, zha_impl):
    """bf16 prefill: with a workspace the window comes from the tensor-core
    window kernel's partials and the ZHA kernel runs its small-CTA prefill
    shape; without, the ZHA kernel attends the window itself."""
    lens, top_p = [20000, 13001], 0.8
    g, K, V, r, Kd, Vd, rd, tree = _setup(MODEL, lens, 20480, top_p, seed=130)
    trees = _trees(g, K, V, r, lens)
    q0, nq = 12000, 1001
    pos = (q0 + torch.arange(nq, dtype=torch.int64))[None].expand(2, nq)
    Q, _, _ = synth.make_queries(MODEL, K, pos.contiguous(), seed=131)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((2, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    ws = (torch.empty(R.recsa_prefill_workspace_bytes(g, nq), dtype=torch.uint8, device="cuda")
          if workspace else None)
    R.recsa_prefill(g, Qd, Kd, Vd, tree, q0, nq, O, trace, workspace=ws)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    G = g.n_q_heads // g.n_kv_heads
    rng = np.random.default_rng(9)
    for s in range(2):
        for i in [0, 1, 63, 64, 500, nq - 1] + list(rng.integers(0, nq, 4)):
            for h in range(0, g.n_q_heads, 3):
                Kh, Vh, src = trees[(s, h // G)]
                check_query_zha(st, O_[s, i, h], tr[s, i, h], to_np(Q[s, i, h]), q0 + i, Kh, Vh,
                                src, og, top_p, g.k)
    st.check(torch.bfloat16, f"zha {zha_impl} prefill model small workspace={workspace}")


# ---------------------------------------------------------------------------
# Several reference queries pooled on the tensor cores (R >= 4, bf16, d = 128):
# one pass over each leaf's K and V (the scores [B x d] x [d x R] and the
# pooling [R x B] x [B x d] as tcgen05 products with split fp32 operands)
# ---------------------------------------------------------------------------

def _model_variant(B, b):
    return synth.Workload(**{**MODEL.__dict__, "leaf_block": B, "branching": b})


@pytest.mark.parametrize("Rn,B", [(16, 64), (20, 64), (16, 32), (16, 16)])
def test_zha_multiref_tc_tree_matches_oracle(Rn, B):
    """Every node of a model-shaped multi-reference tree (level 1 on the
    tensor-core pooler, higher levels pooling its keys) against the float64
    oracle, at the fp32 tolerance: two sequences of ragged lengths, so the
    last tile of a sequence holds fewer than 128 / B leaves."""
    w = _model_variant(B, 16 if B == 64 else 8)
    lens = [20000, 13001]
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_multi(w, lens, 20480, 0.9, Rn, seed=200 + Rn + B)
    st = Stats()
    for s, L in enumerate(lens):
        for h in (0, 5):
            Kh, Vh = to_np(K[s, h, :L]), to_np(V[s, h, :L])
            levels = oracle.build_tree_multi(Kh, Vh, Rq.double().numpy(), g.leaf_block,
                                             g.branching)
            for lev, (kk, vv) in enumerate(levels, start=1):
                gk, gv = read_tree_level(g, tree, lev)
                n = kk.shape[0]
                st.add(to_np(gk[s, h, :n]), kk)
                st.add(to_np(gv[s, h, :n]), vv)
    st.check(torch.float32, f"multiref tc tree R={Rn} B={B}")


@pytest.mark.parametrize("key_format", [R.KEYS_FP8, R.KEYS_NVFP4])
def test_zha_multiref_tc_lowprec_tree_codes(key_format):
    """Level-1 FP8 / NVFP4 key rows written from the tensor-core pooler are the
    oracle's rounding of the float64 pooled keys, up to one step at a rounding
    midpoint (recsa_testlib.fp8_row_flips / nvfp4_row_flips)."""
    L, Rn = 6000, 16
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_fp8(MODEL, [L], 6144, 0.9, Rn, seed=210,
                                               key_format=key_format)
    Rn_np = Rq.double().numpy()
    d = g.head_dim
    for h in (0, 3):
        Kh = to_np(K[0, h, :L])
        n = L // g.leaf_block
        flips = 0
        if key_format == R.KEYS_FP8:
            codes, scales, _ = read_tree_level_fp8(g, tree, 1)
            got = E4M3_TABLE[codes[0, h, :n].cpu().numpy().astype(np.int64)]
            sc = scales[0, h, :n].cpu().numpy().astype(np.float64)
        else:
            codes, bsc, rsc, _ = read_tree_level_nvfp4(g, tree, 1)
            c = codes[0, h, :n].cpu().numpy().astype(np.int64)
            el = np.stack([E2M1_TABLE[c & 0xF], E2M1_TABLE[c >> 4]], axis=-1).reshape(n, Rn, d)
            sb = E4M3_TABLE[bsc[0, h, :n].cpu().numpy().astype(np.int64)]
            rs = rsc[0, h, :n].cpu().numpy().astype(np.float64)
        for j in range(n):
            for ref in range(Rn):
                x = oracle.pool_keys(Kh[j * g.leaf_block:(j + 1) * g.leaf_block], Rn_np[ref])
                if key_format == R.KEYS_FP8:
                    flips += fp8_row_flips(x, got[j, ref], sc[j, ref])
                else:
                    fe, fb = nvfp4_row_flips(x, el[j, ref], sb[j, ref], rs[j, ref])
                    flips += fe + fb
        assert flips <= max(2, 0.01 * n * Rn * d), flips


def test_zha_multiref_tc_append_matches_build():
    """Appending tokens (level 1 pooled on CUDA cores) gives, to fp32 rounding,
    the nodes a fresh build pooled on the tensor cores (R = 16)."""
    w, top_p, Rn = MODEL, 0.9, 16
    lens0 = [4000, 4031]
    steps = 70
    cap = 4096 + 256
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_multi(w, lens0, cap, top_p, Rn, seed=220)
    Kw, Vw = Kd.clone(), Vd.clone()
    Kw[0, :, 4000:] = 0
    Vw[0, :, 4000:] = 0
    Kw[1, :, 4031:] = 0
    Vw[1, :, 4031:] = 0
    lens_d = torch.tensor(lens0, dtype=torch.int64, device="cuda")
    for step in range(steps):
        kn = torch.stack([Kd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        vn = torch.stack([Vd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        R.recsa_append(g, Kw, Vw, kn, vn, lens_d, Rd, 0, tree)
    new_lens = [L + steps for L in lens0]
    fresh = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, new_lens, Rd, 0, fresh)
    torch.cuda.synchronize()
    for lev in range(1, R.recsa_num_levels(g, max(new_lens)) + 1):
        a_k, a_v = read_tree_level(g, tree, lev)
        b_k, b_v = read_tree_level(g, fresh, lev)
        for s in range(2):
            n = new_lens[s] // (g.leaf_block * g.branching ** (lev - 1))
            torch.testing.assert_close(a_k[s, :, :n], b_k[s, :, :n], rtol=0, atol=2e-6)
            torch.testing.assert_close(a_v[s, :, :n], b_v[s, :, :n], rtol=0, atol=1e-6)


def test_zha_multiref_tc_decode_model(zha_impl):
    """Routing over a tensor-core-pooled tree (R = 16) on both ZHA kernels,
    checked against the oracle with the routing rule of check_query_zha."""
    lens, top_p, Rn = [20000, 13001], 0.9, 16
    g, K, V, Rq, Kd, Vd, Rd, tree = _setup_multi(MODEL, lens, 20480, top_p, Rn, seed=230)
    nq = 2
    pos = torch.tensor([[L - 1] * nq for L in lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(MODEL, K, pos, seed=231, n_needles=2)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((2, nq, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens_d, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    G = g.n_q_heads // g.n_kv_heads
    for s, L in enumerate(lens):
        for h in (0, 7, 21, 30):
            Kh, Vh = to_np(K[s, h // G, :L]), to_np(V[s, h // G, :L])
            src = oracle.LazyMultiTree(Kh, Vh, Rq.double().numpy(), g.leaf_block, g.branching)
            for i in range(nq):
                check_query_zha(st, O_[s, i, h], tr[s, i, h], to_np(Q[s, i, h]), L - 1, Kh, Vh,
                                src, og, top_p, g.k)
    st.check(torch.bfloat16, f"zha {zha_impl} multiref tc decode model")
