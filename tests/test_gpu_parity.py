"""Parity of the CUDA path (through the C ABI) with the float64 CPU oracle.

Sizes span several tiles and ragged tails while the oracle still finishes in
seconds; tolerances and the selection rule are stated in recsa_testlib.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from hierarchical_sparse_attention_recsa_b200 import build_lib, synth
from hierarchical_sparse_attention_recsa_b200 import recsa as R

from recsa_testlib import (Stats, alloc_tree, check_query, geometry, oracle_geometry,
                           read_tree_level, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_lib.build()
    R.lib()


@pytest.fixture(params=["cluster-auto", "split-1,1", "split-1,2", "split-1,4", "split-2,1",
                        "split-4,1", "split-4,2", "generic"])
def decode_impl(request):
    """Select the decode kernel: the cluster kernel with its automatic launch
    shape or a forced one ("split-HPC,S": HPC query heads per CTA, S candidate
    shares per head group), or the generic one-CTA-per-query kernel."""
    keys = ("RECSA_DECODE_SPLIT", "RECSA_DECODE_GENERIC")
    old = {k: os.environ.get(k) for k in keys}
    for k in keys:
        os.environ.pop(k, None)
    if request.param == "generic":
        os.environ["RECSA_DECODE_GENERIC"] = "1"
    elif request.param != "cluster-auto":
        os.environ["RECSA_DECODE_SPLIT"] = request.param.split("-")[1]
    R.recsa_reload_switches()
    yield request.param
    for k, v in old.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v
    R.recsa_reload_switches()


@pytest.fixture(params=["warp", "window", "window-mma", "leaf-tc", "tree-tc", "generic"])
def prefill_impl(request):
    """Select the prefill path: the warp-per-(query, head) kernel alone (no
    workspace), the window kernel (tcgen05; "window-mma": the mma.sync one)
    plus the warp kernel attending the kept leaves (a workspace of the window
    partials' size; bf16 only, fp32 falls back to the warp kernel), the
    tensor-core kept-leaf path with the warp
    traversal ("leaf-tc") or with the tree levels as tensor-core tiles
    ("tree-tc"; bf16, where the window kernel runs; fp32 falls back to the
    warp traversal) -- both with a workspace of recsa_prefill_workspace_bytes
    -- or the generic kernel."""
    keys = ("RECSA_PREFILL_GENERIC", "RECSA_PREFILL_PATH")
    old = {k: os.environ.pop(k, None) for k in keys}
    if request.param == "generic":
        os.environ["RECSA_PREFILL_GENERIC"] = "1"
    elif request.param == "window-mma":
        os.environ["RECSA_PREFILL_PATH"] = "1"
    elif request.param == "leaf-tc":
        os.environ["RECSA_PREFILL_PATH"] = "2"
    elif request.param == "tree-tc":
        os.environ["RECSA_PREFILL_PATH"] = "3"
    R.recsa_reload_switches()
    yield request.param
    for k, v in old.items():
        os.environ.pop(k, None)
        if v is not None:
            os.environ[k] = v
    R.recsa_reload_switches()


def _prefill(g, impl, Q, K, V, tree, q0, nq, O, trace=None):
    ws = None
    if impl in ("window", "window-mma"):
        # exactly the window partials: the window + traversal path
        n = g.batch * nq * g.n_q_heads * (g.head_dim + 2) * 4
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    elif impl in ("leaf-tc", "tree-tc"):
        ws = torch.empty(R.recsa_prefill_workspace_bytes(g, nq), dtype=torch.uint8,
                         device="cuda")
    R.recsa_prefill(g, Q, K, V, tree, q0, nq, O, trace, workspace=ws)


def _setup(w, lens, capacity, seed=0, k=None, rope=1):
    batch = len(lens)
    g = geometry(w, capacity, batch, k=k, rope=rope)
    K, V, r = synth.make_kv(w, capacity, seed=seed, device="cpu", batch=batch)
    Kd, Vd, rd = K.cuda(), V.cuda(), r.cuda()
    tree = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, lens, rd, 0, tree)
    torch.cuda.synchronize()
    return g, K, V, r, Kd, Vd, rd, tree


def _oracle_trees(g, K, V, r, lens):
    trees = {}
    for s, L in enumerate(lens):
        for h in range(g.n_kv_heads):
            Kh, Vh = to_np(K[s, h, :L]), to_np(V[s, h, :L])
            trees[(s, h)] = (Kh, Vh, oracle.build_tree(Kh, Vh, r.double().numpy(),
                                                       g.leaf_block, g.branching))
    return trees


def _check_tree(g, tree, trees, dtype):
    st = Stats()
    for (s, h), (_, _, levels) in trees.items():
        for lev, (kk, vv) in enumerate(levels, start=1):
            gk, gv = read_tree_level(g, tree, lev)
            n = kk.shape[0]
            st.add(to_np(gk[s, h, :n]), kk)
            st.add(to_np(gv[s, h, :n]), vv)
    st.check(dtype, "tree")
    return st


# ---------------------------------------------------------------------------
# Tiny single-layer tree (fp32, L=4096, 4 q heads / 1 KV head, d=64)
# ---------------------------------------------------------------------------

TINY = synth.WORKLOADS["tiny-4k"]


@pytest.fixture(scope="module")
def tiny():
    L = TINY.length
    g, K, V, r, Kd, Vd, rd, tree = _setup(TINY, [L], L)
    trees = _oracle_trees(g, K, V, r, [L])
    return g, K, V, r, Kd, Vd, rd, tree, trees


def test_tree_tiny(tiny):
    g, K, V, r, Kd, Vd, rd, tree, trees = tiny
    _check_tree(g, tree, trees, torch.float32)


def test_decode_tiny_256_queries(tiny, decode_impl):
    g, K, V, r, Kd, Vd, rd, tree, trees = tiny
    L, nq = TINY.length, TINY.n_q
    pos = torch.full((1, nq), L - 1, dtype=torch.int64)
    Q, kind, _ = synth.make_queries(TINY, K, pos, seed=1, n_needles=16)
    assert int((kind == 1).sum()) == 16
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    ti = R.recsa_trace_ints(g)
    trace = torch.zeros((1, nq, g.n_q_heads, ti), dtype=torch.int32, device="cuda")
    lens = torch.tensor([L], dtype=torch.int64, device="cuda")
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, levels = trees[(0, 0)]
    src = oracle.FullTree(levels)
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for i in range(nq):
        for h in range(g.n_q_heads):
            check_query(st, O_[0, i, h], tr[0, i, h], to_np(Q[0, i, h]), L - 1, Kh, Vh, src, og,
                        g.k)
    st.check(torch.float32, "decode tiny")
    assert st.clear > 0.8 * nq * g.n_q_heads


def test_prefill_tiny_all_positions(tiny, prefill_impl):
    g, K, V, r, Kd, Vd, rd, tree, trees = tiny
    L = TINY.length
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=2)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    ti = R.recsa_trace_ints(g)
    trace = torch.zeros((1, L, g.n_q_heads, ti), dtype=torch.int32, device="cuda")
    _prefill(g, prefill_impl, Qd, Kd, Vd, tree, 0, L, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, levels = trees[(0, 0)]
    src = oracle.FullTree(levels)
    rng = np.random.default_rng(0)
    B, W = g.leaf_block, g.window
    sample = sorted(set([0, 1, B - 1, B, W - 2, W - 1, W, W + 1, W + B - 1, W + B, 2 * W + 7,
                         L - 2, L - 1] + list(rng.integers(0, L, 60))))
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for t in sample:
        for h in range(g.n_q_heads):
            check_query(st, O_[0, t, h], tr[0, t, h], to_np(Q[0, t, h]), t, Kh, Vh, src, og, g.k)
    st.check(torch.float32, "prefill tiny")


# ---------------------------------------------------------------------------
# Model-shaped layer, small cache (bf16, 32 q heads / 8 KV heads, d=128)
# ---------------------------------------------------------------------------

MODEL = synth.WORKLOADS["qwen3-4b-131k"]


@pytest.fixture(scope="module")
def model_small():
    lens = [20000, 13001]               # ragged: not multiples of B = 64
    g, K, V, r, Kd, Vd, rd, tree = _setup(MODEL, lens, 20480, seed=3)
    trees = _oracle_trees(g, K, V, r, lens)
    return g, lens, K, V, r, Kd, Vd, rd, tree, trees


def test_tree_model_small(model_small):
    g, lens, K, V, r, Kd, Vd, rd, tree, trees = model_small
    _check_tree(g, tree, trees, torch.bfloat16)


def test_decode_model_small(model_small, decode_impl):
    g, lens, K, V, r, Kd, Vd, rd, tree, trees = model_small
    nq = 3
    pos = torch.tensor([[L - 1] * nq for L in lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(MODEL, K, pos, seed=4, n_needles=2)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    ti = R.recsa_trace_ints(g)
    trace = torch.zeros((2, nq, g.n_q_heads, ti), dtype=torch.int32, device="cuda")
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
                Kh, Vh, levels = trees[(s, h // G)]
                check_query(st, O_[s, i, h], tr[s, i, h], to_np(Q[s, i, h]), L - 1, Kh, Vh,
                            oracle.FullTree(levels), og, g.k)
    st.check(torch.bfloat16, "decode model small")


def test_prefill_model_small(model_small, prefill_impl):
    g, lens, K, V, r, Kd, Vd, rd, tree, trees = model_small
    q0, nq = 12000, 1001                # ends at 13001 = the shorter sequence's length
    pos = (q0 + torch.arange(nq, dtype=torch.int64))[None].expand(2, nq)
    Q, _, _ = synth.make_queries(MODEL, K, pos.contiguous(), seed=5)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    ti = R.recsa_trace_ints(g)
    trace = torch.zeros((2, nq, g.n_q_heads, ti), dtype=torch.int32, device="cuda")
    _prefill(g, prefill_impl, Qd, Kd, Vd, tree, q0, nq, O, trace)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    G = g.n_q_heads // g.n_kv_heads
    rng = np.random.default_rng(1)
    for s in range(2):
        for i in [0, 1, 63, 64, 500, nq - 1] + list(rng.integers(0, nq, 4)):
            for h in range(0, g.n_q_heads, 3):
                Kh, Vh, levels = trees[(s, h // G)]
                check_query(st, O_[s, i, h], tr[s, i, h], to_np(Q[s, i, h]), q0 + i, Kh, Vh,
                            oracle.FullTree(levels), og, g.k)
    st.check(torch.bfloat16, "prefill model small")


# ---------------------------------------------------------------------------
# k >= every candidate count: dense causal attention
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("wname,rope", [("tiny-4k", 1), ("tiny-4k", 0), ("qwen3-4b-131k", 1)])
def test_keep_all_is_dense(wname, rope, prefill_impl):
    w = synth.WORKLOADS[wname]
    L = 1500 if w.head_dim == 64 else 700
    g, K, V, r, Kd, Vd, rd, tree = _setup(w, [L], L, seed=6, k=R.KEEP_ALL, rope=rope)
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(w, K, pos, seed=7)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    _prefill(g, prefill_impl, Qd, Kd, Vd, tree, 0, L, O)
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
    st.check(w.dtype, "keep-all")


# ---------------------------------------------------------------------------
# Append: incremental maintenance equals a fresh build
# ---------------------------------------------------------------------------

def test_append_matches_build_and_oracle():
    w = MODEL
    lens0 = [4000, 4031]
    steps = 200
    cap = 4096 + 256
    g, K, V, r, Kd, Vd, rd, tree = _setup(w, lens0, cap, seed=8)
    lens_d = torch.tensor(lens0, dtype=torch.int64, device="cuda")
    # The synthetic cache already holds the tokens to append at positions >= len.
    Kw, Vw = Kd.clone(), Vd.clone()
    Kw[0, :, 4000:] = 0
    Vw[0, :, 4000:] = 0
    Kw[1, :, 4031:] = 0
    Vw[1, :, 4031:] = 0
    og = oracle_geometry(g)
    G = g.n_q_heads // g.n_kv_heads
    st_out = Stats()
    for step in range(steps):
        kn = torch.stack([Kd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        vn = torch.stack([Vd[s, :, lens0[s] + step] for s in range(2)]).contiguous()
        R.recsa_append(g, Kw, Vw, kn, vn, lens_d, rd, 0, tree)
        if step in (23, 64, 199):        # decode right after an append
            lens_now = [L + step + 1 for L in lens0]
            pos = torch.tensor([[L - 1] for L in lens_now], dtype=torch.int64)
            Q, _, _ = synth.make_queries(w, K, pos, seed=9 + step)
            O = torch.empty_like(Q).cuda()
            trace = torch.zeros((2, 1, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                                device="cuda")
            R.recsa_decode(g, Q.cuda(), Kw, Vw, tree, lens_d, 1, O, trace)
            torch.cuda.synchronize()
            tr = trace.cpu().numpy()
            for s in range(2):
                Kh_all = to_np(K[s, :, :lens_now[s]])
                Vh_all = to_np(V[s, :, :lens_now[s]])
                for h in range(0, g.n_q_heads, 5):
                    Kh, Vh = Kh_all[h // G], Vh_all[h // G]
                    src = oracle.LazyTree(Kh, Vh, r.double().numpy(), g.leaf_block, g.branching)
                    check_query(st_out, to_np(O[s, 0, h]), tr[s, 0, h], to_np(Q[s, 0, h]),
                                lens_now[s] - 1, Kh, Vh, src, og, g.k)
    torch.cuda.synchronize()
    st_out.check(torch.bfloat16, "decode after append")
    new_lens = [L + steps for L in lens0]
    assert lens_d.cpu().tolist() == new_lens
    for s in range(2):
        assert torch.equal(Kw[s, :, :new_lens[s]], Kd[s, :, :new_lens[s]])
        assert torch.equal(Vw[s, :, :new_lens[s]], Vd[s, :, :new_lens[s]])
    fresh = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, new_lens, rd, 0, fresh)
    torch.cuda.synchronize()
    for lev in range(1, R.recsa_num_levels(g, max(new_lens)) + 1):
        a_k, a_v = read_tree_level(g, tree, lev)
        b_k, b_v = read_tree_level(g, fresh, lev)
        for s in range(2):
            n = new_lens[s] // (g.leaf_block * g.branching ** (lev - 1))
            torch.testing.assert_close(a_k[s, :, :n], b_k[s, :, :n], rtol=0, atol=1e-6)
            torch.testing.assert_close(a_v[s, :, :n], b_v[s, :, :n], rtol=0, atol=1e-6)
    trees = _oracle_trees(g, K, V, r, new_lens)
    _check_tree(g, tree, trees, torch.bfloat16)


@pytest.mark.parametrize("nq", [1, 2])
def test_decode_step_equals_append_then_decode(nq):
    """The fused step (one launch) gives the same outputs, cache, tree and
    lengths as recsa_append followed by recsa_decode, across leaf and level-2
    completions, and matches the oracle on sampled steps."""
    w = MODEL
    lens0 = [4000, 4031]
    steps = 130
    cap = 4096 + 256
    g, K, V, r, Kd, Vd, rd, tree_a = _setup(w, lens0, cap, seed=12)
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
        pos = torch.tensor([[L - 1] * nq for L in lens_now], dtype=torch.int64)
        Q, _, _ = synth.make_queries(w, K, pos, seed=100 + step)
        Qd = Q.cuda()
        Oa = torch.empty_like(Qd)
        Ob = torch.empty_like(Qd)
        trace = torch.zeros((2, nq, g.n_q_heads, ti), dtype=torch.int32, device="cuda")
        R.recsa_decode_step(g, Qd, Ka, Va, kn, vn, la, rd, 0, tree_a, nq, Oa, trace)
        R.recsa_append(g, Kb, Vb, kn, vn, lb, rd, 0, tree_b)
        R.recsa_decode(g, Qd, Kb, Vb, tree_b, lb, nq, Ob)
        torch.cuda.synchronize()
        assert torch.equal(Oa, Ob), step
        assert la.cpu().tolist() == lens_now
        if step in (31, 95, steps - 1):
            tr = trace.cpu().numpy()
            for s in range(2):
                Kh_all = to_np(K[s, :, :lens_now[s]])
                Vh_all = to_np(V[s, :, :lens_now[s]])
                for h in range(0, g.n_q_heads, 9):
                    Kh, Vh = Kh_all[h // G], Vh_all[h // G]
                    src = oracle.LazyTree(Kh, Vh, r.double().numpy(), g.leaf_block, g.branching)
                    check_query(st, to_np(Oa[s, nq - 1, h]), tr[s, nq - 1, h],
                                to_np(Q[s, nq - 1, h]), lens_now[s] - 1, Kh, Vh, src, og, g.k)
    st.check(torch.bfloat16, "decode step")
    assert torch.equal(Ka, Kb) and torch.equal(Va, Vb)
    assert torch.equal(tree_a[256:], tree_b[256:])


def test_decode_step_at_capacity_flags_and_decodes_without_append():
    w = MODEL
    cap = 320
    g, K, V, r, Kd, Vd, rd, tree = _setup(w, [cap, 200], cap, seed=13)
    lens = torch.tensor([cap, 200], dtype=torch.int64, device="cuda")
    kn = Kd[:, :, 0].contiguous()
    vn = Vd[:, :, 0].contiguous()
    Q = torch.randn((2, 1, g.n_q_heads, g.head_dim), device="cuda").to(Kd.dtype)
    O = torch.empty_like(Q)
    K_before = Kd.clone()
    R.recsa_decode_step(g, Q, Kd, Vd, kn, vn, lens, rd, 0, tree, 1, O)
    assert R.recsa_tree_error(g, tree, clear=True) == R.DEVERR_APPEND_FULL
    assert lens.cpu().tolist() == [cap, 201]
    assert torch.equal(Kd[0], K_before[0])                    # full sequence untouched
    Ob = torch.empty_like(Q)
    R.recsa_decode(g, Q, Kd, Vd, tree, lens, 1, Ob)
    torch.cuda.synchronize()
    assert torch.equal(O[0], Ob[0])                           # decoded at len - 1
    assert torch.equal(O[1], Ob[1])                           # appended, then decoded


def test_append_at_capacity_sets_flag_and_keeps_len():
    w = MODEL
    cap = 256
    g, K, V, r, Kd, Vd, rd, tree = _setup(w, [cap], cap, seed=10)
    lens_d = torch.tensor([cap], dtype=torch.int64, device="cuda")
    kn = torch.zeros((1, g.n_kv_heads, g.head_dim), dtype=Kd.dtype, device="cuda")
    before = Kd.clone()
    assert R.recsa_tree_error(g, tree) == 0
    R.recsa_append(g, Kd, Vd, kn, kn, lens_d, rd, 0, tree)
    assert R.recsa_tree_error(g, tree, clear=True) == R.DEVERR_APPEND_FULL
    assert R.recsa_tree_error(g, tree) == 0
    assert lens_d.item() == cap
    assert torch.equal(before, Kd)


def test_decode_empty_sequence_gives_zeros():
    w = MODEL
    g, K, V, r, Kd, Vd, rd, tree = _setup(w, [0, 100], 512, seed=11)
    lens_d = torch.tensor([0, 100], dtype=torch.int64, device="cuda")
    Q = torch.randn((2, 1, g.n_q_heads, g.head_dim), device="cuda").to(Kd.dtype)
    O = torch.full_like(Q, 7.0)
    R.recsa_decode(g, Q, Kd, Vd, tree, lens_d, 1, O)
    torch.cuda.synchronize()
    assert torch.all(O[0] == 0)
    assert torch.all(O[1] != 7.0)


def test_bounded_wait_expiry_reports_status_and_context_stays_usable():
    """Failure detection without a fault: RECSA_TEST_EXPIRE_WAIT makes the
    decode kernel's chain threads end with a wait on a barrier that nothing
    completes.  The wait runs out (50 ms), the launch finishes, the tree header
    carries RECSA_DEVERR_WAIT_TIMEOUT, and the next launch runs normally."""
    w = MODEL
    lens = [3000, 2500]
    g, K, V, r, Kd, Vd, rd, tree = _setup(w, lens, 4096, seed=14)
    pos = torch.tensor([[L - 1] for L in lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(w, K, pos, seed=15)
    Qd = Q.cuda()
    lens_d = torch.tensor(lens, dtype=torch.int64, device="cuda")
    O1, O2 = torch.empty_like(Qd), torch.empty_like(Qd)
    assert R.recsa_tree_error(g, tree) == 0
    os.environ["RECSA_TEST_EXPIRE_WAIT"] = "1"
    R.recsa_reload_switches()
    try:
        R.recsa_decode(g, Qd, Kd, Vd, tree, lens_d, 1, O1)
        torch.cuda.synchronize()
    finally:
        os.environ.pop("RECSA_TEST_EXPIRE_WAIT", None)
        R.recsa_reload_switches()
    assert R.recsa_tree_error(g, tree, clear=True) & R.DEVERR_WAIT_TIMEOUT
    assert R.recsa_tree_error(g, tree) == 0
    R.recsa_decode(g, Qd, Kd, Vd, tree, lens_d, 1, O2)
    torch.cuda.synchronize()
    assert R.recsa_tree_error(g, tree) == 0
    # the expiring wait came after the work: both launches wrote the same output
    assert torch.equal(O1, O2)
    og = oracle_geometry(g)
    trees = _oracle_trees(g, K, V, r, lens)
    st = Stats()
    G = g.n_q_heads // g.n_kv_heads
    for s, L in enumerate(lens):
        for h in range(0, g.n_q_heads, 7):
            Kh, Vh, levels = trees[(s, h // G)]
            check_query(st, to_np(O2[s, 0, h]), None, to_np(Q[s, 0, h]), L - 1, Kh, Vh,
                        oracle.FullTree(levels), og, g.k)
    st.check(torch.bfloat16, "decode after an expired wait")
