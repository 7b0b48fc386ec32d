"""Parity of per-KV-group shared selection (geometry mode RECSA_MODE_GROUP)
with the float64 oracle, through the C ABI.

The G query heads of a KV head share one selection per level (group score =
sum of the heads' softmax probabilities over the level's candidates) and each
head attends as in RecSA.  The selection check is bit-exact where the k-th and
(k+1)-th group scores are more than GROUP_GAP apart at every level, and a
validity check plus an output comparison under the GPU's selection elsewhere
(recsa_testlib.check_group).
"""

import os

import numpy as np
import pytest
import torch

import oracle
from hierarchical_sparse_attention_recsa_b200 import build_lib, synth
from hierarchical_sparse_attention_recsa_b200 import recsa as R

from recsa_testlib import Stats, alloc_tree, check_group, geometry, oracle_geometry, to_np

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny-4k"]
MODEL = synth.WORKLOADS["qwen3-4b-131k"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_lib.build()
    R.lib()


@pytest.fixture(params=["cluster-auto", "cluster-4,1", "generic"])
def decode_impl(request):
    """Decode on the cluster kernel (all G heads in each CTA; automatic
    candidate shares, or one share) or on the generic kernel."""
    keys = ("RECSA_DECODE_SPLIT", "RECSA_DECODE_GENERIC")
    old = {k: os.environ.get(k) for k in keys}
    for k in keys:
        os.environ.pop(k, None)
    if request.param == "generic":
        os.environ["RECSA_DECODE_GENERIC"] = "1"
    elif request.param == "cluster-4,1":
        os.environ["RECSA_DECODE_SPLIT"] = "4,1"
    R.recsa_reload_switches()
    yield request.param
    for k, v in old.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v
    R.recsa_reload_switches()


def _setup(w, lens, capacity, seed=0, k=None, rope=1):
    batch = len(lens)
    g = geometry(w, capacity, batch, k=k, rope=rope)
    g.mode = R.MODE_GROUP
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


def test_group_decode_tiny(decode_impl):
    L, nq = TINY.length, TINY.n_q
    g, K, V, r, Kd, Vd, rd, tree = _setup(TINY, [L], L, seed=40)
    trees = _trees(g, K, V, r, [L])
    pos = torch.full((1, nq), L - 1, dtype=torch.int64)
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=41, n_needles=16)
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
        check_group(st, O_[0, i], tr[0, i], to_np(Q[0, i]), L - 1, Kh, Vh, src, og, g.k)
    st.check(torch.float32, f"group {decode_impl} decode tiny")
    assert st.clear > 0.6 * nq


def test_group_prefill_tiny():
    L = TINY.length
    g, K, V, r, Kd, Vd, rd, tree = _setup(TINY, [L], L, seed=42)
    trees = _trees(g, K, V, r, [L])
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(TINY, K, pos, seed=43)
    Qd = Q.cuda()
    O = torch.empty_like(Qd)
    trace = torch.zeros((1, L, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    ws = torch.empty(R.recsa_prefill_workspace_bytes(g, L), dtype=torch.uint8, device="cuda")
    R.recsa_prefill(g, Qd, Kd, Vd, tree, 0, L, O, trace, workspace=ws)
    torch.cuda.synchronize()
    og = oracle_geometry(g)
    Kh, Vh, src = trees[(0, 0)]
    rng = np.random.default_rng(5)
    B, W = g.leaf_block, g.window
    sample = sorted(set([0, 1, B - 1, B, W - 1, W, W + 1, W + B, 2 * W + 7, L - 1] +
                        list(rng.integers(0, L, 40))))
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    for t in sample:
        check_group(st, O_[0, t], tr[0, t], to_np(Q[0, t]), t, Kh, Vh, src, og, g.k)
    st.check(torch.float32, "group prefill tiny")


def test_group_decode_model_small(decode_impl):
    lens = [20000, 13001]
    g, K, V, r, Kd, Vd, rd, tree = _setup(MODEL, lens, 20480, seed=44)
    trees = _trees(g, K, V, r, lens)
    nq = 3
    pos = torch.tensor([[L - 1] * nq for L in lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(MODEL, K, pos, seed=45, n_needles=2)
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
            for kv in range(g.n_kv_heads):
                Kh, Vh, src = trees[(s, kv)]
                hs = slice(kv * G, (kv + 1) * G)
                check_group(st, O_[s, i, hs], tr[s, i, hs], to_np(Q[s, i, hs]), L - 1, Kh, Vh,
                            src, og, g.k)
    st.check(torch.bfloat16, f"group {decode_impl} decode model small")


@pytest.mark.parametrize("wname,rope", [("tiny-4k", 1), ("tiny-4k", 0), ("qwen3-4b-131k", 1)])
def test_group_keep_all_is_dense(wname, rope):
    w = synth.WORKLOADS[wname]
    L = 1500 if w.head_dim == 64 else 700
    g, K, V, r, Kd, Vd, rd, tree = _setup(w, [L], L, seed=46, k=R.KEEP_ALL, rope=rope)
    pos = torch.arange(L, dtype=torch.int64)[None]
    Q, _, _ = synth.make_queries(w, K, pos, seed=47)
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
    st.check(w.dtype, "group keep-all")


def test_group_decode_step_equals_append_then_decode(decode_impl):
    w = MODEL
    lens0 = [4000, 4031]
    steps = 70
    cap = 4096 + 256
    g, K, V, r, Kd, Vd, rd, tree_a = _setup(w, lens0, cap, seed=48)
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
        Q, _, _ = synth.make_queries(w, K, pos, seed=300 + step)
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
                for kv in (0, g.n_kv_heads - 1):
                    src = oracle.LazyTree(Kh_all[kv], Vh_all[kv], r.double().numpy(),
                                          g.leaf_block, g.branching)
                    hs = slice(kv * G, (kv + 1) * G)
                    check_group(st, to_np(Oa[s, 0, hs]), tr[s, 0, hs], to_np(Q[s, 0, hs]),
                                lens_now[s] - 1, Kh_all[kv], Vh_all[kv], src, og, g.k)
    st.check(torch.bfloat16, f"group {decode_impl} decode step")
    assert torch.equal(Ka, Kb) and torch.equal(Va, Vb)
    assert torch.equal(tree_a[256:], tree_b[256:])
