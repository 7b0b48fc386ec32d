"""The selection variants on GQA group sizes other than the workloads' G = 4:
G = 1 (one query head per KV head), G = 2 and G = 8, with bf16 K/V at d = 64
and d = 128.  ZHA routing runs on its own kernel and on the generic kernel;
per-KV-group selection on the cluster kernel (G = 1, 2: all heads in a CTA)
and on the generic kernel (G = 8, which the cluster kernel does not take).
Compared with the float64 oracle as in test_gpu_zha / test_gpu_group."""

import os

import pytest
import torch

import oracle
from hierarchical_sparse_attention_recsa_b200 import build_lib, synth
from hierarchical_sparse_attention_recsa_b200 import recsa as R

from recsa_testlib import (Stats, alloc_tree, check_group, check_query_zha, geometry,
                           oracle_geometry, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_lib.build()
    R.lib()


def _workload(hq, hkv, d):
    return synth.Workload(f"gqa{hq}x{hkv}-d{d}", 6000, d, hq, hkv, 32, 8, 8, 256,
                          torch.bfloat16, True, batch=2, n_q=2)


def _env(generic):
    os.environ.pop("RECSA_ZHA_GENERIC", None)
    os.environ.pop("RECSA_DECODE_GENERIC", None)
    if generic:
        os.environ["RECSA_ZHA_GENERIC"] = "1"
        os.environ["RECSA_DECODE_GENERIC"] = "1"
    R.recsa_reload_switches()


def _run(w, g, lens, seed):
    K, V, r = synth.make_kv(w, w.length, seed=seed, device="cpu", batch=len(lens))
    Kd, Vd = K.cuda(), V.cuda()
    tree = alloc_tree(g)
    R.recsa_build(g, Kd, Vd, lens, r.cuda(), 0, tree)
    pos = torch.tensor([[L - 1] * w.n_q for L in lens], dtype=torch.int64)
    Q, _, _ = synth.make_queries(w, K, pos, seed=seed + 1, n_needles=1)
    O = torch.empty_like(Q).cuda()
    trace = torch.zeros((len(lens), w.n_q, g.n_q_heads, R.recsa_trace_ints(g)),
                        dtype=torch.int32, device="cuda")
    R.recsa_decode(g, Q.cuda(), Kd, Vd, tree,
                   torch.tensor(lens, dtype=torch.int64, device="cuda"), w.n_q, O, trace)
    torch.cuda.synchronize()
    trees = {}
    for s, L in enumerate(lens):
        for h in range(g.n_kv_heads):
            Kh, Vh = to_np(K[s, h, :L]), to_np(V[s, h, :L])
            trees[(s, h)] = (Kh, Vh, oracle.FullTree(
                oracle.build_tree(Kh, Vh, r.double().numpy(), g.leaf_block, g.branching)))
    return Q, to_np(O), trace.cpu().numpy(), trees


@pytest.mark.parametrize("hq,hkv,d", [(2, 2, 64), (4, 2, 128), (8, 1, 64), (16, 2, 128)])
@pytest.mark.parametrize("generic", [False, True])
def test_zha_group_sizes(hq, hkv, d, generic):
    _env(generic)
    try:
        w = _workload(hq, hkv, d)
        lens = [6000, 4321]
        g = geometry(w, w.length, 2, top_p=0.8)
        Q, O_, tr, trees = _run(w, g, lens, seed=110)
        og = oracle_geometry(g)
        G = hq // hkv
        st = Stats()
        for s, L in enumerate(lens):
            for i in range(w.n_q):
                for h in range(hq):
                    Kh, Vh, src = trees[(s, h // G)]
                    check_query_zha(st, O_[s, i, h], tr[s, i, h], to_np(Q[s, i, h]), L - 1, Kh,
                                    Vh, src, og, 0.8, g.k)
        st.check(torch.bfloat16, f"zha G={G} d={d} generic={generic}")
    finally:
        _env(False)


@pytest.mark.parametrize("hq,hkv,d", [(2, 2, 64), (4, 2, 128), (8, 1, 64), (16, 2, 128)])
@pytest.mark.parametrize("generic", [False, True])
def test_group_selection_sizes(hq, hkv, d, generic):
    _env(generic)
    try:
        w = _workload(hq, hkv, d)
        lens = [6000, 4321]
        g = geometry(w, w.length, 2)
        g.mode = R.MODE_GROUP
        Q, O_, tr, trees = _run(w, g, lens, seed=120)
        og = oracle_geometry(g)
        G = hq // hkv
        st = Stats()
        for s, L in enumerate(lens):
            for i in range(w.n_q):
                for kv in range(hkv):
                    Kh, Vh, src = trees[(s, kv)]
                    hs = slice(kv * G, (kv + 1) * G)
                    check_group(st, O_[s, i, hs], tr[s, i, hs], to_np(Q[s, i, hs]), L - 1, Kh,
                                Vh, src, og, g.k)
        st.check(torch.bfloat16, f"group G={G} d={d} generic={generic}")
    finally:
        _env(False)
