"""Parity at the workloads' full sizes, on sampled outputs the oracle computes
one by one (its tree is built lazily from each sampled head's cache).

* 524K (32q/8kv, d=128, B64 b16 k8 W512, 4 levels): decode at batch 4 after an
  append, and the fused append + decode step the benchmark times, in its
  launch configuration (cluster size chosen automatically); full causal prefill of one sequence in 64K-query
  chunks with the tensor-core window workspace, as the benchmark runs it.
* 131K: decode (3 levels).
* 1M (b32, 3 levels): decode with needle and mixture queries.
* 2M (B32 b8 k16 W1024, 6 levels): decode, and the 65536-query chunked
  prefill at the end of the context; entries read per query are checked
  against the closed form from the selection trace.

Tolerances and the selection rule are those of recsa_testlib.
"""

import numpy as np
import pytest
import torch

import oracle
from hierarchical_sparse_attention_recsa_b200 import build_lib, synth
from hierarchical_sparse_attention_recsa_b200 import recsa as R

from recsa_testlib import Stats, alloc_tree, check_query, geometry, oracle_geometry, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_lib.build()
    R.lib()


def _host_head(K, V, s, g, n):
    return (K[s, g, :n].float().cpu().numpy(), V[s, g, :n].float().cpu().numpy())


def _decode_case(wname, batch, appended=1, samples=((0, 0), (0, 13), (0, 31)), seed=0,
                 fused=False):
    w = synth.WORKLOADS[wname]
    L = w.length
    cap = L + 64
    g = geometry(w, cap, batch)
    K, V, r = synth.make_kv(w, cap, seed=seed, device="cuda", batch=batch)
    tree = alloc_tree(g)
    R.recsa_build(g, K, V, [L] * batch, r, 0, tree)
    lens = torch.full((batch,), L, dtype=torch.int64, device="cuda")
    n = L + appended
    pos = torch.full((batch, 1), n - 1, dtype=torch.int64, device="cuda")
    Q, kind, _ = synth.make_queries(w, K, pos, seed=seed + 1, n_needles=None)
    O = torch.empty_like(Q)
    trace = torch.zeros((batch, 1, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    for i in range(appended):
        kn = K[:, :, L + i].contiguous()
        vn = V[:, :, L + i].contiguous()
        if fused and i == appended - 1:
            # the step the benchmark times: append and decode in one launch
            R.recsa_decode_step(g, Q, K, V, kn, vn, lens, r, 0, tree, 1, O, trace)
        else:
            R.recsa_append(g, K, V, kn, vn, lens, r, 0, tree)
    if not fused:
        R.recsa_decode(g, Q, K, V, tree, lens, 1, O, trace)
    torch.cuda.synchronize()
    assert lens.cpu().tolist() == [n] * batch
    og = oracle_geometry(g)
    G = g.n_q_heads // g.n_kv_heads
    O_, tr = to_np(O), trace.cpu().numpy()
    st = Stats()
    heads = {}
    for s, h in samples:
        kv = h // G
        if (s, kv) not in heads:
            Kh, Vh = _host_head(K, V, s, kv, n)
            heads[(s, kv)] = (Kh, Vh, oracle.LazyTree(Kh, Vh, r.double().cpu().numpy(),
                                                       g.leaf_block, g.branching))
        Kh, Vh, src = heads[(s, kv)]
        check_query(st, O_[s, 0, h], tr[s, 0, h], to_np(Q[s, 0, h]), n - 1, Kh, Vh, src, og, g.k)
    st.check(w.dtype, f"decode {wname}")
    return st


def test_decode_524k_batch4_bench_config():
    _decode_case("qwen3-4b-524k", 4, samples=((0, 0), (0, 4), (0, 27), (1, 9), (1, 10), (1, 22),
                                               (2, 18), (2, 3), (2, 31), (3, 31), (3, 30),
                                               (3, 12)))


def test_decode_step_524k_batch4_bench_call():
    """The exact call the benchmark times: recsa_decode_step for the batch,
    here after 63 plain appends so the step itself completes a leaf block and
    pools it in-kernel."""
    _decode_case("qwen3-4b-524k", 4, appended=64, fused=True,
                 samples=((0, 1), (0, 17), (1, 8), (1, 30), (2, 23), (2, 5), (3, 29),
                          (3, 14)), seed=2)


def test_decode_131k():
    _decode_case("qwen3-4b-131k", 1, samples=((0, 0), (0, 7), (0, 13), (0, 22), (0, 26),
                                              (0, 31)), seed=3)


def test_decode_1m_needles_and_mixtures():
    _decode_case("decode-1m", 8, samples=((0, 0), (0, 3), (1, 17), (2, 9), (4, 30), (7, 21)),
                 seed=5)


def test_decode_2m_six_levels():
    st = _decode_case("stress-2m", 1, samples=((0, 0), (0, 12), (0, 19), (0, 31)), seed=7)
    assert st.clear + st.near_tie == 4


def test_prefill_524k_bench_config():
    """Full causal prefill of one 524K sequence in 64K-query chunks with a
    workspace, as the benchmark runs it, every chunk traced.  Sampled
    positions from every chunk are checked on all G heads of three KV groups
    with the selection rule of recsa_testlib.check_query: kept ids bit-exact
    where every level's gap is clear, the oracle re-run under the GPU's
    selection elsewhere; no sample is dropped."""
    w = synth.WORKLOADS["qwen3-4b-524k"]
    L = w.length
    g = geometry(w, L, 1)
    K, V, r = synth.make_kv(w, L, seed=11, device="cuda", batch=1)
    tree = alloc_tree(g)
    R.recsa_build(g, K, V, [L], r, 0, tree)
    chunk = 65536
    ws = torch.empty(R.recsa_prefill_workspace_bytes(g, chunk), dtype=torch.uint8, device="cuda")
    trace = torch.zeros((1, chunk, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    rng = np.random.default_rng(0)
    sample_t = sorted(set([0, 511, 512, 575, 576, 4095, 65535, 65536, L - 1] +
                          [int(c0 + x) for c0 in range(0, L, chunk)
                           for x in rng.integers(0, chunk, 2)]))
    picked = {}
    for c0 in range(0, L, chunk):
        pos = (c0 + torch.arange(chunk, device="cuda", dtype=torch.int64))[None]
        Q, _, _ = synth.make_queries(w, K, pos, seed=40 + c0 // chunk)
        O = torch.empty_like(Q)
        R.recsa_prefill(g, Q, K, V, tree, c0, chunk, O, trace, workspace=ws)
        for t in sample_t:
            if c0 <= t < c0 + chunk:
                picked[t] = (Q[0, t - c0].float().cpu().numpy(),
                             O[0, t - c0].float().cpu().numpy(), trace[0, t - c0].cpu().numpy())
    torch.cuda.synchronize()
    assert sorted(picked) == sample_t
    og = oracle_geometry(g)
    G = g.n_q_heads // g.n_kv_heads
    st = Stats()
    for kv in (0, 5, 7):
        Kh, Vh = _host_head(K, V, 0, kv, L)
        src = oracle.LazyTree(Kh, Vh, r.double().cpu().numpy(), g.leaf_block, g.branching)
        for t, (q, o, tr) in picked.items():
            for h in range(kv * G, kv * G + G):
                check_query(st, o[h].astype(np.float64), tr[h], q[h].astype(np.float64), t, Kh,
                            Vh, src, og, g.k)
    assert st.clear + st.near_tie == len(sample_t) * 3 * G
    st.check(w.dtype, "prefill 524K")


def test_prefill_2m_last_64k_chunk_and_counts():
    """The 65536-query chunked prefill at the end of the 2M context; entries
    read per query (from the trace of a traced sub-range) equal the closed form
    and stay within the O(log L) bound."""
    w = synth.WORKLOADS["stress-2m"]
    L = w.length
    nq = w.extra["prefill_queries"]
    q0 = L - nq
    g = geometry(w, L, 1)
    K, V, r = synth.make_kv(w, L, seed=13, device="cuda", batch=1)
    tree = alloc_tree(g)
    R.recsa_build(g, K, V, [L], r, 0, tree)
    pos = (q0 + torch.arange(nq, device="cuda", dtype=torch.int64))[None]
    Q, _, _ = synth.make_queries(w, K, pos, seed=14)
    O = torch.empty_like(Q)
    ws = torch.empty(R.recsa_prefill_workspace_bytes(g, nq), dtype=torch.uint8, device="cuda")
    R.recsa_prefill(g, Q, K, V, tree, q0, nq, O, workspace=ws)
    # traced sub-range at the very end (same kernels, smaller trace buffer)
    nt = 256
    trace = torch.zeros((1, nt, g.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    O2 = torch.empty_like(Q[:, -nt:])
    R.recsa_prefill(g, Q[:, -nt:].contiguous(), K, V, tree, L - nt, nt, O2, trace,
                    workspace=ws)
    torch.cuda.synchronize()
    torch.testing.assert_close(O2.float(), O[:, -nt:].float(), rtol=0, atol=0)
    og = oracle_geometry(g)
    tr = trace.cpu().numpy()
    levels = len(oracle.level_counts(L, g.leaf_block, g.branching))
    bound = levels * (g.branching * g.k + g.branching - 1) + g.leaf_block * g.k + g.window + \
        g.leaf_block - 1
    for i in range(nt):
        cf = oracle.closed_form_counts(L - nt + i, og)
        for h in range(0, g.n_q_heads, 7):
            rec = tr[0, i, h]
            assert int(rec[1]) == cf["entries"] and int(rec[2]) == cf["keys_read"]
            assert int(rec[1]) <= bound
    # sampled outputs of the full chunk against the oracle, with the trace's selection
    G = g.n_q_heads // g.n_kv_heads
    Kh, Vh = _host_head(K, V, 0, 0, L)
    src = oracle.LazyTree(Kh, Vh, r.double().cpu().numpy(), g.leaf_block, g.branching)
    st = Stats()
    O_ = to_np(O2)
    for i in (0, 100, nt - 1):
        for h in range(G):
            check_query(st, O_[0, i, h], tr[0, i, h], to_np(Q[0, nq - nt + i, h]), L - nt + i,
                        Kh, Vh, src, og, g.k)
    st.check(w.dtype, "prefill 2M")
