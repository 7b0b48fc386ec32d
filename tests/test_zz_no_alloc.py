"""recsa_prefill_static: the prefill entry point for callers that cannot hand the
library any device memory beyond the call's tensors -- a runtime whose device
memory is planned ahead and owned by its own arena, or a C host with no device
allocator on its call path.  It keeps its scratch (the window partials) in a
fixed device array instead of a caller workspace.

Checked here through the C ABI, in every selection mode:
  * RecSA: the output equals, bit for bit, recsa_prefill given a caller
    workspace of exactly the window partials' size (the same kernels on the
    same inputs), on two calls in a row -- the larger query range first, then
    a smaller one at another position, so a row the second call failed to
    write would still hold the first call's nonzero partials -- and the second
    call's sampled outputs and traced selections match the float64 oracle;
  * ZHA and per-KV-group selection: equal, bit for bit, to recsa_prefill
    without a workspace (those modes keep no window partials), on two calls;
  * a request beyond the array's size is refused before any device work.
The file name sorts last so that a run stopping at the first failure has
already run every other test."""

import ctypes

import pytest
import torch

import oracle
from hierarchical_sparse_attention_recsa_b200 import build_lib, synth
from hierarchical_sparse_attention_recsa_b200 import recsa as R

from recsa_testlib import Stats, check_query, oracle_geometry, to_np

SCRATCH_BYTES = 4 << 20        # bytes of the fixed scratch


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return R.lib()


def _geom(batch, capacity, mode=R.MODE_RECSA):
    w = synth.WORKLOADS["qwen3-4b-131k"]
    return w, R.Geometry(head_dim=w.head_dim, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                         leaf_block=w.leaf_block, branching=w.branching, k=w.k, window=w.window,
                         batch=batch, capacity=capacity, dtype=R.DTYPE_BF16, rope_enabled=1,
                         rope_base=w.rope_base, mode=mode,
                         top_p=0.9 if mode == R.MODE_ZHA else 0.0)


def _window_partial_bytes(g, n_q):
    # one fp32 row of head_dim + 2 (normalised output, max, sum) per query head
    return g.batch * n_q * g.n_q_heads * (g.head_dim + 2) * 4


def test_static_prefill_rejects_oversize_before_device_work(lib):
    _, g = _geom(batch=2, capacity=1 << 20)
    cg = g.c()
    ok = ctypes.c_void_p(1 << 20)            # aligned fake pointers: never dereferenced
    n_q = SCRATCH_BYTES // (2 * g.n_q_heads * (g.head_dim + 2) * 4) + 1
    assert lib.recsa_prefill_static(ctypes.byref(cg), ok, ok, ok, ok, 0, n_q, ok, None,
                                    None) == 4
    # a NULL output is refused too
    assert lib.recsa_prefill_static(ctypes.byref(cg), ok, ok, ok, ok, 0, 8, None, None,
                                    None) == 2


def _setup(mode, seed):
    lens = [6000]
    cap = 6144
    w, g = _geom(batch=1, capacity=cap, mode=mode)
    K, V, r = synth.make_kv(w, cap, seed=seed, device="cuda", batch=1)
    tree = torch.zeros(R.recsa_tree_bytes(g), dtype=torch.uint8, device="cuda")
    R.recsa_build(g, K, V, lens, r, 0, tree)
    return w, g, K, V, r, tree


# 252 queries x 32 heads x (128 + 2) fp32 is the largest range the scratch holds
RANGES = [(5748, 252), (1000, 200)]


@pytest.mark.gpu
def test_static_prefill_equals_workspace_prefill_on_two_calls(lib):
    w, g, K, V, r, tree = _setup(R.MODE_RECSA, seed=21)
    ti = R.recsa_trace_ints(g)
    for call, (q0, nq) in enumerate(RANGES):
        pos = (q0 + torch.arange(nq, device="cuda", dtype=torch.int64))[None].expand(1, nq)
        Q, _, _ = synth.make_queries(w, K, pos.contiguous(), seed=30 + call)
        ws = torch.empty(_window_partial_bytes(g, nq), dtype=torch.uint8, device="cuda")
        O_ref = torch.empty_like(Q)
        R.recsa_prefill(g, Q, K, V, tree, q0, nq, O_ref, workspace=ws)
        O_static = torch.full_like(Q, float("nan"))
        trace = torch.zeros((1, nq, g.n_q_heads, ti), dtype=torch.int32, device="cuda")
        R.recsa_prefill_static(g, Q, K, V, tree, q0, nq, O_static, trace)
        torch.cuda.synchronize()
        assert torch.equal(O_static, O_ref), (call, (O_static.float() - O_ref.float()).abs().max())
    # the second call against the oracle: sampled queries, two heads of two KV groups
    og = oracle_geometry(g)
    G = g.n_q_heads // g.n_kv_heads
    q0, nq = RANGES[-1]
    O_, tr = to_np(O_static), trace.cpu().numpy()
    st = Stats()
    for kv in (0, 6):
        Kh, Vh = to_np(K[0, kv, :6000]), to_np(V[0, kv, :6000])
        src = oracle.LazyTree(Kh, Vh, r.double().cpu().numpy(), g.leaf_block, g.branching)
        for i in (0, 1, 63, 64, 137, nq - 1):
            for h in (kv * G, kv * G + G - 1):
                check_query(st, O_[0, i, h], tr[0, i, h], to_np(Q[0, i, h]), q0 + i, Kh, Vh,
                            src, og, g.k)
    st.check(torch.bfloat16, "static prefill vs oracle")


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [R.MODE_ZHA, R.MODE_GROUP])
def test_static_prefill_other_modes_equal_plain_prefill(lib, mode):
    w, g, K, V, r, tree = _setup(mode, seed=23)
    for call, (q0, nq) in enumerate(RANGES):
        pos = (q0 + torch.arange(nq, device="cuda", dtype=torch.int64))[None].expand(1, nq)
        Q, _, _ = synth.make_queries(w, K, pos.contiguous(), seed=50 + call)
        O_ref = torch.empty_like(Q)
        R.recsa_prefill(g, Q, K, V, tree, q0, nq, O_ref)
        O_static = torch.full_like(Q, float("nan"))
        R.recsa_prefill_static(g, Q, K, V, tree, q0, nq, O_static)
        torch.cuda.synchronize()
        assert torch.isfinite(O_static.float()).all()
        assert torch.equal(O_static, O_ref), (mode, call)
