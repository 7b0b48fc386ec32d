"""recsa_prefill_static: the prefill entry point for callers that cannot hand the
library any device memory beyond the call's tensors -- a runtime whose device
memory is planned ahead and owned by its own arena, or a C host with no device
allocator on its call path.  It keeps its scratch (the window partials) in a
fixed device array instead of a caller workspace.

Checked here through the C ABI: its output matches recsa_prefill with a caller
workspace, within the bf16 tolerance the parity tests use, on two calls in a
row with different query ranges (the array keeps the previous call's
contents), and a request beyond the array's size is refused before any device
work.  The file name sorts last so that a run stopping at the first failure
has already run every other test."""

import ctypes

import pytest
import torch

from hierarchical_sparse_attention_recsa_b200 import build_lib, synth
from hierarchical_sparse_attention_recsa_b200 import recsa as R

SCRATCH_BYTES = 4 << 20        # bytes of the fixed scratch


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return R.lib()


def _geom(batch, capacity):
    w = synth.WORKLOADS["qwen3-4b-131k"]
    return w, R.Geometry(head_dim=w.head_dim, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                         leaf_block=w.leaf_block, branching=w.branching, k=w.k, window=w.window,
                         batch=batch, capacity=capacity, dtype=R.DTYPE_BF16, rope_enabled=1,
                         rope_base=w.rope_base)


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


@pytest.mark.gpu
def test_static_prefill_matches_workspace_prefill_on_two_calls(lib):
    lens = [6000]
    cap = 6144
    w, g = _geom(batch=1, capacity=cap)
    K, V, r = synth.make_kv(w, cap, seed=21, device="cuda", batch=1)
    tree = torch.zeros(R.recsa_tree_bytes(g), dtype=torch.uint8, device="cuda")
    R.recsa_build(g, K, V, lens, r, 0, tree)
    # 252 queries x 32 heads x (128 + 2) fp32 is the largest range the scratch holds
    for call, (q0, nq) in enumerate([(1000, 200), (5748, 252)]):
        pos = (q0 + torch.arange(nq, device="cuda", dtype=torch.int64))[None].expand(1, nq)
        Q, _, _ = synth.make_queries(w, K, pos.contiguous(), seed=30 + call)
        ws = torch.empty(R.recsa_prefill_workspace_bytes(g, nq), dtype=torch.uint8,
                         device="cuda")
        O_ref = torch.empty_like(Q)
        R.recsa_prefill(g, Q, K, V, tree, q0, nq, O_ref, workspace=ws)
        O_static = torch.full_like(Q, float("nan"))
        R.recsa_prefill_static(g, Q, K, V, tree, q0, nq, O_static)
        torch.cuda.synchronize()
        err = (O_static.float() - O_ref.float()).abs()
        assert torch.isfinite(O_static.float()).all()
        assert err.max().item() <= 2e-2, (call, err.max().item())
        assert err.mean().item() <= 2e-3, (call, err.mean().item())
