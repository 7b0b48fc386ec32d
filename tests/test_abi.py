"""The C-ABI library loads, exports every declared entry point, and its host-side
logic (geometry checks, level counts, tree sizing, argument errors) behaves as
include/recsa.h states.  No call here reaches the device."""

import ctypes
import os
import re

import pytest

from hierarchical_sparse_attention_recsa_b200 import recsa as R
from hierarchical_sparse_attention_recsa_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return R.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "recsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(recsa_[a-z_]+)\s*\(", text)))


def geo(**kw):
    base = dict(head_dim=128, n_q_heads=32, n_kv_heads=8, leaf_block=64, branching=16, k=8,
                window=512, batch=4, capacity=524288 + 512)
    base.update(kw)
    return R.Geometry(**base)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(R.EXPORTS) == set(names), names
    for n in names:
        assert hasattr(lib, n), n


def test_struct_layout_matches_header(lib):
    # 12 int32/float fields, one int64, then top_p, n_ref, key_format, reserved: 72 bytes.
    assert ctypes.sizeof(R.CGeometry) == 72
    assert R.CGeometry.capacity.offset == 48
    assert R.CGeometry.top_p.offset == 56
    assert R.CGeometry.n_ref.offset == 60
    assert R.CGeometry.key_format.offset == 64
    assert R.CGeometry.reserved.offset == 68


def test_status_strings(lib):
    for code in R.STATUS:
        assert R.recsa_status_string(code)


@pytest.mark.parametrize("kw", [
    dict(),
    dict(head_dim=64, n_q_heads=4, n_kv_heads=1, leaf_block=16, k=4, window=64, batch=1,
         capacity=4096, dtype=R.DTYPE_F32),
    dict(branching=32, batch=8, capacity=1048576 + 256),
    dict(leaf_block=32, branching=8, k=16, window=1024, batch=1, capacity=2097152 + 128),
    dict(k=R.KEEP_ALL, capacity=8192, rope_enabled=0),
    dict(mode=R.MODE_ZHA, top_p=0.9),
    dict(mode=R.MODE_ZHA, top_p=1.0, k=R.KEEP_ALL, capacity=8192),
    dict(mode=R.MODE_GROUP),
    dict(mode=R.MODE_ZHA, top_p=0.9, n_ref=16), dict(n_ref=0), dict(n_ref=1),
    dict(mode=R.MODE_ZHA, top_p=0.9, key_format=R.KEYS_FP8),
    dict(mode=R.MODE_ZHA, top_p=0.9, n_ref=16, key_format=R.KEYS_FP8),
    dict(mode=R.MODE_ZHA, top_p=0.9, n_ref=4, key_format=R.KEYS_NVFP4),
])
def test_valid_geometries(lib, kw):
    R.recsa_validate(geo(**kw))


@pytest.mark.parametrize("kw", [
    dict(head_dim=96), dict(n_q_heads=24), dict(n_q_heads=12, n_kv_heads=4),
    dict(branching=1), dict(window=0), dict(k=0), dict(leaf_block=0), dict(batch=0),
    dict(capacity=0), dict(dtype=7), dict(rope_base=1.0), dict(n_kv_heads=0),
    dict(mode=3), dict(mode=-1), dict(n_ref=2), dict(mode=R.MODE_GROUP, n_ref=4),
    dict(mode=R.MODE_ZHA, top_p=0.5, n_ref=65), dict(n_ref=-1), dict(mode=R.MODE_ZHA, top_p=0.0),
    dict(key_format=R.KEYS_FP8), dict(mode=R.MODE_GROUP, key_format=R.KEYS_FP8),
    dict(mode=R.MODE_ZHA, top_p=0.5, key_format=3), dict(key_format=R.KEYS_NVFP4), dict(mode=R.MODE_ZHA, top_p=1.5),
    dict(mode=R.MODE_ZHA, top_p=float("nan")),
])
def test_invalid_geometries(lib, kw):
    with pytest.raises(R.RecsaError) as e:
        R.recsa_validate(geo(**kw))
    assert e.value.status == 1


def test_num_levels(lib):
    assert R.recsa_num_levels(geo(head_dim=64, leaf_block=16, branching=16), 4096) == 3
    assert R.recsa_num_levels(geo(), 524288) == 4
    assert R.recsa_num_levels(geo(leaf_block=32, branching=8), 2097152) == 6
    assert R.recsa_num_levels(geo(), 63) == 0
    assert R.recsa_num_levels(geo(), 64) == 1


def expected_tree_bytes(g: R.Geometry) -> int:
    """Layout documented in include/recsa.h, recomputed independently."""
    def up(x):
        return (x + 255) // 256 * 256
    kk = min(g.k, g.capacity)
    rows = min(max(g.branching * kk + g.branching, g.leaf_block * kk + g.window + g.leaf_block),
               g.capacity + g.branching + 1)
    if g.mode == R.MODE_ZHA:  # true positions: one row per position
        rows = max(rows, g.capacity + 1)
    total = up(256 + rows * (g.head_dim // 2) * 8)
    span = g.leaf_block
    while g.capacity // span >= 1:
        n = g.capacity // span
        rows = g.batch * g.n_kv_heads * n
        row_bytes = rows * g.head_dim * 4
        nr = max(g.n_ref, 1)
        if g.key_format == R.KEYS_FP8:   # one byte per key element, then fp32 row scales
            total += up(rows * nr * g.head_dim) + up(rows * nr * 4) + up(row_bytes)
        elif g.key_format == R.KEYS_NVFP4:   # half a byte, E4M3 per 16, fp32 per row
            total += (up(rows * nr * g.head_dim // 2) + up(rows * nr * g.head_dim // 16) +
                      up(rows * nr * 4) + up(row_bytes))
        else:
            total += up(row_bytes * nr) + up(row_bytes)
        span *= g.branching
    return total


@pytest.mark.parametrize("kw", [dict(), dict(batch=1, capacity=4096 + 17), dict(k=R.KEEP_ALL),
                                dict(mode=R.MODE_ZHA, top_p=0.5),
                                dict(mode=R.MODE_ZHA, top_p=0.5, n_ref=16),
                                dict(mode=R.MODE_ZHA, top_p=0.5, key_format=R.KEYS_FP8),
                                dict(mode=R.MODE_ZHA, top_p=0.5, n_ref=4,
                                     key_format=R.KEYS_FP8),
                                dict(mode=R.MODE_ZHA, top_p=0.5, n_ref=3,
                                     key_format=R.KEYS_NVFP4)])
def test_tree_bytes(lib, kw):
    g = geo(**kw)
    assert R.recsa_tree_bytes(g) == expected_tree_bytes(g)


@pytest.mark.parametrize("mode", ["recsa", "zha", "group"])
def test_prefill_workspace_bytes(lib, mode):
    # ZHA and group selection: one fp32 window partial (normalised output, max,
    # sum) per query head.  RecSA: the tensor-core kept-leaf path's
    # intermediates, each section 256-byte aligned: the window + summary
    # partial per query head, one partial per (query head, kept-leaf slot), the
    # kept-leaf records (int2) and counts, the per-leaf counts and offsets
    # (int32 per (sequence, KV head, leaf)) and the pairs (int2 per slot).
    extra = {"recsa": {}, "zha": dict(mode=R.MODE_ZHA, top_p=0.9),
             "group": dict(mode=R.MODE_GROUP)}[mode]
    g = geo(batch=2, capacity=4096, **extra)
    rows = 2 * 100 * 32
    part = rows * (128 + 2) * 4
    if mode != "recsa":
        assert R.recsa_prefill_workspace_bytes(g, 100) == part
        return
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    kmax, buckets = 8, 2 * 8 * (4096 // 64)
    # the tree levels' tiles: the level's scores (c_max = min(b k + b - 1,
    # largest level) = 64 candidates), the kept nodes of two levels, the runs of
    # the next level (int4 + int2 per run, k + 1 runs a query head) and the
    # count per query head, the runs grouped by parent (int4), and per-parent
    # counts and offsets: 64 and 4 nodes at levels 1 and 2 -> 64 / 16 + 1 and
    # 4 / 16 + 1 parents per (sequence, KV head); and per run its partial
    # (d fp32) and its (max, sum)
    cmax, runs, parents = 64, rows * (kmax + 1), 2 * 8 * ((64 // 16 + 1) + (4 // 16 + 1))
    tree = (up(rows * cmax * 4) + up(2 * rows * kmax * 4) + up(runs * 16) + up(runs * 8) +
            up(rows * 4) + up(runs * 16) + 2 * up(parents * 4) + up(runs * 128 * 4) +
            up(runs * 8))
    want = (up(part) + up(rows * kmax * 128 * 4) + up(rows * kmax * 8) + up(rows * kmax * 8) +
            up(rows * 4) + 2 * up(buckets * 4) + up(rows * kmax * 8) + up(tree))
    assert R.recsa_prefill_workspace_bytes(g, 100) == want


def test_trace_ints(lib):
    assert R.recsa_trace_ints(geo(k=8)) == 4 + 32 + 16 * 8
    with pytest.raises(R.RecsaError):
        R.recsa_trace_ints(geo(k=100))


def _call(lib, name, *args):
    return getattr(lib, name)(*args)


def test_argument_errors_return_before_device(lib):
    g = geo(batch=1, capacity=4096)
    cg = g.c()
    ok = ctypes.c_void_p(1 << 20)            # aligned fake pointers: never dereferenced
    mis = ctypes.c_void_p((1 << 20) + 8)
    lens = (ctypes.c_int64 * 1)(4096)
    r = ctypes.c_void_p(1 << 20)
    # NULL pointers
    assert lib.recsa_build(ctypes.byref(cg), None, ok, lens, r, 0, ok, None) == 2
    assert lib.recsa_decode(ctypes.byref(cg), ok, ok, ok, ok, None, 1, ok, None, None) == 2
    assert lib.recsa_prefill(ctypes.byref(cg), ok, ok, ok, None, 0, 1, ok, None, None, 0, None) == 2
    assert lib.recsa_append(ctypes.byref(cg), ok, ok, ok, ok, None, r, 0, ok, None) == 2
    # misaligned tree (needs 256) and K (needs 16)
    assert lib.recsa_build(ctypes.byref(cg), ok, ok, lens, r, 0, mis, None) == 3
    assert lib.recsa_prefill(ctypes.byref(cg), ok, ctypes.c_void_p((1 << 20) + 4), ok, ok, 0, 1,
                             ok, None, None, 0, None) == 3
    # lengths and query ranges beyond capacity
    bad = (ctypes.c_int64 * 1)(4097)
    assert lib.recsa_build(ctypes.byref(cg), ok, ok, bad, r, 0, ok, None) == 4
    assert lib.recsa_prefill(ctypes.byref(cg), ok, ok, ok, ok, 4000, 97, ok, None, None, 0, None) == 4
    # a workspace smaller than recsa_prefill_workspace_bytes
    assert lib.recsa_prefill(ctypes.byref(cg), ok, ok, ok, ok, 0, 8, ok, None, ok, 16, None) == 4
    # trace with k beyond the trace limit
    g2 = geo(batch=1, capacity=4096, k=100).c()
    assert lib.recsa_decode(ctypes.byref(g2), ok, ok, ok, ok, ok, 1, ok, ok, None) == 5
    # zero queries: nothing to do
    assert lib.recsa_prefill(ctypes.byref(cg), ok, ok, ok, ok, 0, 0, ok, None, None, 0, None) == 0


def test_zha_capacity_limit(lib):
    """A ZHA tree's RoPE table has a row per position: capacity below 2^24."""
    ok = geo(mode=R.MODE_ZHA, top_p=0.5, batch=1, capacity=(1 << 24) - 2)
    assert R.recsa_tree_bytes(ok) > 0
    with pytest.raises(R.RecsaError) as e:
        R.recsa_tree_bytes(geo(mode=R.MODE_ZHA, top_p=0.5, batch=1, capacity=(1 << 24) + 10))
    assert e.value.status == 5
    # RecSA's table covers only candidate-local indices: no such limit
    assert R.recsa_tree_bytes(geo(batch=1, capacity=(1 << 24) + 10)) > 0
