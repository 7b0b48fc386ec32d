"""Host logic of bench.py that needs no GPU: the DRAM-traffic figures are read
from a committed ncu summary only while the kernel sources hash to the value
the summary records, and only for the workload it was captured on; the
algorithmic bytes of a decode launch (the roofline numerator) agree with a
hand-worked trace."""

import hashlib
import os

import numpy as np

import bench
from hierarchical_sparse_attention_recsa_b200 import recsa as R
from hierarchical_sparse_attention_recsa_b200 import synth


def _sources_sha(names):
    csrc = os.path.join(os.path.dirname(os.path.abspath(R.__file__)), "csrc")
    h = hashlib.sha256()
    for f in names:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _full(workload=None):
    w = synth.WORKLOADS[workload or bench.WORKLOAD]
    return (workload or bench.WORKLOAD), w.length, w.batch


def test_decode_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "decode.md"
    prof.write_text("text\ntraffic_bytes_per_launch: 12345\n"
                    f"source_sha256: {_sources_sha(bench.DECODE_SOURCES)}\n")
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(prof))
    assert bench.measured_traffic(*_full()) == 12345.0
    # another workload, length or batch: no figure
    name, L, batch = _full()
    assert bench.measured_traffic(name, L // 2, batch) is None
    assert bench.measured_traffic(name, L, batch + 1) is None
    # a source changed since the capture: no figure
    prof.write_text("traffic_bytes_per_launch: 12345\nsource_sha256: " + "0" * 64 + "\n")
    assert bench.measured_traffic(*_full()) is None
    # no capture at all
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(tmp_path / "missing.md"))
    assert bench.measured_traffic(*_full()) is None


def test_variant_traffic_per_leg(tmp_path, monkeypatch):
    prof = tmp_path / "variants.md"
    prof.write_text("traffic_bytes_per_launch[zha]: 111\n"
                    "traffic_bytes_per_launch[group]: 222\n"
                    f"source_sha256: {_sources_sha(bench.VARIANT_SOURCES)}\n")
    monkeypatch.setattr(bench, "VARIANT_PROFILE", str(prof))
    assert bench.measured_variant_traffic("zha", *_full()) == 111.0
    assert bench.measured_variant_traffic("group", *_full()) == 222.0
    assert bench.measured_variant_traffic("zha_multiref", *_full()) is None
    prof.write_text("traffic_bytes_per_launch[zha]: 111\nsource_sha256: " + "f" * 64 + "\n")
    assert bench.measured_variant_traffic("zha", *_full()) is None


def test_committed_summaries_parse():
    # the committed summaries carry the two fields the gates read
    for path in (bench.TRAFFIC_PROFILE, bench.VARIANT_PROFILE):
        text = open(path).read()
        assert "source_sha256: " in text and "traffic_bytes_per_launch" in text


def test_decode_bytes_from_a_hand_worked_trace():
    """B = 4, b = 2, W = 4, k = 1, two query heads on one KV head, d = 4,
    bf16; one sequence of 20 tokens, so t = 19, a = 4 and levels 3/2/1 hold
    1/2/4 visible nodes.  Head 0 keeps nodes 0, 0, 1 and head 1 nodes 0, 1, 3
    (levels 3, 2, 1).  Distinct rows by hand:
      keys scored   level 3 {0}, level 2 {0, 1}, level 1 {0, 1} | {2, 3}  -> 7
      unselected    level 3 {}, level 2 {1} | {0}, level 1 {0} | {2}      -> 4
      exact tokens  leaves {1, 3} (8 tokens) + window [16, 19] (4)        -> 12
    """
    from hierarchical_sparse_attention_recsa_b200 import counts
    B, b, W, k, G, d, elem = 4, 2, 4, 1, 2, 4, 2
    ints = 4 + 32 + 16 * k
    tr = np.zeros((1, 1, G, ints), dtype=np.int32)
    kept = {0: {3: 0, 2: 0, 1: 1}, 1: {3: 0, 2: 1, 1: 3}}
    for h in range(G):
        tr[0, 0, h, 0] = 3
        for lev in (1, 2, 3):
            tr[0, 0, h, 4 + 16 + lev - 1] = 1
            tr[0, 0, h, counts.TRACE_HEAD + (lev - 1) * k] = kept[h][lev]
    lens = np.array([20])
    r = counts.decode_bytes_from_trace(tr, lens, B, b, W, G, d, elem, k)
    assert (r["key_rows"], r["val_rows"], r["tok_rows"]) == (7, 4, 12)
    qo = 2 * 1 * 1 * G * d * elem
    assert r["bytes"] == qo + 7 * d * 4 + 4 * d * 4 + 12 * d * elem * 2 == 400
    # ZHA routing: no summary values in the softmax; R key rows per node of
    # FP8 codes plus a scale
    z = counts.decode_bytes_from_trace(tr, lens, B, b, W, G, d, elem, k, summary_values=False,
                                       keys_per_node=3, key_row_bytes=d + 4)
    assert z["bytes"] == qo + 7 * 3 * (d + 4) + 12 * d * elem * 2


def test_oracle_runs_on_every_host_core():
    """cpu_baseline and the reference arm time the oracle with one worker
    process per host core and report that count."""
    cpu = bench.CpuPool("tiny-4k")
    try:
        res = bench.cpu_baseline(cpu, seconds=0.3)
        assert res["cores"] == bench.host_cores() >= 1
        assert res["value"] > 0 and res["kind"] == "oracle"
        args = type("A", (), dict(workload="tiny-4k", warmup=1, steps=2))()
        ref = bench.run_reference(args, 0, 1, cpu)
        assert ref["impl"] == "reference" and ref["cpu_baseline"]["cores"] == cpu.cores
        assert ref["value"] > 0 and ref["e2e"]["value"] == ref["value"]
    finally:
        cpu.close()
