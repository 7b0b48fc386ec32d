"""Host logic of bench.py that needs no GPU: the DRAM-traffic figures are read
from a committed ncu summary only while the kernel sources hash to the value
the summary records, and only for the workload it was captured on."""

import hashlib
import os

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
