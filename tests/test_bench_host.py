"""Host logic of bench.py that needs no GPU."""
import bench
from packed_kv_attention_b200 import synth


def _current_hash():
    import hashlib
    import os
    h = hashlib.sha256()
    for f in bench.TRAFFIC_SOURCES:
        with open(os.path.join(bench.ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def test_traffic_record_is_reported_only_for_the_sources_it_was_taken_from(monkeypatch):
    """The ncu DRAM bytes bench.py reports for the attention kernel belong to
    the sources they were captured from: with the current sources' hash the
    record is reported, with any other hash it is null (stale counters are
    never reported)."""
    w = synth.WORKLOADS["infinity_8b"]
    m = dict(bench.MEASURED_TRAFFIC)
    cur = _current_hash()
    expect = m["bytes"] if m["sources_sha256_16"] == cur else None
    assert bench.measured_traffic(w, m["bits"], m["lq"], m["rope"]) == expect
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {**m, "sources_sha256_16": cur})
    assert bench.measured_traffic(w, m["bits"], m["lq"], m["rope"]) == m["bytes"]
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {**m, "sources_sha256_16": "0" * 16})
    assert bench.measured_traffic(w, m["bits"], m["lq"], m["rope"]) is None


def test_traffic_record_is_only_for_its_workload(monkeypatch):
    m = {**bench.MEASURED_TRAFFIC, "sources_sha256_16": _current_hash()}
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", m)
    w = synth.WORKLOADS["infinity_8b"]
    assert bench.measured_traffic(w, 2, m["lq"], m["rope"]) is None
    assert bench.measured_traffic(synth.WORKLOADS["sweep"], m["bits"], m["lq"], m["rope"]) is None
    assert bench.measured_traffic(w, m["bits"], m["lq"], True) is None
