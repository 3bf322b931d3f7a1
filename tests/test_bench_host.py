"""Host logic of bench.py that needs no GPU."""
import bench
from packed_kv_attention_b200 import synth


def test_traffic_record_matches_the_committed_attention_sources():
    """The ncu DRAM bytes bench.py reports for the attention kernel were taken
    from these sources: a change to them without a new capture makes the record
    (and this test) fail instead of reporting stale traffic."""
    w = synth.WORKLOADS["infinity_8b"]
    m = bench.MEASURED_TRAFFIC
    assert bench.measured_traffic(w, m["bits"], m["lq"], m["rope"]) == m["bytes"]


def test_traffic_record_is_only_for_its_workload():
    m = bench.MEASURED_TRAFFIC
    w = synth.WORKLOADS["infinity_8b"]
    assert bench.measured_traffic(w, 2, m["lq"], m["rope"]) is None
    assert bench.measured_traffic(synth.WORKLOADS["sweep"], m["bits"], m["lq"], m["rope"]) is None
    assert bench.measured_traffic(w, m["bits"], m["lq"], True) is None
