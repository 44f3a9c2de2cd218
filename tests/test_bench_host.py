"""Host-side pieces of bench.py (no GPU): the roofline denominators and the DRAM-traffic lookup,
which must report null once a kernel's source has changed since its counters were taken."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_peaks_come_from_the_measured_file():
    import bench
    peak, kind = bench.measured_peaks()
    tpeak, tkind = bench.measured_tensor_peak()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        assert (peak, kind) == (float(d["hbm_gbs"]), "measured")
        assert (tpeak, tkind) == (float(d["bf16_tflops"]), "measured")
    else:
        assert kind == tkind == "fallback"


def test_traffic_is_reported_only_for_the_source_it_was_taken_on():
    import bench
    src = {"tq3_encode": "tq3_mma.cu", "tq3_decode": "tq3_rows.cu", "rpbh_quantize": "rpbh_lanes.cu",
           "rpbh_rotate": "rpbh_lanes.cu", "rpbh_linear": "rpbh_linear.cu", "tq3_attention": "tq3_attn.cu"}
    lines = [l.split() for l in open(os.path.join(ROOT, "profiles", "traffic.txt")) if l.strip() and not l.startswith("#")]
    assert lines
    for name, workload, sha, _, value in lines:
        assert workload in bench.WORKLOADS
        cur = hashlib.sha256(open(os.path.join(ROOT, "weight_quantization_b200", "csrc", src[name]), "rb").read())
        got = bench.traffic_bytes(name, workload)
        if cur.hexdigest()[:16] == sha:
            assert got == float(value)
        else:
            assert got is None
    assert bench.traffic_bytes("no_such_kernel", "kv") is None
    assert bench.traffic_bytes("tq3_decode", "no_such_workload") is None


def test_oracle_timing_is_pinned_to_one_core_and_restored():
    import bench
    before = os.sched_getaffinity(0)
    with bench.OneCore() as pin:
        if pin.pinned:
            assert len(os.sched_getaffinity(0)) == 1
    assert os.sched_getaffinity(0) == before
    info = bench.host_cpu()
    assert info["nproc"] == len(before) and isinstance(info["cpu"], str)
