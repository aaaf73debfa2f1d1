"""Host-side pieces of bench.py that need no GPU: the provenance rule of the reported DRAM traffic
and the parsing of the clock samples."""
import hashlib
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_only_for_the_captured_source(bench):
    srcs = [b"kernel source", b"helpers"]
    sha = hashlib.sha256(b"kernel source" + b"helpers").hexdigest()
    rec = {"source_sha256": sha, "dram_bytes_per_launch": 12345}
    assert bench.traffic_from_record(rec, srcs) == 12345
    # any change to either file (or their order) withdraws the figure
    assert bench.traffic_from_record(rec, [b"kernel source!", b"helpers"]) is None
    assert bench.traffic_from_record(rec, [b"helpers", b"kernel source"]) is None
    assert bench.traffic_from_record({"dram_bytes_per_launch": 1}, srcs) is None
    assert bench.traffic_from_record(None, srcs) is None


def test_committed_traffic_record_names_its_sources(bench):
    import json
    rec = json.load(open(os.path.join(ROOT, "profiles", "attend_main_decode_attention_traffic.json")))
    assert rec["source_files"] == ["kv_cache_vector_encode_b200/csrc/" + s for s in bench.TRAFFIC_SOURCES]
    assert rec["dram_bytes_per_launch"] > 0
    # the captured case is scaled to a bench launch in proportion to the attended tokens
    scaled = (rec["dram_read_mb_captured"] + rec["dram_write_mb_captured"]) * 1e6 * rec["scale_to_bench_launch"]
    assert abs(scaled - rec["dram_bytes_per_launch"]) <= 1e-6 * scaled


def test_clock_samples_parse(bench):
    cs = bench.ClockSampler(0)
    cs._parse("1965, 1965, 0, 0, 0, 1")                       # NVML child: 0/1 flags
    cs._parse("1800, 1965, Not Active, Not Active, Not Active, Active")   # nvidia-smi words
    cs._parse("garbage")
    cs._parse("x, y, 0, 0, 0, 0")
    s = cs.summary()
    assert s["samples"] == 2
    assert s["sm_max_mhz"] == 1965.0 and s["sm_mhz_min"] == 1800.0
    assert s["reasons"] == ["sw_power_cap"]
    assert bench.ClockSampler(0).summary()["samples"] == 0
