"""Host-side logic of bench.py, on CPU: the clock summary of the timed
region, the DRAM-traffic lookup that is void once a kernel's sources
change, and the CUDA-runtime lookup behind the graph's event nodes."""
import json
import os

import bench


def _sampler(smi_rows, nvml_rows):
    s = object.__new__(bench.ClockSampler)      # no nvidia-smi process, no NVML thread
    s.samples = smi_rows
    s.nvml_samples = nvml_rows
    return s


def test_clock_summary_merges_both_sources_inside_the_region():
    smi = [(10.0, "0, 1965, 1965, 900.5, 0x4, Not Active, Not Active, Not Active, Active"),
           (99.0, "0, 900, 1965, 300.0, 0x0, Active, Not Active, Not Active, Not Active")]
    nvml = [(10.1, 1800.0, 1965.0, {"sw_power_cap"}),
            (10.2, 1500.0, 1965.0, set()),
            (50.0, 100.0, 1965.0, {"hw_slowdown"})]              # outside [t0, t1]
    out = _sampler(smi, nvml).summary(9.0, 11.0)
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1800.0                               # median of 1965, 1800, 1500
    assert out["sm_mhz_range"] == [1500.0, 1965.0]
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]                    # the later rows are outside
    assert "NVML every 10 ms: 2" in out["sources"]


def test_clock_summary_takes_nearby_rows_for_a_short_region():
    smi = [(10.45, "0, 1700, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active")]
    out = _sampler(smi, []).summary(10.0, 10.2)
    assert out["samples"] == 1 and out["sm_mhz"] == 1700.0 and out["reasons"] == []


def test_traffic_lookup_is_void_once_sources_change(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_text("__global__ void k() {}\n")
    import hashlib
    digest = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    entry = {"k": {"read": 1000, "write": 24, "sources": digest, "files": ["k.cu"]}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(entry))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("k") == 1024
    assert bench.measured_traffic("other") is None
    src.write_text("__global__ void k() { /* changed */ }\n")
    assert bench.measured_traffic("k") is None


def test_stored_traffic_matches_the_current_sources():
    # profiles/traffic.json is refreshed with every capture; each entry names
    # the files its kernel is built from, and all of them exist.
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    kernels = [k for k in table if not k.startswith("_")]
    assert bench.ATTN_KERNEL in kernels and "append_gather_kernel<16>" in kernels
    for k in kernels:
        for rel in table[k]["files"]:
            assert os.path.exists(os.path.join(bench.ROOT, rel)), (k, rel)


def test_event_record_entry_point_lookup_does_not_raise():
    f = bench._external_event_record()
    assert f is None or callable(f)
