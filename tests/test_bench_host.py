"""Host logic of bench.py that needs no GPU: the DRAM-traffic lookup (an entry is used
only while its kernel sources are unchanged), the clock-sample summary (only samples
inside the timed region count; throttle reasons are collected), and the workload config
that the JSON line carries."""
import datetime as dt
import hashlib
import json
import os

import bench
from exact_io_aware_83_b200.inputs import DECODE_WORKLOADS, WORKLOADS


def _write_traffic(root, source_text, recorded_text):
    os.makedirs(os.path.join(root, "profiles"))
    os.makedirs(os.path.join(root, "src"))
    with open(os.path.join(root, "src", "k.cuh"), "w") as f:
        f.write(source_text)
    entry = {"kernel": "k", "workload": "w", "dram_bytes_per_launch": 1234,
             "sources": ["src/k.cuh"],
             "sources_sha256": [hashlib.sha256(recorded_text.encode()).hexdigest()]}
    with open(os.path.join(root, "profiles", "dram_traffic.json"), "w") as f:
        json.dump({"entries": [entry]}, f)


def test_traffic_used_while_the_source_is_unchanged(tmp_path, monkeypatch):
    _write_traffic(str(tmp_path), "kernel v1", "kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._profile_traffic("k", "w") == 1234
    assert bench._profile_traffic("k", "other") is None
    assert bench._profile_traffic("other", "w") is None


def test_traffic_dropped_once_the_source_changes(tmp_path, monkeypatch):
    _write_traffic(str(tmp_path), "kernel v2", "kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._profile_traffic("k", "w") is None


def test_committed_traffic_entries_name_existing_sources():
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        entries = json.load(f)["entries"]
    assert entries
    for e in entries:
        assert e["dram_bytes_per_launch"] == e["dram_bytes_read"] + e["dram_bytes_write"]
        for src in e["sources"]:
            assert os.path.exists(os.path.join(bench.ROOT, src)), src


def test_smi_clock_summary_keeps_the_timed_region_only(tmp_path):
    s = bench._SmiSampler.__new__(bench._SmiSampler)
    s.file = open(tmp_path / "c.csv", "w+")
    s.proc = object()  # stands for the nvidia-smi process
    t0 = dt.datetime(2026, 1, 1, 12, 0, 0)
    s.t0, s.t1 = t0, t0 + dt.timedelta(seconds=1)
    rows = [
        (-0.5, 900, "Not Active", "Not Active"),     # before the region: ignored
        (0.1, 1900, "Not Active", "Active"),         # sw_power_cap active
        (0.3, 1950, "Not Active", "Not Active"),
        (0.6, 1930, "Not Active", "Not Active"),
        (1.5, 300, "Active", "Not Active"),          # after the region: ignored
    ]
    for off, mhz, hw, cap in rows:
        ts = (t0 + dt.timedelta(seconds=off)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        s.file.write(f"{ts}, {mhz}, 1965, 900.0, 0x0, {hw}, Not Active, Not Active, {cap}\n")
    out = s.summary()
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1930
    assert out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]


class _FakeNvml:
    """Read-only NVML queries with scripted answers (no GPU involved)."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80

    def __init__(self, clocks, reasons):
        self.clocks, self.reasons, self.i = clocks, reasons, 0

    def nvmlDeviceGetClockInfo(self, h, which):
        return self.clocks[min(self.i, len(self.clocks) - 1)]

    def nvmlDeviceGetPowerUsage(self, h):
        return 950000

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        r = self.reasons[min(self.i, len(self.reasons) - 1)]
        self.i += 1
        return r


def test_nvml_clock_sampler_polls_during_the_region():
    import threading
    import time
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.period = 0.001
    s.samples = []
    s.source = "nvml"
    s.nvml = _FakeNvml([1965, 1950, 1940], [0x0, 0x4, 0x0])
    s.handle = None
    s.max_mhz = 1965.0
    s._stop = threading.Event()
    s._thread = None
    s.start()
    time.sleep(0.05)
    s.stop()
    out = s.summary()
    assert out["samples"] >= 3
    assert out["sm_max_mhz"] == 1965.0 and out["sm_mhz"] == 1940
    assert out["reasons"] == ["sw_power_cap"]
    assert out["power_w_max"] == 950.0


def test_default_workload_is_the_long_context_target():
    # the parser's default, read from the source of main() without running it
    import inspect
    assert WORKLOADS["long_8k_causal"].N == 8192
    assert 'default="long_8k_causal"' in inspect.getsource(bench.main)


def test_exponential_counts_of_the_workloads():
    w = WORKLOADS["long_8k_causal"]
    assert w.score_pairs() == 2 * 16 * 8192 * 8193 / 2
    assert WORKLOADS["d256_4k_stress"].score_pairs() == 2 * 8 * 4096 * 4096
    win = WORKLOADS["window_8k_1k"]
    assert win.score_pairs() == win.fwd_flops() / (4 * win.d)


def test_strong_scaling_parts_cover_the_workload():
    w = WORKLOADS["long_8k_causal"]
    seen = []
    for rank in range(8):
        for host, bm, B, Hq, Hkv in bench._parts(w, 8, rank, "strong"):
            assert host[0].shape == (B, Hq, w.N, w.d) and host[1].shape == (B, Hkv, w.N, w.d)
            seen.append(B * Hkv)
    assert sum(seen) == w.B * w.Hkv


def test_config_names_the_workload():
    c = bench._config(WORKLOADS["gpt_2k_causal"], 1)
    assert c["workload"] == "gpt_2k_causal" and c["global_batch"] == 8 and c["causal"]
    c = bench._config(WORKLOADS["blocksparse_8k_causal"], 2)
    assert c["global_batch"] == 4 and c["parallelism"] == "dp2"
    assert c["block_mask"]["density"] == 0.25 and 0.2 < c["block_mask"]["enabled_pairs_share_of_causal"] < 0.35
    c = bench._config(WORKLOADS["window_8k_1k"], 1)
    assert c["window"] == [1023, 0]
    c = bench._config(DECODE_WORKLOADS["decode_64k_gqa"], 1)
    assert c["cache_len"] == 65536 and c["passes"] == "decode"


def test_backward_kernel_names_follow_the_library_dispatch():
    import re
    src = open(os.path.join(os.path.dirname(bench.__file__), "exact_io_aware_83_b200", "csrc",
                            "fa_bwd.cuh")).read()
    assert int(re.search(r"constexpr int kQ128MinN = (\d+);", src).group(1)) == bench.Q128_MIN_N
    expect = {"gpt_2k_causal": "fa_bwd_main_kernel", "long_8k_causal": "fa_bwd_q128_kernel",
              "gqa_4k_causal_fwd": "fa_bwd_q128_kernel", "d256_4k_stress": "fa_bwd_pair_kernel",
              "window_8k_1k": "fa_bwd_main_kernel", "dropout_8k_causal": "fa_bwd_main_kernel",
              "blocksparse_8k_causal": "fa_bwd_main_kernel"}
    for name, kernel in expect.items():
        assert bench._bwd_kernel_name(WORKLOADS[name]) == kernel, name
