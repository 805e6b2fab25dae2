"""Host logic of the benchmark that needs no GPU.

These cover the rebuild's algorithmic bytes (a hand count), the NVML clock
sampler (a fake NVML module: reason bits, median clock, no NVML at all),
the traffic record that is reported only for the kernel source it was
captured on, and the choice between the measured and the fallback HBM
peak.
"""

import json
import sys
import time
import types

import bench
from block_sparse_attention_kv_b200 import synth


def test_rebuild_bytes_hand_count():
    # keys read (128 bf16 channels = 256 B per token), 64 B of INT4 codes
    # per block, 128 x (fp32 scale + int32 zero point) per (sequence, head)
    w = synth.custom("rb", 2, 4, 2, [100, 33], [32, 16], 64, seed=3)
    d = synth.make_layer(w, 0, "cpu")
    assert [int(b) for b in d.block_size] == [32, 16]
    expect = (100 * 256 + 4 * 64 + 1024) + (100 * 256 + 7 * 64 + 1024) \
        + (33 * 256 + 2 * 64 + 1024) + (33 * 256 + 3 * 64 + 1024)
    assert bench.rebuild_bytes(d) == expect


def _fake_nvml(clocks, reasons):
    seq = iter(zip(clocks, reasons))
    last = [clocks[-1], reasons[-1]]

    def clock_info(h, which):
        try:
            c, r = next(seq)
            last[0], last[1] = c, r
        except StopIteration:
            pass
        return last[0]

    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByIndex = lambda i: ("gpu", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, which: 1965
    m.nvmlDeviceGetClockInfo = clock_info
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: last[1]
    return m


def _sample(monkeypatch, clocks, reasons):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(clocks, reasons))
    s = bench.ClockSampler(0, period=0.0005)
    assert s.ok
    s.start()
    deadline = time.time() + 5
    while len(s.sm) < 2 * len(clocks) and time.time() < deadline:
        time.sleep(0.002)
    return s.stop()


def test_clock_sampler_reasons_and_median(monkeypatch):
    # NVML clock-event bits: 0x4 software power cap, 0x8 hardware slowdown,
    # 0x40 hardware thermal slowdown; 0x1 (idle) is not reported
    out = _sample(monkeypatch, [1965, 1900, 1965], [0x0, 0x4 | 0x1, 0x8 | 0x40])
    assert out["sm_max_mhz"] == 1965
    assert out["sm_mhz"] == 1965.0           # the last value repeats, so it is the median
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]
    assert out["samples"] >= 3


def test_clock_sampler_quiet_run(monkeypatch):
    out = _sample(monkeypatch, [1965], [0x0])
    assert out["reasons"] == [] and out["sm_mhz"] == 1965.0


def test_clock_sampler_without_nvml(monkeypatch):
    m = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no NVML")

    m.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", m)
    s = bench.ClockSampler(0)
    assert not s.ok
    s.start()
    assert s.stop() is None                  # no clocks key rather than invented ones


def test_traffic_reported_only_for_its_source(monkeypatch, tmp_path):
    rec = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    rec.write_text(json.dumps({"source_sha": bench.kernel_source_hash(),
                               "dram_bytes_per_launch": 9.0e6}))
    assert bench.recorded_traffic() == 9.0e6
    rec.write_text(json.dumps({"source_sha": "0" * 16, "dram_bytes_per_launch": 9.0e6}))
    assert bench.recorded_traffic() is None
    rec.unlink()
    assert bench.recorded_traffic() is None


def test_kernel_source_hash_follows_the_code_not_the_comments(monkeypatch, tmp_path):
    a, b = tmp_path / "a.cu", tmp_path / "b.cuh"
    a.write_text('int f(int x) {  // doubles x\n  return 2 * x;\n}\nconst char* s = "a // b";\n')
    b.write_text("/* header */\n#define N 4\n")
    monkeypatch.setattr(bench, "KERNEL_SOURCES", [str(a), str(b)])
    h0 = bench.kernel_source_hash()
    assert len(h0) == 16
    # comments, blank lines and indentation: the same code, the same hash
    a.write_text('// f doubles its argument\n\nint f(int x) {\n    return 2 * x;   /* twice */\n}\n'
                 'const char* s = "a // b";\n')
    b.write_text("/* another\n   header */\n#define N 4\n")
    assert bench.kernel_source_hash() == h0
    # a token, a string literal's contents or a directive's line: another hash
    for src_a, src_b in [('int f(int x) { return 3 * x; }\nconst char* s = "a // b";\n', "#define N 4\n"),
                         ('int f(int x) { return 2 * x; }\nconst char* s = "a // c";\n', "#define N 4\n"),
                         ('int f(int x) { return 2 * x; }\nconst char* s = "a // b";\n', "#define N 4 int\n")]:
        a.write_text(src_a)
        b.write_text(src_b)
        assert bench.kernel_source_hash() != h0


def test_code_text_strips_comments_only():
    src = 'a = 1; // c1\nb = "/* not a comment */"; /* c2 */ c = \'/\';\n\n  d\t=  2;\n'
    assert bench.code_text(src) == 'a = 1;\nb = "/* not a comment */"; c = \'/\';\nd = 2;'


def test_hbm_peak_measured_else_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6531.5}))
    assert bench.hbm_peak() == (6531.5, "measured")


def test_clocks_rejected():
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": []}
    assert bench.clocks_rejected(ok) == []
    assert bench.clocks_rejected(None) == []
    capped = {"sm_mhz": 1300.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.clocks_rejected(capped) == []           # kept and noted
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected({**ok, "reasons": [r, "sw_power_cap"]}) == [r]
    locked = {"sm_mhz": 1200.0, "sm_max_mhz": 1965, "reasons": []}
    assert bench.clocks_rejected(locked) == ["sm clock below 85 % of max with no reason"]
    assert bench.clocks_rejected({**locked, "sm_mhz": 1900.0}) == []
