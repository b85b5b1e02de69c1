"""Host logic behind the bench line, on the CPU: the DRAM-traffic figures read from the committed ncu
summaries (and dropped once a kernel's sources change), and the clock record parsed from
nvidia-smi samples (median SM clock, maximum clock, throttle reasons seen while active)."""
import hashlib
import os
import re
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

MARKER = re.compile(r"<!-- bench-traffic kernel=(\S+) per_unit_bytes=(\d+) unit=(\S+) sha1=(\w+) sources=(\S+) -->")


def _write_marker(root, kernel, per_unit, sources):
    h = hashlib.sha1()
    for s in sources:
        h.update(open(os.path.join(root, s), "rb").read())
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", "k.md"), "w") as f:
        f.write(f"<!-- bench-traffic kernel={kernel} per_unit_bytes={per_unit} unit=chunk_head "
                f"sha1={h.hexdigest()[:16]} sources={','.join(sources)} -->\n")


def test_traffic_scales_with_units_and_goes_stale(tmp_path, monkeypatch):
    src = tmp_path / "kern.cuh"
    src.write_text("// version 1\n")
    _write_marker(str(tmp_path), "my_kernel", 1000, ["kern.cuh"])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    got, note = bench.kernel_traffic("my_kernel", 16)
    assert got == 16000 and "1000 B per chunk_head x 16" in note
    assert bench.kernel_traffic("other_kernel", 16) == (None, "no capture")
    src.write_text("// version 2\n")  # the kernel changed since the capture
    got, note = bench.kernel_traffic("my_kernel", 16)
    assert got is None and "stale" in note


def test_committed_markers_parse_and_name_existing_sources():
    found = set()
    for name in sorted(os.listdir(os.path.join(ROOT, "profiles"))):
        for m in MARKER.finditer(open(os.path.join(ROOT, "profiles", name)).read()):
            found.add(m.group(1))
            assert int(m.group(2)) > 0
            for s in m.group(5).split(","):
                assert os.path.isfile(os.path.join(ROOT, s)), s
    assert {"tc_intra", "tc_inter", "decode_step"} <= found


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


class _FakeThread:
    def join(self, timeout=None):
        pass


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.proc, s.t, s.lines = _FakeProc(), _FakeThread(), lines
    return s


def test_clock_record_median_max_and_reasons(monkeypatch):
    monkeypatch.setattr(bench.time, "sleep", lambda _: None)
    lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1900, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 800.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    rec = _sampler(lines).stop()
    assert rec["sm_mhz"] == 1950 and rec["sm_max_mhz"] == 1965 and rec["samples"] == 3
    assert rec["reasons"] == ["sw_power_cap"]
    rec = _sampler(["0, 1200, 1965, 500, 0x8, Not Active, Active, Not Active, Not Active"]).stop()
    assert rec["reasons"] == ["hw_thermal_slowdown"]


@pytest.mark.parametrize("lines, reason", [([], "no samples")])
def test_clock_record_without_samples(monkeypatch, lines, reason):
    monkeypatch.setattr(bench.time, "sleep", lambda _: None)
    assert _sampler(lines).stop()["reasons"] == [reason]
    assert bench.ClockSampler(0).stop()["reasons"] == ["nvidia-smi unavailable"]
