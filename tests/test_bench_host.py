"""Host-side logic of bench.py that needs no GPU: the code digest that ties a committed
ncu summary to the kernel code it was taken on, the reading of nvidia-smi clock samples,
and the format of the committed summaries."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _write(folder, name, text):
    with open(os.path.join(folder, name), "w") as f:
        f.write(text)


def test_code_digest_ignores_comments_and_layout(tmp_path):
    a, b = tmp_path / "a", tmp_path / "b"
    a.mkdir()
    b.mkdir()
    _write(a, "k.cu", "// the kernel\nint f(int x) {\n  return x + 1;  // one more\n}\n")
    _write(b, "k.cu", "/* reworded\n   comment */ int f(int x) { return x + 1; }\n\n// trailing note\n")
    _write(a, "h.cuh", "constexpr int kN = 4;\n")
    _write(b, "h.cuh", "constexpr int kN = 4;  // four\n")
    assert bench.code_digest(["k.cu", "h.cuh"], str(a)) == bench.code_digest(["h.cuh", "k.cu"], str(b))


def test_code_digest_sees_code_changes(tmp_path):
    _write(tmp_path, "k.cu", "int f(int x) { return x + 1; }\n")
    d0 = bench.code_digest(["k.cu"], str(tmp_path))
    _write(tmp_path, "k.cu", "int f(int x) { return x + 2; }\n")
    assert bench.code_digest(["k.cu"], str(tmp_path)) != d0
    # the same text split differently over two files is a different set of sources
    _write(tmp_path, "a.cu", "int f(int x) {")
    _write(tmp_path, "b.cu", " return x + 2; }\n")
    assert bench.code_digest(["a.cu", "b.cu"], str(tmp_path)) != bench.code_digest(["k.cu"], str(tmp_path))


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_samples_median_and_reasons():
    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 950.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    r = s.stop()
    assert r["sm_mhz"] == 1900.0 and r["sm_max_mhz"] == 1965.0 and r["samples"] == 3
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvidia_smi():
    r = bench.ClockSampler(0).stop()
    assert r["sm_mhz"] is None and r["reasons"] == ["nvidia-smi unavailable"]


@pytest.mark.parametrize("kernel", sorted(bench.PROFILE_OF))
def test_committed_summaries_carry_bytes_and_digest(kernel):
    import re
    path = os.path.join(ROOT, "profiles", bench.PROFILE_OF[kernel])
    text = open(path).read()
    assert re.search(r"DRAM bytes per value\s+[0-9.]+", text)
    m = re.search(r"kernel code sha256 \(([^)]*)\): ([0-9a-f]{64})", text)
    assert m, path
    for f in m.group(1).split():
        assert os.path.exists(os.path.join(ROOT, "lossless_float_weight_b200", "csrc", f)), f
    assert "Command" in text and "--clock-control none" in text
