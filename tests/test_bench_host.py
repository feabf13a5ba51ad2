"""Host-side logic of bench.py that needs no GPU: the clock sampler's parsing of nvidia-smi
samples, the ncu traffic table's source-hash keying, and the single-rank max."""
import hashlib
import os

import bench


class _FakeProc:
    def __init__(self, out):
        self.out = out

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.out, ""


def test_clock_sampler_parses_samples_and_reasons():
    lines = [
        "0, 1965, 1965, 420.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1850, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, N/A, 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = bench.ClockSampler(0)
    s.proc = _FakeProc("\n".join(lines) + "\n")
    r = s.stop()
    assert r["samples"] == 3
    assert r["sm_mhz"] == 1850.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_sampler_flags_slowdowns():
    s = bench.ClockSampler(0)
    s.proc = _FakeProc("0, 1200, 1965, 700, 0x8, Active, Not Active, Active, Not Active\n")
    assert s.stop()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_sampler_without_samples():
    s = bench.ClockSampler(0)
    assert s.stop() is None  # never started
    s.proc = _FakeProc("")
    assert s.stop() is None


def test_ncu_traffic_is_keyed_to_the_kernel_source():
    for kind, (path, digest, nbytes) in bench.NCU_TRAFFIC.items():
        with open(os.path.join(bench.ROOT, path), "rb") as f:
            current = hashlib.sha256(f.read()).hexdigest()
        got = bench.ncu_traffic(kind)
        # the stored figure is reported only while the source it was measured on is unchanged
        assert got == (nbytes if current == digest else None)
        assert nbytes > 0


def test_ncu_traffic_stale_key_reports_nothing(monkeypatch):
    key = bench.synth.DECODE.name
    path, digest, nbytes = bench.NCU_TRAFFIC[key]
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, (path, "0" * 64, nbytes))
    assert bench.ncu_traffic(key) is None
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, ("no/such/file.cu", digest, nbytes))
    assert bench.ncu_traffic(key) is None
    assert bench.ncu_traffic("a workload nobody measured") is None


def test_prefill_algorithmic_bytes():
    w = bench.synth.LONG_8K
    # q, k, v, O: 2 * 8192 * 16 * 128 * 2 bytes each; LSE 2 * 16 * 8192 * 4 bytes
    assert bench.prefill_bytes(w) == 4 * 67108864 + 1048576
    g = bench.synth.LONG_8K_GQA
    assert bench.prefill_bytes(g) == 2 * 134217728 + 2 * 33554432 + 2097152


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks([1.5, 2.0], None) == [1.5, 2.0]


def test_step_peak_is_sustained_for_long_timed_regions():
    measured = {"bf16_tflops": 1631.8, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6545.6}
    assert bench.step_tensor_peak(measured, 27.0) == (1631.8, False)
    assert bench.step_tensor_peak(measured, 2700.0) == (1400.0, True)
    assert bench.step_tensor_peak(measured, bench.LONG_REGION_MS) == (1400.0, True)
    # a peaks file without the sustained figure falls back to the recipe's one
    assert bench.step_tensor_peak({"bf16_tflops": 1631.8}, 2700.0) == (bench.FALLBACK["bf16_tflops_sustained"], True)
