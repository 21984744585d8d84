"""Host-side pieces of bench.py on CPU: the NVML clock sampler against a fake
NVML (it only reads clocks and clock-event reasons; it never sets anything)."""
import time
from types import SimpleNamespace

import bench


class FakeNVML:
    NVML_CLOCK_SM = 1

    def __init__(self, pcis, clocks, reasons):
        self.pcis, self.clocks, self.reasons = pcis, clocks, reasons
        self.calls = []

    def nvmlInit(self):
        pass

    def nvmlDeviceGetCount(self):
        return len(self.pcis)

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetPciInfo(self, h):
        d, b, s = self.pcis[h]
        return SimpleNamespace(domain=d, bus=b, device=s)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.calls.append(h)
        return self.clocks[h]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons[h]


def _fake():
    return FakeNVML([(0, 0x1B, 0), (0, 0x43, 0), (0, 0x52, 0)], clocks=[1000, 1965, 1500],
                    reasons=[0x8, 0x4, 0x20])


def test_sampler_picks_the_nvml_device_with_the_cuda_device_pci_address():
    nv = _fake()
    with bench.ClockSampler(0, period_s=0.001, pci=(0, 0x43, 0), nvml=nv) as clk:
        time.sleep(0.02)
    s = clk.summary()
    assert s["nvml_device"] == "pci" and set(nv.calls) == {1}
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] >= 1


def test_sampler_falls_back_to_the_index_without_a_pci_match():
    nv = _fake()
    with bench.ClockSampler(2, period_s=0.001, pci=(0, 0x99, 0), nvml=nv) as clk:
        time.sleep(0.02)
    s = clk.summary()
    assert s["nvml_device"] == "index" and set(nv.calls) == {2}
    assert s["reasons"] == ["sw_thermal_slowdown"]


def test_sampler_without_nvml_reports_no_samples():
    class Broken(FakeNVML):
        def nvmlInit(self):
            raise RuntimeError("no NVML")
    with bench.ClockSampler(0, pci=(0, 0x1B, 0), nvml=Broken([], [], [])) as clk:
        pass
    assert clk.summary()["samples"] == 0 and clk.summary()["sm_mhz"] is None


def test_reference_arm_prints_one_contract_line(capsys, monkeypatch):
    """`bench.py --impl reference` (the oracle on the host cores) on rank 0: one JSON line with the
    contract's keys, the same metric and workload as the GPU arm, and zero host-device bytes."""
    import json
    monkeypatch.setenv("RANK", "0")
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0", "--M", "256"])
    assert bench.run_reference(args) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["value"] > 0 and d["steps"] == 1
    assert d["config"]["workload"].startswith("qwen3_8b_projections") and d["config"]["M"] == 256
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
