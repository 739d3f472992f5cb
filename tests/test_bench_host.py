"""Host-side logic of bench.py (CPU only): metric names, the byte accounting
behind the roofline, the gate on the committed ncu traffic figure, and the
clock sampler's summary against a fake NVML."""
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from activation_sparse_predictor_b200 import synth  # noqa: E402

HEADLINE = "llama2_70b_reglu_8192x28672_q4_0"


def test_metric_names():
    assert bench.metric_name(HEADLINE, 1) == bench.METRIC
    other = bench.metric_name("falcon40b_relu_8192x32768_f16", 64)
    assert "falcon40b_relu_8192x32768_f16" in other and "batch 64" in other
    assert bench.metric_name(HEADLINE, 16) != bench.METRIC


def test_weight_row_bytes():
    # Q4_0: 16 bytes of nibbles + one binary16 scale per 32 weights
    assert bench.weight_row_bytes("q4_0", 8192) == 8192 // 32 * (16 + 2) == 4608
    assert bench.weight_row_bytes("f16", 8192) == 16384
    assert bench.weight_row_bytes("f32", 512) == 2048


def test_headline_layer_bytes():
    w = synth.WORKLOADS[HEADLINE]
    listed, down = 7260, 2800  # rows per layer (typical of the headline run)
    by = bench.layer_algorithmic_bytes(w, listed, down, 1)
    d, F, H, r = w.d_model, w.d_ff, w.hot, w.rank
    row = (d // 32) * 18  # one Q4_0 row with its scales
    # predictor: P1 [r][d] and the non-hot rows of P2 [F][r], fp16, plus the bias
    assert by["pred_u"] >= r * d * 2
    assert by["pred_z"] >= (F - H) * r * 2 + (F - H) * 4
    # gate + up rows of every listed neuron, down rows of the nonzero ones
    assert by["ffn_up"] >= listed * 2 * row
    assert by["ffn_down"] == down * row
    total = sum(by.values())
    assert 140e6 < total < 150e6  # about 144 MB per layer at this shape
    # bytes scale with the layer evaluations and the rows actually read
    by2 = bench.layer_algorithmic_bytes(w, 2 * listed, 2 * down, 2)
    assert sum(by2.values()) == pytest.approx(2 * total)
    # second-level sparsity (ReGLU): W_up rows only where the gate fired
    by3 = bench.layer_algorithmic_bytes(w, listed, down, 1, rows_second=down)
    assert total - sum(by3.values()) == pytest.approx((listed - down) * row)
    relu = synth.WORKLOADS["falcon40b_relu_8192x32768_f16"]
    by4 = bench.layer_algorithmic_bytes(relu, 1000, 100, 1)
    assert by4["ffn_up"] == pytest.approx(1000 * (16384 + 8) + (4 * 8192 + 4 * 1024))


def test_traffic_figure_follows_the_kernel_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "PROFILES", str(prof))
    assert bench.measured_traffic_per_layer(HEADLINE) is None  # no summary
    sha = bench.kernel_source_sha256()
    (prof / f"fused_stack_{HEADLINE}_ncu.md").write_text(
        f"# summary\n\n- source_sha256: `{sha}`\n- dram_bytes_per_layer: `153114112`\n")
    assert bench.measured_traffic_per_layer(HEADLINE) == 153114112.0
    (prof / f"fused_stack_{HEADLINE}_ncu.md").write_text(
        f"- source_sha256: `{'0' * 64}`\n- dram_bytes_per_layer: `153114112`\n")
    assert bench.measured_traffic_per_layer(HEADLINE) is None  # other sources


class _FakeNvml(types.SimpleNamespace):
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, reasons):
        super().__init__()
        self._clocks, self._reasons, self._i = list(clocks), reasons, 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        return ("handle", bus)

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("handle", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        v = self._clocks[min(self._i, len(self._clocks) - 1)]
        self._i += 1
        return v

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self._reasons


def _sampler(monkeypatch, clocks, reasons):
    import torch
    monkeypatch.setitem(sys.modules, "pynvml", _FakeNvml(clocks, reasons))
    props = types.SimpleNamespace(pci_domain_id=0, pci_bus_id=0x1B, pci_device_id=0)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda dev: props)
    s = bench.ClockSampler(0)
    assert s.ok
    for _ in range(len(clocks)):
        s._sample()
    return s.summary()


def test_clock_summary_reports_median_and_reasons(monkeypatch):
    out = _sampler(monkeypatch, [1965, 1900, 1965, 1800, 1965], 0x4 | 0x40)
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert out["samples"] == 5


def test_clock_summary_without_nvml(monkeypatch):
    import torch
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda dev: (_ for _ in ()).throw(RuntimeError("no device")))
    s = bench.ClockSampler(0)
    assert not s.ok
    out = s.summary()
    assert out["sm_mhz"] is None and out["reasons"] == []


def test_l2_mode_by_stack_size():
    # the tiny workload (8.4 MB) fits in L2: timed step by step after a flush
    assert bench.l2_mode_for(synth.WORKLOADS["tiny_relu_512x2048_f32"], 1,
                             bench.B200_L2_BYTES) == "flushed"
    w = synth.WORKLOADS[HEADLINE]
    assert bench.l2_mode_for(w, w.n_layers, bench.B200_L2_BYTES) == "streamed"
    assert "L2" in bench.run_config(w, 1, "per_token", 80, 1)["l2"]


def test_cold_tier_is_named_in_the_config():
    w = synth.WORKLOADS["llama2_70b_reglu_8192x28672_q4_0"]
    plain = bench.run_config(w, 1, "per_token", 8, 1)
    cold = bench.run_config(w, 1, "per_token", 8, 1, cold_tier="host")
    assert "cold_tier" not in plain
    assert "host memory" in cold["cold_tier"]
    assert {k: v for k, v in cold.items() if k != "cold_tier"} == plain
