"""Host-side logic of bench.py, on CPU: the recorded-traffic lookup, the clock
sampler's summary, and the reference arm (the oracle) on the tiny workload."""

import json
import os
import shutil
import types

import pytest

import bench


def test_recorded_traffic_only_for_the_recorded_source(tmp_path, monkeypatch):
    # a table written for one kernel source: its value is used only while the
    # source keeps the recorded sha256, and only for the recorded workload
    import hashlib
    root = tmp_path
    (root / "profiles").mkdir()
    csrc = root / "bit_mixture_experts_route_b200" / "csrc"
    csrc.mkdir(parents=True)
    src = csrc / "grouped_gemm_decode.cu"
    src.write_bytes(b"// kernel source\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    (root / "profiles" / "kernel_traffic.txt").write_text(
        "# kernel_source  sha256  workload  bytes_per_launch\n"
        f"grouped_gemm_decode.cu {sha} olmoe-decode:T=64 157830656\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.recorded_traffic("grouped_gemm_decode.cu", "olmoe-decode:T=64") == 157830656
    assert bench.recorded_traffic("grouped_gemm_decode.cu", "olmoe-decode:T=7") is None
    assert bench.recorded_traffic("no_such_kernel.cu", "olmoe-decode:T=64") is None
    src.write_bytes(b"// kernel source\n// edited\n")
    assert bench.recorded_traffic("grouped_gemm_decode.cu", "olmoe-decode:T=64") is None


def _line(ts, sm, reasons=("Not Active",) * 4):
    return ", ".join([ts, "0", str(sm), "1965", "900.0", "0x0", *reasons])


def test_clock_summary_keeps_the_timed_region_and_reports_reasons():
    c = bench.ClockSampler(0)
    t0 = c._stamp("2026/12/02 10:00:01.000")
    c.t0, c.t1 = t0, t0 + 1.0
    c.lines = [
        _line("2026/12/02 10:00:00.500", 600),                        # before: dropped
        _line("2026/12/02 10:00:01.100", 1965),
        _line("2026/12/02 10:00:01.500", 1950,
              ("Not Active", "Not Active", "Not Active", "Active")),  # power cap
        _line("2026/12/02 10:00:01.900", 1965),
        _line("2026/12/02 10:00:03.000", 300,
              ("Active", "Not Active", "Not Active", "Not Active")),  # after: dropped
        "garbage line",
    ]
    s = c.summary()
    assert s["samples"] == 3 and s["samples_outside_timed_region"] == 2
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_without_samples():
    c = bench.ClockSampler(0)
    c.lines = []
    assert c.summary()["samples"] == 0


def _args(**kw):
    a = dict(gpus=1, steps=2, warmup=1, impl="reference", config="tiny", tokens=None,
             layers=None, algo="auto", weights="nf4", lora=0, backward=False,
             no_cpu_baseline=False, seed=0)
    a.update(kw)
    return types.SimpleNamespace(**a)


def test_reference_arm_prints_one_line(capsys, monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    shape, T, layers = bench.CONFIGS["tiny"]
    bench.run_reference(_args(), shape, T, layers)
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "tiny"


def test_reference_arm_is_silent_on_other_ranks(capsys, monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    shape, T, layers = bench.CONFIGS["tiny"]
    bench.run_reference(_args(), shape, T, layers)
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("weights,lora,backward", [("nf4", 0, False), ("int4", 0, False),
                                                   ("mxfp4", 0, False), ("nf4", 16, False),
                                                   ("nf4", 0, True)])
def test_gate_up_bytes_accounting(weights, lora, backward):
    # the per-launch algorithmic bytes, from the formats' per-weight sizes
    sh, T = bench.moe_synth.OLMOE, 64
    wl = object.__new__(bench.Workload)
    wl.shape, wl.T, wl.fmt, wl.lora, wl.backward = sh, T, weights, lora, backward
    per_w = 0.5 + {"nf4": 4 / 64, "int4": 4 / 128, "mxfp4": 1 / 32}[weights]
    out = T * sh.k * (2 * sh.I * 4 if (lora or backward) else sh.I * 2)
    assert wl.gate_up_bytes(64) == pytest.approx(64 * 2 * sh.I * sh.H * per_w + T * sh.H * 2 + out)
    if lora:
        M = T * sh.k
        want = 64 * lora * (sh.H + 2 * sh.I) * 2 + M * sh.H * 2 + 2 * M * 2 * sh.I * 4
        assert wl.lora_bytes(64) == want


def test_a_device_fault_is_not_taken_for_a_capture_failure():
    # graph capture failures are recorded and the eager timing is reported;
    # a fault on the device must surface instead (the context is lost)
    assert bench._cuda_fault(RuntimeError("CUDA error: unspecified launch failure"))
    assert bench._cuda_fault(RuntimeError("CUDA error: an illegal memory access was encountered"))
    assert bench._cuda_fault(RuntimeError("CUDA error: misaligned address"))
    assert not bench._cuda_fault(RuntimeError("operation not permitted when stream is capturing"))
    assert not bench._cuda_fault(RuntimeError("moe_layer_forward: workspace too small"))
