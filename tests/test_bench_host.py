"""Host-side arithmetic of bench.py (no GPU): the algorithmic bytes behind
the roofline line, per weight format, and the workloads' linears."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synthetic  # noqa: E402


def shape(fmt, M=76, K=2560, N=9728):
    return synthetic.LinearShape("t", M, K, N, fmt=fmt)


def test_weight_bytes_per_format():
    N, K = 9728, 2560
    assert bench.weight_bytes(shape("w4a4")) == N * K // 2
    assert bench.weight_bytes(shape("int8_tensorwise")) == N * K
    assert bench.weight_bytes(shape("convrot_int8")) == N * K
    # 4-bit indices + one e4m3 scale per 16 + the 16-level fp32 codebook
    assert bench.weight_bytes(shape("asym_w4a8")) == N * K // 2 + N * K // 16 + 64


def test_algorithmic_bytes():
    s = shape("w4a4", M=16)
    x, w, sw, b, y = 2 * 16 * 2560, 9728 * 2560 // 2, 4 * 9728, 2 * 9728, 2 * 16 * 9728
    assert bench.alg_bytes(s) == x + w + sw + b + y
    # the GEMM launch reads the activation codes as bytes and their scales instead of x
    assert bench.gemm_alg_bytes(s) == w + 16 * 2560 + 4 * 16 + 6 * 9728 + y


@pytest.mark.parametrize("workload,fmt,count", [("qwen3_4b_w4a8", "asym_w4a8", 14), ("small_m_w4a8", "asym_w4a8", 20),
                                                ("qwen3_4b_mixed", None, 14), ("edit20b_int8", "int8_tensorwise", 2)])
def test_workload_formats(workload, fmt, count):
    shapes = synthetic.workload_shapes(workload)
    assert len(shapes) == count
    if fmt:
        assert all(s.fmt == fmt for s in shapes)
    else:  # mixed: attention in ConvRot INT8, MLP in W4A4
        assert {s.fmt for s in shapes} == {"convrot_int8", "w4a4"}
    assert all(s.K % 256 == 0 and s.N % 8 == 0 for s in shapes)
    assert workload in bench.WORKLOAD_DESC


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler_with(tmp_path, smi_lines, nvml):
    c = bench.ClockSampler(0)
    c.nvml_ok = False
    if smi_lines is not None:
        path = tmp_path / "clocks.csv"
        path.write_text("".join(l + "\n" for l in smi_lines))
        c.path, c.fh, c.proc = str(path), open(os.devnull, "w"), _DoneProc()
    c.nvml_samples = nvml
    return c


def test_clock_record_merges_both_readers(tmp_path):
    smi = ["0, 1965, 1965, 700.5, 0x0, Not Active, Not Active, Not Active, Not Active",
           "0, 1950, 1965, 800.0, 0x4, Not Active, Not Active, Not Active, Active"]
    # few NVML samples: the nvidia-smi record leads, NVML beside it, reasons united
    r = _sampler_with(tmp_path, smi, [(1965.0, 1965.0, ["hw_slowdown"])]).stop()
    assert r["source"].startswith("nvidia-smi") and r["samples"] == 2 and r["sm_mhz"] == 1957.5
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap"] and r["nvml"]["samples"] == 1
    # enough NVML samples from inside the timed steps: they lead
    r = _sampler_with(tmp_path, smi, [(1965.0, 1965.0, [])] * 3 + [(1900.0, 1965.0, [])]).stop()
    assert r["source"].startswith("NVML") and r["samples"] == 4 and r["sm_min_mhz"] == 1900.0
    assert r["reasons"] == ["sw_power_cap"] and r["nvidia_smi"]["samples"] == 2
    # no reader at all (a host without a GPU): no record
    assert _sampler_with(tmp_path, None, []).stop() is None
