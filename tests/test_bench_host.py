"""Host-side arithmetic of bench.py, on the CPU: launch counts, algorithmic bytes and
FLOPs, the roofline's bound and fraction, the traffic record's source check, and the
clock summary.  The expected values are worked out by hand from the layer's shapes
(the per-stage formulas of the design notes) or taken from the ncu launch lists."""
import json
import os

import pytest

import bench
from routed_grouped_gemm_softmax_b200.inputs import CONFIGS

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1200.0}


def test_kernels_per_forward_match_the_launch_lists():
    # one forward's kernels, as listed by ncu on the GPU:
    # decode: logits, top-k + grouping, the layer GEMM (x rows gathered by the GEMM,
    # both expert GEMMs and the combine in one launch)
    assert bench.kernels_per_forward(CONFIGS["decode"]) == 3
    # prefill/skewed: prep, tensor-core logits, certify, count, scan, scatter, gather,
    # the layer GEMM, combine
    assert bench.kernels_per_forward(CONFIGS["prefill"]) == 9
    assert bench.kernels_per_forward(CONFIGS["skewed"]) == 9
    # fp8: the large-batch router and grouping, quantiser, gather, two GEMMs, combine
    assert bench.kernels_per_forward(CONFIGS["fp8"]) == 11
    # tiny (T = 64, 16 rows per expert): the large-batch router, the layer GEMM
    # gathering its x rows, the combine kernel
    assert bench.kernels_per_forward(CONFIGS["tiny"]) == 8
    # with the library's plan bits: the gather kernel (no direct A rows), two GEMM
    # launches and the combine inside the second
    assert bench.kernels_per_forward(CONFIGS["decode"], plan=1 | 4) == 2 + 1 + 2
    assert bench.kernels_per_forward(CONFIGS["prefill"], plan=2 | 8) == 6 + 1 + 1 + 1
    assert bench.kernels_per_forward(CONFIGS["prefill"], plan=2 | 8 | 16) == 6 + 1 + 1


def test_stage_work_bf16_by_hand():
    cfg = CONFIGS["tiny"].replace(name="w", T=4, H=256, I=128, E=4, top_k=2)
    w = bench.stage_work(cfg, [3, 0, 5, 0])  # two experts touched, A = 8 rows
    assert w["_D"] == 2
    # gate/up: 2 experts x (gate + up) x I x H bf16 + 8 rows of x in + 8 rows of h out
    assert w["gemm_gate_up"]["bytes"] == 2 * 2 * 128 * 256 * 2 + 8 * 256 * 2 + 8 * 128 * 2 == 268288
    assert w["gemm_gate_up"]["flops"] == 2 * 8 * 256 * 256
    # down: 2 experts x H x I bf16 + 8 rows of h in + 8 rows of y out
    assert w["gemm_down"]["bytes"] == 2 * 256 * 128 * 2 + 8 * 128 * 2 + 8 * 256 * 2 == 137216
    assert w["gemm_down"]["flops"] == 2 * 8 * 128 * 256
    # combine: y in, gates in, out
    assert w["combine"]["bytes"] == 8 * 256 * 2 + 8 * 4 + 4 * 256 * 2
    # router: x, router_w, indices + gates
    assert w["route"]["bytes"] == 4 * 256 * 2 + 256 * 4 * 2 + 8 * 8


def test_stage_work_fp8_by_hand():
    cfg = CONFIGS["fp8"].replace(name="w8", T=4, H=256, I=256, E=4, top_k=2)
    w = bench.stage_work(cfg, [8, 0, 0, 0])  # one expert, A = 8
    # e4m3 gate + up (1 byte) + a 2 x 2 grid of fp32 block scales each; x and h rows
    # as codes + one fp32 scale per 128 values
    weights = 2 * 256 * 256 + 2 * (2 * 2 * 4)
    rows = 8 * 256 + 8 * 2 * 4
    assert w["gemm_gate_up"]["bytes"] == weights + rows + rows == 135328
    assert w["gemm_down"]["bytes"] == (256 * 256 + 2 * 2 * 4) + rows + 8 * 256 * 2


def test_roofline_picks_the_binding_resource():
    work = {"g": {"bytes": 6e9, "flops": 1e12}, "t": {"bytes": 1e9, "flops": 3e12}}
    r = bench.roofline_for("g", work, 2.0, PEAKS, "measured", False, "none")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(3000.0) and r["frac"] == pytest.approx(0.5)
    r = bench.roofline_for("t", work, 4.0, PEAKS, "measured", False, "none")
    assert r["bound"] == "tensor" and r["peak"] == 1500.0
    assert r["achieved"] == pytest.approx(750.0) and r["frac"] == pytest.approx(0.5)
    # a kernel timed inside a long run takes the sustained peak; fp8 doubles it
    assert bench.roofline_for("t", work, 4.0, PEAKS, "measured", True, "none")["peak"] == 1200.0
    assert bench.roofline_for("t", work, 4.0, PEAKS, "measured", False, "none", fp8=True)["peak"] == 3000.0


def test_recorded_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    rec = {"decode": {"gemm_gate_up": {"dram_bytes_per_launch": 123, "sources": "aaaa"}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda stage: "aaaa")
    assert bench.recorded_traffic("decode", "gemm_gate_up") == 123
    assert bench.recorded_traffic("decode", "gemm_down") is None
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda stage: "bbbb")  # the kernel changed
    assert bench.recorded_traffic("decode", "gemm_gate_up") is None


def test_kernel_sources_hash_covers_the_stage_files():
    for stage, files in bench.STAGE_SOURCES.items():
        csrc = os.path.join(bench.ROOT, "routed_grouped_gemm_softmax_b200", "csrc")
        assert all(os.path.exists(os.path.join(csrc, f)) for f in files), stage
        assert len(bench.kernel_sources_hash(stage)) == 16


def _sampler():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.lines, s.samples, s.thread, s.max_mhz = [], [], None, None
    return s


def test_clock_summary_from_nvidia_smi_lines():
    s = _sampler()
    s.lines = [
        "2026/12/02 10:00:00.000, 1100, 1965, 300.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 10:00:01.000, 1900, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:01.050, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:01.100, 1700, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage",
    ]
    import datetime as dt
    t0 = dt.datetime(2026, 12, 2, 10, 0, 1).timestamp()
    c = s.summary(t0, t0 + 0.1)
    assert c["samples"] == 3 and c["sm_mhz"] == 1800.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]


def test_clock_summary_from_nvml_samples():
    s = _sampler()
    s.thread, s.max_mhz = object(), 1965.0
    s.bits = (0x8, 0x40, 0x20, 0x4)  # hw slowdown, hw thermal, sw thermal, sw power cap
    s.samples = [(0.5, 1000.0, 0x0), (1.0, 1965.0, 0x0), (1.001, 1900.0, 0x4), (1.002, 1500.0, 0x40), (2.0, 1.0, 0x8)]
    c = s.summary(1.0, 1.5)
    assert c["samples"] == 3 and c["sm_mhz"] == 1900.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_layer_work_matches_the_config_table():
    # whole-layer bytes and FLOPs of the four workloads, as tabulated from their shapes:
    # Decode D x 6.29 MB + 1.2 MB, 0.82 GFLOP; Prefill 1.61 GB + 35 MB (all 256 experts),
    # 206.2 + 4.3 GFLOP; Skewed 2.21 GB + 135 MB, 1700.8 + 4.3 GFLOP; FP8 11.28 GB of
    # e4m3 weights and scales + 33 MB, 721.6 + 3.8 GFLOP
    dec = bench.layer_work(CONFIGS["decode"], [1] * 103 + [0] * 153)
    assert dec["bytes"] == 103 * 6291456 + 1180672
    assert dec["flops"] / 1e9 == pytest.approx(0.822, abs=1e-3)
    pre = bench.layer_work(CONFIGS["prefill"], [1] * 256)
    assert pre["bytes"] / 1e9 == pytest.approx(1.61 + 0.035, abs=0.01)
    assert pre["flops"] / 1e9 == pytest.approx(206.2 + 4.3, abs=0.1)
    skw = bench.layer_work(CONFIGS["skewed"], [1] * 64)
    assert skw["bytes"] / 1e9 == pytest.approx(2.21 + 0.135, abs=0.01)
    assert skw["flops"] / 1e9 == pytest.approx(1700.8 + 4.3, abs=0.1)
    f8 = bench.layer_work(CONFIGS["fp8"], [1] * 256)
    assert f8["bytes"] / 1e9 == pytest.approx(11.28 + 0.033, abs=0.01)
    assert f8["flops"] / 1e9 == pytest.approx(721.6 + 3.8, abs=0.1)
    # the expert-ordered copy of x, h and y: written once, read once
    assert dec["implementation_bytes"] == 2 * (128 * 2048 * 2) + 2 * (128 * 512 * 2) + 2 * (128 * 2048 * 2)


def test_layer_roofline_bound_and_fraction():
    cfg = CONFIGS["decode"]
    counts = [1] * 103 + [0] * 153
    r = bench.layer_roofline(cfg, counts, 0.1, PEAKS, "measured", False)
    b = bench.layer_work(cfg, counts)["bytes"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(b / 1e-4 / 1e9, abs=0.1)
    assert r["frac"] == pytest.approx(r["achieved"] / 6000.0, abs=1e-4)
    r = bench.layer_roofline(CONFIGS["skewed"], [1] * 64, 2.0, PEAKS, "measured", False)
    assert r["bound"] == "tensor" and r["peak"] == 1500.0


def test_alu_bound_router_stage():
    # the small-batch router is fp32 FMA chains on the CUDA cores: reported against
    # 148 SMs x 128 lanes x 2 FLOPs x 1965 MHz = 74.4 TFLOP/s
    assert bench.alu_peak_tflops(1965.0) == pytest.approx(74.45, abs=0.01)
    w = bench.stage_work(CONFIGS["decode"], [1] * 103 + [0] * 153)
    assert w["route"]["alu"] and not bench.stage_work(CONFIGS["prefill"], [1] * 256)["route"]["alu"]
    peaks = dict(PEAKS, sm_max_mhz=1965.0)
    r = bench.roofline_for("route", w, 0.02, peaks, "measured", False, "none")
    assert r["bound"] == "alu" and r["unit"] == "TFLOP/s" and r["peak"] == pytest.approx(74.4, abs=0.1)
    assert r["achieved"] == pytest.approx(2.0 * 16 * 2048 * 256 / 2e-5 / 1e12, abs=1e-3)


def test_load_peaks_carries_the_sm_clock():
    p, kind = bench.load_peaks()
    assert kind in ("measured", "fallback") and p["sm_max_mhz"] > 0
    assert all(k in p for k in bench.FALLBACK_PEAKS)


def test_stage_work_mx_and_shared_by_hand():
    # MX: e2m1 weights at half a byte plus one e8m0 byte per 32 along K; e4m3 activation
    # codes plus one byte per 32 values
    cfg = CONFIGS["fp8"].replace(name="wmx", T=4, H=512, I=512, E=4, top_k=2, dtype="mx")
    w = bench.stage_work(cfg, [8, 0, 0, 0])  # one expert, A = 8
    weights = 2 * (512 * 512 // 2 + 512 * 512 // 32)
    rows = 8 * 512 + 8 * 512 // 32
    assert w["gemm_gate_up"]["bytes"] == weights + rows + rows == 286976
    assert w["gemm_down"]["bytes"] == (512 * 256 + 512 * 16) + rows + 8 * 512 * 2
    # a shared expert of 2 x I columns: its weights, x and h rows, and FLOPs on top
    sh = CONFIGS["tiny"].replace(name="wsh", T=4, H=256, I=128, E=4, top_k=2, shared_mult=2)
    base = bench.stage_work(sh.replace(shared_mult=0), [3, 0, 5, 0])
    ws = bench.stage_work(sh, [3, 0, 5, 0])
    assert ws["gemm_gate_up"]["bytes"] - base["gemm_gate_up"]["bytes"] == 2 * 256 * 256 * 2 + 4 * 256 * 2 + 4 * 256 * 2
    assert ws["gemm_gate_up"]["flops"] - base["gemm_gate_up"]["flops"] == 2.0 * 4 * 256 * 2 * 256
    assert ws["gemm_down"]["flops"] - base["gemm_down"]["flops"] == 2.0 * 4 * 256 * 256
    assert ws["combine"]["bytes"] - base["combine"]["bytes"] == 2 * 4 * 256 * 2


def test_layer_work_mx_is_about_half_of_fp8():
    f8 = bench.layer_work(CONFIGS["fp8"], [1] * 256)
    mx = bench.layer_work(CONFIGS["fp8"].replace(name="mx", dtype="mx"), [1] * 256)
    # 3 matrices of 2048 x 7168 per expert: 0.5 + 1/32 bytes per weight against 1 byte + fp32 per 128x128
    per_mx = 3 * (2048 * 7168 // 2 + 2048 * 7168 // 32)
    per_f8 = 3 * 2048 * 7168 + 3 * 16 * 56 * 4
    assert mx["bytes"] - f8["bytes"] == 256 * (per_mx - per_f8)
    assert mx["flops"] == f8["flops"]


def test_kernels_per_forward_variants():
    assert bench.kernels_per_forward(bench.WORKLOADS["mx"]) == 11   # as fp8 (T > 64: the standalone combine)
    assert bench.kernels_per_forward(bench.WORKLOADS["mx"].replace(T=16)) == 2 + 2 + 2 + 1  # no fused combine
    assert bench.kernels_per_forward(bench.WORKLOADS["prefill_shared"]) == 9   # the shared expert adds none
