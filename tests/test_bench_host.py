"""The benchmark's work model and roofline arithmetic, on the CPU.

`roofline.achieved` is algorithmic work per launch over the measured launch time, and
`frac` is that over the measured peak; these tests recount the work from the layer shapes
(independently of the bench's helpers) and check the per-kernel aggregation over one step's
launch list."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

D, H, DH, L = bench.D, bench.H, bench.DH, bench.L
K = 1639


def test_projection_flops_from_shapes():
    n_in = 2 * H * DH + H * DH + 2 * H        # q, k, v heads and the two gate columns
    assert n_in == 6176
    assert bench.flops_inproj(K, False) == 2 * K * D * n_in
    assert bench.flops_inproj(K, True) == 2 * K * D * (n_in - H * DH)   # no q rows
    assert bench.flops_outproj(K) == 2 * K * H * DH * D


def test_scan_flops_per_token_head():
    C, d = 64, 128
    # the chunked form's count per chunk, 6 C^2 d_k + 4 C^2 d_v + C^3 / 3 + 6 C d_k d_v,
    # spread over the chunk's C tokens
    per_chunk = 6 * C * C * d + 4 * C * C * d + C ** 3 / 3 + 6 * C * d * d
    assert bench.scan_flops_per_token_head() == pytest.approx(per_chunk / C, rel=1e-15)
    assert 180e3 < bench.scan_flops_per_token_head() < 185e3


def test_group_model_counts_each_layer():
    F, B = bench.group_model(K)
    n_in = 3 * H * DH + 2 * H
    flops = 0
    weights = 0
    for l in range(L):
        last = l == L - 1
        rows = n_in - (H * DH if last else 0)
        flops += 2 * K * D * rows
        weights += rows * D * 2
        if not last:
            flops += 2 * K * H * DH * D
            weights += D * H * DH * 2
    flops += L * K * H * bench.scan_flops_per_token_head()
    assert F == pytest.approx(flops, rel=1e-12)
    assert B == weights + K * D * 2 + L * H * DH * DH * 4


def _one_step_names():
    names = []
    for l in range(L):
        last = l == L - 1
        names += ["rmsnorm", "in_proj", "scan_prep", "scan_chain"]
        if not last:
            names += ["scan_out", "out_proj"]
    return names


def test_kernel_rooflines_aggregate_one_step():
    names = _one_step_names()
    avg_ms = [0.01 * (i + 1) for i in range(len(names))]
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    r = bench.kernel_rooflines(names, avg_ms, K, peaks)
    assert r["in_proj"]["launches_per_step"] == L and r["out_proj"]["launches_per_step"] == L - 1
    assert r["scan_out"]["launches_per_step"] == L - 1
    # in-proj: FLOPs of all its launches (the last without q) over their summed time
    t = sum(a for n, a in zip(names, avg_ms) if n == "in_proj")
    fl = (L - 1) * bench.flops_inproj(K, False) + bench.flops_inproj(K, True)
    assert r["in_proj"]["achieved"] == pytest.approx(fl / (t * 1e-3) / 1e12)
    assert r["in_proj"]["frac"] == pytest.approx(r["in_proj"]["achieved"] / 1000.0)
    assert r["in_proj"]["flops_per_launch"] == pytest.approx(fl / L)
    # RMSNorm: bf16 input for the first layer, fp32 for the others, bf16 output
    t = sum(a for n, a in zip(names, avg_ms) if n == "rmsnorm")
    by = K * D * (2 + 2) + (L - 1) * K * D * (4 + 2)
    assert r["rmsnorm"]["achieved"] == pytest.approx(by / (t * 1e-3) / 1e9)
    assert r["rmsnorm"]["unit"] == "GB/s" and r["in_proj"]["unit"] == "TFLOP/s"
    # chain: the final fp32 state of every head
    assert r["scan_chain"]["bytes_per_launch"] == H * DH * DH * 4
    for v in r.values():
        assert v["us_per_step"] > 0


def test_kernel_rooflines_with_the_folded_norm():
    """The step as launched now: the first layer's RMSNorm only (the later layers' is folded
    into the residual GEMM before them), then per layer the projection, the fused scan and
    (but for the last) the output projection.  Layers still count from the projections: the
    last one's projection and scan use the last layer's work."""
    names = ["rmsnorm"]
    for l in range(L):
        names += ["in_proj", "scan_fused"] + (["out_proj"] if l < L - 1 else [])
    avg_ms = [0.01 * (i + 1) for i in range(len(names))]
    r = bench.kernel_rooflines(names, avg_ms, K, {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0})
    assert r["rmsnorm"]["launches_per_step"] == 1
    assert r["rmsnorm"]["bytes_per_launch"] == K * D * (2 + 2)    # bf16 h in, bf16 out
    fl = (L - 1) * bench.flops_inproj(K, False) + bench.flops_inproj(K, True)
    assert r["in_proj"]["flops_per_launch"] == pytest.approx(fl / L)
    by = sum(bench.kernel_work("scan_fused", l, K)[1] for l in range(L))
    assert r["scan_fused"]["bytes_per_launch"] == pytest.approx(by / L)
    assert bench.kernel_work("scan_fused", L - 1, K)[1] < bench.kernel_work("scan_fused", 0, K)[1]


def test_job_throughput_is_all_ranks_over_the_slowest():
    assert bench.job_throughput(K, 4, 2.0) == pytest.approx(4 * K / 2e-3)


def test_clock_summary_from_nvidia_smi_lines():
    """The clocks key: median SM clock under load, the max clock, and every throttle reason
    that was active in any sample (a run that saw a hardware or thermal slowdown is rejected
    by the driver, so none may be lost); malformed lines are skipped."""
    lines = [
        "0, 1965, 1965, 812.3, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1800, 1965, 1001.0, 0x0000000000000008, Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage",
    ]
    r = bench.ClockSampler.summarize("\n".join(lines) + "\n")
    assert r["samples"] == 3
    assert r["sm_mhz"] == 1950.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap"]
    empty = bench.ClockSampler.summarize("")
    assert empty["sm_mhz"] is None and empty["samples"] == 0 and empty["reasons"] == []
