"""Host logic of the benchmark line (no GPU): algorithmic work per launch, DRAM traffic
scaled from the committed small-case capture, and the choice of the roofline kernels."""
import os
import re
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from linear_lsh_sketch_race_b200 import inputs as I  # noqa: E402

WL = I.WORKLOADS[I.HEADLINE]
PEAKS = {"bf16_tflops_sustained": 1000.0, "bf16_tflops": 1500.0, "hbm_gbs": 6000.0}


def test_sweep_work_is_the_forward_work_per_token_head():
    f_fwd, _ = bench.flops_per_token_head(WL)
    assert bench.kernel_work("tc_causal_sweep", WL) == f_fwd * WL.H * WL.N
    # LR (d + 1) terms: state build + readout; d L P terms: q and k projections
    LR = WL.L * WL.R
    assert f_fwd == 4 * LR * (WL.d + 1) + 4 * WL.d * WL.L * WL.P


def test_backward_sides_do_the_forward_sweeps_work():
    w = bench.kernel_work("tc_causal_sweep", WL)
    assert bench.kernel_work("tc_bwd_q", WL) == w
    assert bench.kernel_work("tc_bwd_k", WL) == w
    assert bench.kernel_work("tc_bwd_finalize", WL) is None


def test_traffic_scales_with_token_heads_and_only_for_the_captured_configuration():
    t = bench.kernel_traffic("tc_causal_sweep", WL)
    t2 = bench.kernel_traffic("tc_causal_sweep", WL.replace(N=WL.N // 2))
    assert t == pytest.approx(2 * t2)
    assert bench.kernel_traffic("tc_causal_sweep", WL.replace(N=131072, H=8)) == \
        pytest.approx(698.695e6 + 247.275e6)
    assert bench.kernel_traffic("tc_bwd_q", WL.replace(N=131072, H=8)) == \
        pytest.approx(1442.38e6 + 532.65e6)
    assert bench.kernel_traffic("tc_causal_sweep", WL.replace(P=6)) is None
    assert bench.kernel_traffic("tc_bwd_finalize", WL) is None


def _profile_mb(name):
    text = open(os.path.join(ROOT, "profiles", name)).read()
    m = re.search(r"dram read / write \| ([\d,.]+) MB / ([\d,.]+) MB", text)
    return float(m.group(1).replace(",", "")) + float(m.group(2).replace(",", ""))


def _pipe_profile_mb(side):
    """DRAM read + write (MB) of one instantiation in the pipelined backward's summary."""
    text = open(os.path.join(ROOT, "profiles", "tc_bwd_pipe__causal_h8_n131072_L16_P8.md")).read()
    m = re.search(r"`k_bwd_pipe<%d>`[^|]*\|[^|]*\| ([\d,.]+) MB \| ([\d,.]+) MB" % side, text)
    return float(m.group(1).replace(",", "")) + float(m.group(2).replace(",", ""))


def test_traffic_constants_match_the_committed_capture_summaries():
    sweep = _profile_mb("tc_causal_sweep__causal_h8_n131072_L16_P8.md")
    small = WL.replace(N=131072, H=8)
    assert bench.kernel_traffic("tc_causal_sweep", small) / 1e6 == pytest.approx(sweep, abs=1)
    assert bench.kernel_traffic("tc_bwd_q", small) / 1e6 == pytest.approx(_pipe_profile_mb(0), abs=1)
    assert bench.kernel_traffic("tc_bwd_k", small) / 1e6 == pytest.approx(_pipe_profile_mb(1), abs=1)


def test_roofline_takes_the_dominant_kernel_and_keeps_the_forward_sweep():
    # per step: two sweeps of 80 ms, backward sides of 220 / 210 ms, finalize 60 ms
    ktimes = {"tc_causal_sweep": (160.0, 2), "tc_bwd_q": (220.0, 1), "tc_bwd_k": (210.0, 1),
              "tc_bwd_finalize": (60.0, 2), "tc_normalize": (2.5, 1)}
    roof, fwd = bench.roofline_lines(ktimes, WL, PEAKS, "test")
    assert roof["kernel"] == "tc_bwd_q"
    assert roof["ms_per_launch"] == pytest.approx(220.0)
    assert roof["achieved"] == pytest.approx(
        bench.kernel_work("tc_bwd_q", WL) / 0.220 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1000.0)
    assert roof["share_of_step"] == pytest.approx(220.0 / 652.5)
    assert fwd["kernel"] == "tc_causal_sweep"
    assert fwd["ms_per_launch"] == pytest.approx(80.0)
    # forward-only step: the sweep is the dominant kernel and no second object is added
    roof, fwd = bench.roofline_lines({"tc_causal_sweep": (80.0, 1), "tc_normalize": (2.5, 1)},
                                     WL, PEAKS, "test")
    assert roof["kernel"] == "tc_causal_sweep" and fwd is None
    # nothing with known work: no roofline
    assert bench.roofline_lines({"tc_normalize": (2.5, 1)}, WL, PEAKS, "test") == (None, None)


def test_reported_chunk_is_the_one_the_kernels_run():
    assert bench.chunk_ran(WL, "auto") == 128          # tensor-core sweep, 128-token chunks
    assert bench.chunk_ran(WL, "simt") == 32
    assert bench.chunk_ran(I.WORKLOADS[I.SMALL], "auto") == 32   # float32: CUDA-core tiles
