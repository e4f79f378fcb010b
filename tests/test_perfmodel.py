"""Host-side bookkeeping of bench.py's roofline: the per-segment work model (no GPU).

The counts are checked against the layer shapes of the bench architecture enumerated layer by
layer (input projection 32 -> 2048, conv_pre 2048 -> 1024 k7, seven upsamplers, AMP stages of
three residual blocks with k = 3 / 7 / 11 and three dilations, conv_post 8 -> 1 k7), and
against the stage-1 figure bench.py reports per GEMM launch (55.05 GFLOP).
"""
from __future__ import annotations

import os

import pytest

from bigvgan_waveform_decoder_b200 import perfmodel as PM
from bigvgan_waveform_decoder_b200 import synthetic as S

B, N = 2, 400   # the bench workload


def _layers(arch):
    """(segment, Cin, Cout, taps, output samples per item) of every convolution, in order."""
    out = [("in_proj", arch.latent_channels, arch.latent_dim, 1, N),
           ("conv_pre", arch.latent_dim, arch.decoder_dim, 7, N)]
    C, L = arch.decoder_dim, N
    for i, (r, K) in enumerate(zip(arch.rates, arch.kernels)):
        # a transposed conv: every input sample meets all K taps once
        out.append((f"ups{i}", C, C // 2, K, L))
        C, L = C // 2, L * r
        for k, dils in zip(arch.rb_kernels, arch.rb_dilations):
            for _ in dils:
                out.append((f"amp{i}", C, C, k, L))   # dilated conv
                out.append((f"amp{i}", C, C, k, L))   # conv with dilation 1
    out.append(("post", C, 1, 7, L))
    return out


def test_segment_order_matches_the_library():
    names = [s.name for s in PM.segments(S.Arch(), B, N)]
    assert names == ["in_proj", "conv_pre"] + [f"{p}{i}" for i in range(7) for p in ("ups", "amp")] + ["post"]


def test_conv_flops_match_the_layer_enumeration():
    arch = S.Arch()
    want = {}
    for seg, cin, cout, k, l in _layers(arch):
        want[seg] = want.get(seg, 0.0) + 2.0 * cin * cout * k * l * B
    for s in PM.segments(arch, B, N):
        assert s.conv_flops == pytest.approx(want[s.name], rel=1e-12), s.name


def test_stage1_gemm_launch_work():
    """One GEMM launch of AMP stage 1 is one conv layer of all three blocks: 55.05 GFLOP."""
    amp1 = next(s for s in PM.segments(S.Arch(), B, N) if s.name == "amp1")
    assert amp1.conv_flops / 6 == pytest.approx(2 * 256 * 256 * (3 + 7 + 11) * 20000, rel=1e-12)
    assert amp1.conv_flops / 6 == pytest.approx(55.05e9, rel=1e-3)


def test_activation_flops_count_18_activations_per_stage():
    arch = S.Arch()
    for i, s in enumerate(s for s in PM.segments(arch, B, N) if s.name.startswith("amp")):
        C = arch.decoder_dim >> (i + 1)
        L = N
        for r in arch.rates[: i + 1]:
            L *= r
        assert s.act_flops == pytest.approx(18 * PM.ACT_FLOPS * C * L * B, rel=1e-12)
        assert s.sines == pytest.approx(18 * PM.ACT_SINES * C * L * B, rel=1e-12)


def test_roofline_time_takes_the_slowest_pipe():
    seg = PM.Segment("x", conv_flops=2e12, act_flops=1e11, sines=0, bytes=1e9, tensor=True)
    # tensor 2e12 / 500e12 = 4 ms; fp32 1e11 / 50e12 = 2 ms; bytes 1e9 / 5000e9 = 0.2 ms
    assert PM.roofline_time(seg, 500.0, 50.0, 5000.0) == pytest.approx(4e-3)
    seg.tensor = False   # CUDA-core segment: both parts on the fp32 pipe
    assert PM.roofline_time(seg, 500.0, 50.0, 5000.0) == pytest.approx(2.1e12 / 50e12)


def test_fp32_peak_from_unit_counts():
    assert PM.fp32_peak_tflops(1965.0) == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)


def test_bench_launches_directly_under_a_profiler(monkeypatch):
    """bench.py replays decodes from CUDA graphs unless a profiler has injected itself into the
    CUDA runtime (Nsight Compute sets its transport variables in the program it starts)."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    for k in bench.PROFILER_ENV:
        monkeypatch.delenv(k, raising=False)
    assert bench.graphs_allowed()
    for k in bench.PROFILER_ENV:
        monkeypatch.setenv(k, "1")
        assert not bench.graphs_allowed(), k
        monkeypatch.delenv(k)
    assert bench.graphs_allowed()
