"""Algorithmic work of each decode segment and its roofline time (host-side bookkeeping).

Segments, in launch order: in_proj, conv_pre, then ups{i} and amp{i} for every stage, then
post (final activation + conv_post + clamp).  For each segment:
  * conv_flops  -- 2 x multiply-adds of the convolutions as defined (a transposed conv counts
                   2 * Cin * Cout * K per input sample; no zero-insertion work is counted);
  * act_flops   -- anti-aliased SnakeBeta: per channel-sample 24 (2x polyphase upsample, 6
                   taps per phase) + 8 (two SnakeBeta evaluations) + 24 (12-tap decimator) = 56
                   flops, plus 2 sines counted separately (SFU);
  * bytes       -- compulsory HBM traffic: input and output activations once, weights once
                   (fp32), plus the two extra residual-block outputs a fused mean reads.
Roofline time: the slower of the pipes the segment needs, with the activation on the fp32
CUDA-core pipe and the convolution on the tensor pipe (tensor-core segments) or on the same
fp32 pipe (CUDA-core segments, whose two parts therefore add):
  t_roof = max(conv / P_conv, act / P_fp32, bytes / BW)          (tensor-core segment)
  t_roof = max((conv + act) / P_fp32, bytes / BW)                (CUDA-core segment)
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass

import numpy as np

ACT_FLOPS = 56
ACT_SINES = 2
F32 = 4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@dataclass
class Segment:
    name: str
    conv_flops: float
    act_flops: float
    sines: float
    bytes: float
    tensor: bool = False

    @property
    def flops(self) -> float:
        return self.conv_flops + self.act_flops


def segments(arch, B: int, N: int, tc_stages=(), pre_tc: bool = False) -> list[Segment]:
    """Segments of one decode; `tc_stages` are the AMP stages whose convolutions run on the
    tensor cores, `pre_tc` whether conv_pre does."""
    out = []
    BN = B * N
    Cz, D, C0 = arch.latent_channels, arch.latent_dim, arch.decoder_dim
    out.append(Segment("in_proj", 2.0 * Cz * D * BN, 0, 0, F32 * ((Cz + D) * BN + Cz * D + D)))
    kp = getattr(arch, "conv_pre_kernel", 7)
    out.append(Segment("conv_pre", 2.0 * D * C0 * kp * BN, 0, 0,
                       F32 * ((D + C0) * BN + D * C0 * kp + C0), tensor=pre_tc))
    C, L = C0, N
    nrb = len(arch.rb_kernels)
    for i, (r, K) in enumerate(zip(arch.rates, arch.kernels)):
        Co = C // 2
        reads = 1 if i == 0 else nrb
        out.append(Segment(f"ups{i}", 2.0 * C * Co * K * L * B, 0, 0,
                           F32 * (reads * C * L * B + Co * L * r * B + C * Co * K + Co)))
        C, L = Co, L * r
        conv = 0.0
        wts = 0
        nact = 0
        for j, k in enumerate(arch.rb_kernels):
            nd = len(arch.rb_dilations[j])
            conv += 2 * nd * 2.0 * C * C * k * L * B
            wts += 2 * nd * (C * C * k + C) + 2 * nd * 2 * C
            nact += 2 * nd
        csl = C * L * B
        out.append(Segment(f"amp{i}", conv, nact * ACT_FLOPS * csl, nact * ACT_SINES * csl,
                           F32 * (2 * csl + wts), tensor=i in tc_stages))
    kq = getattr(arch, "conv_post_kernel", 7)
    out.append(Segment("post", 2.0 * C * kq * L * B, ACT_FLOPS * C * L * B, ACT_SINES * C * L * B,
                       F32 * (nrb * C * L * B + L * B + C * kq + 1)))
    return out


def measured_peaks() -> dict:
    """Measured peaks when present, else the recorded fallback figures."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0, "source": "fallback"}


def fp32_peak_tflops(sm_mhz: float, sms: int = 148) -> float:
    """fp32 FMA pipe: 128 lanes per SM, 2 flops per FMA."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def roofline_time(seg: Segment, p_conv_tflops: float, p_fp32_tflops: float, bw_gbs: float) -> float:
    tb = seg.bytes / (bw_gbs * 1e9)
    if seg.tensor:
        return max(seg.conv_flops / (p_conv_tflops * 1e12), seg.act_flops / (p_fp32_tflops * 1e12), tb)
    return max(seg.flops / (p_fp32_tflops * 1e12), tb)


def totals(segs) -> dict:
    return {"flops": float(sum(s.flops for s in segs)), "bytes": float(sum(s.bytes for s in segs)),
            "conv_flops": float(sum(s.conv_flops for s in segs))}


__all__ = ["Segment", "segments", "measured_peaks", "fp32_peak_tflops", "roofline_time", "totals",
           "np"]
