"""An independent restatement of the decode as a composition of library routines.

Used only to pin the oracle (tests/test_oracle_pins.py): every convolution here is
``torch.nn.functional`` in fp64 on the CPU, the weight norm is torch's ``_weight_norm``,
the filter is ``scipy.signal.firwin`` with a Kaiser window, and the padding is
``F.pad(mode="replicate")``.  It shares no code with the oracle's C loops, so an index,
sign or transposition mistake in either one shows up as a mismatch.

Sources: FastVideo "minimax_h3_audio_vae" page, ``MLXMiniMaxH3AudioVAE.decode`` (block
wiring) and ``kaiser_sinc_filter1d`` (filter design); diffusers "AutoencoderKLMiniMaxH3Audio"
page (constructor defaults).  The block body and activation details follow the same readings
as the oracle (listed in the design notes).
"""
from __future__ import annotations

import math

import numpy as np
import scipy.signal as ss
import torch
import torch.nn.functional as F


def lib_filter(K: int = 12, cutoff: float = 0.25, half_width: float = 0.3) -> np.ndarray:
    """Kaiser windowed-sinc low-pass designed by scipy (firwin), Kaiser beta by scipy."""
    atten = ss.kaiser_atten(K // 2, 4 * half_width)
    beta = ss.kaiser_beta(atten)
    return ss.firwin(K, cutoff, window=("kaiser", beta), fs=1.0)


def _t(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float64))


def wn(v, g) -> torch.Tensor:
    v = _t(v)
    g = _t(g).reshape(-1, *([1] * (v.dim() - 1)))
    return torch._weight_norm(v, g, 0)


def act(x: torch.Tensor, alpha, beta, taps: torch.Tensor) -> torch.Tensor:
    """x [B, C, L]; 2x upsample (replicate pad 5, transposed conv, gain 2, crop 15/15),
    SnakeBeta, 2x low-pass decimation (replicate pad 5/6, stride-2 conv)."""
    B, Cc, L = x.shape
    K = taps.numel()
    f = taps.view(1, 1, K).expand(Cc, 1, K)
    xp = F.pad(x, (K // 2 - 1, K // 2 - 1), mode="replicate")
    u = 2.0 * F.conv_transpose1d(xp, f, stride=2, groups=Cc)
    u = u[..., 15:-15]
    a = _t(alpha).view(1, -1, 1)
    b = _t(beta).view(1, -1, 1)
    s = u + torch.sin(a * u) ** 2 / (b + 1e-9)
    sp = F.pad(s, (K // 2 - 1, K // 2), mode="replicate")
    return F.conv1d(sp, f, stride=2, groups=Cc)


def amp_stage(arch, w: dict, stage: int, h: torch.Tensor, taps: torch.Tensor) -> torch.Tensor:
    nrb = len(arch.rb_kernels)
    acc = torch.zeros_like(h)
    for j, k in enumerate(arch.rb_kernels):
        rb = f"decoder.resblocks.{stage * nrb + j}"
        x = h
        for m, d in enumerate(arch.rb_dilations[j]):
            p1, p2 = f"{rb}.convs1.{m}", f"{rb}.convs2.{m}"
            t = act(x, w[f"{rb}.activations.{2 * m}.act.alpha"],
                    w[f"{rb}.activations.{2 * m}.act.beta"], taps)
            t = F.conv1d(t, wn(w[p1 + ".weight_v"], w[p1 + ".weight_g"]), _t(w[p1 + ".bias"]),
                         padding=d * (k - 1) // 2, dilation=d)
            t = act(t, w[f"{rb}.activations.{2 * m + 1}.act.alpha"],
                    w[f"{rb}.activations.{2 * m + 1}.act.beta"], taps)
            t = F.conv1d(t, wn(w[p2 + ".weight_v"], w[p2 + ".weight_g"]), _t(w[p2 + ".bias"]),
                         padding=(k - 1) // 2)
            x = x + t
        acc = acc + x
    return acc / nrb


def decode(arch, w: dict, latents, clamp: bool = True) -> np.ndarray:
    taps = torch.as_tensor(lib_filter().astype(np.float32).astype(np.float64))
    z = _t(latents)
    if arch.latents_std is not None:
        z = z * _t(arch.latents_std).view(1, -1, 1)
    if arch.latents_mean is not None:
        z = z + _t(arch.latents_mean).view(1, -1, 1)
    h = F.conv1d(z, _t(w["dec_in_proj.weight"]), _t(w["dec_in_proj.bias"]))
    h = F.conv1d(h, wn(w["decoder.conv_pre.weight_v"], w["decoder.conv_pre.weight_g"]),
                 _t(w["decoder.conv_pre.bias"]), padding=3)
    for i, (r, K) in enumerate(zip(arch.rates, arch.kernels)):
        p = f"decoder.ups.{i}.0"
        h = F.conv_transpose1d(h, wn(w[p + ".weight_v"], w[p + ".weight_g"]), _t(w[p + ".bias"]),
                               stride=r, padding=(K - r) // 2)
        h = amp_stage(arch, w, i, h, taps)
    h = act(h, w["decoder.activation_post.act.alpha"], w["decoder.activation_post.act.beta"], taps)
    bias = w.get("decoder.conv_post.bias")
    h = F.conv1d(h, wn(w["decoder.conv_post.weight_v"], w["decoder.conv_post.weight_g"]),
                 _t(bias) if bias is not None else None, padding=3)
    if clamp:
        h = torch.clamp(h, -1.0, 1.0)
    return h.numpy()


def stage_amp(arch, w: dict, stage: int, x) -> np.ndarray:
    taps = torch.as_tensor(lib_filter().astype(np.float32).astype(np.float64))
    return amp_stage(arch, w, stage, _t(x), taps).numpy()


__all__ = ["lib_filter", "wn", "act", "decode", "stage_amp", "math"]
