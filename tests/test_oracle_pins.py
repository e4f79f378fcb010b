"""Pins of the fp64 CPU oracle against things other than itself.

Each test checks one oracle function against a closed form, a brute-force definition, an
invariant of the method, or an independent library routine (numpy / scipy / torch fp64),
chosen so that a dropped term, a wrong sign or index, or a transposed operand fails.

Sources: FastVideo "minimax_h3_audio_vae" page (``MLXMiniMaxH3AudioVAE.decode``,
``kaiser_sinc_filter1d``); diffusers "AutoencoderKLMiniMaxH3Audio" page (``decode``:
output ``[B,1,800N]`` clamped to [-1,1]; stereo as batch items); diffusers
"AutoencoderKLMiniMaxH3" page (per-channel denormalisation).
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest
import scipy.signal as ss
import scipy.special as sp
import torch
import torch.nn.functional as F

import oracle
from bigvgan_waveform_decoder_b200 import synthetic as S
from tests import lib_ref

HERE = os.path.dirname(os.path.abspath(__file__))
pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def rng(seed=0):
    return np.random.Generator(np.random.PCG64(seed))


# ------------------------------------------------------------------------------------------
# Kaiser-sinc filter (MLX page, kaiser_sinc_filter1d)
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("x", [0.0, 1e-3, 0.5, 1.0, 4.6638, 10.0, 30.0])
def test_bessel_i0_matches_scipy(x):
    assert oracle.bessel_i0(x) == pytest.approx(float(sp.i0(x)), rel=1e-14)


@pytest.mark.parametrize("K,cutoff,hw", [(12, 0.25, 0.3), (11, 0.25, 0.3), (24, 0.125, 0.15),
                                         (12, 0.2, 0.1)])
def test_kaiser_sinc_matches_scipy_firwin(K, cutoff, hw):
    """The page's design is the Kaiser windowed-sinc FIR that scipy.signal.firwin implements
    (window * 2fc sinc(2fc t), normalised to unit DC gain); Kaiser's attenuation/beta rules
    are scipy's kaiser_atten / kaiser_beta with numtaps K/2 and width 4*half_width."""
    taps, A, beta = oracle.kaiser_sinc_filter(cutoff, hw, K)
    A_ref = ss.kaiser_atten(K // 2, 4 * hw)
    assert A == pytest.approx(A_ref, rel=1e-14)
    assert beta == pytest.approx(ss.kaiser_beta(A_ref), rel=1e-14, abs=1e-15)
    ref = ss.firwin(K, cutoff, window=("kaiser", ss.kaiser_beta(A_ref)), fs=1.0)
    np.testing.assert_allclose(taps, ref, rtol=0, atol=1e-14)


def test_kaiser_sinc_invariants():
    taps, A, beta = oracle.kaiser_sinc_filter(0.25, 0.3, 12)
    # Kaiser design values at the activation's parameters
    assert A == pytest.approx(2.285 * 5 * math.pi * 1.2 + 7.95, rel=1e-15)
    assert A > 50 and beta == pytest.approx(0.1102 * (A - 8.7), rel=1e-15)
    # symmetric, unit DC gain
    np.testing.assert_allclose(taps, taps[::-1], atol=0)
    assert taps.sum() == pytest.approx(1.0, abs=1e-15)
    # the two polyphase halves of a symmetric even-length filter are mirror images of each
    # other, so each carries exactly half the DC gain: the 2x upsampler's gain of 2 restores
    # a constant exactly
    assert taps[0::2].sum() == pytest.approx(0.5, abs=1e-15)
    assert taps[1::2].sum() == pytest.approx(0.5, abs=1e-15)
    # a low-pass at a quarter of the sample rate: ~1 near DC, strongly attenuated near Nyquist
    w, H = ss.freqz(taps, worN=[0.0, 0.02 * np.pi, 0.9 * np.pi, np.pi])
    assert abs(H[0]) == pytest.approx(1.0, abs=1e-14)
    assert abs(H[1]) == pytest.approx(1.0, abs=1e-3)
    assert abs(H[2]) < 1e-2 and abs(H[3]) < 1e-2


def test_kaiser_sinc_golden_fixture():
    """Stored taps (written by tests/golden/make_golden.py from the oracle) must match a fresh
    scipy design, so the fixture itself is pinned by a library routine."""
    path = os.path.join(HERE, "golden", "kaiser_sinc_k12_c0.25_hw0.3.txt")
    vals = np.loadtxt(path)
    np.testing.assert_allclose(vals, lib_ref.lib_filter(), atol=1e-15)
    np.testing.assert_allclose(vals, oracle.kaiser_sinc_filter(0.25, 0.3, 12)[0], atol=0)


# ------------------------------------------------------------------------------------------
# weight norm (MLX page, _wn_weight(weight_v, weight_g))
# ------------------------------------------------------------------------------------------

def test_weight_norm_conv_matches_torch():
    r = rng(1)
    v = r.standard_normal((6, 5, 3)).astype(np.float32)
    g = r.uniform(0.5, 2.0, (6, 1, 1)).astype(np.float32)
    w = oracle.weight_norm(v, g)
    ref = torch._weight_norm(torch.as_tensor(v, dtype=torch.float64),
                             torch.as_tensor(g, dtype=torch.float64), 0).numpy()
    np.testing.assert_allclose(w, ref, rtol=1e-14, atol=1e-15)
    # ||w_o|| = g_o over (in, k), per output channel
    np.testing.assert_allclose(np.linalg.norm(w.reshape(6, -1), axis=1), g.reshape(-1),
                               rtol=1e-12)


def test_weight_norm_transposed_conv_is_per_input_channel():
    """A ConvTranspose1d weight is stored [in, out, k]; torch's weight_norm (dim 0) on that
    module normalises per input channel -- the stored tensor's first axis."""
    torch.manual_seed(0)
    m = torch.nn.ConvTranspose1d(4, 3, 5).double()
    m = torch.nn.utils.parametrizations.weight_norm(m, name="weight", dim=0)
    with torch.no_grad():
        m.parametrizations.weight.original0.uniform_(0.5, 2.0)
    g = m.parametrizations.weight.original0.detach().numpy().astype(np.float32)
    v = m.parametrizations.weight.original1.detach().numpy().astype(np.float32)
    w = oracle.weight_norm(v, g)
    ref = torch._weight_norm(torch.as_tensor(v, dtype=torch.float64),
                             torch.as_tensor(g, dtype=torch.float64), 0).numpy()
    np.testing.assert_allclose(w, ref, rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(w.reshape(4, -1), axis=1), g.reshape(-1), rtol=1e-12)


def test_weight_norm_identity_and_zero():
    r = rng(2)
    v = r.standard_normal((3, 4, 2)).astype(np.float32)
    g = np.linalg.norm(v.astype(np.float64).reshape(3, -1), axis=1).astype(np.float32)
    w = oracle.weight_norm(v, g)
    np.testing.assert_allclose(w, v, rtol=1e-6)  # g = ||v|| (to fp32) gives w = v
    w0 = oracle.weight_norm(v, np.zeros(3, np.float32))
    assert np.all(w0 == 0.0)


# ------------------------------------------------------------------------------------------
# convolutions (MLX page, _conv1d / _conv_transpose1d)
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("Cin,Cout,K,stride,pad,dil,L", [
    (3, 4, 1, 1, 0, 1, 9), (5, 2, 3, 1, 1, 1, 17), (4, 4, 7, 1, 3, 1, 12),
    (2, 3, 11, 1, 25, 5, 40), (3, 3, 3, 1, 5, 5, 7), (2, 2, 12, 2, 0, 1, 31),
    (3, 2, 7, 1, 3, 1, 2),
])
def test_conv1d_matches_torch(Cin, Cout, K, stride, pad, dil, L):
    r = rng(3)
    x = r.standard_normal((Cin, L))
    w = r.standard_normal((Cout, Cin, K))
    b = r.standard_normal(Cout)
    y = oracle.conv1d(x, w, b, stride=stride, pad=pad, dil=dil)
    ref = F.conv1d(torch.as_tensor(x)[None], torch.as_tensor(w), torch.as_tensor(b),
                   stride=stride, padding=pad, dilation=dil)[0].numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def _convT_brute(x, w, stride, pad):
    """Insert stride-1 zeros between samples, pad K-1-pad zeros each side, correlate with the
    flipped kernel transposed to [out, in, k]."""
    Cin, L = x.shape
    _, Cout, K = w.shape
    z = np.zeros((Cin, (L - 1) * stride + 1))
    z[:, ::stride] = x
    q = K - 1 - pad
    z = np.pad(z, ((0, 0), (q, q)))
    wf = np.transpose(w, (1, 0, 2))[:, :, ::-1]
    Lout = z.shape[1] - K + 1
    y = np.zeros((Cout, Lout))
    for o in range(Cout):
        for c in range(Cin):
            y[o] += np.correlate(z[c], wf[o, c], mode="valid")
    return y


@pytest.mark.parametrize("r,K", [(5, 9), (2, 4), (3, 3), (4, 8)])
def test_conv_transpose1d_brute_force_and_torch(r, K):
    rg = rng(4)
    pad = (K - r) // 2
    for Cin, Cout, L in [(3, 2, 1), (4, 3, 7), (2, 5, 13)]:
        x = rg.standard_normal((Cin, L))
        w = rg.standard_normal((Cin, Cout, K))
        y = oracle.conv_transpose1d(x, w, None, stride=r, pad=pad)
        np.testing.assert_allclose(y, _convT_brute(x, w, r, pad), rtol=1e-12, atol=1e-12)
        ref = F.conv_transpose1d(torch.as_tensor(x)[None], torch.as_tensor(w), stride=r,
                                 padding=pad)[0].numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
        if (K - r) % 2 == 0:
            assert y.shape[1] == L * r  # padding (K-r)/2 gives exactly r samples per input


# ------------------------------------------------------------------------------------------
# SnakeBeta closed form
# ------------------------------------------------------------------------------------------

def test_snake_beta_closed_form():
    a, b = 1.3, 0.9
    x = np.array([0.0, math.pi / 2 / a, math.pi / a, 7 * math.pi / a, -3 * math.pi / 2 / a])
    y = oracle.snake_beta(x, a, b)
    inv = 1.0 / (b + 1e-9)
    assert y[0] == 0.0
    assert y[1] == pytest.approx(x[1] + inv, rel=1e-15)          # sin^2(pi/2) = 1
    assert y[2] == pytest.approx(x[2], abs=1e-14)                 # sin^2(k pi) = 0
    assert y[3] == pytest.approx(x[3], abs=1e-13)
    assert y[4] == pytest.approx(x[4] + inv, rel=1e-14)
    # small alpha: x + alpha^2 x^2 / beta
    xs = np.linspace(-2, 2, 9)
    ys = oracle.snake_beta(xs, 1e-4, b)
    np.testing.assert_allclose(ys - xs, (1e-4 * xs) ** 2 / (b + 1e-9), rtol=1e-6, atol=1e-20)
    # alpha = 0: identity
    np.testing.assert_array_equal(oracle.snake_beta(xs, 0.0, b), xs)


# ------------------------------------------------------------------------------------------
# anti-aliased activation (MLX page, _activation1d; readings of the up/down samplers)
# ------------------------------------------------------------------------------------------

def _up_brute(x, taps):
    """Replicate-pad 5, zero-stuff by 2, full convolution with the taps, gain 2, crop 15."""
    xp = np.pad(x, 5, mode="edge")
    z = np.zeros(2 * xp.size - 1)
    z[::2] = xp
    full = 2.0 * np.convolve(z, taps)
    return full[15:15 + 2 * x.size]


def test_upsample2_brute_force_and_torch():
    taps = oracle.act_taps()
    r = rng(5)
    for L in (1, 2, 3, 6, 17):
        x = r.standard_normal(L)
        u = oracle.upsample2(x, taps)
        np.testing.assert_allclose(u, _up_brute(x, taps), rtol=1e-13, atol=1e-14)
        t = torch.as_tensor(x).view(1, 1, L)
        ref = 2.0 * F.conv_transpose1d(F.pad(t, (5, 5), mode="replicate"),
                                       torch.as_tensor(taps).view(1, 1, 12), stride=2)
        np.testing.assert_allclose(u, ref[0, 0, 15:-15].numpy(), rtol=1e-13, atol=1e-14)


def test_downsample2_matches_torch():
    taps = oracle.act_taps()
    r = rng(6)
    for L2 in (2, 4, 10, 34):
        s = r.standard_normal(L2)
        y = oracle.downsample2(s, taps)
        t = torch.as_tensor(s).view(1, 1, L2)
        ref = F.conv1d(F.pad(t, (5, 6), mode="replicate"), torch.as_tensor(taps).view(1, 1, 12),
                       stride=2)[0, 0].numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-14)
        assert y.size == L2 // 2


def test_activation_constant_and_low_frequency():
    taps = oracle.act_taps()
    # alpha = 0: SnakeBeta is the identity; a constant passes unchanged, edges included
    c = np.full(37, 0.731)
    np.testing.assert_allclose(oracle.activation1d(c, 0.0, 1.0, taps), c, rtol=1e-6)
    # the same with fp64 taps is exact up to rounding (polyphase halves sum to 1/2 each)
    t64, _, _ = oracle.kaiser_sinc_filter(0.25, 0.3, 12)
    np.testing.assert_allclose(oracle.activation1d(c, 0.0, 1.0, t64), c, rtol=1e-14)
    # tiny alpha ~ identity
    np.testing.assert_allclose(oracle.activation1d(c, 1e-7, 1.0, t64), c, rtol=1e-12)
    # a slow sinusoid passes with gain ~ 1 away from the edges
    n = np.arange(400)
    x = np.sin(2 * np.pi * 0.01 * n)
    y = oracle.activation1d(x, 0.0, 1.0, t64)
    np.testing.assert_allclose(y[20:-20], x[20:-20], atol=2e-3)


def test_activation_matches_library_composition():
    taps = oracle.act_taps()
    r = rng(7)
    x = 3.0 * r.standard_normal((1, 3, 29))
    alpha = [0.9, 1.1, 1.2]
    beta = [1.05, 0.85, 1.0]
    ref = lib_ref.act(torch.as_tensor(x), alpha, beta, torch.as_tensor(taps)).numpy()[0]
    for c in range(3):
        y = oracle.activation1d(x[0, c], alpha[c], beta[c], taps)
        np.testing.assert_allclose(y, ref[c], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------------------------------
# AMP stage and decode (MLX page, MLXMiniMaxH3AudioVAE.decode)
# ------------------------------------------------------------------------------------------

def test_amp_stage_matches_library_composition(small_arch):
    w = S.make_weights(small_arch, 11)
    for stage, L in [(0, 23), (3, 40), (6, 9)]:
        C = small_arch.stage_channels(stage)
        x = S.make_stage_input(2, C, L, 5 + stage)
        y = oracle.amp_stage(small_arch, w, stage, x)
        ref = lib_ref.stage_amp(small_arch, w, stage, x.astype(np.float64))
        np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-10)


def test_amp_stage_zero_weights_is_identity(small_arch):
    w = dict(S.make_weights(small_arch, 12))
    for k in list(w):
        if ".resblocks." in k and (k.endswith("weight_g") or k.endswith(".bias")):
            w[k] = np.zeros_like(w[k])
    x = S.make_stage_input(1, small_arch.stage_channels(2), 31, 3)
    y = oracle.amp_stage(small_arch, w, 2, x)
    np.testing.assert_array_equal(y, x.astype(np.float64))


def test_decode_matches_library_composition(small_arch):
    w = S.make_weights(small_arch, 13)
    z = S.make_latents(2, 5, small_arch.latent_channels, 13)
    y = oracle.decode(small_arch, w, z, clamp=False)
    ref = lib_ref.decode(small_arch, w, z, clamp=False)
    assert y.shape == (2, 1, 800 * 5)
    scale = np.abs(ref).max()
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-10 * scale)


def test_decode_default_arch_matches_library_composition():
    """Full-width default architecture, one short item (the B=1, N=4 workload)."""
    arch, w, z = S.workload_inputs(0)
    y = oracle.decode(arch, w, z, clamp=False)
    ref = lib_ref.decode(arch, w, z, clamp=False)
    scale = np.abs(ref).max()
    np.testing.assert_allclose(y, ref, rtol=1e-9, atol=1e-11 * scale)
    yc = oracle.decode(arch, w, z, clamp=True)
    np.testing.assert_array_equal(yc, np.clip(y, -1.0, 1.0))


@pytest.mark.parametrize("n", [1, 2, 3, 4, 40])
def test_decode_length_is_800n(small_arch, n):
    w = S.make_weights(small_arch, 14)
    z = S.make_latents(1, n, small_arch.latent_channels, n)
    y = oracle.decode(small_arch, w, z)
    assert y.shape == (1, 1, 800 * n)
    assert np.all(np.abs(y) <= 1.0)


def test_decode_batch_independence(small_arch):
    """Stereo is carried as two batch items that decode independently (bit-exact)."""
    w = S.make_weights(small_arch, 15)
    z = S.make_latents(3, 4, small_arch.latent_channels, 15)
    y = oracle.decode(small_arch, w, z, clamp=False)
    for b in range(3):
        yb = oracle.decode(small_arch, w, z[b:b + 1], clamp=False)
        np.testing.assert_array_equal(y[b], yb[0])


def test_decode_shift_equivariance(small_arch):
    """Shifting the latents by one frame shifts the waveform by one hop (800 samples),
    away from the replicate/zero-padded ends."""
    w = S.make_weights(small_arch, 16)
    # the receptive field spans about +-31 latent frames (stage 0's residual blocks alone
    # reach +-90 samples at 5 samples per frame), so compare frames 34..65 of 100
    z = S.make_latents(1, 101, small_arch.latent_channels, 16)
    y0 = oracle.decode(small_arch, w, z[:, :, :-1], clamp=False)
    y1 = oracle.decode(small_arch, w, z[:, :, 1:], clamp=False)
    # a one-frame shift: y1[t] = y0[t + 800] in the interior
    lo, hi = 34 * 800, 65 * 800
    np.testing.assert_allclose(y1[0, 0, lo:hi], y0[0, 0, lo + 800:hi + 800], rtol=1e-12,
                               atol=1e-12 * np.abs(y0).max())


def test_decode_linear_without_snake_and_bias(small_arch):
    w = dict(S.make_weights(small_arch, 17))
    for k in list(w):
        if k.endswith(".alpha"):
            w[k] = np.zeros_like(w[k])
        if k.endswith(".bias"):
            w[k] = np.zeros_like(w[k])
    # inputs on disjoint channels and power-of-two scales, so the combined fp32 input is exact
    za = S.make_latents(1, 3, small_arch.latent_channels, 1)
    zb = S.make_latents(1, 3, small_arch.latent_channels, 2)
    za[:, 2:] = 0.0
    zb[:, :2] = 0.0
    ya = oracle.decode(small_arch, w, za, clamp=False)
    yb = oracle.decode(small_arch, w, zb, clamp=False)
    yab = oracle.decode(small_arch, w, 0.5 * za + 2.0 * zb, clamp=False)
    np.testing.assert_allclose(yab, 0.5 * ya + 2.0 * yb, rtol=1e-9,
                               atol=1e-11 * np.abs(yab).max())


def test_decode_denormalisation(small_arch):
    """decode with latents_mean/std == decode of (x * std + mean) without them."""
    mean, std = S.make_denorm(small_arch.latent_channels, 3)
    arch_dn = S.Arch(**{**small_arch.__dict__, "latents_mean": mean, "latents_std": std})
    w = S.make_weights(small_arch, 18)
    z = S.make_latents(2, 3, small_arch.latent_channels, 18)
    y = oracle.decode(arch_dn, w, z, clamp=False)
    zd = z.astype(np.float64) * np.array(std)[None, :, None] + np.array(mean)[None, :, None]
    ref = lib_ref.decode(small_arch, w, zd, clamp=False)
    np.testing.assert_allclose(y, ref, rtol=1e-9, atol=1e-10 * np.abs(ref).max())


def test_decode_clamp_and_nan():
    """Clamp is inclusive at +-1 and lets NaN through (checked on a tiny synthetic tail)."""
    arch = S.Arch(latent_channels=2, latent_dim=8, decoder_dim=128)
    w = dict(S.make_weights(arch, 19))
    w["decoder.conv_post.bias"] = np.array([5.0], np.float32)
    w["decoder.conv_post.weight_g"] = np.zeros((1, 1, 1), np.float32)
    z = S.make_latents(1, 1, 2, 19)
    y = oracle.decode(arch, w, z)
    assert np.all(y == 1.0)
    w["decoder.conv_post.bias"] = np.array([np.nan], np.float32)
    assert np.all(np.isnan(oracle.decode(arch, w, z)))


def test_missing_and_misshaped_weights_raise(small_arch):
    w = dict(S.make_weights(small_arch, 20))
    z = S.make_latents(1, 1, small_arch.latent_channels, 0)
    bad = dict(w)
    del bad["decoder.conv_pre.weight_g"]
    with pytest.raises(RuntimeError, match="missing"):
        oracle.decode(small_arch, bad, z)
    bad = dict(w)
    bad["decoder.ups.2.0.weight_v"] = bad["decoder.ups.2.0.weight_v"][:, :, :3].copy()
    with pytest.raises(RuntimeError, match="shape"):
        oracle.decode(small_arch, bad, z)
