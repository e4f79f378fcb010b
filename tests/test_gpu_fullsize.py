"""GPU parity at the full benchmark sizes, on outputs the oracle can compute window by window.

Every output sample of the decode depends only on latents within its receptive field: about
+-31 latent frames (stage 0's residual blocks alone reach +-90 samples at 5 samples per frame).
The oracle therefore decodes a window of latent frames around the samples under test; the
samples farther than the receptive field from the window's cut edges are exact (a true
sequence end is not a cut edge).  Likewise one AMP stage reaches +-90 samples of its input.

The GPU runs the full workload in the launch configuration bench.py times.  Tolerances are
those of the tensor-core path (rel L2 <= 2e-3, max abs <= 1e-2), on the pre-clamp waveform.
"""
from __future__ import annotations

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from bigvgan_waveform_decoder_b200 import binding as Bd  # noqa: E402
from bigvgan_waveform_decoder_b200 import synthetic as S  # noqa: E402
from tests.test_gpu_parity import check  # noqa: E402

pytestmark = pytest.mark.gpu

RF_FRAMES = 32          # receptive-field radius of the decode, in latent frames (rounded up)
RF_STAGE = 96           # receptive-field radius of one AMP stage, in samples (rounded up)
HOP = 800


def windows(N, n_mid=1):
    """(lo, hi, keep_lo, keep_hi) latent-frame windows: the sequence start, middle(s), end."""
    w = 2 * RF_FRAMES + 4
    out = [(0, w, 0, w - RF_FRAMES)]
    for k in range(n_mid):
        c = (k + 1) * N // (n_mid + 1)
        out.append((c - w // 2, c + w // 2, c - w // 2 + RF_FRAMES, c + w // 2 - RF_FRAMES))
    out.append((N - w, N, N - w + RF_FRAMES, N))
    return out


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _decode_windows(dev, index, items):
    arch, w, z = S.workload_inputs(index)
    B, _, N = z.shape
    d = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=B, max_frames=N, no_clamp=True)
    y = d.decode(torch.from_numpy(z).to(dev)).cpu().numpy()
    d.check_device_error()
    d.close()
    assert y.shape == (B, 1, HOP * N)
    for b in items:
        for lo, hi, klo, khi in windows(N):
            ref = oracle.decode(arch, w, z[b:b + 1, :, lo:hi], clamp=False)[0, 0]
            seg = ref[(klo - lo) * HOP:(khi - lo) * HOP]
            got = y[b, 0, klo * HOP:khi * HOP]
            check(got, seg, Bd.MH3A_BF16X3, f"workload {index} item {b} frames {klo}-{khi}",
                  waveform=True)


def test_decode_10s_stereo_sampled(dev):
    """B=2, N=400 (the bench workload): windows at the start, middle and end of both items."""
    _decode_windows(dev, 3, items=(0, 1))


def test_decode_20s_batched_denormalised_sampled(dev):
    """B=16, N=800 with per-channel latent denormalisation: items 0 and 15."""
    _decode_windows(dev, 4, items=(0, 15))


def test_amp_stage0_full_size_sampled(dev):
    """The single-AMP-stage workload: x [2, 512, 2000], stage 0."""
    arch, w, x = S.workload_inputs(1)
    B, C, L = x.shape
    d = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=2, max_frames=200)
    y = d.amp_stage(torch.from_numpy(x).to(dev), 0).cpu().numpy()
    d.check_device_error()
    d.close()
    width = 2 * RF_STAGE + 64
    for b in range(B):
        for lo in (0, L // 2 - width // 2, L - width):
            hi = lo + width
            ref = oracle.amp_stage(arch, w, 0, x[b:b + 1, :, lo:hi])[0]
            klo = lo if lo == 0 else lo + RF_STAGE
            khi = hi if hi == L else hi - RF_STAGE
            check(y[b, :, klo:khi], ref[:, klo - lo:khi - lo], Bd.MH3A_BF16X3,
                  f"AMP stage 0 item {b} samples {klo}-{khi}")


@pytest.mark.parametrize("B,N", [(2, 7), (1, 1)])
def test_decode_bench_arch_short_odd_lengths(dev, B, N):
    """The bench architecture at short, odd latent lengths, compared over the whole output.  Every
    tile of every tensor-core kernel is a ragged edge tile here: the split-K conv_pre and the
    projection fused into its operand split, odd-length upsampler input splits (no paired
    loads), the grouped rate-5 upsamplers and the fused activation_post + conv_post."""
    arch = S.Arch()
    w = S.workload_weights(3, arch)
    z = S.make_latents(B, N, arch.latent_channels, 11)
    d = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=B, max_frames=N, no_clamp=True)
    y = d.decode(torch.from_numpy(z).to(dev)).cpu().numpy()
    d.check_device_error()
    d.close()
    assert y.shape == (B, 1, HOP * N)
    ref = oracle.decode(arch, w, z, clamp=False)
    for b in range(B):
        check(y[b, 0], ref[b, 0], Bd.MH3A_BF16X3, f"bench arch B={B} N={N} item {b}", waveform=True)
