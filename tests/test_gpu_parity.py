"""GPU parity: the CUDA library (through its C ABI) against the fp64 CPU oracle, on the same
seeded inputs.

Tolerances (relative L2 = ||y - y_oracle|| / ||y_oracle||, on the pre-clamp waveform or the
stage output):
  * FP32 CUDA-core path: rel L2 <= 1e-5;
  * BF16X3 tensor-core path: rel L2 <= 2e-3, and max |y - y_oracle| <= 1e-2 both on the signal
    as computed (the pre-clamp waveform of a decode, or an AMP stage's output) and on the
    clamped waveform the caller receives.
The clamped waveform is also checked as clamp(pre-clamp) == clamped output, bit for bit, which
with the 1-Lipschitz clamp bounds its error by the pre-clamp error sample by sample.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from bigvgan_waveform_decoder_b200 import binding as Bd  # noqa: E402
from bigvgan_waveform_decoder_b200 import synthetic as S  # noqa: E402

pytestmark = pytest.mark.gpu

TOL = {Bd.MH3A_FP32: (1e-5, None), Bd.MH3A_BF16X3: (2e-3, 1e-2)}


def rel_l2(y, ref):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


def check(y, ref, precision, what="", waveform=False):
    """Relative L2 on the signal as computed (for a waveform: before the clamp).  The max-abs
    bound applies to the signal as computed and, for a waveform, also to the clamped output
    the caller receives (clamp(y) vs clamp(y_oracle); the clamp is 1-Lipschitz, so the second
    bound follows from the first, and is kept as the check of what a caller sees)."""
    rl, ma = TOL[precision]
    y = np.asarray(y, np.float64)
    r = rel_l2(y, ref)
    m_raw = float(np.max(np.abs(y - ref)))
    m = float(np.max(np.abs(np.clip(y, -1, 1) - np.clip(ref, -1, 1)))) if waveform else m_raw
    log = os.environ.get("MH3A_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"case": what, "precision": int(precision), "rel_l2": r,
                                "max_abs": m, "max_abs_preclamp": m_raw,
                                "ref_absmax": float(np.max(np.abs(ref)))}) + "\n")
    assert np.all(np.isfinite(y)), what
    assert r <= rl, f"{what}: rel L2 {r:.3e} > {rl:.1e} (max abs {m:.3e})"
    if ma is not None:
        assert m_raw <= ma, f"{what}: max abs {m_raw:.3e} > {ma:.1e} (rel L2 {r:.3e})"
        assert m <= ma, f"{what}: clamped max abs {m:.3e} > {ma:.1e} (rel L2 {r:.3e})"
    return r, m_raw


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(scope="module")
def full_weights():
    return S.workload_weights(0, S.Arch())


_decoders = {}


def decoder(arch, weights, precision, max_batch=2, max_frames=64, no_clamp=True, key=None):
    k = key or (id(weights), arch, precision, max_batch, max_frames, no_clamp)
    if k not in _decoders:
        _decoders[k] = Bd.Decoder(arch, weights, precision=precision, max_batch=max_batch,
                                  max_frames=max_frames, no_clamp=no_clamp)
    return _decoders[k]


# AMP stage sizes: several time tiles plus a ragged tail, oracle time a few seconds each
STAGE_CASES = [(0, 2, 150), (1, 2, 503), (2, 1, 2999), (3, 2, 3001), (4, 1, 10007), (5, 2, 9001),
               (6, 1, 40003)]


@pytest.mark.parametrize("stage,B,L", STAGE_CASES)
@pytest.mark.parametrize("precision", [Bd.MH3A_FP32, Bd.MH3A_BF16X3])
def test_amp_stage_matches_oracle(dev, full_weights, stage, B, L, precision):
    arch = S.Arch()
    C = arch.stage_channels(stage)
    x = S.make_stage_input(B, C, L, 100 + stage)
    ref = oracle.amp_stage(arch, full_weights, stage, x)
    d = decoder(arch, full_weights, precision, max_batch=2, max_frames=64)
    y = d.amp_stage(torch.from_numpy(x).to(dev), stage)
    torch.cuda.synchronize()
    d.check_device_error()
    if precision == Bd.MH3A_BF16X3:
        assert d.stage_uses_tensor_cores(stage)
    check(y.cpu().numpy(), ref, precision, f"stage {stage}")


@pytest.mark.parametrize("precision", [Bd.MH3A_FP32, Bd.MH3A_BF16X3])
def test_decode_small_matches_oracle(dev, full_weights, precision):
    """The B=1, N=4 workload (seed 0), pre-clamp and clamped."""
    arch, w, z = S.workload_inputs(0)
    ref = oracle.decode(arch, w, z, clamp=False)
    d = decoder(arch, w, precision, max_batch=2, max_frames=64, no_clamp=True)
    zt = torch.from_numpy(z).to(dev)
    y = d.decode(zt).cpu().numpy()
    check(y, ref, precision, "decode N=4", waveform=True)
    dc = decoder(arch, w, precision, max_batch=2, max_frames=64, no_clamp=False)
    yc = dc.decode(zt).cpu().numpy()
    d.check_device_error()
    dc.check_device_error()
    np.testing.assert_array_equal(yc, np.clip(y, -1.0, 1.0))
    assert yc.shape == (1, 1, 3200) and np.all(np.abs(yc) <= 1.0)


@pytest.mark.parametrize("precision", [Bd.MH3A_FP32, Bd.MH3A_BF16X3])
def test_decode_stereo_1s_matches_oracle(dev, precision):
    """The B=2, N=40 workload (1 s stereo, seed 2)."""
    arch, w, z = S.workload_inputs(2)
    ref = oracle.decode(arch, w, z, clamp=False)
    d = decoder(arch, w, precision, max_batch=2, max_frames=64, no_clamp=True)
    y = d.decode(torch.from_numpy(z).to(dev)).cpu().numpy()
    check(y, ref, precision, "decode B=2 N=40", waveform=True)


@pytest.mark.parametrize("N", [1, 2, 3, 7])
def test_decode_short_and_ragged(dev, full_weights, N):
    arch = S.Arch()
    z = S.make_latents(1, N, 32, 50 + N)
    ref = oracle.decode(arch, full_weights, z, clamp=False)
    d = decoder(arch, full_weights, Bd.MH3A_FP32, max_batch=2, max_frames=64)
    y = d.decode(torch.from_numpy(z).to(dev)).cpu().numpy()
    assert y.shape == (1, 1, 800 * N)
    check(y, ref, Bd.MH3A_FP32, f"decode N={N}", waveform=True)


def test_batch_independence_and_determinism(dev, full_weights):
    arch = S.Arch()
    z = S.make_latents(2, 5, 32, 77)
    d = decoder(arch, full_weights, Bd.MH3A_BF16X3, max_batch=2, max_frames=64)
    zt = torch.from_numpy(z).to(dev)
    y2 = d.decode(zt).cpu().numpy()
    y2b = d.decode(zt).cpu().numpy()
    np.testing.assert_array_equal(y2, y2b)
    for b in range(2):
        y1 = d.decode(zt[b:b + 1].contiguous()).cpu().numpy()
        np.testing.assert_array_equal(y1[0], y2[b])


@pytest.mark.parametrize("prec", [Bd.MH3A_FP32, Bd.MH3A_BF16X3], ids=["FP32", "BF16X3"])
@pytest.mark.parametrize("out_kind", ["pinned", "pinned_odd_offset", "pageable"])
def test_decode_host_matches_device(dev, full_weights, prec, out_kind):
    """Host-buffer decode == device decode bit for bit, whether the waveform reaches host memory
    through the last kernel's direct stores (pinned output, also 4 bytes off an 8-byte boundary)
    or through a copy (pageable output)."""
    arch = S.Arch()
    z = S.make_latents(2, 6, 32, 78)
    d = decoder(arch, full_weights, prec, max_batch=2, max_frames=64)
    yd = d.decode(torch.from_numpy(z).to(dev)).cpu().numpy()
    zp = torch.from_numpy(z).pin_memory()
    n = 2 * 800 * 6
    if out_kind == "pinned":
        yp = torch.full((2, 1, 800 * 6), float("nan"), dtype=torch.float32).pin_memory()
    elif out_kind == "pinned_odd_offset":
        big = torch.full((n + 1,), float("nan"), dtype=torch.float32).pin_memory()
        yp = big[1:].view(2, 1, 800 * 6)
        assert yp.data_ptr() % 8 == 4
    else:
        yp = torch.full((2, 1, 800 * 6), float("nan"), dtype=torch.float32)
    d.decode_host(zp, yp)
    np.testing.assert_array_equal(yp.numpy(), yd)
    if out_kind == "pinned_odd_offset":
        assert np.isnan(big[0].item())   # nothing written before the buffer


def test_denormalised_decode(dev, full_weights):
    """Per-channel latents_mean/std folded into the input projection."""
    mean, std = S.make_denorm(32, 4)
    arch = S.Arch(latents_mean=mean, latents_std=std)
    z = S.make_latents(2, 3, 32, 4)
    ref = oracle.decode(arch, full_weights, z, clamp=False)
    d = Bd.Decoder(arch, full_weights, precision=Bd.MH3A_FP32, max_batch=2, max_frames=8,
                   no_clamp=True)
    y = d.decode(torch.from_numpy(z).to(dev)).cpu().numpy()
    check(y, ref, Bd.MH3A_FP32, "denormalised decode", waveform=True)
    d.close()


def test_shape_limits_are_enforced(dev, full_weights):
    arch = S.Arch()
    d = decoder(arch, full_weights, Bd.MH3A_FP32, max_batch=2, max_frames=64)
    z = torch.zeros((3, 32, 4), device=dev)
    with pytest.raises(Bd.MH3AError) as e:
        d.decode(z)
    assert e.value.status == 3
    z = torch.zeros((1, 32, 65), device=dev)
    with pytest.raises(Bd.MH3AError):
        d.decode(z)
    x = torch.zeros((2, 512, 64 * 2 * 5 * 2), device=dev)
    with pytest.raises(Bd.MH3AError):
        d.amp_stage(x, 0)


def test_launch_counter_counts_kernels(dev, full_weights):
    arch = S.Arch()
    d = decoder(arch, full_weights, Bd.MH3A_BF16X3, max_batch=2, max_frames=64)
    before = d.launch_count()
    d.decode(torch.zeros((1, 32, 2), device=dev))
    torch.cuda.synchronize()
    n = d.launch_count() - before
    assert 10 <= n <= 128
