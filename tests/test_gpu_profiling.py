"""The timing entry points bench.py builds on: per-segment events (mh3a_set_profiling /
mh3a_segment_times), per-kernel events of one AMP stage (mh3a_set_kernel_profiling /
mh3a_stage_kernel_times) and the tensor-core queries.  The events must not change the decode's
output, and the times they report must be consistent with the whole decode's."""
from __future__ import annotations

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from bigvgan_waveform_decoder_b200 import binding as Bd  # noqa: E402
from bigvgan_waveform_decoder_b200 import synthetic as S  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dec():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    arch = S.Arch()
    d = Bd.Decoder(arch, S.workload_weights(0, arch), precision=Bd.MH3A_BF16X3, max_batch=2, max_frames=40)
    z = torch.from_numpy(S.make_latents(2, 40, arch.latent_channels, 17)).cuda()
    yield arch, d, z
    d.close()


def _timed(d, z):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    y = d.decode(z)
    e1.record()
    e1.synchronize()
    return y, e0.elapsed_time(e1)


def test_segment_events_leave_the_output_unchanged_and_add_up(dec):
    arch, d, z = dec
    y_plain = d.decode(z).clone()
    d.set_profiling(True)
    try:
        y, total = _timed(d, z)
        seg = np.asarray(d.segment_times(), dtype=np.float64)
    finally:
        d.set_profiling(False)
    d.check_device_error()
    assert torch.equal(y, y_plain)
    nst = len(arch.rates)
    # input projection, conv_pre, (upsampler, AMP stage) per stage, output conv
    assert seg.shape == (2 + 2 * nst + 1,)
    assert np.all(seg >= 0.0) and np.all(np.isfinite(seg))
    # the segments tile the decode between its first and last event
    assert seg.sum() <= total * 1.05 + 0.05
    assert seg.sum() >= total * 0.5
    # the AMP stages dominate a decode
    amp = seg[3:3 + 2 * nst:2]
    assert amp.sum() > 0.5 * seg.sum()


def test_kernel_events_of_one_stage(dec):
    arch, d, z = dec
    y_plain = d.decode(z).clone()
    d.set_kernel_profiling(1)
    try:
        y = d.decode(z)
        act, gemm = d.stage_kernel_times(1)
        # only the selected stage was recorded
        with pytest.raises(Bd.MH3AError):
            d.stage_kernel_times(2)
    finally:
        d.set_kernel_profiling(-1)
    d.check_device_error()
    assert torch.equal(y, y_plain)
    assert act > 0.0 and gemm > 0.0
    # the stage's six GEMM launches outweigh its six activation launches
    assert gemm > act


def test_kernel_events_of_the_fused_stage(dec):
    arch, d, z = dec
    last = len(arch.rates) - 1
    d.set_kernel_profiling(last)
    try:
        d.decode(z)
        act, gemm = d.stage_kernel_times(last)
    finally:
        d.set_kernel_profiling(-1)
    d.check_device_error()
    # one fused launch runs the whole 8-channel stage: reported as GEMM time, no activation launch
    assert act == 0.0 and gemm > 0.0


def test_out_of_range_queries_are_rejected(dec):
    arch, d, z = dec
    nst = len(arch.rates)
    with pytest.raises(Bd.MH3AError):
        d.stage_kernel_times(nst)
    with pytest.raises(Bd.MH3AError):
        d.stage_kernel_times(-1)
    assert Bd.load().mh3a_stage_uses_tensor_cores(d.handle, nst) == -1
    assert Bd.load().mh3a_segment_uses_tensor_cores(d.handle, 2 + 2 * nst + 1) == -1


def test_tensor_core_queries_follow_the_precision(dec):
    arch, d, z = dec
    nst = len(arch.rates)
    assert all(d.stage_uses_tensor_cores(i) for i in range(nst))
    # every AMP segment of a 3xBF16 handle is on the tensor cores, so are conv_pre and the
    # upsamplers
    assert all(d.segment_uses_tensor_cores(3 + 2 * i) for i in range(nst))
    assert d.segment_uses_tensor_cores(1)
    f32 = Bd.Decoder(arch, S.workload_weights(0, arch), precision=Bd.MH3A_FP32, max_batch=1, max_frames=4)
    try:
        assert not any(f32.stage_uses_tensor_cores(i) for i in range(nst))
        assert not any(f32.segment_uses_tensor_cores(s) for s in range(2 + 2 * nst + 1))
    finally:
        f32.close()
