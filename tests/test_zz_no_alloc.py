"""mh3a_amp_stage_static, the AMP-stage call for callers that cannot allocate device memory
while they run (a real-time audio thread, or a host whose device memory belongs to another
framework's budget).  It keeps its intermediate buffers in a fixed array inside the library's
device image instead of the handle's workspace.

Checked through the C ABI against the workspace entry point mh3a_amp_stage, on two calls in a
row with different inputs, within the parity tolerances the other GPU tests use, and bit for bit
at the stage where both run the same fused kernel.  The handle
used for the static calls is created with the smallest workspace (max_batch = max_frames = 1),
so those calls cannot be reading the handle's workspace.  This file is collected last.
"""
from __future__ import annotations

import ctypes as C

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from bigvgan_waveform_decoder_b200 import binding as Bd  # noqa: E402
from bigvgan_waveform_decoder_b200 import synthetic as S  # noqa: E402

pytestmark = pytest.mark.gpu

TOL = {Bd.MH3A_FP32: (1e-5, None), Bd.MH3A_BF16X3: (2e-3, 1e-2)}
LIMIT = 2796160  # MH3A_STATIC_SCRATCH_MAX_ELEMS
FUSED_STAGES = (6,)  # stages the decode runs as one fused kernel in BF16X3 mode (8 channels)


def _static_fn():
    lib = Bd.load()
    f = lib.mh3a_amp_stage_static
    f.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p]
    f.restype = C.c_int
    return f


def _close(y, ref, precision, what):
    y = y.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    rl, ma = TOL[precision]
    r = float(np.linalg.norm(y - ref) / np.linalg.norm(ref))
    m = float(np.max(np.abs(y - ref)))
    assert np.all(np.isfinite(y)), what
    assert r <= rl, f"{what}: rel L2 {r:.3e}"
    if ma is not None:
        assert m <= ma, f"{what}: max abs {m:.3e}"


@pytest.mark.parametrize("precision", [Bd.MH3A_FP32, Bd.MH3A_BF16X3])
def test_static_scratch_stage_matches_workspace_stage(precision):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    f = _static_fn()
    arch = S.Arch()
    w = S.workload_weights(0, arch)
    ref_dec = Bd.Decoder(arch, w, precision=precision, max_batch=2, max_frames=64)
    small = Bd.Decoder(arch, w, precision=precision, max_batch=1, max_frames=1)
    stream = torch.cuda.current_stream().cuda_stream
    try:
        # every stage width: several time tiles plus a ragged tail
        for stage, B, L in [(0, 2, 150), (1, 2, 503), (2, 1, 2999), (3, 2, 3001), (4, 1, 10007),
                            (5, 2, 9001), (6, 1, 40003)]:
            C_ = arch.stage_channels(stage)
            for call in range(2):
                x = torch.from_numpy(S.make_stage_input(B, C_, L, 900 + 10 * stage + call)).to(dev)
                ref = ref_dec.amp_stage(x, stage)
                out = torch.full_like(x, float("nan"))
                st = f(small.handle, x.data_ptr(), B, L, stage, out.data_ptr(), stream)
                assert st == 0, Bd.load().mh3a_last_error().decode()
                torch.cuda.synchronize()
                # a bounded pipeline wait that gave up would leave stale scratch behind
                small.check_device_error()
                ref_dec.check_device_error()
                _close(out, ref, precision, f"stage {stage} call {call}")
                if precision == Bd.MH3A_BF16X3 and stage in FUSED_STAGES:
                    # the same fused kernel as mh3a_amp_stage: identical bits
                    assert torch.equal(out, ref), f"stage {stage} call {call}: not bit-identical"
        # beyond the static limit: rejected on the host with a clear message, output untouched
        C0 = arch.stage_channels(0)
        L_big = LIMIT // C0 + 1
        x = torch.zeros((1, C0, L_big), device=dev)
        out = torch.full_like(x, 7.0)
        st = f(small.handle, x.data_ptr(), 1, L_big, 0, out.data_ptr(), stream)
        assert st == 3
        assert "static scratch limit" in Bd.load().mh3a_last_error().decode()
        torch.cuda.synchronize()
        assert bool(torch.all(out == 7.0))
    finally:
        small.close()
        ref_dec.close()
