"""A handle whose device memory comes from another framework's allocator (torch's caching
allocator here) decodes exactly like one whose memory comes from cudaMalloc, and gives every
allocation back when it is destroyed."""
from __future__ import annotations

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from bigvgan_waveform_decoder_b200 import binding as Bd  # noqa: E402
from bigvgan_waveform_decoder_b200 import synthetic as S  # noqa: E402

pytestmark = pytest.mark.gpu


def test_torch_allocator_handle_matches_default():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    live = {}

    def alloc(n):
        p = torch.cuda.caching_allocator_alloc(n, device=0)
        live[p] = n
        return p

    def release(p):
        live.pop(p)
        torch.cuda.caching_allocator_delete(p)

    arch = S.Arch()
    w = S.workload_weights(0, arch)
    z = torch.from_numpy(S.make_latents(2, 6, arch.latent_channels, 31)).to(dev)
    ref = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=2, max_frames=8)
    d = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=2, max_frames=8, allocator=(alloc, release))
    assert len(live) == 2
    try:
        y_ref = ref.decode(z).cpu().numpy()
        y = d.decode(z).cpu().numpy()
        d.check_device_error()
        np.testing.assert_array_equal(y, y_ref)
    finally:
        d.close()
        ref.close()
    assert live == {}
