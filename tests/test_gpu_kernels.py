"""Which kernels run: the stage entry point launches the decode's own kernels.

mh3a_amp_stage is the per-stage boundary call whose parity tests stand for the decode's AMP
stages, so it must run exactly the kernels the decode runs for that stage, not a separate
implementation.  The kernel names come from the CUDA profiler (CUPTI, through torch.profiler),
which records every kernel the process launches, the library's included; the library's own
launch counter is checked alongside.
"""
from __future__ import annotations

import re

import pytest

torch = pytest.importorskip("torch")

from bigvgan_waveform_decoder_b200 import binding as Bd  # noqa: E402
from bigvgan_waveform_decoder_b200 import synthetic as S  # noqa: E402

pytestmark = pytest.mark.gpu

# kernels of the fp32 CUDA-core path: none of them may run in a BF16X3 AMP stage
SIMT_CONV = ("k_conv_simt", "k_convT_simt", "k_conv_tc")


def kernel_names(fn):
    """Names of the CUDA kernels launched while fn() runs (after a synchronize)."""
    from torch.profiler import ProfilerActivity, profile

    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    names = []
    for e in prof.events():
        if str(getattr(e, "device_type", "")).endswith("CUDA") and "mh3a::" in e.name:
            names.append(e.name)
    return names


def short(name: str) -> str:
    """'void mh3a::(anonymous namespace)::k_gemm_ps<1, 256, 4, 8, 1>(...)' -> 'k_gemm_ps<1, 256, 4, 8, 1>'."""
    m = re.search(r"::(k_\w+(?:<[^>]*>)?)", name)
    return m.group(1) if m else name


@pytest.fixture(scope="module")
def setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    arch = S.Arch()
    w = S.workload_weights(0, arch)
    d = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=1, max_frames=8)
    z = torch.from_numpy(S.make_latents(1, 8, arch.latent_channels, 5)).to(dev)
    d.decode(z)   # warm-up outside the profiler
    torch.cuda.synchronize()
    decode_kernels = {short(n) for n in kernel_names(lambda: d.decode(z))}
    if not decode_kernels:
        pytest.skip("the CUDA profiler recorded no kernels in this environment")
    yield dev, arch, d, decode_kernels
    d.close()


@pytest.mark.parametrize("stage", range(7))
def test_amp_stage_runs_the_decode_kernels(setup, stage):
    dev, arch, d, decode_kernels = setup
    C = arch.stage_channels(stage)
    L = min(arch.stage_length(stage, 8), 4000)
    x = torch.from_numpy(S.make_stage_input(1, C, L, 40 + stage)).to(dev)
    n0 = d.launch_count()
    names = [short(n) for n in kernel_names(lambda: d.amp_stage(x, stage))]
    launched = d.launch_count() - n0
    d.check_device_error()
    assert d.stage_uses_tensor_cores(stage) == 1
    assert len(names) == launched, (names, launched)
    stage_kernels = set(names) - {"k_mean3"}
    assert not any(k.startswith(SIMT_CONV) for k in stage_kernels), stage_kernels
    # every kernel of the stage call is one the decode itself launches
    assert stage_kernels <= decode_kernels, stage_kernels - decode_kernels
    assert any(k.startswith("k_gemm_ps") or k.startswith("k_amp_") for k in stage_kernels), stage_kernels
