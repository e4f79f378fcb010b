"""Graph replay of decodes (mh3a_set_graph_mode): the first decode for a (B, N, input, output)
launches directly, the second captures the launches into a CUDA graph, later ones replay it.  A replay must produce exactly
the direct decode's output and count the same kernels, follow new contents of the same input
buffer, and every other path (a new shape, a replaced cache slot, the host-buffer entry point,
the default stream, graph mode switched off) must stay exact."""
from __future__ import annotations

import pytest

torch = pytest.importorskip("torch")

from bigvgan_waveform_decoder_b200 import binding as Bd  # noqa: E402
from bigvgan_waveform_decoder_b200 import synthetic as S  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def decs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    arch = S.Arch()
    w = S.workload_weights(0, arch)
    eager = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=2, max_frames=24)
    graph = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=2, max_frames=24)
    graph.set_graph_mode(True)
    yield arch, eager, graph
    graph.close()
    eager.close()


def _lat(arch, B, N, seed):
    return torch.from_numpy(S.make_latents(B, N, arch.latent_channels, seed)).cuda()


def test_replay_matches_direct_decode_and_counts_the_same_kernels(decs):
    arch, eager, graph = decs
    s = torch.cuda.Stream()
    z = _lat(arch, 2, 20, 41)
    y = torch.empty((2, 1, 800 * 20), device="cuda")
    ref = eager.decode(z).clone()
    n0 = eager.launch_count()
    eager.decode(z)
    per_decode = eager.launch_count() - n0
    torch.cuda.synchronize()
    for call in range(4):   # direct, capture, then two replays
        c0 = graph.launch_count()
        with torch.cuda.stream(s):
            y.fill_(float("nan"))
            graph.decode(z, out=y, stream=s)
        s.synchronize()
        assert graph.launch_count() - c0 == per_decode, f"call {call}"
        assert torch.equal(y, ref), f"call {call}"
    # new contents of the same input buffer: the replay reads them
    z.copy_(_lat(arch, 2, 20, 42))
    ref2 = eager.decode(z)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        graph.decode(z, out=y, stream=s)
    s.synchronize()
    assert torch.equal(y, ref2)
    graph.check_device_error()


def test_decode_kernel_count(decs):
    """The launches of one BF16X3 decode at the default architecture: the fused projection and
    conv_pre (2); seven upsamplers, five of them after a standalone input split (12: the last
    layers of the 32- and 16-channel stages write upsamplers 5 and 6's operands themselves);
    six AMP stages of six layers, each an activation and a GEMM (72); the fused 8-channel stage
    and the fused tail (2)."""
    arch, eager, _ = decs
    z = _lat(arch, 1, 6, 43)
    eager.decode(z)
    torch.cuda.synchronize()
    n0 = eager.launch_count()
    eager.decode(z)
    torch.cuda.synchronize()
    assert eager.launch_count() - n0 == 2 + 12 + 72 + 2


def test_several_shapes_and_slot_replacement(decs):
    arch, eager, graph = decs
    s = torch.cuda.Stream()
    # six distinct (B, N, buffers) against four cache slots: first uses launch directly, second
    # uses capture (and replace slots), third uses replay or capture again
    shapes = [(1, 7), (2, 9), (1, 16), (2, 24), (1, 3), (2, 11)]
    bufs = [(_lat(arch, B, N, 50 + i), torch.empty((B, 1, 800 * N), device="cuda")) for i, (B, N) in enumerate(shapes)]
    torch.cuda.synchronize()
    for rnd in range(3):
        for (B, N), (z, y) in zip(shapes, bufs):
            with torch.cuda.stream(s):
                graph.decode(z, out=y, stream=s)
            s.synchronize()
            assert torch.equal(y, eager.decode(z)), f"round {rnd} shape {(B, N)}"
    graph.check_device_error()


def test_default_stream_and_host_entry_point(decs):
    arch, eager, graph = decs
    z = _lat(arch, 2, 12, 61)
    # the legacy default stream cannot be captured: the launches run directly
    assert torch.equal(graph.decode(z, stream=None), eager.decode(z))
    # the host-buffer entry point goes through the handle's own staging buffers
    zh = z.cpu().pin_memory()
    yh = torch.empty((2, 1, 800 * 12)).pin_memory()
    yh_ref = torch.empty((2, 1, 800 * 12)).pin_memory()
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    for _ in range(3):
        graph.decode_host(zh, yh, stream=s)
    eager.decode_host(zh, yh_ref)
    assert torch.equal(yh, yh_ref)
    graph.check_device_error()


def test_switching_graph_mode_off(decs):
    arch, eager, graph = decs
    s = torch.cuda.Stream()
    z = _lat(arch, 1, 10, 71)
    y = torch.empty((1, 1, 8000), device="cuda")
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for _ in range(2):   # the second call leaves a captured graph behind
            graph.decode(z, out=y, stream=s)
    graph.set_graph_mode(False)
    try:
        y2 = torch.empty_like(y)
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            graph.decode(z, out=y2, stream=s)
        s.synchronize()
        ref = eager.decode(z)
        assert torch.equal(y, ref) and torch.equal(y2, ref)
    finally:
        graph.set_graph_mode(True)
    graph.check_device_error()
