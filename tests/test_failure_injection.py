"""Failure injection on the host: device allocations that fail inside mh3a_create.

mh3a_create_with_allocator takes the handle's device memory from a caller-supplied allocator.
Here the allocator is a fake that fails on a chosen call, so the failure happens on the host
with no GPU involved: the call must report MH3A_ERR_ALLOC, hand back NULL, and return through
`release` every allocation it had obtained.  Both allocations are made before any device copy,
so these cases run on a machine without a GPU; the case where both allocations succeed reaches
the weight upload and is run only where there is no CUDA device (it then fails there).
"""
from __future__ import annotations

import ctypes as C

import pytest

from bigvgan_waveform_decoder_b200 import binding as Bd
from bigvgan_waveform_decoder_b200 import synthetic as S


class FakeAllocator:
    """Hands out 256-byte aligned host buffers (never touched by the library before the failing
    call) and fails on call number `fail_at` (1-based); records what is outstanding."""

    def __init__(self, fail_at: int, misalign: bool = False):
        self.fail_at = fail_at
        self.misalign = misalign
        self.calls = 0
        self.live = {}
        self.released = []
        self._keep = []

    def alloc(self, nbytes, user):
        self.calls += 1
        if self.calls == self.fail_at:
            return None
        buf = C.create_string_buffer(min(nbytes, 1 << 12) + 512)
        addr = (C.addressof(buf) + 255) & ~255
        if self.misalign:
            addr += 16
        self._keep.append(buf)
        self.live[addr] = nbytes
        return addr

    def release(self, ptr, user):
        self.released.append(ptr)
        self.live.pop(ptr, None)

    def struct(self):
        self._fns = (Bd.ALLOC_FN(self.alloc), Bd.RELEASE_FN(self.release))
        return Bd.mh3a_allocator(self._fns[0], self._fns[1], None)


@pytest.fixture(scope="module")
def small():
    arch = S.Arch(latent_channels=4, latent_dim=32, decoder_dim=128)
    return arch, S.make_weights(arch, 1)


def _create(arch, weights, allocator):
    cfg, keep = Bd.make_config(arch, max_batch=1, max_frames=2)
    tab, keep2 = Bd.make_table(weights)
    h = C.c_void_p(12345)
    a = allocator.struct() if allocator is not None else None
    st = Bd.load().mh3a_create_with_allocator(C.byref(cfg), tab, len(weights),
                                              C.byref(a) if a is not None else None, C.byref(h))
    return st, h


def test_first_allocation_fails(small):
    arch, w = small
    fa = FakeAllocator(fail_at=1)
    st, h = _create(arch, w, fa)
    assert st == 5 and not h.value
    assert fa.calls == 1 and fa.released == [] and fa.live == {}
    assert "weights" in Bd.load().mh3a_last_error().decode()


def test_second_allocation_fails_and_the_first_is_released(small):
    arch, w = small
    fa = FakeAllocator(fail_at=2)
    st, h = _create(arch, w, fa)
    assert st == 5 and not h.value
    assert fa.calls == 2
    assert len(fa.released) == 1 and fa.live == {}
    assert "workspace" in Bd.load().mh3a_last_error().decode()


def test_misaligned_allocation_is_refused_and_released(small):
    arch, w = small
    fa = FakeAllocator(fail_at=99, misalign=True)
    st, h = _create(arch, w, fa)
    assert st == 5 and not h.value
    assert fa.calls == 1 and len(fa.released) == 1 and fa.live == {}


def test_allocator_without_functions_is_rejected(small):
    arch, w = small
    cfg, keep = Bd.make_config(arch)
    tab, keep2 = Bd.make_table(w)
    h = C.c_void_p()
    empty = Bd.mh3a_allocator()
    assert Bd.load().mh3a_create_with_allocator(C.byref(cfg), tab, len(w), C.byref(empty), C.byref(h)) == 1
    assert not h.value


def test_failed_upload_releases_both_allocations(small):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("runs only without a CUDA device: the upload must fail")
    arch, w = small
    fa = FakeAllocator(fail_at=99)
    st, h = _create(arch, w, fa)
    assert st == 6 and not h.value
    assert fa.calls == 2 and len(fa.released) == 2 and fa.live == {}
