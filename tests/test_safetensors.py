"""mh3a_create_from_safetensors: a decoder built from the audio VAE's single checkpoint file
(FastVideo "minimax_h3_audio_vae" page, `mlx_h3_audio_vae_from_file`: decode prefixes
"dec_in_proj." / "decoder.", three required keys, fp32 storage).

Synthetic files in the safetensors layout (8-byte little-endian header length, JSON header,
data) are written here from seeded random weights.  Every malformed-file case fails before any
device work, so these run without a GPU; a well-formed file on a machine without a GPU gets as far
as the weight upload (the first device copy) and fails there, which shows that parsing, the
prefix filter and the table handed to mh3a_create all passed.  The GPU test at the end checks
that a handle built from the file decodes exactly like one built from the same tensors."""
from __future__ import annotations

import ctypes as C
import json
import struct

import numpy as np
import pytest

from bigvgan_waveform_decoder_b200 import binding as Bd
from bigvgan_waveform_decoder_b200 import synthetic as S

from .test_failure_injection import FakeAllocator

_DT = {"F32": (np.float32, 4), "F16": (np.float16, 2), "BF16": (np.uint16, 2), "F64": (np.float64, 8)}


def write_st(path, tensors, dtypes=None, metadata=None, header_patch=None, tail=b""):
    """tensors: name -> array; dtypes: name -> format dtype (default F32).  header_patch(h) may
    edit the header dict before it is written; tail is appended after the data."""
    dtypes = dtypes or {}
    header, blobs, off = {}, [], 0
    for name, a in tensors.items():
        dt = dtypes.get(name, "F32")
        arr = np.ascontiguousarray(a, dtype=_DT[dt][0])
        b = arr.tobytes()
        header[name] = {"dtype": dt, "shape": list(arr.shape), "data_offsets": [off, off + len(b)]}
        blobs.append(b)
        off += len(b)
    if metadata is not None:
        header["__metadata__"] = metadata
    if header_patch is not None:
        header_patch(header)
    text = json.dumps(header).encode()
    with open(path, "wb") as f:
        f.write(struct.pack("<Q", len(text)))
        f.write(text)
        for b in blobs:
            f.write(b)
        f.write(tail)


@pytest.fixture(scope="module")
def small():
    arch = S.Arch(latent_channels=4, latent_dim=32, decoder_dim=128)
    return arch, S.make_weights(arch, 5)


def _create(arch, path, allocator=None):
    cfg, keep = Bd.make_config(arch, max_batch=1, max_frames=2)
    h = C.c_void_p(12345)
    a = C.byref(allocator) if allocator is not None else None
    st = Bd.load().mh3a_create_from_safetensors(C.byref(cfg), str(path).encode(), a, C.byref(h))
    return st, h, Bd.load().mh3a_last_error().decode()


def _no_gpu():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("runs only without a CUDA device: the weight upload must fail")


def test_well_formed_file_reaches_the_weight_upload(small, tmp_path):
    _no_gpu()
    arch, w = small
    p = tmp_path / "ok.safetensors"
    # other components' tensors in other dtypes and ranks are skipped unread; metadata and unknown
    # fields are ignored
    extra = {"encoder.block.0.weight_v": np.ones((2, 3, 4, 5)), "mean_proj.weight": np.ones((3, 2))}
    write_st(p, {**w, **extra}, dtypes={"encoder.block.0.weight_v": "BF16", "mean_proj.weight": "F16"},
             metadata={"format": "pt", "note": 'a "quoted" \u00e9 value'},
             header_patch=lambda h: h["decoder.conv_pre.bias"].update({"extra_field": [1, {"x": None}]}))
    # host buffers stand in for the two device allocations, so the call gets to the first copy
    fa = FakeAllocator(fail_at=99)
    st, h, err = _create(arch, p, fa.struct())
    assert st == 6 and not h.value, err   # the upload fails: there is no device
    assert fa.calls == 2 and fa.live == {}


def test_missing_required_key(small, tmp_path):
    arch, w = small
    p = tmp_path / "missing.safetensors"
    write_st(p, {k: v for k, v in w.items() if k != "decoder.conv_post.weight_v"})
    st, h, err = _create(arch, p)
    assert st == 4 and not h.value
    assert "decoder.conv_post.weight_v" in err


def test_decoder_tensor_not_fp32_is_refused(small, tmp_path):
    arch, w = small
    p = tmp_path / "f16.safetensors"
    write_st(p, w, dtypes={"decoder.conv_pre.weight_g": "F16"})
    st, h, err = _create(arch, p)
    assert st == 7 and not h.value
    assert "decoder.conv_pre.weight_g" in err and "F16" in err


def test_decoder_tensor_with_four_dims_is_refused(small, tmp_path):
    arch, w = small
    p = tmp_path / "rank4.safetensors"
    write_st(p, {**w, "decoder.conv_pre.extra": np.zeros((1, 2, 3, 4))})
    st, h, err = _create(arch, p)
    assert st == 7 and not h.value


@pytest.mark.parametrize("case", ["length_past_end", "zero_length", "truncated_json", "not_object",
                                  "text_after", "offsets_vs_shape", "offsets_past_end", "missing_field",
                                  "negative_shape", "float_offset"])
def test_malformed_files_are_rejected(small, tmp_path, case):
    arch, w = small
    p = tmp_path / f"{case}.safetensors"
    name = "decoder.conv_pre.bias"
    if case == "length_past_end":
        write_st(p, w)
        raw = bytearray(p.read_bytes())
        raw[:8] = struct.pack("<Q", len(raw))
        p.write_bytes(bytes(raw))
    elif case == "zero_length":
        p.write_bytes(struct.pack("<Q", 0))
    elif case in ("truncated_json", "not_object", "text_after"):
        text = {"truncated_json": b'{"decoder.conv_pre.bias": {"dtype": "F32", "shape": [4',
                "not_object": b'["decoder.conv_pre.bias"]',
                "text_after": b'{} {}'}[case]
        p.write_bytes(struct.pack("<Q", len(text)) + text)
    elif case == "offsets_vs_shape":
        write_st(p, w, header_patch=lambda h: h[name]["shape"].append(2))
    elif case == "offsets_past_end":
        write_st(p, w, header_patch=lambda h: h[name].update(
            {"data_offsets": [h[name]["data_offsets"][0], h[name]["data_offsets"][1] + (1 << 30)]}))
    elif case == "missing_field":
        write_st(p, w, header_patch=lambda h: h[name].pop("dtype"))
    elif case == "negative_shape":
        write_st(p, w, header_patch=lambda h: h[name].update({"shape": [-4]}))
    elif case == "float_offset":
        write_st(p, w, header_patch=lambda h: h[name].update({"data_offsets": [0.5, 4]}))
    st, h, err = _create(arch, p)
    assert st == 1 and not h.value, (case, st, err)
    assert err


def test_unreadable_path_and_null_arguments(small, tmp_path):
    arch, w = small
    st, h, err = _create(arch, tmp_path / "does_not_exist.safetensors")
    assert st == 1 and not h.value and "cannot open" in err
    cfg, keep = Bd.make_config(arch)
    out = C.c_void_p()
    assert Bd.load().mh3a_create_from_safetensors(None, b"x", None, C.byref(out)) == 1
    assert Bd.load().mh3a_create_from_safetensors(C.byref(cfg), None, None, C.byref(out)) == 1


@pytest.mark.gpu
def test_file_handle_decodes_like_the_table_handle(tmp_path):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    arch = S.Arch()
    w = S.workload_weights(0, arch)
    p = tmp_path / "diffusion_pytorch_model.safetensors"
    # the released file also holds encoder tensors, which are skipped
    write_st(p, {**w, "encoder.block.0.weight_v": np.ones((4, 2, 7), np.float32)}, metadata={"format": "pt"})
    z = torch.from_numpy(S.make_latents(2, 9, arch.latent_channels, 77)).cuda()
    a = Bd.Decoder(arch, w, max_batch=2, max_frames=9)
    b = Bd.Decoder(arch, str(p), max_batch=2, max_frames=9)
    try:
        assert torch.equal(a.decode(z), b.decode(z))
        b.check_device_error()
    finally:
        b.close()
        a.close()
