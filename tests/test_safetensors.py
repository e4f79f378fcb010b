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


# ---------------------------------------------------------------------------------------------
# config.json (mh3a_config_from_json, binding.load_config, Decoder.from_component_dir)
# ---------------------------------------------------------------------------------------------

def _released_like_config(**over):
    """The diffusers constructor arguments with their defaults (the pages say these mirror the
    released audio_vae/config.json), plus diffusers' bookkeeping keys."""
    c = {"_class_name": "AutoencoderKLMiniMaxH3Audio", "_diffusers_version": "0.0.0",
         "encoder_dim": 64, "encoder_rates": [2, 4, 4, 5, 5], "latent_dim": 2048, "latent_channels": 32,
         "num_attention_heads": 8, "decoder_dim": 1024, "decoder_rates": [5, 5, 2, 2, 2, 2, 2],
         "decoder_kernel_sizes": [9, 9, 4, 4, 4, 4, 4], "resblock_kernel_sizes": [3, 7, 11],
         "resblock_dilation_sizes": [[1, 3, 5], [1, 3, 5], [1, 3, 5]], "sampling_rate": 32000,
         "latents_mean": None, "latents_std": None}
    c.update(over)
    return c


def _cfg_status(path, cap=64, with_buffers=True):
    cfg = Bd.mh3a_config()
    m = np.zeros(max(cap, 1), np.float32)
    s = np.zeros(max(cap, 1), np.float32)
    fp = C.POINTER(C.c_float)
    st = Bd.load().mh3a_config_from_json(str(path).encode(), C.byref(cfg),
                                         m.ctypes.data_as(fp) if with_buffers else None,
                                         s.ctypes.data_as(fp) if with_buffers else None, cap)
    return st, cfg, m, s, Bd.load().mh3a_last_error().decode()


def test_released_like_config_gives_the_defaults(tmp_path):
    p = tmp_path / "config.json"
    p.write_text(json.dumps(_released_like_config()))
    a = Bd.load_config(p)
    d = S.Arch()
    assert (a.latent_channels, a.latent_dim, a.decoder_dim) == (d.latent_channels, d.latent_dim, d.decoder_dim)
    assert a.rates == tuple(d.rates) and a.kernels == tuple(d.kernels)
    assert a.rb_kernels == tuple(d.rb_kernels) and a.rb_dilations == tuple(tuple(r) for r in d.rb_dilations)
    assert a.sampling_rate == 32000 and a.latents_mean is None and a.latents_std is None


def test_config_with_statistics_and_a_smaller_architecture(tmp_path):
    rng = np.random.default_rng(3)
    mean = rng.uniform(-0.5, 0.5, 4).tolist()
    std = rng.uniform(0.5, 1.5, 4).tolist()
    p = tmp_path / "config.json"
    p.write_text(json.dumps(_released_like_config(
        latent_channels=4, latent_dim=32, decoder_dim=128, decoder_rates=[8, 5, 4, 5],
        decoder_kernel_sizes=[16, 11, 8, 11], resblock_kernel_sizes=[3, 5],
        resblock_dilation_sizes=[[1, 2], [1, 3]], latents_mean=mean, latents_std=std)))
    a = Bd.load_config(p)
    assert a.latent_channels == 4 and a.rates == (8, 5, 4, 5) and a.kernels == (16, 11, 8, 11)
    assert a.rb_kernels == (3, 5) and a.rb_dilations == ((1, 2), (1, 3))
    np.testing.assert_array_equal(a.latents_mean, np.float32(mean))
    np.testing.assert_array_equal(a.latents_std, np.float32(std))


@pytest.mark.parametrize("case,expect", [
    ({"decoder_rates": [5, 5, 2, 2, 2, 16]}, 2),                                 # stage count, no kernels
    ({"decoder_kernel_sizes": [9, 9, 4]}, 2),                                    # 3 kernels, 7 stages
    ({"decoder_rates": [2] * 9, "decoder_kernel_sizes": [4] * 9}, 2),            # beyond MAX_STAGES
    ({"resblock_dilation_sizes": [[1, 3, 5], [1, 3]]}, 2),                       # 2 rows for 3 blocks
    ({"resblock_dilation_sizes": [[1, 3, 5], [1, 3], [1, 5, 7]]}, 2),            # ragged rows
    ({"resblock_kernel_sizes": [3, 7]}, 2),                                      # block count, no dilations
    ({"latents_mean": [0.0] * 31}, 3),                                           # 31 values for 32 channels
    ({"latent_dim": -2048}, 1),
    ({"latent_channels": 32.5}, 1),
    ({"decoder_rates": "5,5,2"}, 1),
])
def test_bad_configs_are_rejected(tmp_path, case, expect):
    p = tmp_path / "config.json"
    p.write_text(json.dumps(_released_like_config(**case)))
    st, cfg, m, s, err = _cfg_status(p)
    assert st == expect, (case, st, err)
    assert err


def test_malformed_config_and_small_buffers(tmp_path):
    p = tmp_path / "config.json"
    p.write_text('{"latent_dim": 2048,')
    assert _cfg_status(p)[0] == 1
    p.write_text(json.dumps(_released_like_config(latents_mean=[0.1] * 32)))
    assert _cfg_status(p, cap=16)[0] == 3                      # 32 values, room for 16
    assert _cfg_status(p, cap=64, with_buffers=False)[0] == 3   # statistics but no buffers
    st, cfg, m, s, err = _cfg_status(p, cap=64)
    assert st == 0 and bool(cfg.latents_mean) and not bool(cfg.latents_std)
    np.testing.assert_array_equal(m[:32], np.float32([0.1] * 32))
    assert _cfg_status(tmp_path / "nothing.json")[0] == 1


def test_component_dir_needs_the_weights_file(tmp_path):
    (tmp_path / "config.json").write_text(json.dumps(_released_like_config()))
    with pytest.raises(FileNotFoundError):
        Bd.Decoder.from_component_dir(tmp_path)


@pytest.mark.gpu
def test_component_dir_decodes_like_the_table_handle(tmp_path):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    rng = np.random.default_rng(9)
    mean = rng.uniform(-0.5, 0.5, 32).astype(np.float32)
    std = rng.uniform(0.5, 1.5, 32).astype(np.float32)
    arch = S.Arch(latents_mean=mean, latents_std=std)
    w = S.workload_weights(0, S.Arch())
    (tmp_path / "config.json").write_text(json.dumps(_released_like_config(
        latents_mean=mean.tolist(), latents_std=std.tolist())))
    write_st(tmp_path / "diffusion_pytorch_model.safetensors", w, metadata={"format": "pt"})
    z = torch.from_numpy(S.make_latents(2, 8, 32, 78)).cuda()
    a = Bd.Decoder(arch, w, max_batch=2, max_frames=8)
    b = Bd.Decoder.from_component_dir(tmp_path, max_batch=2, max_frames=8)
    try:
        assert torch.equal(a.decode(z), b.decode(z))
        b.check_device_error()
    finally:
        b.close()
        a.close()
