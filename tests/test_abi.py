"""Host-side checks of the C ABI (no GPU): the library loads, exports every entry point that
include/mh3a.h declares, and rejects bad configurations and weight tables before any device
work."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from bigvgan_waveform_decoder_b200 import binding as Bd
from bigvgan_waveform_decoder_b200 import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    txt = open(os.path.join(ROOT, "include", "mh3a.h")).read()
    return sorted(set(re.findall(r"MH3A_API\s+[^;(]*?\b(mh3a_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    lib = Bd.load()
    syms = header_symbols()
    assert len(syms) >= 12
    for s in syms:
        assert hasattr(lib, s), s
    assert set(Bd.EXPORTS) <= set(syms)


def test_default_config_matches_constructor_defaults():
    cfg = Bd.mh3a_config()
    Bd.load().mh3a_default_config(C.byref(cfg))
    assert (cfg.latent_channels, cfg.latent_dim, cfg.decoder_dim, cfg.n_stages) == (32, 2048, 1024, 7)
    assert list(cfg.rates)[:7] == [5, 5, 2, 2, 2, 2, 2]
    assert list(cfg.kernels)[:7] == [9, 9, 4, 4, 4, 4, 4]
    assert list(cfg.rb_kernels)[:3] == [3, 7, 11]
    assert [list(r)[:3] for r in cfg.rb_dilations][:3] == [[1, 3, 5]] * 3
    assert cfg.sampling_rate == 32000 and cfg.precision == Bd.MH3A_BF16X3


def test_status_strings():
    lib = Bd.load()
    for code, text in Bd.STATUS.items():
        assert lib.mh3a_status_string(code).decode() == text


def _create(arch, weights, **kw):
    cfg, keep = Bd.make_config(arch, **kw)
    tab, keep2 = Bd.make_table(weights)
    h = C.c_void_p()
    st = Bd.load().mh3a_create(C.byref(cfg), tab, len(weights), C.byref(h))
    return st, h, cfg


@pytest.fixture(scope="module")
def small():
    arch = S.Arch(latent_channels=4, latent_dim=32, decoder_dim=128)
    return arch, S.make_weights(arch, 1)


def test_create_rejects_bad_configs(small):
    arch, w = small
    lib = Bd.load()
    bad_arches = [
        S.Arch(latent_channels=4, latent_dim=32, decoder_dim=128, rates=(5, 5, 2, 2, 2, 2, 3),
               kernels=(9, 9, 4, 4, 4, 4, 5)),          # hop != 800
        S.Arch(latent_channels=4, latent_dim=32, decoder_dim=128, kernels=(9, 8, 4, 4, 4, 4, 4)),
        S.Arch(latent_channels=4, latent_dim=32, decoder_dim=96),   # not divisible by 2^7
        S.Arch(latent_channels=4, latent_dim=32, decoder_dim=128, rb_kernels=(3, 6, 11)),
    ]
    for a in bad_arches:
        st, h, _ = _create(a, w)
        assert st == 2 and not h.value
    st, h, _ = _create(arch, w, precision=9)
    assert st == 2
    st, h, _ = _create(arch, w, max_batch=0)
    assert st == 2
    assert lib.mh3a_create(None, None, 0, None) == 1


def test_create_rejects_missing_and_misshaped_weights(small):
    arch, w = small
    for key in ("dec_in_proj.weight", "decoder.conv_pre.weight_v", "decoder.ups.3.0.bias",
                "decoder.resblocks.7.convs2.1.weight_g",
                "decoder.resblocks.20.activations.5.act.beta",
                "decoder.activation_post.act.alpha", "decoder.conv_post.weight_v"):
        bad = dict(w)
        del bad[key]
        st, h, _ = _create(arch, bad)
        assert st == 4 and not h.value, key
    bad = dict(w)
    bad["decoder.ups.2.0.weight_v"] = np.zeros((8, 8, 4), np.float32)
    st, h, _ = _create(arch, bad)
    assert st == 3
    bad = dict(w)
    bad["decoder.resblocks.4.activations.0.act.alpha"] = np.ones(3, np.float32)
    st, h, _ = _create(arch, bad)
    assert st == 3


def test_null_handle_calls_are_rejected():
    lib = Bd.load()
    assert lib.mh3a_decode(None, None, 1, 1, None, None) == 1
    assert lib.mh3a_amp_stage(None, None, 1, 1, 0, None, None) == 1
    assert lib.mh3a_launch_count(None) == -1
    lib.mh3a_destroy(None)
